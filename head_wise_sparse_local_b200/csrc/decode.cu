// rtp_decode_attn: one decode step of the head-wise sparse attention layer.
//
// Pipeline (all on the caller's stream, scratch in the caller's workspace):
//   1. score_kernel   streams the 16-d indexer-key cache once (two 16-byte
//                     loads per token), forms s_j = q~ . k~_j / 4 for the G
//                     query heads of a retrieval KV head, stores the fp32
//                     scores and a per-chunk maximum.
//   2. hist_kernel    softmax mass of every score, exp(s - max) in 2^-40 fixed
//                     point, into a 2048-bucket histogram ordered by score;
//                     the last CTA of a head finds the bucket where the
//                     cumulative mass (highest scores first) reaches
//                     ceil(p * Z).
//   3. collect_kernel gathers the scores that fall into that bucket; the last
//                     CTA of a head resolves the exact threshold score tau by
//                     8-bit radix passes over the candidates and, when only
//                     some tokens tied at tau fit, the index j_cut of the last
//                     one kept (ties go to the lower index).
//   4. attn_kernel    exact attention.  Sink/window tiles cover every KV head;
//                     selected-row tiles scan a retrieval head's context and
//                     attend the kept rows outside sinks/window.  Each CTA
//                     writes (max, sum, unnormalised o) per query head; the
//                     last CTA of a KV head merges them (log-sum-exp) into out.
// Top-p follows the abstract's observation (3) and the atlas.scime.ai summary
// ("query-adaptive top-p threshold"); sinks + window follow the same summary's
// "Approach"; the 16-d pre-RoPE indexer follows observation (2).
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace rtp {
namespace {

constexpr int kThreads = 256;
constexpr int kScoreChunk = 1024;  // tokens per score CTA
constexpr int kSelChunk = 4096;    // tokens per histogram / collect CTA
constexpr int kSwTile = 128;       // sink/window rows per attention CTA
constexpr int kSelTile = 2048;     // context rows scanned per selected-row CTA
constexpr int kCandSmem = 4096;    // candidates staged in shared memory for the solve

enum : int { kModeThresh = 0, kModeAll = 1, kModeSkip = 2 };

struct DecodeHead {
  unsigned long long target;  // ceil(p * Z), 2^-40 units
  unsigned long long above;   // mass of the buckets above the boundary bucket
  float m;                    // maximum score
  float tau;                  // score of the last kept token
  int bucket;                 // boundary bucket
  int mode;
  int jcut;                   // tokens with score == tau kept iff index <= jcut
  unsigned cnt_above;         // tokens in the buckets above the boundary
  int pad[2];
};

struct DecodeArgs {
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W, max_seq_len, words;
  float top_p, rope_base;
  const void* q_pre;
  const float* w_q;
  void* out;
  const void* k;
  const void* v;
  const void* kidx;
  int* status;
  const int* seq_len;
  uint32_t* sel_bitmask;
  int* sel_count;
  float* logits;
  float* cmax;
  unsigned long long* hmass;
  unsigned* hcnt;
  DecodeHead* heads;
  unsigned* ctl;  // [tick_hist NRt][tick_coll NRt][ncand NRt][tick_attn B*Hkv]
  uint2* cand;
  float* pm;
  float* pl;
  float* po;
  int n_ctl, nch_score_max, n_sw_tiles, n_tiles_max;
  int ret_head[kMaxRetrieval];
  int ret_rank[kMaxRetrieval];
};

__device__ __forceinline__ unsigned* tick_hist(const DecodeArgs& a) { return a.ctl; }
__device__ __forceinline__ unsigned* tick_coll(const DecodeArgs& a) { return a.ctl + a.B * a.NR; }
__device__ __forceinline__ unsigned* ncand(const DecodeArgs& a) { return a.ctl + 2 * a.B * a.NR; }
__device__ __forceinline__ unsigned* tick_attn(const DecodeArgs& a) { return a.ctl + 3 * a.B * a.NR; }

__device__ __forceinline__ bool seq_ok(int L, const DecodeArgs& a) {
  return L >= 1 && L <= a.max_seq_len;
}

// Block-wide max for kThreads threads.
__device__ __forceinline__ float block_max(float v, float* sm) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  float r = sm[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) r = fmaxf(r, sm[w]);
  return r;
}

// "Last CTA of the group" ticket: every CTA of the group calls this once.
__device__ __forceinline__ bool take_ticket(unsigned* counter, unsigned n, int* s_flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned t = atomicAdd(counter, 1u);
    *s_flag = (t == n - 1);
  }
  __syncthreads();
  const bool last = *s_flag;
  if (last) __threadfence();
  return last;
}

// ---------------------------------------------------------------------------
// 1. indexer scores
// ---------------------------------------------------------------------------
template <typename T, int G>
__global__ void __launch_bounds__(kThreads) score_kernel(DecodeArgs a) {
  const int chunk = blockIdx.x;
  const int b = blockIdx.y / a.R, r = blockIdx.y % a.R;
  const int tid = threadIdx.x;
  {  // zero this call's histograms and control words (read by later kernels)
    const size_t cta = (size_t)blockIdx.y * gridDim.x + chunk;
    const size_t n_cta = (size_t)gridDim.x * gridDim.y;
    const size_t n_hist = (size_t)a.B * a.NR * kNumBuckets;
    for (size_t i = cta * kThreads + tid; i < n_hist; i += n_cta * kThreads) {
      a.hmass[i] = 0ull;
      a.hcnt[i] = 0u;
    }
    if (cta == 0)
      for (int i = tid; i < a.n_ctl; i += kThreads) a.ctl[i] = 0u;
  }
  const int L = a.seq_len[b];
  if (!seq_ok(L, a)) {
    if (chunk == 0 && r == 0 && tid == 0) atomicOr(a.status, RTP_DEV_SEQ_LEN);
    return;
  }
  const int j0 = chunk * kScoreChunk;
  if (j0 >= L) return;
  const int h = a.ret_head[r];

  __shared__ float s_q[G][kIdxDim];
  __shared__ float s_red[kThreads / 32];
  if (tid < G * kIdxDim) {
    const int g = tid / kIdxDim, i = tid % kIdxDim;
    const float* w = a.w_q + ((size_t)r * kIdxDim + i) * a.D;
    const T* q = static_cast<const T*>(a.q_pre) + ((size_t)b * a.Hq + h * G + g) * a.D;
    float acc = 0.f;
    for (int d = 0; d < a.D; ++d) acc = fmaf(__ldg(w + d), to_f32(q[d]), acc);
    s_q[g][i] = acc;
  }
  __syncthreads();
  float qr[G][kIdxDim];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < kIdxDim; ++i) qr[g][i] = s_q[g][i];

  const T* kidx = static_cast<const T*>(a.kidx) + ((size_t)b * a.R + r) * a.Lmax * kIdxDim;
  float* lg = a.logits + ((size_t)b * a.NR + (size_t)r * G) * a.Lmax;
  float mx[G];
#pragma unroll
  for (int g = 0; g < G; ++g) mx[g] = -CUDART_INF_F;
  const int j1 = min(L, j0 + kScoreChunk);
#pragma unroll 4
  for (int j = j0 + tid; j < j1; j += kThreads) {
    float kv[kIdxDim];
    load_row<T, kIdxDim>(kidx + (size_t)j * kIdxDim, kv);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < kIdxDim; ++i) s = fmaf(qr[g][i], kv[i], s);
      s = s * kIdxScale + 0.0f;  // exact scaling; +0 turns -0 into +0
      lg[(size_t)g * a.Lmax + j] = s;
      mx[g] = fmaxf(mx[g], s);
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float m = block_max(mx[g], s_red);
    if (tid == 0) a.cmax[((size_t)b * a.NR + r * G + g) * a.nch_score_max + chunk] = m;
  }
}

// ---------------------------------------------------------------------------
// 2. mass histogram + boundary bucket
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) hist_kernel(DecodeArgs a) {
  const int chunk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.NR;
  const int tid = threadIdx.x;
  __shared__ unsigned long long s_mass[kNumBuckets];
  __shared__ unsigned s_cnt[kNumBuckets];
  __shared__ float s_red[kThreads / 32];
  __shared__ unsigned long long s_sa[kThreads / 32];
  __shared__ unsigned s_sc[kThreads / 32];
  __shared__ int s_flag;

  const int L = a.seq_len[b];
  const bool valid = seq_ok(L, a);
  const bool keep_all = a.top_p >= 1.0f;
  float m = -CUDART_INF_F;
  unsigned long long* gm = a.hmass + (size_t)bh * kNumBuckets;
  unsigned* gc = a.hcnt + (size_t)bh * kNumBuckets;
  if (valid && !keep_all) {
    const int nch = (L + kScoreChunk - 1) / kScoreChunk;
    const float* cm = a.cmax + (size_t)bh * a.nch_score_max;
    for (int c = tid; c < nch; c += kThreads) m = fmaxf(m, cm[c]);
    m = block_max(m, s_red);
    const int j0 = chunk * kSelChunk;
    if (j0 < L) {
      for (int i = tid; i < kNumBuckets; i += kThreads) { s_mass[i] = 0ull; s_cnt[i] = 0u; }
      __syncthreads();
      const float* lg = a.logits + (size_t)bh * a.Lmax;
      const int j1 = min(L, j0 + kSelChunk);
      for (int j = j0 + tid; j < j1; j += kThreads) {
        const float s = lg[j];
        const int bk = score_bucket(s);
        atomicAdd(&s_mass[bk], mass_fx(s, m));
        atomicAdd(&s_cnt[bk], 1u);
      }
      __syncthreads();
      for (int i = tid; i < kNumBuckets; i += kThreads) {
        if (s_cnt[i]) {
          atomicAdd(&gm[i], s_mass[i]);
          atomicAdd(&gc[i], s_cnt[i]);
        }
      }
    }
  }
  if (!take_ticket(&tick_hist(a)[bh], gridDim.x, &s_flag)) return;

  DecodeHead* hd = a.heads + bh;
  if (!valid) {
    if (tid == 0) hd->mode = kModeSkip;
    return;
  }
  if (keep_all) {
    if (tid == 0) {
      hd->mode = kModeAll;
      if (a.sel_count) a.sel_count[bh] = L;
    }
    return;
  }
  // Thread t owns buckets NB-1-8t-k, k = 0..7 (highest scores first).
  constexpr int kPer = kNumBuckets / kThreads;
  unsigned long long ms[kPer];
  unsigned cs[kPer];
  unsigned long long my_m = 0ull;
  unsigned my_c = 0u;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int bk = kNumBuckets - 1 - (tid * kPer + k);
    ms[k] = __ldcg(gm + bk);
    cs[k] = __ldcg(gc + bk);
    my_m += ms[k];
    my_c += cs[k];
  }
  unsigned long long ex_m, tot_m;
  unsigned ex_c, tot_c;
  block_excl_scan2<kThreads>(my_m, my_c, ex_m, ex_c, tot_m, tot_c, s_sa, s_sc);
  const double pz = (double)a.top_p * (double)tot_m;
  unsigned long long target = (unsigned long long)ceil(pz);
  if (target > tot_m) target = tot_m;
  if (target < 1ull) target = 1ull;
  __shared__ unsigned long long s_above;
  __shared__ unsigned s_cabove;
  __shared__ int s_bucket;
  if (tid == 0) s_bucket = -1;
  __syncthreads();
  unsigned long long cum = ex_m;
  unsigned cumc = ex_c;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    if (cum < target && cum + ms[k] >= target) {  // exactly one (thread, k) crosses
      s_above = cum;
      s_cabove = cumc;
      s_bucket = kNumBuckets - 1 - (tid * kPer + k);
    }
    cum += ms[k];
    cumc += cs[k];
  }
  __syncthreads();
  if (tid == 0) {
    if (s_bucket < 0) {  // unreachable for target <= Z; keep every token rather than guess
      hd->mode = kModeAll;
      if (a.sel_count) a.sel_count[bh] = L;
    } else {
      hd->target = target;
      hd->above = s_above;
      hd->cnt_above = s_cabove;
      hd->bucket = s_bucket;
      hd->m = m;
      hd->mode = kModeThresh;
    }
  }
}

// ---------------------------------------------------------------------------
// 3. candidates of the boundary bucket + exact threshold
// ---------------------------------------------------------------------------
struct DigitResult {
  int digit;
  unsigned long long above;  // mass (or count) of the digits ranked before `digit`
  unsigned cnt_above;
  unsigned cnt_digit;
};

// One 8-bit radix step over items[0, n).  kMass: items matching (x & mask) ==
// prefix are weighted by their softmax mass and digits are ranked from high to
// low (highest scores first).  !kMass: items with x == key_eq are counted and
// their index digits (y) ranked from low to high (lowest index first).  Finds
// the first digit at which the running total reaches `need`.
template <bool kMass>
__device__ DigitResult radix_step(const uint2* items, int n, uint32_t prefix, uint32_t mask,
                                  uint32_t key_eq, int shift, float m, unsigned long long need,
                                  unsigned long long* h_m, unsigned* h_c, DigitResult* s_res) {
  const int tid = threadIdx.x;
  for (int i = tid; i < 256; i += kThreads) { h_m[i] = 0ull; h_c[i] = 0u; }
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) {
    const uint2 it = items[i];
    if constexpr (kMass) {
      if ((it.x & mask) == prefix) {
        const int dg = (it.x >> shift) & 255;
        atomicAdd(&h_m[dg], mass_fx(key_score(it.x), m));
        atomicAdd(&h_c[dg], 1u);
      }
    } else {
      if (it.x == key_eq && (it.y & mask) == prefix) {
        const int dg = (it.y >> shift) & 255;
        atomicAdd(&h_m[dg], 1ull);
        atomicAdd(&h_c[dg], 1u);
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    const int lane = tid;
    unsigned long long w[8];
    unsigned c[8];
    unsigned long long sw = 0ull;
    unsigned sc = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int dg = kMass ? 255 - (lane * 8 + k) : lane * 8 + k;
      w[k] = h_m[dg];
      c[k] = h_c[dg];
      sw += w[k];
      sc += c[k];
    }
    const unsigned long long incl = warp_incl_scan_u64(sw);
    const unsigned inclc = warp_incl_scan_u32(sc);
    unsigned long long cum = incl - sw;
    unsigned cumc = inclc - sc;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (cum < need && cum + w[k] >= need) {
        s_res->digit = kMass ? 255 - (lane * 8 + k) : lane * 8 + k;
        s_res->above = cum;
        s_res->cnt_above = cumc;
        s_res->cnt_digit = c[k];
      }
      cum += w[k];
      cumc += c[k];
    }
  }
  __syncthreads();
  const DigitResult res = *s_res;
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kThreads) collect_kernel(DecodeArgs a) {
  const int chunk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.NR;
  const int tid = threadIdx.x, lane = tid & 31;
  __shared__ int s_flag;
  __shared__ __align__(16) uint2 s_cand[kCandSmem];
  __shared__ unsigned long long h_m[256];
  __shared__ unsigned h_c[256];
  __shared__ DigitResult s_res;
  __shared__ uint32_t s_kmin[kThreads / 32], s_kmax[kThreads / 32];

  const int L = a.seq_len[b];
  const bool valid = seq_ok(L, a);
  DecodeHead* hd = a.heads + bh;
  const int mode = valid ? hd->mode : kModeSkip;
  uint2* cand = a.cand + (size_t)bh * a.Lmax;
  if (mode == kModeThresh) {
    const int bucket = hd->bucket;
    const float* lg = a.logits + (size_t)bh * a.Lmax;
    const int j0 = chunk * kSelChunk;
    const int j1 = min(L, j0 + kSelChunk);
    for (int jb = j0; jb < j1; jb += kThreads) {
      const int j = jb + tid;
      float s = 0.f;
      bool in = false;
      if (j < j1) {
        s = lg[j];
        in = score_bucket(s) == bucket;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      if (bal) {
        unsigned base = 0;
        if (lane == 0) base = atomicAdd(&ncand(a)[bh], (unsigned)__popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (in) cand[base + __popc(bal & ((1u << lane) - 1u))] = make_uint2(score_key(s), (unsigned)j);
      }
    }
  }
  if (!take_ticket(&tick_coll(a)[bh], gridDim.x, &s_flag)) return;
  if (mode != kModeThresh) return;

  // ---- exact threshold among the candidates (this CTA only) ----
  const int n = (int)__ldcg(&ncand(a)[bh]);
  const float m = hd->m;
  const unsigned long long need0 = hd->target - hd->above;
  const uint2* items = cand;
  if (n <= kCandSmem) {
    for (int i = tid; i < n; i += kThreads) s_cand[i] = __ldcg(cand + i);
    __syncthreads();
    items = s_cand;
  }
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int i = tid; i < n; i += kThreads) {
    const uint32_t k = items[i].x;
    kmin = min(kmin, k);
    kmax = max(kmax, k);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) { s_kmin[tid >> 5] = kmin; s_kmax[tid >> 5] = kmax; }
  __syncthreads();
  kmin = s_kmin[0];
  kmax = s_kmax[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) { kmin = min(kmin, s_kmin[w]); kmax = max(kmax, s_kmax[w]); }

  uint32_t prefix = kmin, mask = 0xffffffffu;
  unsigned long long need = need0;
  unsigned cnt_above_in = 0u;
  unsigned cnt_eq = (unsigned)n;
  const uint32_t diff = kmin ^ kmax;
  if (diff != 0u) {
    const int hb = 31 - __clz(diff);
    mask = (hb == 31) ? 0u : ~((2u << hb) - 1u);
    prefix = kmin & mask;
    for (int shift = (hb / 8) * 8; shift >= 0; shift -= 8) {
      const DigitResult d = radix_step<true>(items, n, prefix, mask, 0u, shift, m, need, h_m, h_c, &s_res);
      need -= d.above;
      cnt_above_in += d.cnt_above;
      cnt_eq = d.cnt_digit;
      prefix |= (uint32_t)d.digit << shift;
      mask |= 0xffu << shift;
    }
  }
  const uint32_t tau_key = prefix;
  const unsigned long long w_tau = mass_fx(key_score(tau_key), m);
  unsigned long long kk = (w_tau > 0ull) ? (need + w_tau - 1ull) / w_tau : (unsigned long long)cnt_eq;
  if (kk < 1ull) kk = 1ull;
  if (kk > cnt_eq) kk = cnt_eq;
  int jcut = INT_MAX;
  if (kk < cnt_eq) {  // only the first kk tied tokens (by index) are kept
    uint32_t ip = 0u, im = 0u;
    unsigned long long want = kk;
    for (int shift = 16; shift >= 0; shift -= 8) {
      const DigitResult d = radix_step<false>(items, n, ip, im, tau_key, shift, 0.f, want, h_m, h_c, &s_res);
      want -= d.above;
      ip |= (uint32_t)d.digit << shift;
      im |= 0xffu << shift;
    }
    jcut = (int)ip;
  }
  if (tid == 0) {
    hd->tau = key_score(tau_key);
    hd->jcut = jcut;
    if (a.sel_count) a.sel_count[bh] = (int)(hd->cnt_above + cnt_above_in + (unsigned)kk);
  }
}

// ---------------------------------------------------------------------------
// 4. attention over sinks/window and kept rows, then the log-sum-exp merge
// ---------------------------------------------------------------------------
template <int D, int G>
struct AttnCfg {
  static constexpr int kLpr = (G == 8 && D == 128) ? 16 : 8;  // lanes per row
  static constexpr int kDpl = D / kLpr;                       // dims per lane
  static constexpr int kGroups = kThreads / kLpr;             // rows in flight per CTA
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) attn_kernel(DecodeArgs a) {
  using C = AttnCfg<D, G>;
  constexpr int LPR = C::kLpr, DPL = C::kDpl, NGRP = C::kGroups;
  constexpr int kWarps = kThreads / 32;
  const int tile = blockIdx.x;
  const int bkv = blockIdx.y;
  const int b = bkv / a.Hkv, h = bkv % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = a.ret_rank[h];
  const bool sel_tile = tile >= a.n_sw_tiles;

  __shared__ float s_q[G][D];
  __shared__ int s_row[kSelTile];
  __shared__ unsigned char s_msk[kSelTile];
  __shared__ int s_wcnt[kWarps];
  __shared__ float s_o[kWarps][G][D];
  __shared__ float s_m[kWarps][G], s_l[kWarps][G];
  __shared__ int s_flag;

  const int L = a.seq_len[b];
  const bool valid = seq_ok(L, a);
  const int s_cnt = valid ? min(a.S, L) : 0;
  const int sw0 = valid ? max(s_cnt, L - a.W) : 0;
  const bool active = valid && (!sel_tile || r >= 0);
  const size_t part0 = (size_t)bkv * a.n_tiles_max + tile;

  if (!valid && tile == 0 && h == 0 && tid == 0) atomicOr(a.status, RTP_DEV_SEQ_LEN);

  if (active) {
    // RoPE'd query at position L-1, pre-scaled by log2(e)/sqrt(D)
    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    for (int i = tid; i < G * (D / 2); i += kThreads) {
      const int g = i / (D / 2), k = i % (D / 2);
      const T* q = static_cast<const T*>(a.q_pre) + ((size_t)b * a.Hq + h * G + g) * D;
      const float x1 = to_f32(q[k]), x2 = to_f32(q[k + D / 2]);
      float c, s;
      rope_cos_sin(L - 1, k, D, a.rope_base, c, s);
      s_q[g][k] = (x1 * c - x2 * s) * qscale;
      s_q[g][k + D / 2] = (x2 * c + x1 * s) * qscale;
    }
    int n_rows = 0;
    int e0 = 0;
    if (!sel_tile) {
      const int n_sw = s_cnt + (L - sw0);
      e0 = tile * kSwTile;
      n_rows = max(0, min(kSwTile, n_sw - e0));
    } else {
      // scan [j0, j0 + kSelTile) for kept rows; record bitmask / list
      const int j0 = (tile - a.n_sw_tiles) * kSelTile;
      float tau[G];
      int jcut[G], mode[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const DecodeHead* hd = a.heads + (size_t)b * a.NR + r * G + g;
        mode[g] = hd->mode;
        tau[g] = hd->tau;
        jcut[g] = hd->jcut;
      }
      const float* lg = a.logits + ((size_t)b * a.NR + (size_t)r * G) * a.Lmax;
      int base = 0;
      for (int it = 0; it < kSelTile; it += kThreads) {
        const int j = j0 + it + tid;
        unsigned msk = 0u;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          bool in = false;
          if (j < L) {
            if (mode[g] == kModeAll) in = true;
            else {
              const float s = lg[(size_t)g * a.Lmax + j];
              in = s > tau[g] || (s == tau[g] && j <= jcut[g]);
            }
          }
          const unsigned word = __ballot_sync(0xffffffffu, in);
          if (a.sel_bitmask && lane == 0 && (j >> 5) < a.words && j0 + it < a.max_seq_len)
            a.sel_bitmask[((size_t)b * a.NR + r * G + g) * a.words + (j >> 5)] = word;
          msk |= (in ? 1u : 0u) << g;
        }
        const bool att = msk != 0u && j >= s_cnt && j < sw0;
        const unsigned bal = __ballot_sync(0xffffffffu, att);
        if (lane == 0) s_wcnt[warp] = __popc(bal);
        __syncthreads();
        int off = base;
        int tot = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          if (w < warp) off += s_wcnt[w];
          tot += s_wcnt[w];
        }
        if (att) {
          const int p = off + __popc(bal & ((1u << lane) - 1u));
          s_row[p] = j;
          s_msk[p] = (unsigned char)msk;
        }
        base += tot;
        __syncthreads();
      }
      n_rows = base;
    }
    __syncthreads();

    // ---- rows: LPR lanes per row, DPL dims per lane ----
    const int grp = tid / LPR, sub = tid % LPR;
    float qv[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int d = 0; d < DPL; ++d) qv[g][d] = s_q[g][sub * DPL + d];
    float mrun[G], lrun[G], o[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mrun[g] = -CUDART_INF_F;
      lrun[g] = 0.f;
#pragma unroll
      for (int d = 0; d < DPL; ++d) o[g][d] = 0.f;
    }
    const T* kbase = static_cast<const T*>(a.k) + ((size_t)b * a.Hkv + h) * a.Lmax * D + sub * DPL;
    const T* vbase = static_cast<const T*>(a.v) + ((size_t)b * a.Hkv + h) * a.Lmax * D + sub * DPL;
    // Every lane runs the same trip count (the shuffles below name the whole
    // warp); rows past n_rows are masked out.
    const int n_iter = (n_rows + NGRP - 1) / NGRP;
    for (int itr = 0; itr < n_iter; ++itr) {
      const int e = itr * NGRP + grp;
      int row = 0;
      unsigned msk = 0u;
      if (e < n_rows) {
        if (!sel_tile) {
          const int idx = e0 + e;
          row = idx < s_cnt ? idx : sw0 + (idx - s_cnt);
          msk = (1u << G) - 1u;
        } else {
          row = s_row[e];
          msk = s_msk[e];
        }
      }
      RawRow<T, DPL> kr, vr;
      kr.load(kbase + (size_t)row * D);  // row 0 always exists (L >= 1)
      vr.load(vbase + (size_t)row * D);
      float sc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float acc = 0.f;
#pragma unroll
        for (int d = 0; d < DPL; ++d) acc = fmaf(qv[g][d], kr.get(d), acc);
        sc[g] = acc;
      }
#pragma unroll
      for (int off = 1; off < LPR; off <<= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], off);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if ((msk >> g) & 1u) {
          const float mn = fmaxf(mrun[g], sc[g]);
          const float al = exp2f(mrun[g] - mn);
          const float p = exp2f(sc[g] - mn);
          lrun[g] = lrun[g] * al + p;
#pragma unroll
          for (int d = 0; d < DPL; ++d) o[g][d] = fmaf(p, vr.get(d), o[g][d] * al);
          mrun[g] = mn;
        }
      }
    }
    // merge the row groups of a warp (lanes differing in bits >= log2(LPR))
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mo = __shfl_xor_sync(0xffffffffu, mrun[g], off);
        const float lo = __shfl_xor_sync(0xffffffffu, lrun[g], off);
        const float mn = fmaxf(mrun[g], mo);
        const float al = (mn == -CUDART_INF_F) ? 0.f : exp2f(mrun[g] - mn);
        const float be = (mn == -CUDART_INF_F) ? 0.f : exp2f(mo - mn);
        lrun[g] = lrun[g] * al + lo * be;
#pragma unroll
        for (int d = 0; d < DPL; ++d) {
          const float oo = __shfl_xor_sync(0xffffffffu, o[g][d], off);
          o[g][d] = o[g][d] * al + oo * be;
        }
        mrun[g] = mn;
      }
    }
    if (lane < LPR) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int d = 0; d < DPL; ++d) s_o[warp][g][lane * DPL + d] = o[g][d];
        if (lane == 0) { s_m[warp][g] = mrun[g]; s_l[warp][g] = lrun[g]; }
      }
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += kThreads) {
      const int g = i / D, d = i % D;
      float mn = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) mn = fmaxf(mn, s_m[w][g]);
      float acc = 0.f, den = 0.f;
      if (mn != -CUDART_INF_F) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float sc = exp2f(s_m[w][g] - mn);
          acc = fmaf(s_o[w][g][d], sc, acc);
          den = fmaf(s_l[w][g], sc, den);
        }
      }
      a.po[(part0 * G + g) * D + d] = acc;
      if (d == 0) {
        a.pm[part0 * G + g] = mn;
        a.pl[part0 * G + g] = den;
      }
    }
  }

  if (!take_ticket(&tick_attn(a)[bkv], gridDim.x, &s_flag)) return;
  if (!valid) return;
  // ---- merge the tiles of this KV head into out ----
  const int n_parts = (r >= 0) ? (int)gridDim.x : a.n_sw_tiles;
  const size_t pbase = (size_t)bkv * a.n_tiles_max;
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, d = i % D;
    float mn = -CUDART_INF_F;
    for (int t = 0; t < n_parts; ++t) mn = fmaxf(mn, __ldcg(a.pm + (pbase + t) * G + g));
    float acc = 0.f, den = 0.f;
    for (int t = 0; t < n_parts; ++t) {
      const float pmv = __ldcg(a.pm + (pbase + t) * G + g);
      if (pmv == -CUDART_INF_F) continue;
      const float sc = exp2f(pmv - mn);
      acc = fmaf(__ldcg(a.po + ((pbase + t) * G + g) * D + d), sc, acc);
      den = fmaf(__ldcg(a.pl + (pbase + t) * G + g), sc, den);
    }
    T* out = static_cast<T*>(a.out) + ((size_t)b * a.Hq + h * G + g) * D + d;
    *out = from_f32<T>(acc / den);
  }
}

template <typename T, int G>
void launch_score(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  score_kernel<T, G><<<grid, kThreads, 0, st>>>(a);
}

template <typename T, int D>
void launch_attn_g(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  switch (a.G) {
    case 1: attn_kernel<T, D, 1><<<grid, kThreads, 0, st>>>(a); break;
    case 2: attn_kernel<T, D, 2><<<grid, kThreads, 0, st>>>(a); break;
    case 4: attn_kernel<T, D, 4><<<grid, kThreads, 0, st>>>(a); break;
    default: attn_kernel<T, D, 8><<<grid, kThreads, 0, st>>>(a); break;
  }
}

template <typename T>
void launch_score_g(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  switch (a.G) {
    case 1: launch_score<T, 1>(a, grid, st); break;
    case 2: launch_score<T, 2>(a, grid, st); break;
    case 4: launch_score<T, 4>(a, grid, st); break;
    default: launch_score<T, 8>(a, grid, st); break;
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

DecodeLayout decode_layout(const Shape& sh) {
  DecodeLayout l;
  const size_t NRt = (size_t)sh.B * sh.NR;
  l.nch_score_max = (sh.Lmax + kScoreChunk - 1) / kScoreChunk;
  l.nch_sel_max = (sh.Lmax + kSelChunk - 1) / kSelChunk;
  l.n_sw_tiles = (sh.S + sh.W + kSwTile - 1) / kSwTile;
  l.n_sel_tiles_max = (sh.Lmax + kSelTile - 1) / kSelTile;
  l.n_tiles_max = l.n_sw_tiles + (sh.R > 0 ? l.n_sel_tiles_max : 0);
  l.n_ctl = (int)(3 * NRt + (size_t)sh.B * sh.Hkv);
  size_t off = 0;
  l.logits = off; off = align256(off + NRt * sh.Lmax * sizeof(float));
  l.cmax = off;   off = align256(off + NRt * l.nch_score_max * sizeof(float));
  l.hmass = off;  off = align256(off + NRt * kNumBuckets * sizeof(unsigned long long));
  l.hcnt = off;   off = align256(off + NRt * kNumBuckets * sizeof(unsigned));
  l.heads = off;  off = align256(off + NRt * sizeof(DecodeHead));
  l.ctl = off;    off = align256(off + (size_t)l.n_ctl * sizeof(unsigned));
  l.cand = off;   off = align256(off + NRt * sh.Lmax * sizeof(uint2));
  const size_t nparts = (size_t)sh.B * sh.Hkv * l.n_tiles_max * sh.G;
  l.pm = off;     off = align256(off + nparts * sizeof(float));
  l.pl = off;     off = align256(off + nparts * sizeof(float));
  l.po = off;     off = align256(off + nparts * sh.D * sizeof(float));
  l.total = off;
  return l;
}

int launch_decode(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* seq_len,
                  int max_seq_len, const float* w_q, void* out, uint32_t* sel_bitmask,
                  int* sel_count, void* ws, const DecodeLayout& lay, cudaStream_t st) {
  DecodeArgs a;
  a.B = sh.B; a.Hq = sh.Hq; a.Hkv = sh.Hkv; a.G = sh.G; a.D = sh.D; a.R = sh.R; a.NR = sh.NR;
  a.Lmax = sh.Lmax; a.S = sh.S; a.W = sh.W;
  a.max_seq_len = max_seq_len > 0 ? max_seq_len : sh.Lmax;
  a.words = (sh.Lmax + 31) / 32;
  a.top_p = sh.top_p; a.rope_base = sh.rope_base;
  a.q_pre = q_pre; a.w_q = w_q; a.out = out;
  a.k = cache->k; a.v = cache->v; a.kidx = cache->kidx; a.status = cache->status;
  a.seq_len = seq_len; a.sel_bitmask = sel_bitmask; a.sel_count = sel_count;
  char* w = static_cast<char*>(ws);
  a.logits = reinterpret_cast<float*>(w + lay.logits);
  a.cmax = reinterpret_cast<float*>(w + lay.cmax);
  a.hmass = reinterpret_cast<unsigned long long*>(w + lay.hmass);
  a.hcnt = reinterpret_cast<unsigned*>(w + lay.hcnt);
  a.heads = reinterpret_cast<DecodeHead*>(w + lay.heads);
  a.ctl = reinterpret_cast<unsigned*>(w + lay.ctl);
  a.cand = reinterpret_cast<uint2*>(w + lay.cand);
  a.pm = reinterpret_cast<float*>(w + lay.pm);
  a.pl = reinterpret_cast<float*>(w + lay.pl);
  a.po = reinterpret_cast<float*>(w + lay.po);
  a.n_ctl = lay.n_ctl; a.nch_score_max = lay.nch_score_max; a.n_sw_tiles = lay.n_sw_tiles;
  a.n_tiles_max = lay.n_tiles_max;
  for (int i = 0; i < kMaxRetrieval; ++i) { a.ret_head[i] = sh.ret_head[i]; a.ret_rank[i] = sh.ret_rank[i]; }

  const int Lh = a.max_seq_len;
  const int nch_score = (Lh + kScoreChunk - 1) / kScoreChunk;
  const int nch_sel = (Lh + kSelChunk - 1) / kSelChunk;
  const int n_sel_tiles = (Lh + kSelTile - 1) / kSelTile;
  if (sh.R > 0) {
    const dim3 gs(nch_score, sh.B * sh.R);
    trace_begin(RTP_STAGE_DECODE_SCORE, st);
    if (sh.dtype == RTP_BF16) launch_score_g<__nv_bfloat16>(a, gs, st);
    else launch_score_g<float>(a, gs, st);
    trace_end(RTP_STAGE_DECODE_SCORE, st);
    const dim3 gh(nch_sel, sh.B * sh.NR);
    trace_begin(RTP_STAGE_DECODE_HIST, st);
    hist_kernel<<<gh, kThreads, 0, st>>>(a);
    trace_end(RTP_STAGE_DECODE_HIST, st);
    trace_begin(RTP_STAGE_DECODE_SELECT, st);
    collect_kernel<<<gh, kThreads, 0, st>>>(a);
    trace_end(RTP_STAGE_DECODE_SELECT, st);
  } else {
    cudaMemsetAsync(a.ctl, 0, (size_t)a.n_ctl * sizeof(unsigned), st);
  }
  const dim3 ga(lay.n_sw_tiles + (sh.R > 0 ? n_sel_tiles : 0), sh.B * sh.Hkv);
  trace_begin(RTP_STAGE_DECODE_ATTN, st);
  if (sh.dtype == RTP_BF16) {
    if (sh.D == 128) launch_attn_g<__nv_bfloat16, 128>(a, ga, st);
    else launch_attn_g<__nv_bfloat16, 64>(a, ga, st);
  } else {
    if (sh.D == 128) launch_attn_g<float, 128>(a, ga, st);
    else launch_attn_g<float, 64>(a, ga, st);
  }
  trace_end(RTP_STAGE_DECODE_ATTN, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("decode launch: ") + cudaGetErrorString(e));
    return RTP_ERR_CUDA;
  }
  return RTP_OK;
}

}  // namespace rtp
