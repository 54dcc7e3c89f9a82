// rtp_prefill_attn: one causal prefill chunk of the head-wise sparse attention
// layer.  Every query row does what a decode step at its position does
// (atlas.scime.ai summary, "Approach"; abstract, observations (2)-(3)).
//
//   select_rows_kernel  retrieval query heads only.  One warp per query row,
//       8 rows per CTA sharing the indexer-key tiles staged in shared memory.
//       Each pass computes a tile's scores for all 8 rows on tensor cores with
//       the decode path's fragments (IdxMma: q~ as bf16 hi + lo parts, the
//       fp32 score to about 2^-17), so a row's scores, and its selection,
//       equal the decode step's at that position bit for bit.
//       The softmax mass exp(s - max) of every score is taken in 2^-36 fixed
//       point (mass36, shared with the decode path; exact integer sums).  The
//       first pass takes the maximum and the scores' mean and spread; the
//       first split sums every key's mass into 8 sub-intervals whose edges go
//       around the boundary a Gaussian score model predicts (a guess that only
//       places them); later (wide) splits bin the few keys inside the boundary
//       interval into 32 sub-intervals in shared memory, until at most kCand
//       tokens remain; a warp-level exact solve finishes (ties to the lower
//       index), in the pass that also writes the row's top-p bitmask.
//   attn_rows_kernel  tensor-core (mma.sync m16n8k16 bf16, fp32 accumulate)
//       flash attention over 64-row query tiles and 64-key tiles, masked by
//       causality, sinks, the window and (retrieval heads) the bitmask; used
//       for local heads that keep a ring of window rows (the tcgen05 kernel in
//       prefill_tc.cu takes every other head).
#include <climits>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace rtp {
namespace {

constexpr int kSelRows = 8;       // query rows (warps) per selection CTA
constexpr int kKeyTile = 512;     // indexer keys staged per step
constexpr int kKeyStages = 2;     // key tiles in flight: the one in use and one ahead
// dynamic shared memory of the selection at indexer width d: the key-tile ring and one tile's scores of the rows
constexpr size_t sel_dyn_smem(int idx) {
  return (size_t)kKeyStages * kKeyTile * idx * sizeof(__nv_bfloat16) + kSelRows * (kKeyTile + 4) * sizeof(float);
}
constexpr int kCand = 160;        // tokens the exact solve takes per row
constexpr int kBQ = 64;           // attention: query rows per CTA (16 per warp)
constexpr int kBK = 64;           // attention: keys per tile

struct PrefillArgs {
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W, T, words;
  int Lk;  // indexer-key rows per (sequence, retrieval head) block
  float top_p, rope_base;
  const void* q_pre;
  const float* w_q;
  void* out;
  const void* k;
  const void* v;
  const void* kidx;
  int* status;
  const int* start_pos;
  float* sel_tau;
  int* sel_jcut;
  int* sel_count;
  uint32_t* mask;  // [B][NR][mask_rows][words] top-p bitmask of rows [mask_t0, mask_t0 + mask_rows)
  int t_base, t_end;         // this launch's query rows [t_base, t_end) of the chunk
  int mask_t0, mask_rows;
  int ring_only;             // attention: only the heads that keep a window ring
  KvMap kv;
  int ret_head[kMaxRetrieval];
  int ret_rank[kMaxRetrieval];
  double inv_freq[64];  // RoPE frequencies, k < D/2
};

__device__ __forceinline__ unsigned long long wsum64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned wsum32(unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float wsumf(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float wmaxf(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ unsigned wminu(unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ unsigned wmaxu(unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------------------------
// tensor-core helpers (mma.sync m16n8k16 bf16, fp32 accumulate; ldmatrix)
// ---------------------------------------------------------------------------

// What a row's warp does with each of its scores in one pass over its keys.
enum : int {
  kOpMax = 0,    // row maximum
  kOpSplit = 1,  // first split: every key's mass into the 8 sub-intervals around the guessed boundary
  kOpRange = 2,  // min/max order key inside the current interval
  kOpCand = 3,   // collect the current interval's tokens for the exact solve; write the bitmask
  kOpTies = 4,   // count tied tokens with index <= probe (index bisection)
  kOpEmit = 5,   // write the top-p bitmask (after exact ties or p >= 1; the
                 // candidate pass writes it itself)
  kOpDone = 6,
  kOpWide = 7    // later splits: the keys inside the current interval into 32 sub-intervals
};
constexpr int kWideBins = 32;

// Per-row selection state (kept identical in every lane of the row's warp).
struct RowSel {
  float m;                   // row maximum score
  unsigned long long need;   // mass still needed inside the current interval
  unsigned cnt_above;        // tokens ordered before the current interval
  unsigned cnt_in;           // tokens inside the current interval
  // current interval: d = m - s in [dlo, dhi) (dhi < 0: no upper bound) and
  // order key in [klo, khi]
  float dlo, dhi;
  unsigned klo, khi;
  bool by_key;               // split on order keys (d can no longer be split)
  bool first;                // first split: also sums the total mass Z
  float th[7];               // thresholds of the 8 sub-intervals (d or key as float bits)
  unsigned kth[7];
  // ties: all remaining tokens share one key; keep the first `need_ties` by index
  unsigned tie_key, need_ties, tie_lo, tie_hi;
  float tau;
  int jcut;
  unsigned count;
  int op;
};

// The edges and interval a split pass tests, loaded from the row's state.
struct SplitView {
  float m, dlo, dhi;
  unsigned klo, khi;
  bool by_key;
  float thr[7];  // d thresholds, or order keys (as bits) when by_key
};
__device__ __forceinline__ SplitView load_split(const RowSel& R) {
  SplitView v;
  v.m = R.m;
  v.dlo = R.dlo;
  v.dhi = R.dhi;
  v.klo = R.klo;
  v.khi = R.khi;
  v.by_key = R.by_key;
#pragma unroll
  for (int e = 0; e < 7; ++e) v.thr[e] = v.by_key ? __uint_as_float(R.kth[e]) : R.th[e];
  return v;
}
// One score inside the interval of a wide split: its exact mass and a count
// into the bin it falls in (the number of the interval's 31 edges it passes;
// edges are d thresholds ascending, or order keys descending, so passing is
// monotone in the edge index and a 5-step search finds the bin).
__device__ __forceinline__ void wide_item(float m, bool by_key, const unsigned* edges, unsigned long long* bm,
                                          unsigned* bc, float sv) {
  const float d = m - sv;
  const unsigned key = score_key(sv);
  int nb = 0;
#pragma unroll
  for (int step = 16; step >= 1; step >>= 1) {
    const int e = nb + step - 1;
    if (e < kWideBins - 1) {
      const unsigned ed = edges[e];
      if (by_key ? key < ed : d >= __uint_as_float(ed)) nb += step;
    }
  }
  atomicAdd(&bm[nb], mass36(sv, m));
  atomicAdd(&bc[nb], 1u);
}

template <int D, int IDX>
__global__ void __launch_bounds__(kSelRows * 32, 3) select_rows_kernel(const __grid_constant__ PrefillArgs a) {
  constexpr int KB = IDX * (int)sizeof(__nv_bfloat16);  // bytes per indexer key
  // dynamic shared memory: a ring of key tiles, then this tile's scores of
  // the CTA's rows
  extern __shared__ __align__(16) unsigned char sel_dsm[];
  auto s_k = reinterpret_cast<__nv_bfloat16 (*)[kKeyTile * IDX]>(sel_dsm);
  auto s_sc = reinterpret_cast<float (*)[kKeyTile + 4]>(sel_dsm + kKeyStages * kKeyTile * IDX * sizeof(__nv_bfloat16));
  __shared__ float s_qi[kSelRows][IDX];
  __shared__ uint2 s_cand[kSelRows][kCand];
  __shared__ unsigned long long s_cw[kSelRows][kCand];
  // Each row's selection state lives in shared memory: a pass loads only the
  // few fields its op tests into registers, and the step between passes works
  // on a copy, which keeps the per-key loops' registers free of it.
  __shared__ RowSel s_rs[kSelRows];
  // later splits: the scores inside the interval, gathered 32 at a time
  __shared__ float s_ring[kSelRows][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / a.NR, hh = bh % a.NR;
  const int r = hh / a.G, g = hh % a.G;
  const int h = a.ret_head[r];
  const int t = a.t_base + blockIdx.x * kSelRows + warp;
  const int start = a.start_pos[b];
  if (start < 0 || start + a.T > a.Lmax) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && hh == 0) atomicOr(a.status, RTP_DEV_POSITION);
    return;  // uniform over the CTA
  }
  const bool row_ok = t < a.t_end;
  const int i = start + t;  // query position; keys [0, i]
  const int i_last = start + min(a.t_end, a.t_base + (int)(blockIdx.x + 1) * kSelRows) - 1;

  // q~ = W_q q_pre with the decode path's association: four quarter sums of
  // D/4 dims each, then butterfly adds.
  float qi[IDX];
  {
    constexpr int DQ = D / 4;
    constexpr int NIT = (IDX * 4 + 31) / 32;
    float part[NIT];
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
      const int task = it * 32 + lane;  // IDX outputs x 4 quarters
      const int o = task >> 2, qd = task & 3;
      float acc = 0.f;
      if (row_ok && o < IDX) {
        const float4* w = reinterpret_cast<const float4*>(a.w_q + ((size_t)r * IDX + o) * D + qd * DQ);
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q_pre) +
                                 (((size_t)b * a.T + t) * a.Hq + h * a.G + g) * D + qd * DQ;
        float wv[DQ], qv[DQ];
#pragma unroll
        for (int k = 0; k < DQ / 4; ++k) {
          const float4 f = __ldg(w + k);
          wv[4 * k] = f.x; wv[4 * k + 1] = f.y; wv[4 * k + 2] = f.z; wv[4 * k + 3] = f.w;
        }
        load_row<__nv_bfloat16, DQ>(q, qv);
#pragma unroll
        for (int k = 0; k < DQ; ++k) acc = fmaf(wv[k], qv[k], acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      part[it] = acc;
    }
#pragma unroll
    for (int o = 0; o < IDX; ++o) qi[o] = __shfl_sync(0xffffffffu, part[o >> 3], (o & 7) * 4);
  }
  {
    // lane l < IDX stores q~[l] (constant register indices only)
    float mine = 0.f;
#pragma unroll
    for (int o = 0; o < IDX; ++o)
      if (lane == o) mine = qi[o];
    if (lane < IDX) s_qi[warp][lane] = mine;
  }
  __syncthreads();
  // Scores on tensor cores with the decode path's fragments (IdxMma): S =
  // K~ Q~^T, q~ split into bf16 hi and lo parts (the products are exact; fp32
  // accumulation), so the score is the fp32 q~ . k~ to about 2^-17 relative
  // and equals the decode step's bit for bit.  Column n of the product is row
  // n of this CTA.
  IdxMma<IDX> mm;
  mm.set_q(s_qi[lane >> 2], lane);
  constexpr float kScale = idx_scale<IDX>();

  if (lane == 0) {
    s_rs[warp] = RowSel{};
    s_rs[warp].op = row_ok ? kOpMax : kOpDone;
    s_rs[warp].m = -CUDART_INF_F;
    s_rs[warp].first = false;
  }
  __syncwarp();
  const RowSel& R = s_rs[warp];
  const __nv_bfloat16* kidx = static_cast<const __nv_bfloat16*>(a.kidx) + ((size_t)b * a.R + r) * a.Lk * IDX;
  uint32_t* mrow = a.mask + (((size_t)b * a.NR + hh) * a.mask_rows + (row_ok ? t - a.mask_t0 : 0)) * a.words;
  // The wide split's bins and edges use the warp's candidate arrays (a row is
  // never in a split pass and a candidate pass at once): exact mass and count
  // per sub-interval, and the 31 edges (d as float bits, or order keys).
  unsigned long long* wd_m = s_cw[warp];
  unsigned* wd_c = reinterpret_cast<unsigned*>(s_cand[warp]);
  unsigned* wd_e = wd_c + kWideBins;
  static_assert(kCand * sizeof(uint2) >= (2 * kWideBins) * sizeof(unsigned), "bins and edges fit");
  static_assert(kCand >= kWideBins, "bin masses fit");
  // After a split: the candidate pass once the boundary interval holds few
  // enough tokens; else a wide split of a d interval while d still separates
  // its tokens (edges written to the warp's edge array), else the range pass,
  // which bounds the interval by the keys present (and finds exact ties)
  // before a wide split on order keys.
  auto next_step = [&](RowSel& rs, unsigned before) {
    if (rs.cnt_in <= (unsigned)kCand) {
      rs.op = kOpCand;
      return;
    }
    if (rs.by_key || rs.dhi < 0.f || rs.cnt_in >= before) {
      rs.op = kOpRange;
      return;
    }
    const float step = (rs.dhi - rs.dlo) * (1.0f / kWideBins);
    const float ed = fminf(rs.dlo + step * (float)(lane + 1), rs.dhi);  // edge `lane` (< 31)
    const bool splits = __shfl_sync(0xffffffffu, ed, 0) > rs.dlo &&
                        __shfl_sync(0xffffffffu, ed, kWideBins - 2) < rs.dhi;
    if (!splits) {
      rs.op = kOpRange;
      return;
    }
    if (lane < kWideBins - 1) wd_e[lane] = __float_as_uint(ed);
    __syncwarp();
    rs.op = kOpWide;
  };

  // pass accumulators
  unsigned long long pm[8];
  unsigned pc[8];
  // the small accumulators of the other ops share three registers:
  //   max: x0 = max score, x1 = sum of s, x2 = sum of s^2 (float bits)
  //   range: x0 = min key, x1 = max key; candidates: x0 = count; ties: x0 = count
  unsigned x0, x1, x2;

  for (int pass = 0; pass < 200; ++pass) {
    const int op = R.op;
    // reset accumulators
#pragma unroll
    for (int q = 0; q < 8; ++q) { pm[q] = 0ull; pc[q] = 0u; }
    x0 = op == kOpMax ? __float_as_uint(-CUDART_INF_F) : (op == kOpRange ? 0xffffffffu : 0u);
    x1 = 0u;  // also 0.f
    x2 = 0u;
    const bool first_split = (op == kOpSplit) && R.first;
    if (op == kOpWide) {
      wd_m[lane] = 0ull;
      wd_c[lane] = 0u;
      __syncwarp();
    }
    unsigned q_head = 0u, q_tail = 0u;  // s_ring[warp] positions (warp-uniform)
    // key tiles [kt, kt + kKeyTile) up to i_last, copied asynchronously
    // kKeyStages - 1 tiles ahead of their use (an empty group past the end)
    auto stage_async = [&](int kt_, int buf) {
      if (kt_ <= i_last) {
        const int n = min(kKeyTile, i_last + 1 - kt_);
        const char* src = reinterpret_cast<const char*>(kidx + (size_t)kt_ * IDX);
        const unsigned dst = (unsigned)__cvta_generic_to_shared(s_k[buf]);
        // whole 16-byte vectors: an odd count of 8-byte keys takes the next key
        // of the block too (the block then has an even row count past it)
        const int nvec = (n * KB + 15) / 16;
        for (int v = threadIdx.x; v < nvec; v += kSelRows * 32)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst + 16u * v), "l"(src + 16 * (size_t)v));
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    __syncthreads();  // the previous pass is done with every buffer
#pragma unroll
    for (int s0 = 0; s0 < kKeyStages - 1; ++s0) stage_async(s0 * kKeyTile, s0);
    int buf = 0;
    for (int kt = 0; kt <= i_last; kt += kKeyTile) {
      asm volatile("cp.async.wait_group %0;" :: "n"(kKeyStages - 2) : "memory");
      __syncthreads();  // tile kt landed for every thread; the previous tile's buffer is free
      stage_async(kt + (kKeyStages - 1) * kKeyTile, buf == 0 ? kKeyStages - 1 : buf - 1);
      // warp w: the scores of keys [64 w, 64 w + 64) of this tile for all rows
#pragma unroll
      for (int half = 0; half < kKeyTile / kSelRows / 16; ++half) {
        const int kb = warp * (kKeyTile / kSelRows) + half * 16;  // first key (M row) of this 16 x 8 tile
        float c[4];
        mm.scores(reinterpret_cast<const unsigned char*>(s_k[buf]) + (size_t)kb * KB, lane, c);
        const int key0 = kb + (lane >> 2), row0 = (lane & 3) * 2;
        s_sc[row0][key0] = c[0] * kScale + 0.0f;  // +0 turns -0 into +0
        s_sc[row0 + 1][key0] = c[1] * kScale + 0.0f;
        s_sc[row0][key0 + 8] = c[2] * kScale + 0.0f;
        s_sc[row0 + 1][key0 + 8] = c[3] * kScale + 0.0f;
      }
      __syncthreads();
      buf = buf + 1 == kKeyStages ? 0 : buf + 1;  // the next tile's buffer
      if (op == kOpDone || kt > i) continue;  // uniform per warp
      // One tight loop per kind of pass over this tile's 16 groups of 32 keys
      // (the row's op is warp-uniform).  Keys past the row (j > i) are off.
      const float* srow = s_sc[warp];
      const int ulim = min(kKeyTile / 32, (i - kt) / 32 + 1);  // groups holding keys <= i
      switch (op) {
        case kOpMax: {
          float fmx = __uint_as_float(x0), fs = __uint_as_float(x1), fs2 = __uint_as_float(x2);
#pragma unroll 8
          for (int u = 0; u < kKeyTile / 32; ++u) {
            const int j = kt + u * 32 + lane;
            if (u < ulim && j <= i) {
              const float sv = srow[u * 32 + lane];
              fmx = fmaxf(fmx, sv);
              fs += sv;
              fs2 = fmaf(sv, sv, fs2);
            }
          }
          x0 = __float_as_uint(fmx);
          x1 = __float_as_uint(fs);
          x2 = __float_as_uint(fs2);
          break;
        }
        case kOpEmit: {
          const float tau = R.tau;
          const int jcut = R.jcut;
#pragma unroll 8
          for (int u = 0; u < kKeyTile / 32; ++u) {
            if (u >= ulim) break;
            const int j = kt + u * 32 + lane;
            const float sv = srow[u * 32 + lane];
            const bool in = j <= i && (sv > tau || (sv == tau && j <= jcut));
            const unsigned wd = __ballot_sync(0xffffffffu, in);
            if (lane == 0) mrow[(kt >> 5) + u] = wd;
          }
          break;
        }
        case kOpSplit: {  // the first split: every key is inside; total mass and d-thresholds
          const SplitView v = load_split(R);
          const float m = v.m;
#pragma unroll 4
          for (int u = 0; u < kKeyTile / 32; ++u) {
            const int j = kt + u * 32 + lane;
            if (u >= ulim || j > i) continue;
            const float sv = srow[u * 32 + lane];
            const float d = m - sv;
            const unsigned long long w = mass36(sv, m);
            pm[7] += w;  // every key: the total mass
            pc[7] += 1u;
#pragma unroll
            for (int e = 0; e < 7; ++e)
              if (d >= v.thr[e]) { pm[e] += w; pc[e] += 1u; }
          }
          break;
        }
        case kOpWide: {
          // a small share of the keys lies inside: gather those scores in the
          // warp's ring and bin them 32 at a time (no divergent lanes)
          const float m = R.m, dlo = R.dlo, dhi = R.dhi;
          const unsigned klo = R.klo, khi = R.khi;
          const bool by_key = R.by_key;
          float* ring = s_ring[warp];
#pragma unroll 4
          for (int u = 0; u < kKeyTile / 32; ++u) {
            if (u >= ulim) break;
            const int j = kt + u * 32 + lane;
            const float sv = srow[u * 32 + lane];
            const float d = m - sv;
            const unsigned key = score_key(sv);
            const bool inside = j <= i && d >= dlo && (dhi < 0.f || d < dhi) && key >= klo && key <= khi;
            const unsigned bal = __ballot_sync(0xffffffffu, inside);
            if (bal == 0u) continue;
            if (inside) ring[(q_tail + __popc(bal & ((1u << lane) - 1u))) & 63u] = sv;
            q_tail += (unsigned)__popc(bal);
            if (q_tail - q_head >= 32u) {
              __syncwarp();
              const float sq = ring[(q_head + lane) & 63u];
              __syncwarp();
              q_head += 32u;
              wide_item(m, by_key, wd_e, wd_m, wd_c, sq);
            }
          }
          break;
        }
        case kOpRange: {
          const float m = R.m, dlo = R.dlo, dhi = R.dhi;
          const unsigned klo = R.klo, khi = R.khi;
#pragma unroll 4
          for (int u = 0; u < kKeyTile / 32; ++u) {
            const int j = kt + u * 32 + lane;
            if (u >= ulim || j > i) continue;
            const float sv = srow[u * 32 + lane];
            const float d = m - sv;
            const unsigned key = score_key(sv);
            if (d >= dlo && (dhi < 0.f || d < dhi) && key >= klo && key <= khi) {
              x0 = min(x0, key);
              x1 = max(x1, key);
            }
          }
          break;
        }
        case kOpTies: {
          const unsigned tie_key = R.tie_key, tie_hi = R.tie_hi;
#pragma unroll 4
          for (int u = 0; u < kKeyTile / 32; ++u) {
            const int j = kt + u * 32 + lane;
            if (u >= ulim || j > i) continue;
            const unsigned key = score_key(srow[u * 32 + lane]);
            if (key == tie_key && (unsigned)j <= tie_hi) x0 += 1u;
          }
          break;
        }
        case kOpCand: {
          const float m = R.m, dlo = R.dlo, dhi = R.dhi;
          const unsigned klo = R.klo, khi = R.khi;
#pragma unroll 2
          for (int u = 0; u < kKeyTile / 32; ++u) {
            if (u >= ulim) break;
            const int j = kt + u * 32 + lane;
            const float sv = srow[u * 32 + lane];
            const float d = m - sv;
            const unsigned key = score_key(sv);
            const bool below_hi = dhi < 0.f || d < dhi;
            const bool inside = j <= i && d >= dlo && below_hi && key >= klo && key <= khi;
            // ordered before every candidate: kept whatever the solve finds
            const bool above = j <= i && (d < dlo || (below_hi && key > khi));
            const unsigned wd = __ballot_sync(0xffffffffu, above);
            if (lane == 0) mrow[(kt >> 5) + u] = wd;
            const unsigned bal = __ballot_sync(0xffffffffu, inside);
            const unsigned slot = x0 + __popc(bal & ((1u << lane) - 1u));
            if (inside && slot < (unsigned)kCand) {
              s_cand[warp][slot] = make_uint2(key, (unsigned)j);
              s_cw[warp][slot] = mass36(sv, m);
            }
            x0 += __popc(bal);
          }
          break;
        }
        default:
          break;
      }
    }
    if (op == kOpWide && q_tail != q_head) {  // the ring's last (< 32) scores
      __syncwarp();
      if (lane < q_tail - q_head) wide_item(R.m, R.by_key, wd_e, wd_m, wd_c, s_ring[warp][(q_head + lane) & 63u]);
    }
    // ---- reduce this pass and choose the next step (warp-uniform) ----
    RowSel rs = R;
    if (op == kOpDone) {
      // nothing
    } else if (op == kOpMax) {
      rs.m = wmaxf(__uint_as_float(x0));
      rs.op = kOpSplit;
      rs.dlo = 0.f;
      rs.dhi = -1.f;
      rs.klo = 0u;
      rs.khi = 0xffffffffu;
      rs.by_key = false;
      rs.first = true;
      rs.cnt_above = 0u;
      rs.need = 0ull;
      // First split: edges around a guess of the boundary's distance below the
      // max. For scores ~ N(mu, sd^2) the softmax-weighted scores are
      // ~ N(mu + sd^2, sd^2), whose upper p-quantile lies z_p sd below
      // mu + sd^2. Large scores beyond the bulk move the boundary towards the
      // max, hence the wider bins on that side. The guess only places the
      // edges: the split stays exact wherever the boundary falls.
      {
        const float n = (float)(i + 1);
        const float mu = __shfl_sync(0xffffffffu, wsumf(__uint_as_float(x1)), 0) / n;
        const float var = fmaxf(__shfl_sync(0xffffffffu, wsumf(__uint_as_float(x2)), 0) / n - mu * mu, 0.f);
        const float sd = sqrtf(var);
        const float c = rs.m - (mu + var - normcdfinvf(a.top_p) * sd);
        const float off[7] = {-0.8f, -0.4f, -0.2f, -0.08f, 0.f, 0.08f, 0.25f};
        const float fixed[7] = {0.5f, 1.f, 2.f, 3.f, 4.5f, 7.f, 12.f};
        const bool ok = isfinite(c) && isfinite(sd);
#pragma unroll
        for (int e = 0; e < 7; ++e) rs.th[e] = ok ? c + off[e] * sd : fixed[e];
      }
      if (a.top_p >= 1.0f) {  // keep everything
        rs.tau = -CUDART_INF_F;
        rs.jcut = INT_MAX;
        rs.count = (unsigned)(i + 1);
        rs.op = kOpEmit;
      }
    } else if (op == kOpSplit) {
#pragma unroll
      for (int e = 0; e < 8; ++e) { pm[e] = wsum64(pm[e]); pc[e] = wsum32(pc[e]); }
      const unsigned long long inside_mass = pm[7];  // first split: every key, Z
      {  // cumulative -> per sub-interval (e = 0 holds the highest scores)
        const unsigned long long tm = pm[7];
        const unsigned tc = pc[7];
        pm[7] = pm[6];
        pc[7] = pc[6];
#pragma unroll
        for (int e = 6; e >= 1; --e) { pm[e] = pm[e - 1] - pm[e]; pc[e] = pc[e - 1] - pc[e]; }
        pm[0] = tm - pm[0];
        pc[0] = tc - pc[0];
      }
      if (first_split) {
        const unsigned long long Z = inside_mass;
        unsigned long long target = (unsigned long long)ceil((double)a.top_p * (double)Z);
        if (target > Z) target = Z;
        if (target < 1ull) target = 1ull;
        rs.need = target;
        rs.cnt_in = (unsigned)(i + 1);
        rs.first = false;
      }
      // sub-intervals are ordered from the highest scores (e = 0) down; the
      // first one that reaches the mass still needed holds the boundary.
      // (Constant indices only, so that these arrays stay in registers.)
      unsigned long long cum = 0ull;
      unsigned cc = 0u, pc_sel = pc[7];
      int sel = 7;
      bool found = false;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (!found && cum + pm[e] >= rs.need) { sel = e; found = true; pc_sel = pc[e]; }
        if (!found) { cum += pm[e]; cc += pc[e]; }
      }
      rs.need -= cum;
      rs.cnt_above += cc;
      const unsigned before = rs.cnt_in;
      rs.cnt_in = pc_sel;
      if (!rs.by_key) {
        float lo = rs.dlo, hi = rs.dhi;
#pragma unroll
        for (int e = 0; e < 7; ++e) {
          if (e == sel - 1) lo = rs.th[e];
          if (e == sel) hi = rs.th[e];
        }
        rs.dlo = lo;
        rs.dhi = hi;
      } else {
        // key sub-intervals: e = 0 holds the highest keys
        unsigned hi = rs.khi, lo = rs.klo;
#pragma unroll
        for (int e = 0; e < 7; ++e) {
          if (e == sel - 1) hi = rs.kth[e] - 1u;
          if (e == sel) lo = rs.kth[e];
        }
        rs.klo = lo;
        rs.khi = hi;
      }
      next_step(rs, before);
    } else if (op == kOpWide) {
      // bins from the highest scores (lane 0) down: the first whose cumulative
      // mass reaches the mass still needed holds the boundary
      __syncwarp();
      const unsigned long long mb = wd_m[lane];
      const unsigned cb = wd_c[lane];
      unsigned long long cm = mb;
      unsigned ck = cb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long tm = __shfl_up_sync(0xffffffffu, cm, o);
        const unsigned tc = __shfl_up_sync(0xffffffffu, ck, o);
        if (lane >= o) {
          cm += tm;
          ck += tc;
        }
      }
      const unsigned ball = __ballot_sync(0xffffffffu, cm >= rs.need);
      const int sel = ball ? __ffs(ball) - 1 : kWideBins - 1;
      const unsigned long long ex_m = __shfl_sync(0xffffffffu, cm - mb, sel);
      const unsigned ex_c = __shfl_sync(0xffffffffu, ck - cb, sel);
      const unsigned in_c = __shfl_sync(0xffffffffu, cb, sel);
      const unsigned my_e = lane < kWideBins - 1 ? wd_e[lane] : 0u;
      const unsigned e_lo = __shfl_sync(0xffffffffu, my_e, sel > 0 ? sel - 1 : 0);
      const unsigned e_hi = __shfl_sync(0xffffffffu, my_e, sel < kWideBins - 1 ? sel : 0);
      rs.need -= ex_m;
      rs.cnt_above += ex_c;
      const unsigned before = rs.cnt_in;
      rs.cnt_in = in_c;
      if (!rs.by_key) {  // bin b: d in [edge b-1, edge b)
        if (sel > 0) rs.dlo = __uint_as_float(e_lo);
        if (sel < kWideBins - 1) rs.dhi = __uint_as_float(e_hi);
      } else {           // bin b: keys in [edge b, edge b-1 - 1]
        if (sel > 0) rs.khi = e_lo - 1u;
        if (sel < kWideBins - 1) rs.klo = e_hi;
      }
      __syncwarp();  // every lane has read the edges before they are rewritten
      next_step(rs, before);
    } else if (op == kOpRange) {
      rs.klo = max(rs.klo, wminu(x0));
      rs.khi = min(rs.khi, wmaxu(x1));
      rs.by_key = true;
      if (rs.klo == rs.khi) {  // exact ties: keep the first ceil(need / w) by index
        const unsigned long long w = mass36(key_score(rs.klo), rs.m);
        unsigned long long kk = w ? (rs.need + w - 1ull) / w : (unsigned long long)rs.cnt_in;
        if (kk < 1ull) kk = 1ull;
        if (kk > rs.cnt_in) kk = rs.cnt_in;
        rs.tie_key = rs.klo;
        rs.need_ties = (unsigned)kk;
        rs.tau = key_score(rs.klo);
        rs.count = rs.cnt_above + (unsigned)kk;
        if (kk == rs.cnt_in) {
          rs.jcut = INT_MAX;
          rs.op = kOpEmit;
        } else {
          rs.tie_lo = 0u;
          rs.tie_hi = (unsigned)i;
          rs.op = kOpTies;
          // first probe
          rs.tie_hi = (rs.tie_lo + (unsigned)i) / 2u;
          rs.kth[0] = (unsigned)i;  // upper end of the bisection range
        }
      } else {
        // edge e (< 31): first key of the (e+1)-th of 32 key sub-intervals from the top
        const unsigned long long span = (unsigned long long)rs.khi - rs.klo + 1ull;
        if (lane < kWideBins - 1)
          wd_e[lane] = (unsigned)(rs.khi + 1ull -
                                  (span * (unsigned long long)(lane + 1) + (kWideBins - 1)) / kWideBins);
        __syncwarp();
        rs.op = kOpWide;
      }
    } else if (op == kOpTies) {
      // bisection on the index: smallest probe with count(ties <= probe) >= need_ties
      const unsigned tie_cnt = wsum32(x0);
      unsigned lo = rs.tie_lo, hi = rs.kth[0];
      if (tie_cnt >= rs.need_ties) hi = rs.tie_hi;
      else lo = rs.tie_hi + 1u;
      rs.tie_lo = lo;
      rs.kth[0] = hi;
      if (lo >= hi) {
        rs.jcut = (int)lo;
        rs.op = kOpEmit;
      } else {
        rs.tie_hi = (lo + hi) / 2u;
      }
    } else if (op == kOpCand) {
      // exact solve: candidate c is kept iff the mass ordered before it is < need
      const int n = (int)min(x0, (unsigned)kCand);
      unsigned kept_n = 0u, tkey = 0xffffffffu;
      __syncwarp();
      for (int c = lane; c < n; c += 32) {
        const uint2 me = s_cand[warp][c];
        unsigned long long before = 0ull;
        for (int o = 0; o < n; ++o) {
          const uint2 ot = s_cand[warp][o];
          if (ot.x > me.x || (ot.x == me.x && ot.y < me.y)) before += s_cw[warp][o];
        }
        if (before < rs.need) {
          ++kept_n;
          tkey = min(tkey, me.x);
        }
      }
      kept_n = wsum32(kept_n);
      tkey = wminu(tkey);
      int jc = -1;
      for (int c = lane; c < n; c += 32) {
        const uint2 me = s_cand[warp][c];
        if (me.x != tkey) continue;
        unsigned long long before = 0ull;
        for (int o = 0; o < n; ++o) {
          const uint2 ot = s_cand[warp][o];
          if (ot.x > me.x || (ot.x == me.x && ot.y < me.y)) before += s_cw[warp][o];
        }
        if (before < rs.need) jc = max(jc, (int)me.y);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) jc = max(jc, __shfl_xor_sync(0xffffffffu, jc, o));
      // the pass wrote the bitmask words with the tokens above the interval;
      // add the kept candidates
      for (int c = lane; c < n; c += 32) {
        const uint2 me = s_cand[warp][c];
        if (me.x > tkey || (me.x == tkey && (int)me.y <= jc)) atomicOr(&mrow[me.y >> 5], 1u << (me.y & 31u));
      }
      __syncwarp();
      rs.tau = key_score(tkey);
      rs.jcut = jc;
      rs.count = rs.cnt_above + kept_n;
      if (lane == 0) {
        if (a.sel_tau) a.sel_tau[((size_t)b * a.NR + hh) * a.T + t] = rs.tau;
        if (a.sel_jcut) a.sel_jcut[((size_t)b * a.NR + hh) * a.T + t] = rs.jcut;
        if (a.sel_count) a.sel_count[((size_t)b * a.NR + hh) * a.T + t] = (int)rs.count;
      }
      rs.op = kOpDone;
    } else if (op == kOpEmit) {
      // last word(s) past i inside the row stay as written (bits > i are zero)
      if (lane == 0) {
        if (a.sel_tau) a.sel_tau[((size_t)b * a.NR + hh) * a.T + t] = rs.tau;
        if (a.sel_jcut) a.sel_jcut[((size_t)b * a.NR + hh) * a.T + t] = rs.jcut;
        if (a.sel_count) a.sel_count[((size_t)b * a.NR + hh) * a.T + t] = (int)rs.count;
      }
      rs.op = kOpDone;
    }
    __syncwarp();
    if (lane == 0) s_rs[warp] = rs;
    __syncwarp();
    if (!__syncthreads_or(rs.op != kOpDone)) break;
  }
}

// ---------------------------------------------------------------------------
// masked causal attention on tensor cores
// ---------------------------------------------------------------------------
template <int D>
struct AttnSmem {
  static constexpr int kStride = D + 8;  // bf16 elements per shared row (pad: no ldmatrix conflicts)
  // two buffers of (K tile, V tile); the Q tile borrows the first K tile
  // until its fragments are in registers
  static_assert(kBQ <= kBK, "the Q tile fits in one K tile");
  static constexpr size_t kBytes = (size_t)(4 * kBK) * kStride * sizeof(__nv_bfloat16);
};

template <int D>
__global__ void __launch_bounds__(128, 3) attn_rows_kernel(const __grid_constant__ PrefillArgs a) {
  constexpr int ST = AttnSmem<D>::kStride;
  constexpr int KS = D / 16;  // k-steps of Q K^T
  constexpr int NO = D / 8;   // n8 tiles of the output
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* s_q = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* s_kv = s_q;  // buffer u: K at s_kv + 2u kBK ST, V right after
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int bq = blockIdx.y;
  const int b = bq / a.Hq, hq = bq % a.Hq;
  const int h = hq / a.G, g = hq % a.G;
  const int r = a.ret_rank[h];
  if (a.ring_only && !((a.kv.ring_mask >> h) & 1ull)) return;  // the tensor-core kernel's head
  const int start = a.start_pos[b];
  if (start < 0 || start + a.T > a.Lmax) return;  // flagged by the selection kernel / host
  const int t0 = a.t_base + blockIdx.x * kBQ;
  const int hh = r >= 0 ? r * a.G + g : 0;

  // ---- Q tile: RoPE at each row's position, scaled by log2(e)/sqrt(D), bf16 ----
  const float qscale = 1.4426950408889634f * rsqrtf((float)D);
  for (int e = threadIdx.x; e < kBQ * (D / 2); e += blockDim.x) {
    const int rr = e / (D / 2), kk = e % (D / 2);
    const int t = t0 + rr;
    float y1 = 0.f, y2 = 0.f;
    if (t < a.t_end) {
      const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q_pre) + (((size_t)b * a.T + t) * a.Hq + hq) * D;
      const float x1 = __bfloat162float(q[kk]), x2 = __bfloat162float(q[kk + D / 2]);
      float c, sn;
      rope_cos_sin(start + t, a.inv_freq[kk], c, sn);
      y1 = (x1 * c - x2 * sn) * qscale;
      y2 = (x2 * c + x1 * sn) * qscale;
    }
    s_q[rr * ST + kk] = __float2bfloat16_rn(y1);
    s_q[rr * ST + kk + D / 2] = __float2bfloat16_rn(y2);
  }
  __syncthreads();
  // Q fragments of this warp's 16 rows stay in registers
  unsigned qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int col = ks * 16 + (lane >> 4) * 8;
    ldsm_x4(qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], s_q + row * ST + col);
  }

  // rows of this thread: warp*16 + gq and + 8
  int ti[2], pi[2], wlo[2];
  bool rv[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    ti[x] = t0 + warp * 16 + gq + 8 * x;
    rv[x] = ti[x] < a.t_end;
    pi[x] = start + ti[x];
    wlo[x] = pi[x] - a.W + 1;  // window: keys >= wlo
  }
  const int t_last = min(a.t_end, t0 + kBQ) - 1;
  const int i_max = start + t_last;
  const int i_min = start + t0;
  const uint32_t* mrow[2];
#pragma unroll
  for (int x = 0; x < 2; ++x)
    mrow[x] = a.mask + (((size_t)b * a.NR + hh) * a.mask_rows + (rv[x] ? ti[x] - a.mask_t0 : 0)) * a.words;

  float o[NO][4];
#pragma unroll
  for (int n = 0; n < NO; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mrun[2] = {-CUDART_INF_F, -CUDART_INF_F}, lrun[2] = {0.f, 0.f};

  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);

  // Key tiles in order, local heads jumping from the sinks to the first window
  // tile; each tile's K, V (cp.async, rows past the chunk zero-filled) and
  // mask words are requested one tile ahead.
  auto next_tile = [&](int kt_) {
    int n = kt_ + kBK;
    if (r < 0 && n >= a.S) n = max(n, (max(0, i_min - a.W + 1) / kBK) * kBK);
    return n;
  };
  auto issue_kv = [&](int kt_, int u) {
    const unsigned dk = (unsigned)__cvta_generic_to_shared(s_kv + (size_t)(2 * u) * kBK * ST);
    const unsigned dv = (unsigned)__cvta_generic_to_shared(s_kv + (size_t)(2 * u + 1) * kBK * ST);
    for (int e = threadIdx.x; e < kBK * (D / 8); e += blockDim.x) {
      const int kr = e / (D / 8), c8 = e % (D / 8);
      const int j = kt_ + kr;
      const unsigned sz = j <= i_max ? 16u : 0u;  // 0: zero fill
      const size_t row = a.kv.row(b, h, j <= i_max ? j : 0);
      const unsigned off = (unsigned)((kr * ST + c8 * 8) * sizeof(__nv_bfloat16));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dk + off),
                   "l"(kg + row * D + c8 * 8), "r"(sz));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dv + off),
                   "l"(vg + row * D + c8 * 8), "r"(sz));
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  auto load_mw = [&](int kt_, unsigned (&m_)[2][2]) {
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        const int wd = (kt_ >> 5) + y;
        m_[x][y] = (r >= 0 && rv[x] && wd * 32 <= pi[x]) ? __ldg(mrow[x] + wd) : 0u;
      }
  };
  unsigned mw[2][2];
  load_mw(0, mw);
  __syncthreads();  // every warp holds its Q fragments: the first K tile may overwrite them
  issue_kv(0, 0);
  int ub = 0;
  for (int kt = 0; kt <= i_max; ub ^= 1) {
    const int kn = next_tile(kt);
    unsigned mwn[2][2];
    if (kn <= i_max) {
      issue_kv(kn, ub ^ 1);
      load_mw(kn, mwn);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    const __nv_bfloat16* s_k = s_kv + (size_t)(2 * ub) * kBK * ST;
    const __nv_bfloat16* s_v = s_k + kBK * ST;
    // does any row of the tile keep a key of this tile?
    const bool sink_tile = kt < a.S;
    const bool win_tile = kt + kBK - 1 >= i_min - a.W + 1;
    bool any = false;
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int y = 0; y < 2; ++y) any |= mw[x][y] != 0u;
    if (!__syncthreads_or(any || sink_tile || win_tile)) {  // also: tile kt's K, V visible
      kt = kn;
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 2; ++y) mw[x][y] = mwn[x][y];
      continue;
    }
    // S = Q K^T for this warp's 16 rows x 64 keys
    float sc[kBK / 8][4];
#pragma unroll
    for (int n = 0; n < kBK / 8; ++n) {
      sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        unsigned b0, b1;
        const int krow = n * 8 + (lane & 7);
        const int kcol = ks * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x2(b0, b1, s_k + krow * ST + kcol);
        mma_bf16(sc[n], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
      }
    }
    // mask + tile maximum per row
    float tmax[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
    for (int n = 0; n < kBK / 8; ++n) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int x = c >> 1;
        const int jj = n * 8 + 2 * tq + (c & 1);
        const int j = kt + jj;
        bool ok = rv[x] && j <= pi[x] && (j < a.S || j >= wlo[x]);
        if (!ok && r >= 0 && rv[x] && j <= pi[x]) ok = (mw[x][jj >> 5] >> (jj & 31)) & 1u;
        sc[n][c] = ok ? sc[n][c] : -CUDART_INF_F;
        tmax[x] = fmaxf(tmax[x], sc[n][c]);
      }
    }
    float alpha[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      tmax[x] = fmaxf(tmax[x], __shfl_xor_sync(0xffffffffu, tmax[x], 1));
      tmax[x] = fmaxf(tmax[x], __shfl_xor_sync(0xffffffffu, tmax[x], 2));
      const float mn = fmaxf(mrun[x], tmax[x]);
      alpha[x] = (mn == -CUDART_INF_F) ? 1.f : exp2f(mrun[x] - mn);
      mrun[x] = mn;
    }
    float lsum[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < kBK / 8; ++n) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int x = c >> 1;
        const float p = (sc[n][c] == -CUDART_INF_F) ? 0.f : exp2f(sc[n][c] - mrun[x]);
        sc[n][c] = p;
        lsum[x] += p;
      }
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) lrun[x] = lrun[x] * alpha[x] + lsum[x];
#pragma unroll
    for (int n = 0; n < NO; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kc = 0; kc < kBK / 16; ++kc) {
      const unsigned pa0 = pack_bf16(sc[2 * kc][0], sc[2 * kc][1]);
      const unsigned pa1 = pack_bf16(sc[2 * kc][2], sc[2 * kc][3]);
      const unsigned pa2 = pack_bf16(sc[2 * kc + 1][0], sc[2 * kc + 1][1]);
      const unsigned pa3 = pack_bf16(sc[2 * kc + 1][2], sc[2 * kc + 1][3]);
#pragma unroll
      for (int n = 0; n < NO; ++n) {
        unsigned b0, b1;
        const int vrow = kc * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x2_t(b0, b1, s_v + vrow * ST + n * 8);
        mma_bf16(o[n], pa0, pa1, pa2, pa3, b0, b1);
      }
    }
    __syncthreads();  // this buffer is free for the tile after next
    kt = kn;
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int y = 0; y < 2; ++y) mw[x][y] = mwn[x][y];
  }
  // ---- epilogue ----
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    lrun[x] += __shfl_xor_sync(0xffffffffu, lrun[x], 1);
    lrun[x] += __shfl_xor_sync(0xffffffffu, lrun[x], 2);
  }
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    if (!rv[x]) continue;
    const float inv = 1.f / lrun[x];
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + (((size_t)b * a.T + ti[x]) * a.Hq + hq) * D;
#pragma unroll
    for (int n = 0; n < NO; ++n) {
      const __nv_bfloat162 v2 = __floats2bfloat162_rn(o[n][2 * x] * inv, o[n][2 * x + 1] * inv);
      *reinterpret_cast<__nv_bfloat162*>(orow + n * 8 + 2 * tq) = v2;
    }
  }
}

template <int D>
void set_select_attrs() {
  cudaFuncSetAttribute(select_rows_kernel<D, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_dyn_smem(4));
  cudaFuncSetAttribute(select_rows_kernel<D, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_dyn_smem(8));
  cudaFuncSetAttribute(select_rows_kernel<D, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_dyn_smem(16));
  cudaFuncSetAttribute(select_rows_kernel<D, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_dyn_smem(32));
}

template <int D>
void launch_select_rows(int idx, dim3 gs, cudaStream_t st, const PrefillArgs& a) {
  switch (idx) {
    case 4: select_rows_kernel<D, 4><<<gs, kSelRows * 32, sel_dyn_smem(4), st>>>(a); break;
    case 8: select_rows_kernel<D, 8><<<gs, kSelRows * 32, sel_dyn_smem(8), st>>>(a); break;
    case 32: select_rows_kernel<D, 32><<<gs, kSelRows * 32, sel_dyn_smem(32), st>>>(a); break;
    default: select_rows_kernel<D, 16><<<gs, kSelRows * 32, sel_dyn_smem(16), st>>>(a); break;
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

// Rows whose top-p bitmask the workspace holds at once: the whole chunk when
// that stays under kMaskBudget, else blocks of a multiple of the tcgen05
// attention's 256-row groups (the chunk then runs block by block: selection,
// attention, next block).
constexpr size_t kMaskBudget = size_t(1) << 30;
constexpr int kBlockAlign = 256;

int prefill_block_rows(const Shape& sh, int T) {
  const size_t words = (size_t)(sh.Lmax + 31) / 32;
  const size_t per_row = (size_t)sh.B * (size_t)(sh.NR > 0 ? sh.NR : 1) * words * sizeof(uint32_t);
  size_t rows = kMaskBudget / per_row;
  if (rows >= (size_t)T) return T;
  rows = rows / kBlockAlign * kBlockAlign;
  return rows < (size_t)kBlockAlign ? kBlockAlign : (int)rows;
}

PrefillLayout prefill_layout(const Shape& sh, int T) {
  PrefillLayout l;
  const size_t words = (size_t)(sh.Lmax + 31) / 32;
  const int rows = prefill_block_rows(sh, T);
  l.block_rows = rows;
  l.tmap = align256((size_t)sh.B * sh.NR * rows * words * sizeof(uint32_t));
  l.total = l.tmap + align256(tile_map_bytes(sh, T)) + 256;
  return l;
}

int launch_prefill(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* start_pos,
                   int T, const float* w_q, void* out, uint32_t* sel_bitmask, float* sel_tau,
                   int* sel_jcut, int* sel_count, void* ws, const PrefillLayout& lay, cudaStream_t st) {
  if (sh.dtype != RTP_BF16) {
    set_error("rtp_prefill_attn: the prefill path computes in bf16 (dtype must be RTP_BF16)");
    return RTP_ERR_DTYPE;
  }
  PrefillArgs a;
  a.B = sh.B; a.Hq = sh.Hq; a.Hkv = sh.Hkv; a.G = sh.G; a.D = sh.D; a.R = sh.R; a.NR = sh.NR;
  a.Lmax = sh.Lmax; a.S = sh.S; a.W = sh.W; a.T = T; a.words = (sh.Lmax + 31) / 32; a.Lk = sh.Lk;
  a.top_p = sh.top_p; a.rope_base = sh.rope_base;
  a.q_pre = q_pre; a.w_q = w_q; a.out = out;
  a.k = cache->k; a.v = cache->v; a.kidx = cache->kidx; a.status = cache->status;
  a.start_pos = start_pos;
  a.sel_tau = sel_tau; a.sel_jcut = sel_jcut; a.sel_count = sel_count;
  a.mask = sel_bitmask ? sel_bitmask : static_cast<uint32_t*>(ws);
  a.kv = sh.kv;
  a.ring_only = 0;
  for (int i = 0; i < kMaxRetrieval; ++i) { a.ret_head[i] = sh.ret_head[i]; a.ret_rank[i] = sh.ret_rank[i]; }
  for (int i = 0; i < 64; ++i) a.inv_freq[i] = sh.inv_freq[i];

  // per-device kernel attributes, set once under a mutex (calls may come from
  // several host threads)
  static std::mutex s_mu;
  static bool s_attr[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(s_mu);
  if (dev >= 0 && dev < 64 && !s_attr[dev]) {
    cudaFuncSetAttribute(attn_rows_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)AttnSmem<128>::kBytes);
    cudaFuncSetAttribute(attn_rows_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)AttnSmem<64>::kBytes);
    set_select_attrs<128>();
    set_select_attrs<64>();
    s_attr[dev] = true;
  }
  // The caller's bitmask holds every row; the workspace one block of rows.
  const int blk = sel_bitmask ? T : lay.block_rows;
  for (int t_base = 0; t_base < T; t_base += blk) {
    a.t_base = t_base;
    a.t_end = min(T, t_base + blk);
    a.mask_t0 = sel_bitmask ? 0 : t_base;
    a.mask_rows = sel_bitmask ? T : blk;
    const int n = a.t_end - t_base;
    if (sh.R > 0) {
      const dim3 gs((n + kSelRows - 1) / kSelRows, sh.B * sh.NR);
      trace_begin(RTP_STAGE_PREFILL_INDEX, st);
      if (sh.D == 128) launch_select_rows<128>(sh.idx, gs, st, a);
      else launch_select_rows<64>(sh.idx, gs, st, a);
      trace_end(RTP_STAGE_PREFILL_INDEX, st);
    }
    trace_begin(RTP_STAGE_PREFILL_ATTN, st);
    // full-context heads on tcgen05 tensor cores; local heads that keep a
    // window ring (rows not contiguous in positions) on the mma.sync kernel
    int rc = launch_attn_tc(sh, cache, q_pre, start_pos, T, out, a.mask, a.t_base, a.t_end, a.mask_t0,
                            a.mask_rows, reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + lay.tmap),
                            400ull * 1000 * 1000, st);
    if (rc != RTP_OK) return rc;
    if (sh.kv.ring_mask) {
      a.ring_only = 1;
      const dim3 ga((n + kBQ - 1) / kBQ, sh.B * sh.Hq);
      if (sh.D == 128) attn_rows_kernel<128><<<ga, 128, AttnSmem<128>::kBytes, st>>>(a);
      else attn_rows_kernel<64><<<ga, 128, AttnSmem<64>::kBytes, st>>>(a);
    }
    trace_end(RTP_STAGE_PREFILL_ATTN, st);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("prefill launch: ") + cudaGetErrorString(e));
    return RTP_ERR_CUDA;
  }
  return RTP_OK;
}

}  // namespace rtp
