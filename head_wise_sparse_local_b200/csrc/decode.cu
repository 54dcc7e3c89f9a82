// rtp_decode_attn: one decode step of the head-wise sparse attention layer.
//
// Three kernels on the caller's stream, chained with programmatic dependent
// launch, scratch in the caller's workspace, launched in the order score,
// select, sink/window.  The sink/window stream runs beside the select kernel;
// the stream kernels' CTAs pull their whole share into shared memory with
// asynchronous copies that complete on an mbarrier:
//
//   score_kernel   a chunk of the d-dim indexer-key cache (contiguous rows)
//                  per CTA (d = 16, or 4, 8, 32 for the dimension ablation);
//                  the fp32 scores s_j = q~ . k~_j / sqrt(d) of the G query
//                  heads of a retrieval KV head are formed on tensor cores
//                  (q~ as bf16 high and low parts, as in the prefill) and
//                  written with a per-chunk maximum.
//   select_kernel  one thread-block cluster per (sequence, retrieval q head).
//                  It launches once every score CTA has passed its wait and
//                  prepares its query, then waits for the score kernel to
//                  complete.  The softmax mass
//                  exp(s - max) of every score is taken in 2^-36 fixed point
//                  (integer sums: exact and order independent).  One pass sums
//                  the total mass and the mass and count at or above rungs 1,
//                  2, 4 and 8 below the maximum, and hands every score at or
//                  above the top rung to the leader CTA through distributed
//                  shared memory.  When those scores hold ceil(p * Z), the
//                  leader solves the exact threshold score tau (and, for ties
//                  at tau, the last kept index j_cut) over them.  Otherwise a
//                  lower rung's scores are collected in one more pass, or a
//                  2048-bucket mass histogram finds the boundary bucket whose
//                  scores are solved.  Every CTA then writes its share of the
//                  top-p bitmask and attends, for its query head, the kept
//                  rows of its share that lie outside the sinks and the
//                  window, and leaves its partial (o, max, sum) in L2.  Static
//                  top-k (the pages' fixed-budget baseline) runs the same
//                  solver with every token weighing 1 and the target k.
//   sw_kernel      one cluster per (sequence, KV head) attends the sinks and
//                  the window: S = K Q^T and O^T = V^T P on tensor cores per
//                  16-row tile (bf16; fp32 layers on CUDA cores), rows staged
//                  by cp.async into a padded layout, log-sum-exp merged across
//                  the cluster.  Local heads write their output here; a
//                  retrieval head's clusters wait for the select kernel and
//                  merge its partials into the output.
//
// Every in-kernel wait is either a hardware barrier reached uniformly or a
// bounded wait on a copy barrier (RTP_DEV_TIMEOUT when it gives up).
//
// Top-p follows the abstract's observation (3) and the atlas.scime.ai summary
// ("query-adaptive top-p threshold"); sinks + window follow that summary's
// "Approach"; the 16-d pre-RoPE indexer follows observation (2), the other
// widths the summary's "Surprising findings" (dimension 4); static top-k its
// "Baselines".
#include <algorithm>
#include <atomic>
#include <climits>
#include <mutex>
#include <type_traits>

#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace rtp {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// CTAs per sink/window cluster (one cluster per sequence and KV head).  A
// portable size: the clusters launch beside the select kernel's, and 8-CTA
// clusters find room on SMs where 16-CTA ones would wait for it to finish.
constexpr int kSwCluster = 8;
constexpr int kStreamSmem = 80 * 1024;  // stream kernel: bytes of staged keys (score) or K/V rows (two stages)
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxCS = 16;          // largest select cluster
constexpr int kLgCap = 8192;        // scores a select CTA holds in shared memory
constexpr int kCandSmem = 4096;     // candidates the leader holds in shared memory
constexpr int kBruteMax = kSelThreads;  // exact solve by pairwise ranks up to this many candidates
constexpr int kGroup = 4;           // kept rows a warp attends per memory round trip
constexpr int kPos = kLgCap / kSelThreads;  // positions a select thread owns per staged chunk
constexpr int kTopPerWarp = 16;     // top-rung items a warp hands the leader in the first pass
static_assert(kTopPerWarp <= 32, "the tail gives each top-rung item of a warp its own lane");
constexpr int kSpec = 2;            // of those, rows whose keys and values a warp stages early

// Tokens per score chunk: four (bf16) or two (fp32) keys per thread, 2 KB of
// indexer keys per indexer dim (32 KB at d = 16).
__host__ __device__ constexpr int score_chunk(int esize) { return kThreads * (esize == 2 ? 4 : 2); }
__host__ __device__ constexpr int score_smem(int idx) { return 2 * 2048 * idx; }  // two chunk buffers
__host__ __device__ constexpr int score_ctas_per_sm(int idx) { return idx == 32 ? 1 : 3; }

struct DecodeArgs {
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W, max_seq_len, words;
  int Lk;           // indexer-key rows per (sequence, retrieval head) block
  int lstride;      // row stride of the score scratch (Lmax rounded up to 32)
  float top_p, rope_base;
  int top_k;        // > 0: static top-k instead of top-p
  const void* q_pre;
  const float* w_q;
  void* out;
  const void* k;
  const void* v;
  const void* kidx;
  int* status;
  const int* seq_len;
  uint32_t* mask;   // [B][NR][words] top-p bitmask (caller's sel_bitmask or scratch)
  int* sel_count;   // optional [B][NR]
  float* logits;    // [B][NR][lstride]
  float* cmax;      // [B][NR][nch_score_max]
  float* sw_scratch;  // [B][Hkv][kSwCluster][G][D + 2]: partial of each CTA of a sink/window cluster
  float* sel_scratch; // [B][NR][kMaxCS][D + 3]: partial (o[D], m, l) and kept count of each select CTA
  uint2* cand;      // [B][NR][lstride] boundary-bucket candidates past kCandSmem
  int nch_score_max, n_score_ctas, sel_cs;
  int want_mask;    // 1: the caller asked for the top-p bitmask
  unsigned tx_extra;   // bytes a copy barrier expects beyond its copies (0; 16 when a test arms expiry)
  unsigned long long wait_ns;  // time a bounded wait allows before it gives up
  KvMap kv;
  int ret_head[kMaxRetrieval];
  int ret_rank[kMaxRetrieval];
  double inv_freq[64];  // RoPE frequencies, k < D/2
};


// Split cluster barrier (every thread of every CTA of the cluster calls both).
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" :: "l"(p)); }

__device__ __forceinline__ bool seq_ok(int L, const DecodeArgs& a) {
  return L >= 1 && L <= a.max_seq_len;
}

template <int kN>
__device__ __forceinline__ float block_max(float v, float* sm) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  float r = sm[0];
#pragma unroll
  for (int w = 1; w < kN / 32; ++w) r = fmaxf(r, sm[w]);
  return r;
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned warp_sum_u32(unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// RoPE'd query of the G heads of KV head h at position pos, scaled by
// log2(e)/sqrt(D), into shared memory [G][D].
template <typename T, int D, int G>
__device__ void rope_query(const DecodeArgs& a, int b, int h, int pos, float* s_q) {
  const float qscale = 1.4426950408889634f * rsqrtf((float)D);
  for (int i = threadIdx.x; i < G * (D / 2); i += blockDim.x) {
    const int g = i / (D / 2), k = i % (D / 2);
    const T* q = static_cast<const T*>(a.q_pre) + ((size_t)b * a.Hq + h * G + g) * D;
    const float x1 = to_f32(q[k]), x2 = to_f32(q[k + D / 2]);
    float c, s;
    rope_cos_sin(pos, a.inv_freq[k], c, s);
    s_q[g * D + k] = (x1 * c - x2 * s) * qscale;
    s_q[g * D + k + D / 2] = (x2 * c + x1 * s) * qscale;
  }
}

// ---------------------------------------------------------------------------
// 1a. score CTAs: indexer scores + per-chunk maxima of the retrieval KV heads
// ---------------------------------------------------------------------------
// A persistent grid (at most score_ctas_per_sm per SM) walks the chunks
// (sequence, retrieval KV head, chunk of kChunk tokens) in order, a CTA taking
// every gridDim.x-th.  A chunk's indexer keys (contiguous rows of the key
// cache) arrive in shared memory with one bulk asynchronous copy, two chunks in
// flight per CTA; the scores are formed there.
template <typename T, int D, int G, int IDX>
__device__ __forceinline__ void score_q(const DecodeArgs& a, int b, int r, float* s_q) {
  // q~ = W_q q_pre: four threads per output, a quarter of the dims each
  const int tid = threadIdx.x;
  const int h = a.ret_head[r];
  for (int o4 = tid; o4 < G * IDX * 4; o4 += kThreads) {
    const int o = o4 >> 2, qd = o4 & 3;
    const int g = o / IDX, i = o % IDX;
    constexpr int DQ = D / 4;
    const float4* w = reinterpret_cast<const float4*>(a.w_q + ((size_t)r * IDX + i) * D + qd * DQ);
    const T* q = static_cast<const T*>(a.q_pre) + ((size_t)b * a.Hq + h * G + g) * D + qd * DQ;
    float wv[DQ], qv[DQ];
#pragma unroll
    for (int k = 0; k < DQ / 4; ++k) {
      const float4 f = __ldg(w + k);
      wv[4 * k] = f.x; wv[4 * k + 1] = f.y; wv[4 * k + 2] = f.z; wv[4 * k + 3] = f.w;
    }
    load_row<T, DQ>(q, qv);
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < DQ; ++k) acc = fmaf(wv[k], qv[k], acc);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (qd == 0) s_q[g * IDX + i] = acc;
  }
}

template <typename T, int D, int G, int IDX>
__device__ __forceinline__ void score_ctas(const DecodeArgs& a, unsigned char* dsm, uint64_t* bar) {
  constexpr int kChunk = score_chunk(sizeof(T));
  constexpr int TPT = kChunk / kThreads;        // keys per thread
  constexpr int KB = IDX * sizeof(T);           // bytes per key
  constexpr int kBuf = kChunk * KB;             // bytes of one chunk buffer
  static_assert(2 * kBuf == score_smem(IDX), "chunk buffers");
  constexpr float kScale = idx_scale<IDX>();
  __shared__ __align__(16) float s_q[G * IDX];
  __shared__ float s_ml[kWarps * G];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = a.n_score_ctas / (a.B * a.R);  // chunks per (sequence, retrieval head)
  const int n_all = a.n_score_ctas;
  const uint64_t pol = l2_evict_first();
  if (blockIdx.x >= n_all) {  // no chunk for this CTA
    griddep_wait();
    griddep_launch();
    return;
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
  }
  int cur_br = blockIdx.x / nch;
  score_q<T, D, G, IDX>(a, cur_br / a.R, cur_br % a.R, s_q);  // the caller's inputs: before the wait
  __syncthreads();  // barriers initialised, q~ visible
  griddep_wait();   // rtp_append_kv (and with it the previous decode step) has completed
  griddep_launch();
  // chunk c: keys [j0, jh) of (sequence b, retrieval head r); rows fetched up to
  // the call's maximum length without looking at seq_len (rows past seq_len are
  // in bounds and their scores are never used)
  auto issue = [&](int c, int k) {  // k-th chunk of this CTA -> buffer k & 1
    const int br = c / nch, chunk = c % nch;
    const int j0 = chunk * kChunk, jh = min(a.max_seq_len, j0 + kChunk);
    const unsigned char* src = static_cast<const unsigned char*>(a.kidx) +
                               ((size_t)br * a.Lk + j0) * KB;
    // whole 16-byte units: an odd count of 8-byte keys takes the next key of
    // the block too (Lk is even then, and jh < Lk), never past the block
    const uint32_t bytes = ((uint32_t)(jh - j0) * KB + 15u) & ~15u;
    mbar_expect_tx(bar + (k & 1), bytes + a.tx_extra);
    bulk_g2s(dsm + (size_t)(k & 1) * kBuf, src, bytes, bar + (k & 1), pol);
  };
  if (tid == 0) {
    issue(blockIdx.x, 0);
    if (blockIdx.x + gridDim.x < n_all) issue(blockIdx.x + gridDim.x, 1);
  }
  int k = 0;
  for (int c = blockIdx.x; c < n_all; c += gridDim.x, ++k) {
    const int br = c / nch, chunk = c % nch;
    const int b = br / a.R, r = br % a.R;
    const int L = a.seq_len[b];
    if (br != cur_br) {  // another (sequence, retrieval head): its q~ (uniform over the CTA)
      __syncthreads();
      score_q<T, D, G, IDX>(a, b, r, s_q);
      cur_br = br;
    }
    const bool arrived = mbar_wait_bounded(bar + (k & 1), (uint32_t)(k >> 1) & 1u, a.wait_ns, a.status);
    if (__syncthreads_or(!arrived)) {  // every thread takes the same branch
      // a copy did not complete in time (RTP_DEV_TIMEOUT is set): wait, again
      // with a limit, for the copies in flight before leaving; output invalid
      mbar_wait_bounded(bar + (k & 1), (uint32_t)(k >> 1) & 1u, a.wait_ns, a.status);
      if (c + gridDim.x < n_all)
        mbar_wait_bounded(bar + ((k + 1) & 1), (uint32_t)((k + 1) >> 1) & 1u, a.wait_ns, a.status);
      return;
    }
    const unsigned char* kbuf = dsm + (size_t)(k & 1) * kBuf;
    if (!seq_ok(L, a)) {  // uniform over the CTA
      if (chunk == 0 && r == 0 && tid == 0) atomicOr(a.status, RTP_DEV_SEQ_LEN);
    } else {
      const int j0 = chunk * kChunk;
      const int j1 = min(L, min(a.max_seq_len, j0 + kChunk));
      float* lg = a.logits + ((size_t)b * a.NR + (size_t)r * G) * a.lstride;
      if constexpr (sizeof(T) == 2) {
        // Tensor cores, with exactly the prefill selection's arithmetic: S = K~ Q~^T
        // (16 keys x 8 columns per mma, column n = query head n < G), q~ split
        // into bf16 hi and lo parts accumulated in that order into one fp32
        // accumulator.  A prefill row and the decode step at its position then
        // see bit-identical scores.
        const int t4 = lane & 3, gq = lane >> 2;
        IdxMma<IDX> mm;
        mm.set_q(gq < G ? s_q + gq * IDX : nullptr, lane);
        // this lane's columns 2 t4, 2 t4 + 1 (query heads when < G)
        float mxa = -CUDART_INF_F, mxb = -CUDART_INF_F;
        const bool ca = 2 * t4 < G, cb = 2 * t4 + 1 < G;
        // The warp's tiles are warp, warp + kWarps, ...: all of their products
        // are issued first (independent mma chains overlap their latency),
        // then the scores are stored.  A tile past the chunk's keys reads
        // stale shared memory (inside the buffer) whose scores are dropped.
        constexpr int kTiles = kChunk / 16;
        constexpr int kTPW = kTiles / kWarps;  // tiles per warp
        static_assert(kTiles % kWarps == 0, "whole tiles per warp");
        float cc[kTPW][4];
#pragma unroll
        for (int u = 0; u < kTPW; ++u) mm.scores(kbuf + (size_t)(warp + u * kWarps) * 16 * KB, lane, cc[u]);
#pragma unroll
        for (int u = 0; u < kTPW; ++u) {
          const int kb = (warp + u * kWarps) * 16;  // first key of the tile (chunk-local)
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int j = j0 + kb + gq + 8 * x;
            if (j >= j1) continue;
            const float sa = cc[u][2 * x] * kScale + 0.0f;  // +0 turns -0 into +0
            const float sb = cc[u][2 * x + 1] * kScale + 0.0f;
            if (ca) {
              lg[(size_t)(2 * t4) * a.lstride + j] = sa;
              mxa = fmaxf(mxa, sa);
            }
            if (cb) {
              lg[(size_t)(2 * t4 + 1) * a.lstride + j] = sb;
              mxb = fmaxf(mxb, sb);
            }
          }
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, o));
          mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, o));
        }
        if (gq == 0) {
          if (ca) s_ml[warp * G + 2 * t4] = mxa;
          if (cb) s_ml[warp * G + 2 * t4 + 1] = mxb;
        }
      } else {
        float mx[G];
#pragma unroll
        for (int g = 0; g < G; ++g) mx[g] = -CUDART_INF_F;
#pragma unroll
        for (int t = 0; t < TPT; ++t) {
          const int jl = t * kThreads + tid;
          const int j = j0 + jl;
          if (j >= j1) continue;
          constexpr int NV = KB / 16;  // 16-byte vectors per fp32 key
          uint4 kr[NV];
#pragma unroll
          for (int v = 0; v < NV; ++v) kr[v] = reinterpret_cast<const uint4*>(kbuf + (size_t)jl * KB)[v];
          float kv[IDX];
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            kv[v * 4 + 0] = __uint_as_float(kr[v].x); kv[v * 4 + 1] = __uint_as_float(kr[v].y);
            kv[v * 4 + 2] = __uint_as_float(kr[v].z); kv[v * 4 + 3] = __uint_as_float(kr[v].w);
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4* q4 = reinterpret_cast<const float4*>(s_q + g * IDX);
            float sco = 0.f;
#pragma unroll
            for (int i4 = 0; i4 < IDX / 4; ++i4) {
              const float4 qq = q4[i4];
              sco = fmaf(qq.x, kv[4 * i4], sco);
              sco = fmaf(qq.y, kv[4 * i4 + 1], sco);
              sco = fmaf(qq.z, kv[4 * i4 + 2], sco);
              sco = fmaf(qq.w, kv[4 * i4 + 3], sco);
            }
            sco = sco * kScale + 0.0f;  // +0 turns -0 into +0
            lg[(size_t)g * a.lstride + j] = sco;
            mx[g] = fmaxf(mx[g], sco);
          }
        }
        // one block reduction for the G chunk maxima (-inf for a chunk past seq_len)
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float v = warp_max(mx[g]);
          if (lane == 0) s_ml[warp * G + g] = v;
        }
      }
      __syncthreads();
      if (tid < G) {
        float v = s_ml[tid];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) v = fmaxf(v, s_ml[w * G + tid]);
        a.cmax[((size_t)b * a.NR + r * G + tid) * a.nch_score_max + chunk] = v;
      }
    }
    __syncthreads();  // buffer k & 1 is free
    if (tid == 0 && c + 2 * gridDim.x < n_all) issue(c + 2 * gridDim.x, k + 2);
  }
}

// ---------------------------------------------------------------------------
// 1b. sink/window CTA: rank `crank` of the cluster of (sequence b, KV head h)
// ---------------------------------------------------------------------------
// The CTA's rows (the sinks, then the window, which wraps once in a ring)
// arrive in shared memory by cp.async, 16 bytes per thread, in stages of at
// most kStreamSmem / 2 bytes (K and V), two stages in flight; a bf16 row is
// padded by 16 bytes there.  bf16 layers run the tensor-core tiles below.
// fp32 layers: a half-warp owns a row, lane (half, c) reading dims
// [c*EPL, c*EPL + EPL) of the row's key and value, so a warp covers two rows;
// scores of the G query heads are reduced over the half-warp by shuffles, and
// every lane keeps the running (max, sum) of its half and the weighted value
// sum of its own dims.
template <typename T, int D>
struct SwLane {
  static constexpr int EPL = D / 16;                 // elements per lane per row
  static constexpr int VB = EPL * (int)sizeof(T);    // bytes per lane per row
  static constexpr int NV = VB >= 16 ? VB / 16 : 1;
  using Vec = typename std::conditional<VB >= 16, uint4, uint2>::type;
  Vec v[NV];
  __device__ __forceinline__ void load(const unsigned char* p) {
    const Vec* q = reinterpret_cast<const Vec*>(p);
#pragma unroll
    for (int i = 0; i < NV; ++i) v[i] = q[i];
  }
  __device__ __forceinline__ void to_f32(float (&f)[EPL]) const {
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(v);
#pragma unroll
      for (int i = 0; i < EPL / 2; ++i) {
        const float2 x = __bfloat1622float2(h2[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
      }
    } else {
      const float* x = reinterpret_cast<const float*>(v);
#pragma unroll
      for (int i = 0; i < EPL; ++i) f[i] = x[i];
    }
  }
};

template <typename T, int D, int G>
__device__ __forceinline__ void sw_cta(const DecodeArgs& a, int bkv, int crank, int csw, unsigned char* dsm,
                                       uint64_t* bar) {
  using Lane = SwLane<T, D>;
  constexpr int EPL = Lane::EPL;
  constexpr int RB = D * (int)sizeof(T);             // bytes per cache row
  // Shared-memory row stride: a bf16 row is padded by 16 bytes, so the 8 rows
  // that one ldmatrix phase reads start 4 banks apart (conflict-free) instead
  // of all in the same 4 banks.
  constexpr int RBS = sizeof(T) == 2 ? RB + 16 : RB;
  constexpr int CPW = 2 * RB / 16;                   // 16-byte chunks of a row's K and V
  static_assert((CPW & (CPW - 1)) == 0, "chunks per row: a power of two");
  // rows per stage (K and V of a stage take at most half the buffer; at most
  // 80 rows, 32 for G = 8, which keeps a warp's scores of a stage in registers)
  constexpr int kCapRows = G >= 8 ? 32 : 80;
  constexpr int SR = ((kStreamSmem / 4 / RBS) < kCapRows ? (kStreamSmem / 4 / RBS) : kCapRows) & ~1;
  static_assert(SR >= 2 && SR % 2 == 0, "a stage holds whole row pairs");
  static_assert(2 * SR * RBS <= kStreamSmem / 2, "a stage's K and V fit in half the buffer");
  __shared__ __align__(16) float s_q[G * D];
  __shared__ __align__(16) float s_wo[kWarps][G][D];
  __shared__ float s_wml[kWarps][G][2];
  cg::cluster_group cl = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = lane >> 4, c = lane & 15;
  const int b = bkv / a.Hkv, h = bkv % a.Hkv;
  const int r = a.ret_rank[h];
  const int L = a.seq_len[b];
  if (!seq_ok(L, a)) {  // uniform over the cluster
    if (crank == 0 && h == 0 && tid == 0) atomicOr(a.status, RTP_DEV_SEQ_LEN);
    return;
  }
  // A stage's barrier phase completes with one arrival per thread, made once
  // that thread's copies have landed, plus one from thread 0 (which, when a
  // test arms expiry, also expects bytes that never come).
  if (tid == 0) {
    mbar_init(bar, kThreads + 1);
    mbar_init(bar + 1, kThreads + 1);
  }
  // With a score kernel ahead the appended rows are complete already (this
  // kernel starts after every score CTA has passed its wait): the copies go
  // out first and the query is formed while they fly.  Without one, the query
  // comes first, then the wait for rtp_append_kv.
  const bool waits = a.n_score_ctas == 0;
  if (waits) rope_query<T, D, G>(a, b, h, L - 1, s_q);
  __syncthreads();  // barriers initialised
  if (waits) griddep_wait();

  const int s_cnt = min(a.S, L);
  const int sw0 = max(s_cnt, L - a.W);
  const int n_sw = s_cnt + (L - sw0);      // rows e: sinks e < s_cnt, then window positions
  const int npair_all = (n_sw + 1) / 2;
  const int per = (npair_all + csw - 1) / csw;
  const int e_lo = min(n_sw, 2 * crank * per), e_hi = min(n_sw, 2 * (crank + 1) * per);
  const int n_st = (e_hi - e_lo + SR - 1) / SR;
  const unsigned char* kbase = static_cast<const unsigned char*>(a.k);
  const unsigned char* vbase = static_cast<const unsigned char*>(a.v);
  // Cache row of stage row e.  A ring head's window positions (at or past the
  // sinks whenever the window is not empty) sit in consecutive ring slots from
  // the slot of sw0, wrapping at most once (the ring holds at least W rows).
  const bool fast_ring = ((a.kv.ring_mask >> h) & 1ull) && sw0 >= a.kv.S;
  const int ws0 = fast_ring ? a.kv.S + (sw0 - a.kv.S) % a.kv.ring : 0;
  const size_t seq_row0 = (size_t)b * (size_t)a.kv.rows_per_seq + (size_t)a.kv.row0[h];
  auto row_of = [&](int e) -> size_t {
    if (e >= s_cnt && fast_ring) {
      int sl = ws0 + (e - s_cnt);
      if (sl >= a.kv.S + a.kv.ring) sl -= a.kv.ring;
      return seq_row0 + (size_t)sl;
    }
    return a.kv.row(b, h, e < s_cnt ? e : sw0 + (e - s_cnt));
  };

  // stage st: rows [e_lo + st*SR, ...) into buffer st & 1 (K rows, then V
  // rows, RBS apart), 16 bytes per cp.async; every thread takes part
  auto issue = [&](int st) {
    const int e0 = e_lo + st * SR, e1 = min(e_hi, e0 + SR);
    uint64_t* bb = bar + (st & 1);
    unsigned char* dk = dsm + (size_t)(st & 1) * (kStreamSmem / 2);
    unsigned char* dv = dk + (size_t)SR * RBS;
    const uint64_t pol = l2_evict_first();
    const int nch = (e1 - e0) * CPW;
    for (int i = tid; i < nch; i += kThreads) {
      const int e = e0 + i / CPW, cc = i % CPW;
      const bool isv = cc >= CPW / 2;
      const int off = 16 * (isv ? cc - CPW / 2 : cc);
      const size_t row = row_of(e);
      cp_async16((isv ? dv : dk) + (size_t)(e - e0) * RBS + off, (isv ? vbase : kbase) + row * RB + off, pol);
    }
    cp_async_arrive_noinc(bb);
    if (tid == 0) {
      if (a.tx_extra) mbar_expect_tx(bb, a.tx_extra);
      else mbar_arrive(bb);
    }
  };
  if (n_st > 0) issue(0);
  if (n_st > 1) issue(1);
  if (!waits) rope_query<T, D, G>(a, b, h, L - 1, s_q);
  __syncthreads();  // s_q visible

  int failed = -1;
  if constexpr (sizeof(T) == 2) {
    // Tensor cores.  Per 16-row tile of a stage: S = K Q^T (16 rows x 8
    // columns: query head c < G from q's bf16 high part, column G + c from its
    // low part, so a score is the fp32-query score to about 2^-17), then
    // O^T += V^T P (D x 8: the G heads' weighted values; P in bf16, as the
    // prefill attention rounds it).  A lane owns query heads 2 t4 and
    // 2 t4 + 1 (t4 = lane mod 4) for the tile rows g and g + 8 (g = lane / 4).
    constexpr int KS = D / 16;
    constexpr int NT = (2 * G + 7) / 8;  // n-tiles of S: 1, or 2 for G = 8
    const int t4 = lane & 3, gq = lane >> 2;
    unsigned qb[NT][KS][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int cix = nt * 8 + gq;
      const int hd = cix < G ? cix : cix - G;
      const int part = cix < G ? 0 : (cix < 2 * G ? 1 : 2);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (part < 2) {
          const float* qg = s_q + hd * D + ks * 16 + 2 * t4;
          const float v[4] = {qg[0], qg[1], qg[8], qg[9]};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float hi = __bfloat162float(__float2bfloat16_rn(v[e]));
            x[e] = part == 0 ? hi : v[e] - hi;
          }
        }
        qb[nt][ks][0] = pack_bf16(x[0], x[1]);
        qb[nt][ks][1] = pack_bf16(x[2], x[3]);
      }
    }
    float mh[2] = {-CUDART_INF_F, -CUDART_INF_F}, lh[2] = {0.f, 0.f};
    float oacc[KS][4];
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
    const bool own[2] = {2 * t4 < G, 2 * t4 + 1 < G};
    for (int st = 0; st < n_st; ++st) {
      const bool arrived = mbar_wait_bounded(bar + (st & 1), (uint32_t)(st >> 1) & 1u, a.wait_ns, a.status);
      if (__syncthreads_or(!arrived)) {  // every thread takes the same branch
        failed = st;
        break;
      }
      const int n = min(e_hi, e_lo + (st + 1) * SR) - (e_lo + st * SR);
      const unsigned char* sk = dsm + (size_t)(st & 1) * (kStreamSmem / 2);
      const unsigned char* sv = sk + (size_t)SR * RBS;
      for (int tt = warp; 16 * tt < n; tt += kWarps) {  // warp-uniform
        const int r0 = 16 * tt;
        // S = K Q^T; rows past n read row 0 (their weights are zeroed)
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
        {
          const int rr = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const unsigned char* krow = sk + (size_t)(rr < n ? rr : 0) * RBS + (lane >> 4) * 16;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            unsigned a0, a1, a2, a3;
            ldsm_x4(a0, a1, a2, a3, krow + ks * 32);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(sacc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
          }
        }
        // scores of the lane's heads: high part + low part
        float sc[2][2];  // [row g / g + 8][head 2 t4 + e]
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float lo_part;
          if constexpr (G == 8) lo_part = sacc[NT - 1][i];
          else if constexpr (G == 4) lo_part = __shfl_xor_sync(0xffffffffu, sacc[0][i], 2);
          else if constexpr (G == 2) lo_part = __shfl_xor_sync(0xffffffffu, sacc[0][i], 1);
          else lo_part = sacc[0][i ^ 1];
          sc[i >> 1][i & 1] = (G == 8 ? sacc[0][i] : sacc[0][i]) + lo_part;
        }
        float tmx[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const bool okr = r0 + gq + 8 * x < n;
            sc[x][e] = (own[e] && okr) ? sc[x][e] : -CUDART_INF_F;
          }
          tmx[e] = fmaxf(sc[0][e], sc[1][e]);
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) tmx[e] = fmaxf(tmx[e], __shfl_xor_sync(0xffffffffu, tmx[e], o));
        }
        float pr[2][2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float mn = fmaxf(mh[e], tmx[e]);
          const float al = (mn == -CUDART_INF_F) ? 1.f : exp2f(mh[e] - mn);  // 0 when mh = -inf
          pr[0][e] = (sc[0][e] == -CUDART_INF_F) ? 0.f : exp2f(sc[0][e] - mn);
          pr[1][e] = (sc[1][e] == -CUDART_INF_F) ? 0.f : exp2f(sc[1][e] - mn);
          lh[e] = lh[e] * al + (pr[0][e] + pr[1][e]);
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            oacc[mt][e] *= al;
            oacc[mt][2 + e] *= al;
          }
          mh[e] = mn;
        }
        // B fragments of P (k = 16 rows, n = 8 columns = query heads): lane
        // (g, t4) needs P[rows 2 t4, 2 t4 + 1, 2 t4 + 8, 2 t4 + 9][head g],
        // held by lanes (2 t4) * 4 + g / 2 and (2 t4 + 1) * 4 + g / 2
        const unsigned u0 = pack_bf16(pr[0][0], pr[0][1]);  // row g: heads 2 t4, 2 t4 + 1
        const unsigned u1 = pack_bf16(pr[1][0], pr[1][1]);  // row g + 8
        const int s0 = (2 * t4) * 4 + (gq >> 1), s1 = (2 * t4 + 1) * 4 + (gq >> 1);
        const unsigned x0 = __shfl_sync(0xffffffffu, u0, s0), x1 = __shfl_sync(0xffffffffu, u0, s1);
        const unsigned y0 = __shfl_sync(0xffffffffu, u1, s0), y1 = __shfl_sync(0xffffffffu, u1, s1);
        const unsigned sel = (gq & 1) ? 0x7632u : 0x5410u;
        const unsigned pb0 = gq < G ? __byte_perm(x0, x1, sel) : 0u;
        const unsigned pb1 = gq < G ? __byte_perm(y0, y1, sel) : 0u;
        // O^T += V^T P: V^T fragments by transposing loads of V rows
        {
          const int rr = r0 + (lane & 7) + ((lane >> 4) & 1) * 8;
          const unsigned char* vrow = sv + (size_t)(rr < n ? rr : 0) * RBS + ((lane >> 3) & 1) * 16;
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            unsigned a0, a1, a2, a3;
            ldsm_x4_t(a0, a1, a2, a3, vrow + mt * 32);
            mma_bf16(oacc[mt], a0, a1, a2, a3, pb0, pb1);
          }
        }
      }
      __syncthreads();  // buffer st & 1 is free
      if (st + 2 < n_st) issue(st + 2);
    }
    // the warp's state: l summed over its lanes' rows; O^T fragments to shared memory
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) lh[e] += __shfl_xor_sync(0xffffffffu, lh[e], o);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (!own[e]) continue;
      const int hd = 2 * t4 + e;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        s_wo[warp][hd][mt * 16 + gq] = oacc[mt][e];
        s_wo[warp][hd][mt * 16 + gq + 8] = oacc[mt][2 + e];
      }
      if (gq == 0) {
        s_wml[warp][hd][0] = mh[e];
        s_wml[warp][hd][1] = lh[e];
      }
    }
  } else {
  // this lane's dims of the G RoPE'd queries
  float qr[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) qr[g][e] = s_q[g * D + c * EPL + e];
  float m[G], l[G], o[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -CUDART_INF_F;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[g][e] = 0.f;
  }
  // Per stage: every score of the warp's rows first, then one running-max
  // update per head, then the weights and the weighted values.
  constexpr int PPW = (SR / 2 + kWarps - 1) / kWarps;  // row pairs per warp per stage
  for (int st = 0; st < n_st; ++st) {
    const bool arrived = mbar_wait_bounded(bar + (st & 1), (uint32_t)(st >> 1) & 1u, a.wait_ns, a.status);
    if (__syncthreads_or(!arrived)) {  // every thread takes the same branch
      failed = st;
      break;
    }
    const int n = min(e_hi, e_lo + (st + 1) * SR) - (e_lo + st * SR);
    const unsigned char* sk = dsm + (size_t)(st & 1) * (kStreamSmem / 2);
    const unsigned char* sv = sk + (size_t)SR * RBS;
    float sc[PPW][G];
    float smax[G];
#pragma unroll
    for (int g = 0; g < G; ++g) smax[g] = -CUDART_INF_F;
#pragma unroll
    for (int k = 0; k < PPW; ++k) {
      const int i = 2 * (warp + k * kWarps) + half;
      const bool ok = i < n;  // uniform over the half-warp
      Lane kr;
      kr.load(sk + (size_t)(ok ? i : 0) * RBS + c * Lane::VB);
      float kf[EPL];
      kr.to_f32(kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc = fmaf(qr[g][e], kf[e], acc);
        sc[k][g] = acc;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = sc[k][g];
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        sc[k][g] = ok ? v : -CUDART_INF_F;
        smax[g] = fmaxf(smax[g], sc[k][g]);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mn = fmaxf(m[g], smax[g]);
      if (mn == -CUDART_INF_F) continue;  // nothing in this half-warp yet (uniform over it)
      const float al = exp2f(m[g] - mn);   // 0 while nothing was attended (m = -inf)
      l[g] *= al;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[g][e] *= al;
      m[g] = mn;
    }
#pragma unroll
    for (int k = 0; k < PPW; ++k) {
      const int i = 2 * (warp + k * kWarps) + half;
      if (i >= n) continue;  // uniform over the half-warp
      Lane vr;
      vr.load(sv + (size_t)i * RBS + c * Lane::VB);
      float vf[EPL];
      vr.to_f32(vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pv = exp2f(sc[k][g] - m[g]);
        l[g] += pv;
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[g][e] = fmaf(pv, vf[e], o[g][e]);
      }
    }
    __syncthreads();  // buffer st & 1 is free
    if (st + 2 < n_st) issue(st + 2);
  }
  // the two halves of the warp, then the warps of the CTA
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m[g], 16);
    const float l2 = __shfl_xor_sync(0xffffffffu, l[g], 16);
    const float mn = fmaxf(m[g], m2);
    const float a1 = (m[g] == -CUDART_INF_F) ? 0.f : exp2f(m[g] - mn);
    const float a2 = (m2 == -CUDART_INF_F) ? 0.f : exp2f(m2 - mn);
    l[g] = l[g] * a1 + l2 * a2;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float o2 = __shfl_xor_sync(0xffffffffu, o[g][e], 16);
      o[g][e] = o[g][e] * a1 + o2 * a2;
    }
    m[g] = mn;
    if (half == 0) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) s_wo[warp][g][c * EPL + e] = o[g][e];
    }
    if (lane == 0) {
      s_wml[warp][g][0] = m[g];
      s_wml[warp][g][1] = l[g];
    }
  }
  }
  if (failed >= 0) {
    // a copy did not complete in time (RTP_DEV_TIMEOUT is set): wait, again
    // with a limit, for the stages still in flight before leaving; the
    // output is invalid
    for (int st = failed; st < min(n_st, failed + 2); ++st)
      mbar_wait_bounded(bar + (st & 1), (uint32_t)(st >> 1) & 1u, a.wait_ns, a.status);
    asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's own copies, which always land
  }
  __syncthreads();
  // this CTA's partial (o[D], m, l) per query head -> the cluster's slot in L2
  float* part = a.sw_scratch + ((size_t)bkv * kSwCluster + crank) * (G * (D + 2));
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, d = i % D;
    float mn = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mn = fmaxf(mn, s_wml[w][g][0]);
    float acc = 0.f, den = 0.f;
    if (mn != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = s_wml[w][g][0];
        if (mw == -CUDART_INF_F) continue;
        const float sc = exp2f(mw - mn);
        acc = fmaf(s_wo[w][g][d], sc, acc);
        den = fmaf(s_wml[w][g][1], sc, den);
      }
    }
    part[g * (D + 2) + d] = acc;
    if (d == 0) {
      part[g * (D + 2) + D] = mn;
      part[g * (D + 2) + D + 1] = den;
    }
  }
  cl.sync();  // every rank's partial written (the barrier orders global memory within the cluster)
  // The cluster's merge is spread over its ranks: element i of the G x D
  // outputs goes to rank i mod csw.  A retrieval head adds the kept-row
  // partials of the select kernel's ranks: that kernel was launched ahead of
  // this one and ran beside it; once the wait below returns it has completed.
  // Each thread issues its loads of every partial at once (L2 hits, one round
  // trip).
  const float* parts = a.sw_scratch + (size_t)bkv * kSwCluster * (G * (D + 2));
  const int ncs = r >= 0 ? a.sel_cs : 0;  // select CTAs per retrieval query head (uniform over the cluster)
  if (ncs > 0) griddep_wait();
  for (int i = crank + csw * tid; i < G * D; i += csw * kThreads) {
    const int g = i / D, d = i % D;
    float mq[kSwCluster], lq[kSwCluster], oq[kSwCluster];
    float ms[kMaxCS], ls[kMaxCS], os[kMaxCS];
#pragma unroll
    for (int q = 0; q < kSwCluster; ++q) {
      mq[q] = -CUDART_INF_F;
      lq[q] = 0.f;
      oq[q] = 0.f;
      if (q < csw) {
        const float* pq = parts + (size_t)q * (G * (D + 2)) + g * (D + 2);
        mq[q] = __ldcg(pq + D);
        lq[q] = __ldcg(pq + D + 1);
        oq[q] = __ldcg(pq + d);
      }
    }
    const float* sel = a.sel_scratch + ((size_t)(b * a.NR + (r < 0 ? 0 : r) * G + g) * kMaxCS) * (D + 3);
#pragma unroll
    for (int q = 0; q < kMaxCS; ++q) {
      ms[q] = -CUDART_INF_F;
      ls[q] = 0.f;
      os[q] = 0.f;
      if (q < ncs) {
        const float* pq = sel + (size_t)q * (D + 3);
        ms[q] = __ldcg(pq + D);
        ls[q] = __ldcg(pq + D + 1);
        os[q] = __ldcg(pq + d);
      }
    }
    float mn = -CUDART_INF_F;
#pragma unroll
    for (int q = 0; q < kSwCluster; ++q) mn = fmaxf(mn, mq[q]);
#pragma unroll
    for (int q = 0; q < kMaxCS; ++q) mn = fmaxf(mn, ms[q]);
    float acc = 0.f, den = 0.f;
#pragma unroll
    for (int q = 0; q < kSwCluster; ++q) {
      const float sc = mq[q] == -CUDART_INF_F ? 0.f : exp2f(mq[q] - mn);
      acc = fmaf(oq[q], sc, acc);
      den = fmaf(lq[q], sc, den);
    }
#pragma unroll
    for (int q = 0; q < kMaxCS; ++q) {
      const float sc = ms[q] == -CUDART_INF_F ? 0.f : exp2f(ms[q] - mn);
      acc = fmaf(os[q], sc, acc);
      den = fmaf(ls[q], sc, den);
    }
    T* out = static_cast<T*>(a.out) + ((size_t)b * a.Hq + h * G + g) * D + d;
    *out = from_f32<T>(acc / den);
  }
  // kept-token counts of the head's query heads: the sum over the select ranks
  if (ncs > 0 && crank == 0 && tid < G && a.sel_count != nullptr) {
    const float* sel = a.sel_scratch + ((size_t)(b * a.NR + r * G + tid) * kMaxCS) * (D + 3);
    int cnt = 0;
    for (int q = 0; q < ncs; ++q) cnt += __float_as_int(__ldcg(sel + (size_t)q * (D + 3) + D + 2));
    a.sel_count[b * a.NR + r * G + tid] = cnt;
  }
}

// ---------------------------------------------------------------------------
// 1. the two stream kernels
// ---------------------------------------------------------------------------
// Launch order score -> select -> sink/window.  score_kernel (plain grid)
// waits for rtp_append_kv, then lets the select kernel launch; the select
// kernel lets the sink/window kernel launch at once.  sw_kernel (clusters)
// reads the cache without a wait of its own: it starts only after every score
// CTA has passed its wait, so the appended rows are complete.  A retrieval
// head's clusters wait for the select kernel before their merge; every CTA's
// closing wait makes the kernel's completion imply the select kernel's (and
// with it the score kernel's), which is what the next kernel on the stream
// relies on.
template <typename T, int D, int G, int IDX>
__global__ void __launch_bounds__(kThreads, score_ctas_per_sm(IDX)) score_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ __align__(8) uint64_t s_bar[2];
  score_ctas<T, D, G, IDX>(a, dsm, s_bar);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 2) sw_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ __align__(8) uint64_t s_bar[2];
  griddep_launch();
  const int csw = (int)cg::this_cluster().num_blocks();
  sw_cta<T, D, G>(a, blockIdx.x / csw, (int)cg::this_cluster().block_rank(), csw, dsm, s_bar);
  griddep_wait();
}

// ---------------------------------------------------------------------------
// selection helpers
// ---------------------------------------------------------------------------
// Softmax mass exp(s - max) in 2^-36 fixed point (mass36): integer sums are
// exact and order independent, so the first pass, the histogram and the exact
// solve agree bit for bit.  The histogram accumulates it per bucket as two
// 18-bit halves with 32-bit shared atomics (native and robust to contention):
// with x = mass_x36(s, m), hi = floor(x / 2^18) and x - hi 2^18 are exact in
// fp32, and rounding the remainder gives rint(x) - hi 2^18 because hi 2^18 is
// an even integer.
__device__ __forceinline__ void mass_split36(float s, float m, unsigned& hi, unsigned& lo) {
  const float x = mass_x36(s, m);
  const float hf = floorf(x * 3.814697265625e-06f);  // 2^-18
  hi = (unsigned)hf;
  lo = __float2uint_rn(fmaf(hf, -262144.0f, x));
}

// Weight of an item in the threshold search: its softmax mass in 2^-36 fixed
// point (top-p), or 1 (static top-k: "the shortest prefix whose weight reaches
// k" is then exactly the k highest scores, ties to the lower index).
__device__ __forceinline__ unsigned long long item_w(float s, float m, bool cnt) {
  return cnt ? 1ull : mass36(s, m);
}

struct DigitResult {
  int digit;
  unsigned long long above;
  unsigned cnt_above;
  unsigned cnt_digit;
};

// Items for the exact solve: a list of (order key, index) in shared memory,
// or in global scratch (read through L2: other CTAs of the cluster wrote it).
struct Items {
  const uint2* list;
  bool global;
  __device__ __forceinline__ bool get(int i, uint2& e) const {
    e = global ? __ldcg(list + i) : list[i];
    return true;
  }
};

// One 8-bit radix step.  kMass: items with (key & mask) == prefix, weighted by
// their softmax mass, digits ranked high to low.  !kMass: items with key ==
// key_eq counted, index digits ranked low to high.  Finds the first digit at
// which the running total reaches `need`.
// The general solvers below are rarely reached by a decode step; kept out of
// line so that the common path's code stays compact (each code block a
// launch reaches for the first time costs an instruction fetch from L2).
template <bool kMass>
__device__ __noinline__ DigitResult radix_step(const Items& it, int n, uint32_t prefix, uint32_t mask,
                                  uint32_t key_eq, int shift, float m, bool cntw, unsigned long long need,
                                  unsigned long long* h_m, unsigned* h_c, DigitResult* s_res) {
  const int tid = threadIdx.x;
  for (int i = tid; i < 256; i += blockDim.x) { h_m[i] = 0ull; h_c[i] = 0u; }
  if (tid == 0) *s_res = DigitResult{0, 0ull, 0u, 0u};
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    uint2 e;
    if (!it.get(i, e)) continue;
    if constexpr (kMass) {
      if ((e.x & mask) == prefix) {
        const int dg = (e.x >> shift) & 255;
        atomicAdd(&h_m[dg], item_w(key_score(e.x), m, cntw));
        atomicAdd(&h_c[dg], 1u);
      }
    } else {
      if (e.x == key_eq && (e.y & mask) == prefix) {
        const int dg = (e.y >> shift) & 255;
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

// Exact tau / j_cut among n items whose mass must supply `need` (one CTA).
// Order: key descending, index ascending.  The kept set is the shortest prefix
// whose mass reaches `need`.
__device__ __noinline__ void solve_radix(const Items& it, int n, float m, bool cntw, unsigned long long need,
                            unsigned long long* h_m, unsigned* h_c, DigitResult* s_res,
                            uint32_t* s_kr, float& tau, int& jcut) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  int cnt = 0;
  for (int i = tid; i < n; i += blockDim.x) {
    uint2 e;
    if (!it.get(i, e)) continue;
    kmin = min(kmin, e.x);
    kmax = max(kmax, e.x);
    ++cnt;
  }
  cnt = warp_sum_i(cnt);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) { s_kr[warp] = kmin; s_kr[32 + warp] = kmax; s_kr[64 + warp] = (uint32_t)cnt; }
  __syncthreads();
  kmin = s_kr[0];
  kmax = s_kr[32];
  unsigned n_items = s_kr[64];
  for (int w = 1; w < nw; ++w) {
    kmin = min(kmin, s_kr[w]);
    kmax = max(kmax, s_kr[32 + w]);
    n_items += s_kr[64 + w];
  }
  __syncthreads();

  uint32_t prefix = kmin, mask = 0xffffffffu;
  unsigned cnt_eq = 0u;
  const uint32_t diff = kmin ^ kmax;
  if (diff != 0u) {
    const int hb = 31 - __clz(diff);
    mask = (hb == 31) ? 0u : ~((2u << hb) - 1u);
    prefix = kmin & mask;
    for (int shift = (hb / 8) * 8; shift >= 0; shift -= 8) {
      const DigitResult d = radix_step<true>(it, n, prefix, mask, 0u, shift, m, cntw, need, h_m, h_c, s_res);
      need -= d.above;
      cnt_eq = d.cnt_digit;
      prefix |= (uint32_t)d.digit << shift;
      mask |= 0xffu << shift;
    }
  } else {
    cnt_eq = n_items;  // every item has the same key
  }
  const uint32_t tau_key = prefix;
  const unsigned long long w_tau = item_w(key_score(tau_key), m, cntw);
  unsigned long long kk = (w_tau > 0ull) ? (need + w_tau - 1ull) / w_tau : (unsigned long long)cnt_eq;
  if (kk < 1ull) kk = 1ull;
  if (kk > cnt_eq) kk = cnt_eq;
  int jc = INT_MAX;
  if (kk < cnt_eq) {  // only the first kk tied tokens (by index) are kept
    uint32_t ip = 0u, im = 0u;
    unsigned long long want = kk;
    for (int shift = 16; shift >= 0; shift -= 8) {
      const DigitResult d = radix_step<false>(it, n, ip, im, tau_key, shift, 0.f, cntw, want, h_m, h_c, s_res);
      want -= d.above;
      ip |= (uint32_t)d.digit << shift;
      im |= 0xffu << shift;
    }
    jc = (int)ip;
  }
  tau = key_score(tau_key);
  jcut = jc;
}

// Exact tau / j_cut for n <= blockDim.x list items: item i is kept iff the
// mass of the items ordered before it is below `need`.
__device__ __noinline__ void solve_brute(const uint2* items, int n, float m, bool cntw, unsigned long long need,
                                         uint4* pack, uint32_t* s_min, int* s_jmax, float& tau, int& jcut) {
  // pack[i] = (key, index, mass lo, mass hi): one 16-byte broadcast load per
  // item in the pairwise loop (pack must not overlap items)
  const int tid = threadIdx.x;
  uint2 me = make_uint2(0u, 0u);
  if (tid < n) {
    me = items[tid];
    const unsigned long long w = item_w(key_score(me.x), m, cntw);
    pack[tid] = make_uint4(me.x, me.y, (unsigned)w, (unsigned)(w >> 32));
  }
  if (tid == 0) { *s_min = 0xffffffffu; *s_jmax = -1; }
  __syncthreads();
  bool kept = false;
  if (tid < n) {
    unsigned long long before = 0ull;
#pragma unroll 8
    for (int j = 0; j < n; ++j) {
      const uint4 o = pack[j];
      const unsigned long long ow = ((unsigned long long)o.w << 32) | o.z;
      if (o.x > me.x || (o.x == me.x && o.y < me.y)) before += ow;
    }
    kept = before < need;
    if (kept) atomicMin(s_min, me.x);
  }
  __syncthreads();
  const uint32_t tk = *s_min;
  if (kept && me.x == tk) atomicMax(s_jmax, (int)me.y);
  __syncthreads();
  tau = key_score(tk);
  jcut = *s_jmax;
}

// Rungs m - rung_delta(k) at which the selection sums mass and count in its first
// pass: when the scores at or above one rung hold the target mass and number
// at most kCandSmem, the leader solves over exactly those (no histogram).
constexpr int kRungs = 4;
__host__ __device__ constexpr float rung_delta(int k) { return (float)(1 << k); }  // 1, 2, 4, 8

template <int CS>
struct SelShared {
  unsigned long long pre_m[CS][1 + kRungs];  // per rank: Z, then the mass at or above each rung
  unsigned pre_c[CS][kRungs + 1];            // per rank: count at or above each rung, overflowed warps
  unsigned wcnt[CS * kSelWarps];             // leader: top-rung items per (rank, warp) region
  unsigned long long wpre_m[kSelWarps][1 + kRungs];
  unsigned wpre_c[kSelWarps][kRungs + 1];
  unsigned long long tot_m[1 + kRungs];      // cluster totals
  unsigned tot_c[kRungs + 1];
  unsigned long long slice[CS];   // per-rank slice totals of the histogram
  unsigned long long zpart[CS];   // [0]: mass above the boundary bucket (broadcast)
  int bucket;                     // boundary bucket (broadcast)
  float tau;                      // final threshold (broadcast)
  int jcut;
  unsigned n_cand2;               // leader: items / candidates reserved after the first pass
  float red[kSelWarps];
  unsigned long long scan_a[kSelWarps];
  unsigned scan_c[kSelWarps];
  int cnt[kSelWarps];
};

// Exact tau / j_cut for n <= 32 items by one warp (lane i owns item i): an item
// is kept iff the mass of the items ordered before it is below `need`.
__device__ void solve_warp(const uint2* items, int n, float m, bool cntw, unsigned long long need, float& tau,
                           int& jcut) {
  const int lane = threadIdx.x & 31;
  const uint2 me = lane < n ? items[lane] : make_uint2(0u, 0u);
  const unsigned long long w = lane < n ? item_w(key_score(me.x), m, cntw) : 0ull;
  unsigned long long before = 0ull;
#pragma unroll 4
  for (int j = 0; j < n; ++j) {
    const unsigned ox = __shfl_sync(0xffffffffu, me.x, j);
    const unsigned oy = __shfl_sync(0xffffffffu, me.y, j);
    const unsigned long long ow = __shfl_sync(0xffffffffu, w, j);
    if (ox > me.x || (ox == me.x && oy < me.y)) before += ow;
  }
  const bool kept = lane < n && before < need;
  unsigned tk = kept ? me.x : 0xffffffffu;  // the smallest kept key ...
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tk = min(tk, __shfl_xor_sync(0xffffffffu, tk, o));
  int jm = (kept && me.x == tk) ? (int)me.y : -1;  // ... and its largest kept index
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) jm = max(jm, __shfl_xor_sync(0xffffffffu, jm, o));
  tau = key_score(tk);
  jcut = jm;
}

template <int CS>
struct SelCfg {
  static constexpr size_t kSmem = (size_t)kLgCap * sizeof(float) +
                                  kNumBuckets * (2 * sizeof(unsigned) + sizeof(unsigned long long)) +
                                  kBruteMax * sizeof(unsigned long long) + sizeof(SelShared<CS>);
};
// The histogram's bytes are reused: by the leader for the candidates, then by
// every CTA for its warps' kept-row lists (kLgCap / kSelWarps rows per warp).
static_assert(kNumBuckets * (2 * sizeof(unsigned) + sizeof(unsigned long long)) >= kCandSmem * sizeof(uint2),
              "candidates fit in the histogram's bytes");
static_assert(kNumBuckets * (2 * sizeof(unsigned) + sizeof(unsigned long long)) >= kLgCap * sizeof(int),
              "row lists fit in the histogram's bytes");

// Every kFold scores the 18-bit halves of the histogram are folded into the
// 64-bit bins, so no 32-bit sum can overflow.
constexpr int kFold = 8192;

// Raw vector of one lane's D/32 dims of a cache row.
template <typename T, int D>
struct LaneRaw {
  static constexpr int DL = D / 32;
  static constexpr int VB = DL * sizeof(T);
  using type = typename std::conditional<VB == 16, uint4,
               typename std::conditional<VB == 8, uint2,
               typename std::conditional<VB == 4, unsigned, unsigned short>::type>::type>::type;
};

// ---------------------------------------------------------------------------
// 2. select kernel (cluster per retrieval q head): exact top-p threshold,
// bitmask, and this head's attention over its kept rows outside sinks/window
// ---------------------------------------------------------------------------
template <typename T, int D, int CS>
__global__ void __cluster_dims__(CS, 1, 1) __launch_bounds__(kSelThreads, 2) select_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int kChunk = score_chunk(sizeof(T));
  constexpr int DL = D / 32;
  using Raw = typename LaneRaw<T, D>::type;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int bh = blockIdx.y;
  const int b = bh / a.NR, rq = bh % a.NR;
  const int r = rq / a.G, g = rq % a.G;
  const int h = a.ret_head[r];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(16) unsigned char dsm[];
  float* s_lg = reinterpret_cast<float*>(dsm);                                           // kLgCap
  unsigned* s_hi = reinterpret_cast<unsigned*>(s_lg + kLgCap);                           // 2048
  unsigned* s_lo = s_hi + kNumBuckets;                                                   // 2048
  unsigned long long* s_h = reinterpret_cast<unsigned long long*>(s_lo + kNumBuckets);   // 2048
  uint2* s_cand = reinterpret_cast<uint2*>(s_hi);  // leader, once the histogram is dead
  int* s_rows = reinterpret_cast<int*>(s_hi);      // every CTA, once the selection is done
  unsigned long long* s_w = reinterpret_cast<unsigned long long*>(s_h + kNumBuckets);    // kBruteMax
  SelShared<CS>* sh = reinterpret_cast<SelShared<CS>*>(s_w + kBruteMax);
  __shared__ unsigned long long r_hm[256];
  __shared__ unsigned r_hc[256];
  __shared__ DigitResult s_dres;
  __shared__ uint32_t s_kr[96];
  __shared__ uint32_t s_min;
  __shared__ int s_jmax;
  __shared__ uint2 s_small[32];
  __shared__ __align__(16) T s_spec[kSelWarps][kSpec][2][D];  // early-staged K, V rows per warp
  __shared__ int s_spec_j[kSelWarps][kSpec];
  __shared__ uint2 s_top[kSelWarps][kTopPerWarp];  // this CTA's top-rung items per warp (key, index)
  __shared__ int s_wtop[kSelWarps];
  __shared__ __align__(16) float s_qh[D];
  __shared__ __align__(8) uint64_t s_sbar;     // completion of the bulk copy of this CTA's scores
  __shared__ __align__(16) float s_wo[kSelWarps * D];
  __shared__ float s_wml[kSelWarps * 2];
  // retrieval heads keep the whole context: row pos of head h sits at row0 + pos
  const size_t row0 = a.kv.row(b, h, 0);
  const T* kb = static_cast<const T*>(a.k) + row0 * D;
  const T* vb = static_cast<const T*>(a.v) + row0 * D;

  // This CTA's share of the context comes from the call's maximum length, so
  // the score loads below do not wait for seq_len.
  const int Lh = a.max_seq_len;
  const int per = (((Lh + CS - 1) / CS) + 31) & ~31;
  const int j0 = min(Lh, rank * per);
  const int jh = min(Lh, j0 + per);
  const bool cached = (jh - j0) <= kLgCap;  // uniform over the grid
  const float* lg_g = a.logits + (size_t)bh * a.lstride;
  // Scores are staged in shared memory kLgCap at a time with 16-byte loads
  // issued together (rows are 16-byte aligned, j0 a multiple of 32); when the
  // whole share fits, it is staged once and reused by every pass.
  auto stage = [&](int c0, int c1) {
    const float4* src = reinterpret_cast<const float4*>(lg_g + c0);
    float4* dst = reinterpret_cast<float4*>(s_lg);
    const int nv = (c1 - c0 + 3) >> 2;
#pragma unroll 4
    for (int i = tid; i < nv; i += kSelThreads) dst[i] = __ldcg(src + i);
  };
  // Before waiting for the scores: seq_len and this head's RoPE'd query
  // (scaled by log2(e)/sqrt(D)) from the caller's inputs.  This kernel starts
  // only once every score CTA has passed its wait for rtp_append_kv, so the
  // cache rows it reads are complete.
  const int L = a.seq_len[b];
  if (tid < D / 2 && seq_ok(L, a)) {
    const T* q = static_cast<const T*>(a.q_pre) + ((size_t)b * a.Hq + h * a.G + g) * D;
    const float qx1 = to_f32(q[tid]), qx2 = to_f32(q[tid + D / 2]);
    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    float c, s;
    rope_cos_sin(L - 1, a.inv_freq[tid], c, s);
    s_qh[tid] = (qx1 * c - qx2 * s) * qscale;
    s_qh[tid + D / 2] = (qx2 * c + qx1 * s) * qscale;
  }
  if (rank == 0 && tid == 0) sh->n_cand2 = 0u;
  if (lane < kSpec) s_spec_j[warp][lane] = -1;
  if (tid == 0) mbar_init(&s_sbar, 1);
  griddep_launch();
  cluster_arrive();  // counter zeroed; every CTA of the cluster running
  griddep_wait();    // the score kernel (scores, chunk maxima) has completed
  if (!seq_ok(L, a)) {  // uniform over the cluster; the score kernel flagged it
    cluster_wait();
    return;
  }
  const int nch_h = (Lh + kChunk - 1) / kChunk;
  const float* cm = a.cmax + (size_t)bh * a.nch_score_max;
  const float cm0 = tid < nch_h ? __ldcg(cm + tid) : -CUDART_INF_F;
  // a share that fits is staged once, by one bulk copy (rounded up to whole
  // 16-byte vectors; the score rows are padded to 32 floats)
  const bool bulk = cached && jh > j0;
  if (bulk && tid == 0) {
    const uint32_t bytes = (uint32_t)(((jh - j0) + 3) & ~3) * 4u;
    mbar_expect_tx(&s_sbar, bytes);
    bulk_g2s(s_lg, lg_g + j0, bytes, &s_sbar, l2_evict_first());
  }
  cluster_wait();
  if (bulk && !mbar_wait_bounded(&s_sbar, 0, a.wait_ns, a.status))
    mbar_wait_bounded(&s_sbar, 0, a.wait_ns, a.status);  // the copy, before going on (output invalid)
  const int j1 = min(L, jh);  // j1 <= j0: nothing of this sequence in this CTA's share
  uint32_t* mask = a.mask + (size_t)bh * a.words;
  const bool cntw = a.top_k > 0;  // static top-k: unit weights
  const bool keep_all = !cntw && a.top_p >= 1.0f;
  float tau = -CUDART_INF_F;
  int jcut = INT_MAX;
  bool via_top = false;  // the tail reads only the top-rung items (tier 1, no bitmask)

  if (__builtin_expect(!keep_all, 1)) {  // uniform over the grid
    // maximum score (per-chunk maxima of the score kernel)
    float m;
    {
      const int nch = (L + kChunk - 1) / kChunk;
      float v = tid < nch ? cm0 : -CUDART_INF_F;
      for (int c = tid + kSelThreads; c < nch; c += kSelThreads) v = fmaxf(v, __ldcg(cm + c));
      m = block_max<kSelThreads>(v, sh->red);
    }
    // exp(s - m) 2^36 rounds to 0 below m - 25.65: such scores weigh nothing
    // (top-p); with unit weights every score counts
    const float m_lo = cntw ? -CUDART_INF_F : m - 26.0f;
    SelShared<CS>* lead = cl.map_shared_rank(sh, 0);
    uint2* lead_cand = cl.map_shared_rank(s_cand, 0);

    // ---- pass 1: the exact total mass Z and, for each rung of the ladder
    // m - rung_delta(k), the mass and the count of the scores at or above it ----
    {
      // Z: masses of scores below the lowest rung m - 8 (below 2^25; nearly
      // every score) are summed in 32 bits (at most kLgCap / kSelThreads = 16
      // per thread per chunk, so below 2^29), the rest in 64 bits.
      unsigned long long zs = 0ull, ms[kRungs];
      unsigned zs32 = 0u, cs[kRungs];
#pragma unroll
      for (int k = 0; k < kRungs; ++k) { ms[k] = 0ull; cs[k] = 0u; }
      const float top_lo = m - rung_delta(kRungs - 1);
      unsigned wtop = 0u;  // warp-uniform: this warp's top-rung items so far
      for (int c0 = j0; c0 < j1; c0 += kLgCap) {
        const int c1 = min(j1, c0 + kLgCap);
        if (!cached) {
          __syncthreads();
          stage(c0, c1);
        }
        __syncthreads();
        // this thread's positions c0 + u * kSelThreads + tid, u < kPos: sums,
        // and a bit per position at or above the top rung
        unsigned topbits = 0u;
#pragma unroll 4
        for (int u = 0; u < kPos; ++u) {
          const int j = c0 + u * kSelThreads + tid;
          const float sv = j < c1 ? s_lg[j - c0] : -CUDART_INF_F;
          if (sv > m_lo) {
            const float x = cntw ? 1.0f : mass_x36(sv, m);
            if (sv < top_lo) {  // x < 2^36 e^-8 < 2^25
              zs32 += __float2uint_rn(x);
            } else {
              const unsigned long long w = __float2ull_rn(x);
              zs += w;
#pragma unroll
              for (int k = 0; k < kRungs; ++k)
                if (sv >= m - rung_delta(k)) { ms[k] += w; ++cs[k]; }
              topbits |= 1u << u;
            }
          }
        }
        zs += zs32;
        zs32 = 0u;
        // Scores at or above the top rung go to this warp's region of the
        // leader's item space (kTopPerWarp slots, no atomics); their key and
        // value rows are pulled into L2 meanwhile (the kept rows are among them
        // whenever the leader solves over these items).
        if (__any_sync(0xffffffffu, topbits != 0u)) {
          uint2* region = lead_cand + (rank * kSelWarps + warp) * kTopPerWarp;
          for (int u = 0; u < kPos; ++u) {
            unsigned bal = __ballot_sync(0xffffffffu, (topbits >> u) & 1u);
            while (bal) {  // warp-uniform, one item at a time
              const int src = __ffs(bal) - 1;
              bal &= bal - 1u;
              const int j = c0 + u * kSelThreads + warp * 32 + src;
              if (lane == src && wtop < (unsigned)kTopPerWarp) {
                const uint2 item = make_uint2(score_key(s_lg[j - c0]), (unsigned)j);
                region[wtop] = item;
                s_top[warp][wtop] = item;
              }
              if (wtop < (unsigned)kSpec && cached) {
                // the warp's first rows: keys and values into shared memory
                constexpr int NC = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
                const unsigned dk = (unsigned)__cvta_generic_to_shared(s_spec[warp][wtop][0]);
                const unsigned dv = (unsigned)__cvta_generic_to_shared(s_spec[warp][wtop][1]);
                for (int c = lane; c < 2 * NC; c += 32) {
                  const bool isv = c >= NC;
                  const int cc = isv ? c - NC : c;
                  const char* src_p = reinterpret_cast<const char*>((isv ? vb : kb) + (size_t)j * D) + 16 * cc;
                  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"((isv ? dv : dk) + 16u * cc), "l"(src_p));
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
                if (lane == 0) s_spec_j[warp][wtop] = j;
              } else if (lane == src) {
#pragma unroll
                for (int o = 0; o < D * (int)sizeof(T); o += 128) {
                  prefetch_l2(reinterpret_cast<const char*>(kb + (size_t)j * D) + o);
                  prefetch_l2(reinterpret_cast<const char*>(vb + (size_t)j * D) + o);
                }
              }
              ++wtop;
            }
          }
        }
      }
      // this rank's sums -> every rank of the cluster (the rung sums are zero
      // in most warps: reduce them only where some lane has one)
      zs = warp_sum_u64(zs);
      const bool any_top = __any_sync(0xffffffffu, cs[kRungs - 1] != 0u);
      if (any_top) {
#pragma unroll
        for (int k = 0; k < kRungs; ++k) { ms[k] = warp_sum_u64(ms[k]); cs[k] = warp_sum_u32(cs[k]); }
      }
      if (lane == 0) {
        sh->wpre_m[warp][0] = zs;
#pragma unroll
        for (int k = 0; k < kRungs; ++k) { sh->wpre_m[warp][1 + k] = ms[k]; sh->wpre_c[warp][k] = cs[k]; }
        sh->wpre_c[warp][kRungs] = wtop > (unsigned)kTopPerWarp ? 1u : 0u;
        s_wtop[warp] = (int)min(wtop, (unsigned)kTopPerWarp);
        lead->wcnt[rank * kSelWarps + warp] = wtop;
      }
      __syncthreads();
      if (tid < 1 + kRungs) {
        unsigned long long t = 0ull;
#pragma unroll
        for (int w = 0; w < kSelWarps; ++w) t += sh->wpre_m[w][tid];
#pragma unroll
        for (int q = 0; q < CS; ++q) cl.map_shared_rank(sh, q)->pre_m[rank][tid] = t;
      } else if (tid >= 32 && tid < 32 + kRungs + 1) {
        unsigned t = 0u;
#pragma unroll
        for (int w = 0; w < kSelWarps; ++w) t += sh->wpre_c[w][tid - 32];
#pragma unroll
        for (int q = 0; q < CS; ++q) cl.map_shared_rank(sh, q)->pre_c[rank][tid - 32] = t;
      }
    }
    cl.sync();  // (A) every rank's sums everywhere

    if (tid < 1 + kRungs) {
      unsigned long long t = 0ull;
#pragma unroll
      for (int q = 0; q < CS; ++q) t += sh->pre_m[q][tid];
      sh->tot_m[tid] = t;
    } else if (tid >= 32 && tid < 32 + kRungs + 1) {
      unsigned t = 0u;
#pragma unroll
      for (int q = 0; q < CS; ++q) t += sh->pre_c[q][tid - 32];
      sh->tot_c[tid - 32] = t;
    }
    __syncthreads();
    const unsigned long long Z = sh->tot_m[0];
    unsigned long long Mk[kRungs];
    unsigned Ck[kRungs];
#pragma unroll
    for (int k = 0; k < kRungs; ++k) { Mk[k] = sh->tot_m[1 + k]; Ck[k] = sh->tot_c[k]; }
    unsigned long long target = cntw ? (unsigned long long)a.top_k
                                     : (unsigned long long)ceil((double)a.top_p * (double)Z);
    if (target > Z) target = Z;
    if (target < 1ull) target = 1ull;
    // lowest rung whose scores already hold the target mass: the kept set lies
    // at or above it (every other score is ordered after all of those)
    int kf = -1;
#pragma unroll
    for (int k = kRungs - 1; k >= 0; --k)
      if (Mk[k] >= target) kf = k;
    // tier 1: the first pass already put every score at or above the top rung
    // with the leader, and they hold the target; tier 2: a lower rung's
    // scores hold it and fit (one more pass collects them); else the histogram
    const bool tier1 = Mk[kRungs - 1] >= target && sh->tot_c[kRungs] == 0u;  // no region overflowed
    const bool tier2 = !tier1 && kf >= 0 && Ck[kf] <= (unsigned)kCandSmem;
    // tau is one of the top-rung scores under tier 1, so every kept token is a
    // top-rung item: without a bitmask to write, the tail tests only those
    via_top = tier1 && !a.want_mask;
    float t_lo = m_lo;
#pragma unroll
    for (int k = 0; k < kRungs; ++k)
      if (k == kf) t_lo = m - rung_delta(k);

    uint2* gcand = a.cand + (size_t)bh * a.lstride;
    if (__builtin_expect(tier1 || tier2, 1)) {
      if (__builtin_expect(tier2, 0)) {  // every score at or above rung kf -> the leader
        for (int c0 = j0; c0 < j1; c0 += kLgCap) {
          const int c1 = min(j1, c0 + kLgCap);
          if (!cached) {
            __syncthreads();
            stage(c0, c1);
            __syncthreads();
          }
          unsigned inbits = 0u;
#pragma unroll
          for (int u = 0; u < kPos; ++u) {
            const int j = c0 + u * kSelThreads + tid;
            if (j < c1 && s_lg[j - c0] >= t_lo) inbits |= 1u << u;
          }
          if (__any_sync(0xffffffffu, inbits != 0u)) {
            for (int u = 0; u < kPos; ++u) {
              const bool in = (inbits >> u) & 1u;
              const unsigned bal = __ballot_sync(0xffffffffu, in);
              if (!bal) continue;
              unsigned base = 0u;
              if (lane == 0) base = atomicAdd(&lead->n_cand2, (unsigned)__popc(bal));
              base = __shfl_sync(0xffffffffu, base, 0);
              if (in) {
                const int j = c0 + u * kSelThreads + tid;
                lead_cand[base + __popc(bal & ((1u << lane) - 1u))] = make_uint2(score_key(s_lg[j - c0]), (unsigned)j);
              }
            }
          }
        }
        cl.sync();  // (B) the leader holds every item
      }
      if (rank == 0) {
        int n = (int)Ck[kf];
        bool done = false;
        float t_tau = 0.f;
        int t_jcut = 0;
        if (__builtin_expect(tier1 && Ck[kRungs - 1] <= 32u, 1)) {
          // few items: warp 0 gathers the regions' items at or above rung kf and solves
          // (items below rung kf cannot be kept: the mass before them already
          // reaches the target, so the solve needs no filtering)
          if (warp == 0) {
            constexpr int RPL = kMaxCS * kSelWarps / 32;  // regions per lane
            const int nreg = CS * kSelWarps;
            unsigned cr[RPL], c = 0u;
#pragma unroll
            for (int k = 0; k < RPL; ++k) {
              const int rg = lane * RPL + k;
              cr[k] = rg < nreg ? sh->wcnt[rg] : 0u;
              c += cr[k];
            }
            unsigned off = c;  // exclusive warp prefix of the lanes' counts
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const unsigned v = __shfl_up_sync(0xffffffffu, off, o);
              if (lane >= o) off += v;
            }
            off -= c;
            n = (int)__shfl_sync(0xffffffffu, off + c, 31);
#pragma unroll
            for (int k = 0; k < RPL; ++k)
              for (unsigned i = 0; i < cr[k]; ++i) s_small[off++] = s_cand[(lane * RPL + k) * kTopPerWarp + i];
            __syncwarp();
            solve_warp(s_small, n, m, cntw, target, t_tau, t_jcut);
          }
          done = true;
        } else if (tier1) {
          // gather the regions' items (only those at or above rung kf can be
          // kept) into one list; read everything before writing
          constexpr int kRegions = kMaxCS * kSelWarps;
          constexpr int kRPT = (kRegions + kSelThreads - 1) / kSelThreads;
          static_assert(kRegions * kTopPerWarp <= kCandSmem, "regions fit in the item space");
          const uint32_t klo = score_key(t_lo);
          uint2 it[kRPT][kTopPerWarp];
          unsigned c = 0u;
#pragma unroll
          for (int rr = 0; rr < kRPT; ++rr) {
            const int rg = tid + rr * kSelThreads;
            const int cnt_r = rg < CS * kSelWarps ? (int)sh->wcnt[rg] : 0;
#pragma unroll
            for (int i = 0; i < kTopPerWarp; ++i) {
              it[rr][i] = make_uint2(0u, 0u);
              if (i < cnt_r) {
                it[rr][i] = s_cand[rg * kTopPerWarp + i];
                if (it[rr][i].x >= klo) ++c;
              }
            }
          }
          unsigned long long ex_m, tot_m;
          unsigned off, tot;
          block_excl_scan2<kSelThreads>(0ull, c, ex_m, off, tot_m, tot, sh->scan_a, sh->scan_c);
#pragma unroll
          for (int rr = 0; rr < kRPT; ++rr)
#pragma unroll
            for (int i = 0; i < kTopPerWarp; ++i)
              if (it[rr][i].x >= klo && it[rr][i].x != 0u) s_cand[off++] = it[rr][i];
          __syncthreads();
          n = (int)tot;
        }
        if (done) {
        } else if (n <= 32) {
          if (warp == 0) solve_warp(s_cand, n, m, cntw, target, t_tau, t_jcut);
        } else if (n <= kBruteMax) {
          solve_brute(s_cand, n, m, cntw, target, reinterpret_cast<uint4*>(s_cand + kCandSmem / 2), &s_min, &s_jmax, t_tau, t_jcut);
        } else {
          solve_radix(Items{s_cand, false}, n, m, cntw, target, r_hm, r_hc, &s_dres, s_kr, t_tau, t_jcut);
        }
        if (warp == 0 && lane < CS) {
          SelShared<CS>* rem = cl.map_shared_rank(sh, lane);
          rem->tau = t_tau;
          rem->jcut = t_jcut;
        }
      }
      cl.sync();  // (C) final threshold everywhere (no DSMEM access after this)
    } else {
      // ---- 2048-bucket histogram of the scores at or above the rung ----
      for (int i = tid; i < kNumBuckets; i += kSelThreads) { s_hi[i] = 0u; s_lo[i] = 0u; s_h[i] = 0ull; }
      for (int c0 = j0; c0 < j1; c0 += kLgCap) {
        const int c1 = min(j1, c0 + kLgCap);
        if (!cached) {
          __syncthreads();
          stage(c0, c1);
        }
        __syncthreads();
        for (int f0 = c0; f0 < c1; f0 += kFold) {
          const int f1 = min(c1, f0 + kFold);
          for (int j = f0 + tid; j < f1; j += 4 * kSelThreads) {  // 4 independent scores per step
            float sv[4];
            bool on[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int jj = j + u * kSelThreads;
              on[u] = jj < f1;
              sv[u] = on[u] ? s_lg[jj - c0] : -CUDART_INF_F;
              on[u] = on[u] && sv[u] > m_lo && sv[u] >= t_lo;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (!on[u]) continue;
              unsigned hi, lo;
              if (cntw) {
                hi = 0u;
                lo = 1u;
              } else {
                mass_split36(sv[u], m, hi, lo);
              }
              const int bk = score_bucket(sv[u]);
              if (hi) atomicAdd(&s_hi[bk], hi);
              if (lo) atomicAdd(&s_lo[bk], lo);
            }
          }
          __syncthreads();
          for (int i = tid; i < kNumBuckets; i += kSelThreads) {  // fold into the 64-bit bins
            s_h[i] += ((unsigned long long)s_hi[i] << 18) + s_lo[i];
            s_hi[i] = 0u;
            s_lo[i] = 0u;
          }
          __syncthreads();
        }
      }
      cl.sync();  // (1) every rank's histogram is complete

      // reduce this rank's slice of buckets over the cluster; broadcast its total
      constexpr int NS = kNumBuckets / CS;
      {
        unsigned long long sm_ = 0ull;
        if (tid < NS) {
          const int bk = rank * NS + tid;
#pragma unroll
          for (int q = 0; q < CS; ++q) sm_ += *cl.map_shared_rank(s_h + bk, q);
          r_hm[tid] = sm_;
        }
        unsigned long long ex_m, tot_m;
        unsigned ex_c, tot_c;
        block_excl_scan2<kSelThreads>(sm_, 0u, ex_m, ex_c, tot_m, tot_c, sh->scan_a, sh->scan_c);
        if (tid < CS) cl.map_shared_rank(sh, tid)->slice[rank] = tot_m;
      }
      cl.sync();  // (2) slice totals everywhere

      {  // boundary bucket: the histogram holds every score at or above the
         // rung, whose mass reaches the target; highest buckets live in the
         // highest rank's slice
        int kslice = 0;
        unsigned long long above_slice = 0ull;
        for (int q = CS - 1; q >= 0; --q) {
          if (above_slice + sh->slice[q] >= target) { kslice = q; break; }
          above_slice += sh->slice[q];
        }
        if (rank == kslice && warp == 0) {
          constexpr int PL = NS / 32;
          unsigned long long w8[PL];
          unsigned long long sw = 0ull;
#pragma unroll
          for (int k = 0; k < PL; ++k) {
            w8[k] = r_hm[NS - 1 - (lane * PL + k)];
            sw += w8[k];
          }
          const unsigned long long incl = warp_incl_scan_u64(sw);
          unsigned long long cum = above_slice + incl - sw;
          int found = -1;
          unsigned long long fab = 0ull;
#pragma unroll
          for (int k = 0; k < PL; ++k) {
            if (found < 0 && cum < target && cum + w8[k] >= target) {
              found = rank * NS + NS - 1 - (lane * PL + k);
              fab = cum;
            }
            cum += w8[k];
          }
          const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
          const int src = who ? __ffs(who) - 1 : 0;
          found = who ? __shfl_sync(0xffffffffu, found, src) : -1;
          fab = __shfl_sync(0xffffffffu, fab, src);
          if (lane < CS) {
            SelShared<CS>* rem = cl.map_shared_rank(sh, lane);
            rem->bucket = found;
            rem->zpart[0] = fab;  // mass above the boundary bucket
          }
        }
      }
      cl.sync();  // (3) boundary bucket everywhere; every histogram is dead

      // Candidates of the boundary bucket go straight into the leader's shared
      // memory (order does not matter); past kCandSmem into global scratch.
      // Scores of that bucket below the rung may join: they are ordered after
      // the ones above it, whose mass already covers what is needed.
      const int bucket = sh->bucket;
      const unsigned long long above = sh->zpart[0];
      bool wrote_global = false;
      if (bucket >= 0) {
        for (int c0 = j0; c0 < j1; c0 += kLgCap) {
          const int c1 = min(j1, c0 + kLgCap);
          if (!cached) {
            __syncthreads();
            stage(c0, c1);
            __syncthreads();
          }
          for (int jb = c0; jb < c1; jb += 4 * kSelThreads) {
            float sv[4];
            bool in[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = jb + u * kSelThreads + tid;
              in[u] = false;
              sv[u] = 0.f;
              if (j < c1) {
                sv[u] = s_lg[j - c0];
                in[u] = sv[u] > m_lo && score_bucket(sv[u]) == bucket && (cntw || mass36(sv[u], m) != 0ull);
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const unsigned bal = __ballot_sync(0xffffffffu, in[u]);
              if (bal) {
                unsigned base = 0u;
                if (lane == 0) base = atomicAdd(&lead->n_cand2, (unsigned)__popc(bal));
                base = __shfl_sync(0xffffffffu, base, 0);
                const unsigned slot = base + __popc(bal & ((1u << lane) - 1u));
                if (in[u]) {
                  const uint2 item = make_uint2(score_key(sv[u]), (unsigned)(jb + u * kSelThreads + tid));
                  if (slot < (unsigned)kCandSmem) {
                    lead_cand[slot] = item;
                  } else {
                    gcand[slot] = item;
                    wrote_global = true;
                  }
                }
              }
            }
          }
        }
      }
      if (wrote_global) __threadfence();
      cl.sync();  // (4) candidates complete

      if (rank == 0) {
        float t_tau = -CUDART_INF_F;  // no boundary (unreachable): keep every token
        int t_jcut = INT_MAX;
        if (bucket >= 0) {
          const int n = (int)sh->n_cand2;
          const unsigned long long need = target - above;
          Items items{s_cand, false};
          if (n > kCandSmem) {  // the list continues in global scratch: put its head there too
            for (int i = tid; i < kCandSmem; i += kSelThreads) gcand[i] = s_cand[i];
            __threadfence();
            __syncthreads();
            items = Items{gcand, true};
          }
          if (n <= kBruteMax)
            solve_brute(s_cand, n, m, cntw, need, reinterpret_cast<uint4*>(s_cand + kCandSmem / 2), &s_min, &s_jmax, t_tau, t_jcut);
          else
            solve_radix(items, n, m, cntw, need, r_hm, r_hc, &s_dres, s_kr, t_tau, t_jcut);
        }
        if (tid < CS) {
          SelShared<CS>* rem = cl.map_shared_rank(sh, tid);
          rem->tau = t_tau;
          rem->jcut = t_jcut;
        }
      }
      cl.sync();  // (5) final threshold everywhere (no DSMEM access after this)
    }
    tau = sh->tau;
    jcut = sh->jcut;
  }

  // ---- bitmask, then this head's attention over its kept rows outside
  // sinks/window: each warp lists the rows of its own positions and attends
  // them kGroup at a time (keys and values of a group in one round trip) ----
  const int s_cnt = min(a.S, L);
  const int sw0 = max(s_cnt, L - a.W);
  int* wrows = s_rows + warp * (kLgCap / kSelWarps);
  const uint64_t pol = l2_evict_first();
  __syncthreads();  // s_qh visible
  float qv[DL];
#pragma unroll
  for (int d = 0; d < DL; ++d) qv[d] = s_qh[lane * DL + d];
  float am = -CUDART_INF_F, al = 0.f, ao[DL];
#pragma unroll
  for (int d = 0; d < DL; ++d) ao[d] = 0.f;
  // this warp attends its rows wrows[0, wn) (wn warp-uniform) for query head g
  auto attend_rows = [&](int wn) {
    asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's early copies
    __syncwarp();
    const int sj0 = s_spec_j[warp][0], sj1 = s_spec_j[warp][1];
    for (int i0 = 0; i0 < wn; i0 += kGroup) {  // wn is warp-uniform
      int rw[kGroup];
      Raw kr[kGroup], vr[kGroup];
#pragma unroll
      for (int k = 0; k < kGroup; ++k) {
        kr[k] = Raw();
        vr[k] = Raw();
        rw[k] = (i0 + k < wn) ? wrows[i0 + k] : -1;
        if (rw[k] >= 0) {
          const int sp = rw[k] == sj0 ? 0 : (rw[k] == sj1 ? 1 : -1);
          if (sp >= 0) {
            kr[k] = *reinterpret_cast<const Raw*>(&s_spec[warp][sp][0][lane * DL]);
            vr[k] = *reinterpret_cast<const Raw*>(&s_spec[warp][sp][1][lane * DL]);
          } else {
            kr[k] = ld_stream(reinterpret_cast<const Raw*>(kb + (size_t)rw[k] * D + lane * DL), pol);
            vr[k] = ld_stream(reinterpret_cast<const Raw*>(vb + (size_t)rw[k] * D + lane * DL), pol);
          }
        }
      }
      float sc[kGroup];
#pragma unroll
      for (int k = 0; k < kGroup; ++k) {
        const T* kt = reinterpret_cast<const T*>(&kr[k]);
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < DL; ++d) s = fmaf(qv[d], to_f32(kt[d]), s);
        sc[k] = s;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < kGroup; ++k) sc[k] += __shfl_xor_sync(0xffffffffu, sc[k], o);
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int k = 0; k < kGroup; ++k)
        if (rw[k] >= 0) mx = fmaxf(mx, sc[k]);
      const float mn = fmaxf(am, mx);
      const float alpha = exp2f(am - mn);  // 0 while nothing was attended (am = -inf)
      al *= alpha;
#pragma unroll
      for (int d = 0; d < DL; ++d) ao[d] *= alpha;
#pragma unroll
      for (int k = 0; k < kGroup; ++k) {
        if (rw[k] < 0) continue;
        const float e = exp2f(sc[k] - mn);
        const T* vt = reinterpret_cast<const T*>(&vr[k]);
        al += e;
#pragma unroll
        for (int d = 0; d < DL; ++d) ao[d] = fmaf(e, to_f32(vt[d]), ao[d]);
      }
      am = mn;
    }
  };
  int cnt = 0;
  if (via_top) {
    // this warp's top-rung items (one per lane at most) are its only candidates
    const int nt = s_wtop[warp];
    bool in = false, o = false;
    int jj = 0;
    if (lane < nt) {
      const uint2 e = s_top[warp][lane];
      const float sv = key_score(e.x);
      jj = (int)e.y;
      in = sv > tau || (sv == tau && jj <= jcut);
      o = in && jj >= s_cnt && jj < sw0;
    }
    cnt = in ? 1 : 0;
    const unsigned ob = __ballot_sync(0xffffffffu, o);
    if (o) wrows[__popc(ob & ((1u << lane) - 1u))] = jj;
    __syncwarp();
    attend_rows(__popc(ob));
  } else {
    for (int c0 = j0; c0 < j1; c0 += kLgCap) {
      const int c1 = min(j1, c0 + kLgCap);
      if (!cached) {
        __syncthreads();
        stage(c0, c1);
      }
      __syncthreads();  // staged scores visible; the row lists' bytes are free
      unsigned inbits = 0u, outbits = 0u;
#pragma unroll 4
      for (int u = 0; u < kPos; ++u) {
        const int j = c0 + u * kSelThreads + tid;
        if (j < c1) {
          const float sv = s_lg[j - c0];
          if (keep_all || sv > tau || (sv == tau && j <= jcut)) {
            inbits |= 1u << u;
            if (j >= s_cnt && j < sw0) outbits |= 1u << u;
          }
        }
      }
      cnt += __popc(inbits);
      int wn = 0;
#pragma unroll 2
      for (int u = 0; u < kPos; ++u) {
        const unsigned word = __ballot_sync(0xffffffffu, (inbits >> u) & 1u);
        const int jw = c0 + u * kSelThreads + warp * 32;
        if (lane == 0 && jw < c1) mask[jw >> 5] = word;
        const unsigned ob = __ballot_sync(0xffffffffu, (outbits >> u) & 1u);
        if ((outbits >> u) & 1u) wrows[wn + __popc(ob & ((1u << lane) - 1u))] = jw + lane;
        wn += __popc(ob);
      }
      attend_rows(wn);
    }
  }
  // merge the warps' states into this CTA's partial for query head g
  cnt = warp_sum_i(cnt);
#pragma unroll
  for (int d = 0; d < DL; ++d) s_wo[warp * D + lane * DL + d] = ao[d];
  if (lane == 0) {
    s_wml[warp * 2] = am;
    s_wml[warp * 2 + 1] = al;
    sh->cnt[warp] = cnt;
  }
  __syncthreads();
  float* sp_me = a.sel_scratch + ((size_t)bh * kMaxCS + rank) * (D + 3);
  for (int d = tid; d < D; d += kSelThreads) {
    float mn = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) mn = fmaxf(mn, s_wml[w * 2]);
    float acc = 0.f, den = 0.f;
    if (mn != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < kSelWarps; ++w) {
        const float mw = s_wml[w * 2];
        if (mw == -CUDART_INF_F) continue;
        const float sc = exp2f(mw - mn);
        acc = fmaf(s_wo[w * D + d], sc, acc);
        den = fmaf(s_wml[w * 2 + 1], sc, den);
      }
    }
    sp_me[d] = acc;
    if (d == 0) {
      sp_me[D] = mn;
      sp_me[D + 1] = den;
    }
  }
  if (tid == 0) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) c += sh->cnt[w];
    sp_me[D + 2] = __int_as_float(c);
  }
  // The sink/window kernel, launched after this one, merges every rank's
  // partial with the head's sink/window partial once this grid has completed.
  // No rank touches another's shared memory after the last cluster barrier,
  // so the ranks leave independently.
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------
// Time a bounded wait allows before it gives up (ns).
constexpr unsigned long long kWaitNs = 400ull * 1000 * 1000;

// Test hook (rtp_debug_wait_expiry): per host thread, armed for the next call.
thread_local int t_expiry_polls = 0;

cudaError_t launch_cluster_pdl(void (*k)(DecodeArgs), dim3 grid, dim3 block, size_t smem, int cluster,
                               cudaStream_t st, const DecodeArgs& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k, a);
}

// The two stream kernels: score CTAs (plain grid; part 0), and sink/window
// clusters of kSwCluster CTAs (part 1).  Set up once per device under a mutex.
template <typename T, int D, int G, int IDX>
cudaError_t launch_score(const DecodeArgs& a, int n_sms, cudaStream_t st) {
  return launch_pdl(score_kernel<T, D, G, IDX>, dim3(std::min(a.n_score_ctas, score_ctas_per_sm(IDX) * n_sms)),
                    dim3(kThreads), score_smem(IDX), st, a);
}

template <typename T, int D, int G>
cudaError_t launch_stream(DecodeArgs& a, int n_bkv, int idx, int part, cudaStream_t st) {
  static std::mutex s_mu;
  static std::atomic<int> s_cs[64];  // chosen cluster size; 0 = not set up yet
  static std::atomic<int> s_sms[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) dev = 63;
  int cs = s_cs[dev].load(std::memory_order_acquire);
  if (cs == 0) {
    std::lock_guard<std::mutex> lock(s_mu);
    cs = s_cs[dev].load(std::memory_order_relaxed);
    if (cs == 0) {
      cudaFuncSetAttribute(score_kernel<T, D, G, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, score_smem(4));
      cudaFuncSetAttribute(score_kernel<T, D, G, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, score_smem(8));
      cudaFuncSetAttribute(score_kernel<T, D, G, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, score_smem(16));
      cudaFuncSetAttribute(score_kernel<T, D, G, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, score_smem(32));
      cudaFuncSetAttribute(sw_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem);
      // every decode kernel asks for the largest shared-memory carveout, so
      // their CTAs can share an SM
      cudaFuncSetAttribute(sw_kernel<T, D, G>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
      cudaFuncSetAttribute(score_kernel<T, D, G, 4>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
      cudaFuncSetAttribute(score_kernel<T, D, G, 8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
      cudaFuncSetAttribute(score_kernel<T, D, G, 16>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
      cudaFuncSetAttribute(score_kernel<T, D, G, 32>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
      cudaGetLastError();
      s_sms[dev].store(sms, std::memory_order_relaxed);
      cs = kSwCluster;
      s_cs[dev].store(cs, std::memory_order_release);
    }
  }
  const int n_sms = s_sms[dev].load(std::memory_order_relaxed);
  if (part == 0) {
    trace_begin(RTP_STAGE_DECODE_SCORE, st);
    switch (idx) {
      case 4: e = launch_score<T, D, G, 4>(a, n_sms, st); break;
      case 8: e = launch_score<T, D, G, 8>(a, n_sms, st); break;
      case 32: e = launch_score<T, D, G, 32>(a, n_sms, st); break;
      default: e = launch_score<T, D, G, 16>(a, n_sms, st); break;
    }
    trace_end(RTP_STAGE_DECODE_SCORE, st);
    return e;
  }
  trace_begin(RTP_STAGE_DECODE_LOCAL, st);
  e = launch_cluster_pdl(sw_kernel<T, D, G>, dim3(n_bkv * cs), dim3(kThreads), kStreamSmem, cs, st, a);
  trace_end(RTP_STAGE_DECODE_LOCAL, st);
  return e;
}

template <typename T, int D>
cudaError_t launch_stream_d(DecodeArgs& a, int n_bkv, int idx, int part, cudaStream_t st) {
  switch (a.G) {
    case 1: return launch_stream<T, D, 1>(a, n_bkv, idx, part, st);
    case 2: return launch_stream<T, D, 2>(a, n_bkv, idx, part, st);
    case 4: return launch_stream<T, D, 4>(a, n_bkv, idx, part, st);
    default: return launch_stream<T, D, 8>(a, n_bkv, idx, part, st);
  }
}

// part 0: the score kernel; part 1: the sink/window clusters
cudaError_t launch_stream_any(const Shape& sh, DecodeArgs& a, int part, cudaStream_t st) {
  const int n_bkv = sh.B * sh.Hkv;
  if (sh.dtype == RTP_BF16)
    return sh.D == 128 ? launch_stream_d<__nv_bfloat16, 128>(a, n_bkv, sh.idx, part, st)
                       : launch_stream_d<__nv_bfloat16, 64>(a, n_bkv, sh.idx, part, st);
  return sh.D == 128 ? launch_stream_d<float, 128>(a, n_bkv, sh.idx, part, st)
                     : launch_stream_d<float, 64>(a, n_bkv, sh.idx, part, st);
}

// Select kernel with 16-CTA clusters when the device can keep all of this
// call's clusters resident at once, else 8-CTA clusters (which always fit in
// fewer SMs per GPC): one wave of clusters keeps the kernel as short as one
// cluster's work.
// The per-device attribute set-up and occupancy query run once per device
// under a mutex (calls may come from several host threads); the result is
// published through an atomic, so later calls read it without the lock.
template <typename T, int D>
cudaError_t launch_select(DecodeArgs& a, int n_clusters, cudaStream_t st) {
  static std::mutex s_mu;
  static std::atomic<int> s_max16[64];  // -1 - (clusters resident): 0 = not queried yet
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) dev = 63;  // out-of-range ordinals share the last slot
  int cached = s_max16[dev].load(std::memory_order_acquire);
  if (cached == 0) {
    std::lock_guard<std::mutex> lock(s_mu);
    cached = s_max16[dev].load(std::memory_order_relaxed);
    if (cached == 0) {
      cudaFuncSetAttribute(select_kernel<T, D, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SelCfg<8>::kSmem);
      cudaFuncSetAttribute(select_kernel<T, D, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SelCfg<16>::kSmem);
      cudaFuncSetAttribute(select_kernel<T, D, 16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      cudaFuncSetAttribute(select_kernel<T, D, 8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
      cudaFuncSetAttribute(select_kernel<T, D, 16>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1);
      cfg.blockDim = dim3(kSelThreads);
      cfg.dynamicSmemBytes = SelCfg<16>::kSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, select_kernel<T, D, 16>, &cfg) != cudaSuccess) n = 0;
      cudaGetLastError();  // clear a refused query
      cached = -1 - n;
      s_max16[dev].store(cached, std::memory_order_release);
    }
  }
  const int max16 = cached < 0 ? -1 - cached : 0;
  const int cs = (max16 >= n_clusters) ? 16 : 8;
  a.sel_cs = cs;
  if (cs == 16)
    return launch_pdl(select_kernel<T, D, 16>, dim3(16, n_clusters), dim3(kSelThreads), SelCfg<16>::kSmem, st, a);
  return launch_pdl(select_kernel<T, D, 8>, dim3(8, n_clusters), dim3(kSelThreads), SelCfg<8>::kSmem, st, a);
}

cudaError_t launch_select_any(const Shape& sh, DecodeArgs& a, int n_clusters, cudaStream_t st) {
  if (sh.dtype == RTP_BF16)
    return sh.D == 128 ? launch_select<__nv_bfloat16, 128>(a, n_clusters, st)
                       : launch_select<__nv_bfloat16, 64>(a, n_clusters, st);
  return sh.D == 128 ? launch_select<float, 128>(a, n_clusters, st) : launch_select<float, 64>(a, n_clusters, st);
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

void arm_wait_expiry(int polls) { t_expiry_polls = polls; }

DecodeLayout decode_layout(const Shape& sh) {
  DecodeLayout l;
  const size_t NRt = (size_t)sh.B * sh.NR;
  const int chunk = score_chunk(sh.esize);
  l.nch_score_max = (sh.Lmax + chunk - 1) / chunk;
  const size_t words = (size_t)(sh.Lmax + 31) / 32;
  const size_t lstride = ((size_t)sh.Lmax + 31) & ~size_t(31);
  size_t off = 0;
  l.logits = off;     off = align256(off + NRt * lstride * sizeof(float));
  l.cmax = off;       off = align256(off + NRt * l.nch_score_max * sizeof(float));
  l.mask = off;       off = align256(off + NRt * words * sizeof(uint32_t));  // bitmask when the caller passes none
  l.cand = off;       off = align256(off + NRt * lstride * sizeof(uint2));
  l.sw_scratch = off; off = align256(off + (size_t)sh.B * sh.Hkv * kSwCluster * sh.G * (sh.D + 2) * sizeof(float));
  l.sel_scratch = off; off = align256(off + NRt * kMaxCS * (sh.D + 3) * sizeof(float));
  l.total = off;
  return l;
}

int launch_decode(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* seq_len,
                  int max_seq_len, const float* w_q, void* out, uint32_t* sel_bitmask,
                  int* sel_count, void* ws, const DecodeLayout& lay, cudaStream_t st) {
  DecodeArgs a;
  a.B = sh.B; a.Hq = sh.Hq; a.Hkv = sh.Hkv; a.G = sh.G; a.D = sh.D; a.R = sh.R; a.NR = sh.NR;
  a.Lmax = sh.Lmax; a.S = sh.S; a.W = sh.W; a.Lk = sh.Lk;
  a.max_seq_len = max_seq_len > 0 ? max_seq_len : sh.Lmax;
  a.words = (sh.Lmax + 31) / 32;
  a.lstride = (sh.Lmax + 31) & ~31;
  a.top_p = sh.top_p; a.rope_base = sh.rope_base; a.top_k = sh.top_k;
  a.q_pre = q_pre; a.w_q = w_q; a.out = out;
  a.k = cache->k; a.v = cache->v; a.kidx = cache->kidx; a.status = cache->status;
  a.seq_len = seq_len; a.sel_count = sel_count;
  char* w = static_cast<char*>(ws);
  a.logits = reinterpret_cast<float*>(w + lay.logits);
  a.cmax = reinterpret_cast<float*>(w + lay.cmax);
  a.mask = sel_bitmask ? sel_bitmask : reinterpret_cast<uint32_t*>(w + lay.mask);
  a.want_mask = sel_bitmask != nullptr;
  a.cand = reinterpret_cast<uint2*>(w + lay.cand);
  a.sw_scratch = reinterpret_cast<float*>(w + lay.sw_scratch);
  a.sel_scratch = reinterpret_cast<float*>(w + lay.sel_scratch);
  a.nch_score_max = lay.nch_score_max;
  a.sel_cs = 0;
  a.tx_extra = 0u;
  a.wait_ns = kWaitNs;
  if (t_expiry_polls > 0) {  // test hook: copy barriers that expect bytes that never come
    a.tx_extra = 16u;
    a.wait_ns = 100ull * (unsigned long long)t_expiry_polls;
    t_expiry_polls = 0;
  }
  a.kv = sh.kv;
  for (int i = 0; i < kMaxRetrieval; ++i) { a.ret_head[i] = sh.ret_head[i]; a.ret_rank[i] = sh.ret_rank[i]; }
  for (int i = 0; i < 64; ++i) a.inv_freq[i] = sh.inv_freq[i];

  const int Lh = a.max_seq_len;
  const int chunk = score_chunk(sh.esize);
  a.n_score_ctas = sh.R > 0 ? sh.B * sh.R * ((Lh + chunk - 1) / chunk) : 0;

  // score -> select -> sink/window: the select clusters start as soon as the
  // scores are complete, the sink/window clusters stream beside them and merge
  // the select's partials at their end
  cudaError_t e = cudaSuccess;
  if (a.n_score_ctas > 0) e = launch_stream_any(sh, a, 0, st);
  if (e == cudaSuccess && sh.R > 0) {
    trace_begin(RTP_STAGE_DECODE_SELECT, st);
    e = launch_select_any(sh, a, sh.B * sh.NR, st);
    trace_end(RTP_STAGE_DECODE_SELECT, st);
  }
  if (e == cudaSuccess) e = launch_stream_any(sh, a, 1, st);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("decode launch: ") + cudaGetErrorString(e));
    return RTP_ERR_CUDA;
  }
  return RTP_OK;
}

}  // namespace rtp
