// Prefill attention on the fifth-generation tensor cores (tcgen05 + TMEM).
//
// One CTA per (sequence, query head, 128-row query tile).  Per key tile of 128
// keys: S = Q K^T (128 x 128, fp32 in TMEM), a softmax over S by the thread
// that owns the row (one TMEM lane per thread), then O += P V (128 x D, fp32
// in TMEM).  The layer's masks (causality; sinks and window; for retrieval
// heads the row's top-p bitmask from the selection kernel) are applied to S
// (atlas.scime.ai summary, "Approach"; abstract, observations (2)-(3)).
//
// Roles (256 threads):
//   warp 0, lane 0   stages K and V tiles with TMA (cp.async.bulk.tensor,
//                    128-byte swizzle, boxes of 64 dims x 128 keys), two
//                    stages in flight;
//   warp 1           allocates TMEM; lane 0 issues every tcgen05.mma and
//                    commits its completions to mbarriers;
//   warps 4-7        one thread per query row: read S from TMEM, mask, keep
//                    the running maximum and sum, write P (bf16) to shared
//                    memory, rescale O in TMEM when the maximum grows by more
//                    than 2^8, and finally read O and write the output.
// S has two TMEM buffers, so S of tile j + 1 is computed while tile j's
// softmax runs.  Every wait on an mbarrier is bounded: on expiry the CTA sets
// RTP_DEV_TIMEOUT, stops issuing work, waits (bounded) for what it issued and
// frees its TMEM.
//
// Shared-memory operands use the canonical 128-byte-swizzled layouts of the
// tcgen05 matrix descriptors: K-major (Q, K, P: 8-row atoms of 128-byte rows,
// 16-byte chunk c of row r at chunk c ^ (r mod 8)) and MN-major (V: 8-key
// atoms of 64 dims, the next 64 dims one region further).
#include <cuda.h>  // CUtensorMap and its encoding enums (the encoder is fetched through the runtime)

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace rtp {
namespace {

constexpr int kTcRows = 128;      // query rows per CTA = TMEM lanes
constexpr int kTcKeys = 128;      // keys per tile
constexpr int kTcThreads = 256;
constexpr int kRegion = 128 * 128;  // bytes of a 128-row x 64-dim bf16 region (one TMA box)
constexpr int kTmemCols = 512;
constexpr float kRescale = 8.0f;  // lazy rescale threshold (log2 units)

struct __align__(64) TcArgs {
  CUtensorMap tm_k;  // K cache as [rows][D] bf16, boxes of 64 x 128, 128-byte swizzle
  CUtensorMap tm_v;  // V cache, same
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W, T, words;
  const void* q_pre;
  void* out;
  int* status;
  const int* start_pos;
  const uint32_t* mask;  // [B][NR][mask_rows][words] top-p bitmask of rows [mask_t0, mask_t0 + mask_rows)
  int t_base, t_end, mask_t0, mask_rows;
  int n_heads;            // query heads this launch covers: head_list[0, n_heads)
  unsigned long long wait_ns;
  KvMap kv;
  int ret_rank[kMaxRetrieval];
  int head_list[64];
  double inv_freq[64];
};

template <int D>
struct TcSmem {
  static constexpr int kQ = (D / 64) * kRegion;        // Q: D/64 regions
  static constexpr int kK = (D / 64) * kRegion;        // one K stage
  static constexpr int kV = (D / 64) * kRegion;        // one V stage
  static constexpr int kP = 2 * kRegion;               // P: keys 0-63, 64-127
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQ;             // two stages
  static constexpr int kOffV = kOffK + 2 * kK;         // two stages
  static constexpr int kOffP = kOffV + 2 * kV;
  static constexpr int kBytes = kOffP + kP + 1024;     // + alignment slack
};

// ---------------------------------------------------------------------------
// tcgen05 / TMA primitives
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor: 128-byte swizzle, version 1 (sm_100),
// start address, leading and stride byte offsets in 16-byte units.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, M x N.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
         "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
         "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
         "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
         "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
         "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
         "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
         "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
         "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
         "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
         "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31])));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;"
      :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(pol)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Bounded wait that also gives up once another role of the CTA has aborted.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, const TcArgs& a, volatile int* s_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*s_abort) return false;
    if (global_ns() - t0 > a.wait_ns) {
      *s_abort = 1;
      atomicOr(a.status, RTP_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Key tiles a (head, row tile) attends: all causal tiles for retrieval heads;
// for local heads the tiles holding sinks, then those holding the window.
struct TileSeq {
  int n_a, b0, n;  // tiles [0, n_a), then tiles b0, b0 + 1, ... (n in total)
  __device__ __forceinline__ int start(int j) const { return (j < n_a ? j : b0 + (j - n_a)) * kTcKeys; }
};
__device__ __forceinline__ TileSeq tile_seq(bool local, int S, int W, int i_min, int i_max) {
  TileSeq q;
  const int last = i_max / kTcKeys;
  if (!local) {
    q.n_a = last + 1;
    q.b0 = last + 1;
    q.n = last + 1;
    return q;
  }
  q.n_a = min((S + kTcKeys - 1) / kTcKeys, last + 1);
  q.b0 = max(q.n_a, max(0, i_min - W + 1) / kTcKeys);
  q.n = q.n_a + max(0, last - q.b0 + 1);
  return q;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) attn_tc_kernel(const __grid_constant__ TcArgs a) {
  using SM = TcSmem<D>;
  constexpr int NR = D / 64;  // 64-dim regions
  extern __shared__ __align__(1024) unsigned char dsm_raw[];
  __shared__ __align__(8) uint64_t bar_kv_full[2], bar_kv_empty[2], bar_s_full[2], bar_s_free[2];
  __shared__ __align__(8) uint64_t bar_p_full, bar_o_done, bar_fin;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* dsm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  const uint32_t sQ = smem_u32(dsm + SM::kOffQ), sK = smem_u32(dsm + SM::kOffK);
  const uint32_t sV = smem_u32(dsm + SM::kOffV), sP = smem_u32(dsm + SM::kOffP);

  const int bq = blockIdx.y;
  const int b = bq / a.n_heads, hq = a.head_list[bq % a.n_heads];
  const int h = hq / a.G, g = hq % a.G;
  const int r = a.ret_rank[h];
  const int start = a.start_pos[b];
  if (start < 0 || start + a.T > a.Lmax) return;  // flagged by the selection kernel / host (uniform)
  const int t0 = a.t_base + blockIdx.x * kTcRows;
  const int t_last = min(a.t_end, t0 + kTcRows) - 1;
  const int i_min = start + t0, i_max = start + t_last;
  const TileSeq ts = tile_seq(r < 0, a.S, a.W, i_min, i_max);
  const int hh = r >= 0 ? r * a.G + g : 0;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
      mbar_init(&bar_s_full[s], 1);
      mbar_init(&bar_s_free[s], 128);
    }
    mbar_init(&bar_p_full, 128);
    mbar_init(&bar_o_done, 1);
    mbar_init(&bar_fin, 1);
    s_abort = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&s_tmem)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // ---- Q tile: RoPE at each row's position, scaled by log2(e)/sqrt(D), bf16,
  // into the swizzled K-major layout (rows past the chunk are zero) ----
  {
    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    constexpr int H = D / 2;
    for (int task = tid; task < kTcRows * (H / 8); task += kTcThreads) {
      const int rr = task / (H / 8), c8 = task % (H / 8);  // row, 8-dim chunk of the low half
      const int t = t0 + rr;
      float y1[8], y2[8];
      if (t <= t_last) {
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q_pre) + (((size_t)b * a.T + t) * a.Hq + hq) * D;
        float x1[8], x2[8];
        load_row<__nv_bfloat16, 8>(q + c8 * 8, x1);
        load_row<__nv_bfloat16, 8>(q + H + c8 * 8, x2);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float c, sn;
          rope_cos_sin(start + t, a.inv_freq[c8 * 8 + e], c, sn);
          y1[e] = (x1[e] * c - x2[e] * sn) * qscale;
          y2[e] = (x2[e] * c + x1[e] * sn) * qscale;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) y1[e] = y2[e] = 0.f;
      }
      uint4 lo, hi;
      lo.x = pack_bf16(y1[0], y1[1]); lo.y = pack_bf16(y1[2], y1[3]); lo.z = pack_bf16(y1[4], y1[5]); lo.w = pack_bf16(y1[6], y1[7]);
      hi.x = pack_bf16(y2[0], y2[1]); hi.y = pack_bf16(y2[2], y2[3]); hi.z = pack_bf16(y2[4], y2[5]); hi.w = pack_bf16(y2[6], y2[7]);
      // dims d = c8*8.. (low half) and H + c8*8.. (high half): region d / 64, chunk (d % 64) / 8
      const int d_lo = c8 * 8, d_hi = H + c8 * 8;
      const int reg_lo = d_lo / 64, ch_lo = (d_lo % 64) / 8;
      const int reg_hi = d_hi / 64, ch_hi = (d_hi % 64) / 8;
      *reinterpret_cast<uint4*>(dsm + SM::kOffQ + reg_lo * kRegion + rr * 128 + ((ch_lo ^ (rr & 7)) * 16)) = lo;
      *reinterpret_cast<uint4*>(dsm + SM::kOffQ + reg_hi * kRegion + rr * 128 + ((ch_hi ^ (rr & 7)) * 16)) = hi;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tS[2] = {tmem, tmem + kTcKeys};
  const uint32_t tO = tmem + 2 * kTcKeys;
  const int n = ts.n;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: K and V tiles by TMA ----
      const uint64_t pol = l2_evict_last();
      const size_t rowbase = a.kv.row(b, h, 0);  // full-cache head: position p at rowbase + p
      for (int j = 0; j < n; ++j) {
        const int s = j & 1, k = j >> 1;
        if (!tc_wait(&bar_kv_empty[s], (uint32_t)(k & 1) ^ 1u, a, &s_abort)) break;
        mbar_expect_tx(&bar_kv_full[s], (uint32_t)(2 * NR * kRegion));
        const int y = (int)(rowbase + ts.start(j));
#pragma unroll
        for (int rg = 0; rg < NR; ++rg) {
          tma_load_2d(dsm + SM::kOffK + s * SM::kK + rg * kRegion, &a.tm_k, rg * 64, y, &bar_kv_full[s], pol);
          tma_load_2d(dsm + SM::kOffV + s * SM::kV + rg * kRegion, &a.tm_v, rg * 64, y, &bar_kv_full[s], pol);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      constexpr uint32_t idS = umma_idesc(kTcRows, kTcKeys, false);
      constexpr uint32_t idO = umma_idesc(kTcRows, D, true);
      auto issue_s = [&](int j) {  // S(j) = Q K(j)^T into buffer j & 1
        const int s = j & 1;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int rg = kk / 4, ko = (kk % 4) * 32;
          const uint64_t ad = umma_desc(sQ + rg * kRegion + ko, 16, 1024);
          const uint64_t bd = umma_desc(sK + s * SM::kK + rg * kRegion + ko, 16, 1024);
          umma_f16(tS[s], ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar_s_full[s]);
      };
      bool ok = n > 0 && tc_wait(&bar_kv_full[0], 0u, a, &s_abort);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) {
          const int s1 = (j + 1) & 1, k1 = (j + 1) >> 1;
          if (!tc_wait(&bar_kv_full[s1], (uint32_t)(k1 & 1), a, &s_abort)) break;
          if (!tc_wait(&bar_s_free[s1], (uint32_t)(k1 & 1) ^ 1u, a, &s_abort)) break;
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!tc_wait(&bar_p_full, (uint32_t)(j & 1), a, &s_abort)) break;
        tc_fence_after();
        const int s = j & 1;
#pragma unroll
        for (int kk = 0; kk < kTcKeys / 16; ++kk) {  // O += P V(j)
          const int rg = kk / 4, ko = (kk % 4) * 32;
          const uint64_t ad = umma_desc(sP + rg * kRegion + ko, 16, 1024);
          const uint64_t bd = umma_desc(sV + s * SM::kV + kk * 2048, kRegion, 1024);
          umma_f16(tO, ad, bd, idO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bar_o_done);
        umma_commit(&bar_kv_empty[s]);
      }
      // every MMA this thread issued has completed before TMEM is freed
      umma_commit(&bar_fin);
      mbar_wait_bounded(&bar_fin, 0u, a.wait_ns, a.status);
    }
  } else if (warp >= 4) {
    // ---- softmax: thread = query row ----
    const int row = tid - 128;  // TMEM lane
    const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
    const int t = t0 + row;
    const bool rv = t <= t_last;
    const int pi = start + t;
    const int wlo = pi - a.W + 1;
    const uint32_t* mrow = a.mask + (((size_t)b * a.NR + hh) * a.mask_rows + (rv ? t - a.mask_t0 : 0)) * a.words;
    float m_used = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int kt = ts.start(j);
      const int s = j & 1;
      // every wait's outcome is made warp-uniform: TMEM loads and stores are warp-collective
      if (!__all_sync(0xffffffffu, tc_wait(&bar_s_full[s], (uint32_t)(j >> 1) & 1u, a, &s_abort))) { ok = false; break; }
      tc_fence_after();
      float sv[kTcKeys];
#pragma unroll
      for (int c = 0; c < kTcKeys / 32; ++c) {
        float v[32];
        tmem_ld32(tS[s] + lane_off + c * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = v[e];
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bar_s_free[s]);
      // mask: causal; sinks or window; retrieval heads also keep the top-p set
      uint32_t mw[4] = {0u, 0u, 0u, 0u};
      if (r >= 0 && rv) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int wd = (kt >> 5) + q;
          mw[q] = (wd * 32 <= pi) ? __ldg(mrow + wd) : 0u;
        }
      }
      float tmax = -CUDART_INF_F;
#pragma unroll
      for (int c = 0; c < kTcKeys; ++c) {
        const int jk = kt + c;
        bool keep = rv && jk <= pi && (jk < a.S || jk >= wlo);
        if (r >= 0) keep = keep || (rv && jk <= pi && ((mw[c >> 5] >> (c & 31)) & 1u));
        sv[c] = keep ? sv[c] : -CUDART_INF_F;
        tmax = fmaxf(tmax, sv[c]);
      }
      // lazy rescale: the maximum used moves only when the tile's exceeds it by > 2^8
      float m_new = m_used, f = 1.f;
      if (tmax > m_used + kRescale || (m_used == -CUDART_INF_F && tmax != -CUDART_INF_F)) {
        m_new = tmax;
        f = (m_used == -CUDART_INF_F) ? 0.f : exp2f(m_used - m_new);
      }
      float lsum = 0.f;
      uint32_t pk[kTcKeys / 2];
#pragma unroll
      for (int c = 0; c < kTcKeys; c += 2) {
        const float p0 = sv[c] == -CUDART_INF_F ? 0.f : exp2f(sv[c] - m_new);
        const float p1 = sv[c + 1] == -CUDART_INF_F ? 0.f : exp2f(sv[c + 1] - m_new);
        lsum += p0 + p1;
        pk[c / 2] = pack_bf16(p0, p1);
      }
      l = l * f + lsum;
      m_used = m_new;
      // P's buffer and O are free once PV(j - 1) has completed
      if (j > 0 && !__all_sync(0xffffffffu, tc_wait(&bar_o_done, (uint32_t)((j - 1) & 1), a, &s_abort))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (j > 0 && __any_sync(0xffffffffu, f != 1.f)) {  // rescale O rows (warp-uniform TMEM access)
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tO + lane_off + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tmem_st32(tO + lane_off + c * 32, o);
        }
        tmem_wait_st();
      }
      // last tile: value rows past the query tile's last position may be
      // unwritten cache (their weights are 0, but 0 x NaN would not be)
      if (kt + kTcKeys - 1 > i_max) {
        if (!__all_sync(0xffffffffu, tc_wait(&bar_kv_full[s], (uint32_t)(j >> 1) & 1u, a, &s_abort))) {
          ok = false;
          break;
        }
        if (kt + row > i_max) {
#pragma unroll
          for (int rg = 0; rg < NR; ++rg) {
            uint4* vr = reinterpret_cast<uint4*>(dsm + SM::kOffV + s * SM::kV + rg * kRegion + row * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) vr[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      // P row -> swizzled K-major layout (keys 0-63 in region 0, 64-127 in region 1)
#pragma unroll
      for (int c = 0; c < kTcKeys / 8; ++c) {
        const int rg = c / 8, ch = c % 8;
        uint4 v = make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
        *reinterpret_cast<uint4*>(dsm + SM::kOffP + rg * kRegion + row * 128 + ((ch ^ (row & 7)) * 16)) = v;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bar_p_full);
    }
    // ---- epilogue: O / l -> out ----
    if (ok && n > 0 && __all_sync(0xffffffffu, tc_wait(&bar_o_done, (uint32_t)((n - 1) & 1), a, &s_abort))) {
      tc_fence_after();
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + (((size_t)b * a.T + (rv ? t : 0)) * a.Hq + hq) * D;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tO + lane_off + c * 32, o);
        tmem_wait_ld();
        if (rv) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack_bf16(o[e] * inv, o[e + 1] * inv);
            v.y = pack_bf16(o[e + 2] * inv, o[e + 3] * inv);
            v.z = pack_bf16(o[e + 4] * inv, o[e + 5] * inv);
            v.w = pack_bf16(o[e + 6] * inv, o[e + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + e) = v;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (s_abort && warp == 0 && lane == 0) {
    // copies still in flight after an abort: wait for them (bounded) before leaving
    mbar_wait_bounded(&bar_kv_full[0], 0u, a.wait_ns, a.status);
    mbar_wait_bounded(&bar_kv_full[1], 0u, a.wait_ns, a.status);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------------------
// host: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

bool make_map(CUtensorMap* tm, const void* base, int D, unsigned long long rows) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kTcKeys};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Query heads whose keys and values sit in the full-context layout go to the
// tcgen05 kernel (all of them unless local heads keep a ring).
int launch_attn_tc(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* start_pos, int T,
                   void* out, const uint32_t* mask, int t_base, int t_end, int mask_t0, int mask_rows,
                   unsigned long long wait_ns, cudaStream_t st) {
  TcArgs a;
  const unsigned long long rows = (unsigned long long)sh.B * (unsigned long long)sh.kv.rows_per_seq;
  if (!make_map(&a.tm_k, cache->k, sh.D, rows) || !make_map(&a.tm_v, cache->v, sh.D, rows)) {
    set_error("prefill: could not encode the K/V tensor maps (cuTensorMapEncodeTiled)");
    return RTP_ERR_CUDA;
  }
  a.B = sh.B; a.Hq = sh.Hq; a.Hkv = sh.Hkv; a.G = sh.G; a.D = sh.D; a.R = sh.R; a.NR = sh.NR;
  a.Lmax = sh.Lmax; a.S = sh.S; a.W = sh.W; a.T = T; a.words = (sh.Lmax + 31) / 32;
  a.q_pre = q_pre; a.out = out; a.status = cache->status; a.start_pos = start_pos;
  a.mask = mask; a.t_base = t_base; a.t_end = t_end; a.mask_t0 = mask_t0; a.mask_rows = mask_rows;
  a.wait_ns = wait_ns;
  a.kv = sh.kv;
  for (int i = 0; i < kMaxRetrieval; ++i) a.ret_rank[i] = sh.ret_rank[i];
  for (int i = 0; i < 64; ++i) a.inv_freq[i] = sh.inv_freq[i];
  // heavier heads first: retrieval heads attend every causal tile
  int n = 0;
  for (int pass = 0; pass < 2; ++pass)
    for (int hq = 0; hq < sh.Hq; ++hq) {
      const int h = hq / sh.G;
      if ((sh.kv.ring_mask >> h) & 1ull) continue;  // ring heads: the CUDA-core kernel
      if ((pass == 0) != (sh.ret_rank[h] >= 0)) continue;
      a.head_list[n++] = hq;
    }
  a.n_heads = n;
  if (n == 0) return RTP_OK;
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && !done[dev]) {
      cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSmem<128>::kBytes);
      cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSmem<64>::kBytes);
      done[dev] = true;
    }
  }
  const dim3 grid((t_end - t_base + kTcRows - 1) / kTcRows, sh.B * n);
  if (sh.D == 128) attn_tc_kernel<128><<<grid, kTcThreads, TcSmem<128>::kBytes, st>>>(a);
  else attn_tc_kernel<64><<<grid, kTcThreads, TcSmem<64>::kBytes, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("prefill tcgen05 launch: ") + cudaGetErrorString(e));
    return RTP_ERR_CUDA;
  }
  return RTP_OK;
}

}  // namespace rtp
