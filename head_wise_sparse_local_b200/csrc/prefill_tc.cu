// Prefill attention on the fifth-generation tensor cores (tcgen05 + TMEM).
//
// One CTA per (sequence, query head, 256 query rows), the rows split into two
// slots of 128 (one TMEM lane per row).  The CTA walks the key tiles (128 keys)
// that any of its rows attends, and for each tile and slot: S = Q K^T (128 x
// 128, fp32 in TMEM), a softmax over S by the thread that owns the row, P (bf16)
// written back into S's TMEM columns, then O += P V with P taken from TMEM
// (128 x D, fp32 in TMEM).  The layer's masks (causality; sinks and window;
// for retrieval heads the row's top-p bitmask from the selection kernel) are
// applied to S (atlas.scime.ai summary, "Approach"; abstract, observations
// (2)-(3)).  Tiles in which every row of a slot sees every key need no mask.
//
// The key tiles: the sink tiles and the window tiles of the CTA's rows, and for
// retrieval heads every tile in which some row keeps a token (a per-CTA tile
// map that tile_map_kernel reduces from the selection bitmask); never a tile
// past the last row's position.
//
// Roles (576 threads):
//   warp 0, lane 0   stages K and V tiles with TMA (cp.async.bulk.tensor,
//                    128-byte swizzle, boxes of 64 dims x 128 keys), two
//                    stages in flight;
//   warp 1           allocates TMEM; lane 0 issues every tcgen05.mma and
//                    commits its completions to mbarriers, in the order
//                    S0(i), PV1(i-1), S1(i), PV0(i), so that each slot's
//                    softmax overlaps the other slot's products;
//   warps 2-9, 10-17 the softmax of slot 0 and slot 1, two threads per query
//                    row (each half of the tile's keys): read S from TMEM,
//                    mask, keep the running maximum and sum, write P to TMEM,
//                    rescale O in TMEM when the maximum grows by more than 2^8,
//                    and finally write the output.
// tcgen05.mma operations issued by one thread execute in issue order, so S of
// the next tile may overwrite the TMEM columns that the previous PV read P
// from; a commit after S(i) of a slot also tells that slot's softmax that
// PV(i-1) has completed (its O may be rescaled, its P columns rewritten).
// Every wait on an mbarrier is bounded: on expiry the CTA sets
// RTP_DEV_TIMEOUT, stops issuing work, waits (bounded) for what it issued and
// frees its TMEM.
//
// Shared-memory operands use the canonical 128-byte-swizzled layouts of the
// tcgen05 matrix descriptors: K-major (Q, K: 8-row atoms of 128-byte rows,
// 16-byte chunk c of row r at chunk c ^ (r mod 8)) and MN-major (V: 8-key atoms
// of 64 dims, the next 64 dims one region further).
#include <cuda.h>  // CUtensorMap and its encoding enums (the encoder is fetched through the runtime)

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace rtp {
namespace {

constexpr int kTcRows = 128;      // query rows per slot = TMEM lanes
constexpr int kSlots = 2;
constexpr int kGroupRows = kSlots * kTcRows;  // query rows per CTA
constexpr int kTcKeys = 128;      // keys per tile
constexpr int kTcThreads = 576;  // producer warp, MMA warp, 16 softmax warps
constexpr int kRegion = 128 * 128;  // bytes of a 128-row x 64-dim bf16 region (one TMA box)
constexpr int kTmemCols = 512;
constexpr float kRescale = 8.0f;  // lazy rescale threshold (log2 units)
constexpr int kMaxTileWords = ((1 << 23) / kTcKeys) / 32 + 1;  // tile bitmap words for the largest context

struct __align__(64) TcArgs {
  CUtensorMap tm_k;  // K cache as [rows][D] bf16, boxes of 64 x 128, 128-byte swizzle
  CUtensorMap tm_v;  // V cache, same
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W, T, words;
  const void* q_pre;
  void* out;
  int* status;
  const int* start_pos;
  const uint32_t* mask;  // [B][NR][mask_rows][words] top-p bitmask of rows [mask_t0, mask_t0 + mask_rows)
  const uint32_t* tmap;  // [B][NR][map_groups][map_words] key tiles some row of a 256-row group keeps
  uint32_t* tmap_out;    // the same array, written by tile_map_kernel
  int map_words, map_groups, map_g0;  // words per group; groups per head; group of this launch's first CTA
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
  static constexpr int kQ = (D / 64) * kRegion;        // Q of one slot: D/64 regions
  static constexpr int kK = (D / 64) * kRegion;        // one K stage
  static constexpr int kV = (D / 64) * kRegion;        // one V stage
  static constexpr int kOffQ = 0;                      // two slots
  static constexpr int kOffK = kOffQ + kSlots * kQ;    // two stages
  static constexpr int kOffV = kOffK + 2 * kK;         // two stages
  static constexpr int kOffTiles = kOffV + 2 * kV;     // key-tile bitmap
  static constexpr int kBytes = kOffTiles + kMaxTileWords * 4 + 1024;  // + alignment slack
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
  while (!mbar_try_wait_sleep(bar, parity, kWaitHintNs)) {
    if (*s_abort) return false;
    if (global_ns() - t0 > a.wait_ns) {
      *s_abort = 1;
      atomicOr(a.status, RTP_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// tcgen05.mma of kind::f16 with A from TMEM (P) and B from shared memory (V).
__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      :: "r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
         "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}

__device__ __forceinline__ float max3f(float x, float y, float z) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(x), "f"(y), "f"(z));
  return m;
}

// 2^x by the hardware approximation (relative error about 2^-22; -inf -> +0).
__device__ __forceinline__ float ex2f(float x) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(x));
  return e;
}

// Packed fp32 pairs (one instruction for two lanes of arithmetic).
__device__ __forceinline__ void add2(float& x, float& y, float a, float b) {  // (x, y) += (a, b)
  asm("{\n\t.reg .b64 p, q;\n\tmov.b64 p, {%0, %1};\n\tmov.b64 q, {%2, %3};\n\t"
      "add.rn.f32x2 p, p, q;\n\tmov.b64 {%0, %1}, p;\n\t}"
      : "+f"(x), "+f"(y) : "f"(a), "f"(b));
}
__device__ __forceinline__ void mul2(float& x, float& y, float f) {  // (x, y) *= f
  asm("{\n\t.reg .b64 p, q;\n\tmov.b64 p, {%0, %1};\n\tmov.b64 q, {%2, %2};\n\t"
      "mul.rn.f32x2 p, p, q;\n\tmov.b64 {%0, %1}, p;\n\t}"
      : "+f"(x), "+f"(y) : "f"(f));
}

// 2^x on the FMA pipe, for a share of the softmax weights, so that the MUFU
// pipe (ex2f) does not bound the softmax.  Cody-Waite split x = j + f with
// j = round(x) (by adding 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f by a cubic
// fitted to it in relative error on that interval (Chebyshev-node least
// squares reweighted toward equal ripple: maximum relative error 7.5e-5,
// far below a bf16 weight's rounding); 2^j added to the exponent field.
// Inputs below -125 are taken as -125 (a weight of about 2^-125).
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;  // round(x) in the low mantissa bits of t
  const float f = x - (t - 12582912.f);
  float p = fmaf(0.05517161f, f, 0.24261111f);
  p = fmaf(p, f, 0.69326097f);
  p = fmaf(p, f, 0.99992806f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Walks the set bits of a shared-memory tile bitmap in increasing order.
struct TileCursor {
  const uint32_t* bits;
  int nw, w;
  uint32_t cur;
  __device__ __forceinline__ void init(const uint32_t* b, int n) {
    bits = b;
    nw = n;
    w = 0;
    cur = n > 0 ? b[0] : 0u;
  }
  __device__ __forceinline__ int next() {
    while (cur == 0u) {
      if (++w >= nw) return -1;
      cur = bits[w];
    }
    const int t = w * 32 + (__ffs(cur) - 1);
    cur &= cur - 1u;
    return t;
  }
};

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) attn_tc_kernel(const __grid_constant__ TcArgs a) {
  using SM = TcSmem<D>;
  constexpr int NRG = D / 64;  // 64-dim regions
  extern __shared__ __align__(1024) unsigned char dsm_raw[];
  __shared__ __align__(8) uint64_t bar_k_full[2], bar_k_empty[2], bar_v_full[2], bar_v_empty[2];
  __shared__ __align__(8) uint64_t bar_s_full[kSlots], bar_p_full[kSlots];
  __shared__ __align__(8) uint64_t bar_o_done, bar_fin;
  __shared__ __align__(8) uint64_t bar_pair[kSlots][4];  // the two softmax warps of a row quarter
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort, s_ntiles;
  // the two softmax halves of a row: tile maxima by tile parity, then the sums
  __shared__ float s_xch[kSlots][4][3 * 64];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* dsm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  const uint32_t sQ = smem_u32(dsm + SM::kOffQ), sK = smem_u32(dsm + SM::kOffK);
  const uint32_t sV = smem_u32(dsm + SM::kOffV);
  uint32_t* s_tiles = reinterpret_cast<uint32_t*>(dsm + SM::kOffTiles);

  const int bq = blockIdx.y;
  const int b = bq / a.n_heads, hq = a.head_list[bq % a.n_heads];
  const int h = hq / a.G, g = hq % a.G;
  const int r = a.ret_rank[h];
  const int start = a.start_pos[b];
  if (start < 0 || start + a.T > a.Lmax) return;  // flagged by the selection kernel / host (uniform)
  const int t0 = a.t_base + blockIdx.x * kGroupRows;
  const int t_last = min(a.t_end, t0 + kGroupRows) - 1;
  const int i_lo = start + t0, i_hi = start + t_last;
  const int last_tile = i_hi / kTcKeys;
  const int n_words = last_tile / 32 + 1;
  const int hh = r >= 0 ? r * a.G + g : 0;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_k_full[s], 1);
      mbar_init(&bar_k_empty[s], 1);
      mbar_init(&bar_v_full[s], 1);
      mbar_init(&bar_v_empty[s], 1);
      mbar_init(&bar_s_full[s], 1);
      mbar_init(&bar_p_full[s], 2 * kTcRows);
    }
    mbar_init(&bar_o_done, 1);
    mbar_init(&bar_fin, 1);
    for (int s = 0; s < kSlots; ++s)
      for (int q = 0; q < 4; ++q) mbar_init(&bar_pair[s][q], 64);
    s_abort = 0;
    s_ntiles = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&s_tmem)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  // ---- key tiles: sinks, the rows' windows and (retrieval heads) the tiles
  // some row keeps, none past the last row's tile ----
  {
    const int ns = min((a.S + kTcKeys - 1) / kTcKeys, last_tile + 1);  // sink tiles [0, ns)
    const int w0 = max(0, i_lo - a.W + 1) / kTcKeys;                   // window tiles [w0, last_tile]
    const uint32_t* mp = r >= 0 ? a.tmap + (((size_t)b * a.NR + hh) * a.map_groups + a.map_g0 + blockIdx.x) *
                                               (size_t)a.map_words
                                : nullptr;
    int cnt = 0;
    for (int w = tid; w < n_words; w += kTcThreads) {
      const int lo = w * 32, hi = lo + 31;
      uint32_t v = 0u;
      if (lo < ns) v |= ns - lo >= 32 ? 0xffffffffu : (1u << (ns - lo)) - 1u;
      const int a0 = max(lo, w0), a1 = min(hi, last_tile);
      if (a0 <= a1) v |= a1 - a0 == 31 ? 0xffffffffu : ((1u << (a1 - a0 + 1)) - 1u) << (a0 - lo);
      if (mp) v |= __ldg(mp + w);
      if (hi > last_tile) v &= (1u << (last_tile - lo + 1)) - 1u;  // lo <= last_tile < hi
      s_tiles[w] = v;
      cnt += __popc(v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0 && cnt) atomicAdd(&s_ntiles, cnt);
  }
  // ---- Q of both slots: RoPE at each row's position, scaled by
  // log2(e)/sqrt(D), bf16, into the swizzled K-major layout (rows past the
  // chunk are zero) ----
  {
    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    constexpr int H = D / 2;
    for (int task = tid; task < kGroupRows * (H / 8); task += kTcThreads) {
      const int rr = task / (H / 8), c8 = task % (H / 8);  // row of the CTA, 8-dim chunk of the low half
      const int slot = rr / kTcRows, lr = rr % kTcRows;
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
      unsigned char* qs = dsm + SM::kOffQ + slot * SM::kQ + lr * 128;
      *reinterpret_cast<uint4*>(qs + (d_lo / 64) * kRegion + ((((d_lo % 64) / 8) ^ (lr & 7)) * 16)) = lo;
      *reinterpret_cast<uint4*>(qs + (d_hi / 64) * kRegion + ((((d_hi % 64) / 8) ^ (lr & 7)) * 16)) = hi;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n = s_ntiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: K and V tiles by TMA, each as soon as its stage is
      // free (a K stage frees after the tile's two S products, a V stage after
      // its two PV products) ----
      const uint64_t pol = l2_evict_last();
      const size_t rowbase = a.kv.row(b, h, 0);  // full-cache head: position p at rowbase + p
      TileCursor cur;
      cur.init(s_tiles, n_words);
      for (int i = 0; i < n; ++i) {
        const int kt = cur.next() * kTcKeys;
        const int st = i & 1;
        const uint32_t par = ((uint32_t)(i >> 1) & 1u) ^ 1u;
        const int y = (int)(rowbase + kt);
        if (!tc_wait(&bar_k_empty[st], par, a, &s_abort)) break;
        mbar_expect_tx(&bar_k_full[st], (uint32_t)(NRG * kRegion));
#pragma unroll
        for (int rg = 0; rg < NRG; ++rg)
          tma_load_2d(dsm + SM::kOffK + st * SM::kK + rg * kRegion, &a.tm_k, rg * 64, y, &bar_k_full[st], pol);
        if (!tc_wait(&bar_v_empty[st], par, a, &s_abort)) break;
        mbar_expect_tx(&bar_v_full[st], (uint32_t)(NRG * kRegion));
#pragma unroll
        for (int rg = 0; rg < NRG; ++rg)
          tma_load_2d(dsm + SM::kOffV + st * SM::kV + rg * kRegion, &a.tm_v, rg * 64, y, &bar_v_full[st], pol);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: the warp walks the tiles together (it zeroes the value
    // rows past the CTA's last position in the last tile); lane 0 issues ----
    constexpr uint32_t idS = umma_idesc(kTcRows, kTcKeys, false);
    constexpr uint32_t idO = umma_idesc(kTcRows, D, true);
    const uint32_t tS[2] = {tmem, tmem + kTcKeys};
    const uint32_t tO[2] = {tmem + 2 * kTcKeys, tmem + 3 * kTcKeys};
    // Descriptors: one base per operand, the k-step's offset added to the
    // address field (start address / 16 in the low 14 bits; shared memory is
    // below 256 KB, so the field never carries into the next)
    const uint64_t dq0 = umma_desc(sQ, 16, 1024), dk0 = umma_desc(sK, 16, 1024);
    const uint64_t dv0 = umma_desc(sV, kRegion, 1024);
    auto issue_s = [&](int slot, int st) {  // S(slot) = Q(slot) K(stage st)^T
      if (lane == 0) {
        const uint64_t dq = dq0 + (uint64_t)((slot * SM::kQ) >> 4);
        const uint64_t dk = dk0 + (uint64_t)((st * SM::kK) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(((kk / 4) * kRegion + (kk % 4) * 32) >> 4);
          umma_f16(tS[slot], dq + off, dk + off, idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar_s_full[slot]);
      }
      __syncwarp();
    };
    auto issue_pv = [&](int slot, int st, bool acc) {  // O(slot) += P(slot) V(stage st), P in S's TMEM
      if (lane == 0) {
        const uint64_t dv = dv0 + (uint64_t)((st * SM::kV) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTcKeys / 16; ++kk) {
          // P of keys [64 h, 64 h + 64) sits in S columns [64 h, 64 h + 32)
          const uint32_t pa = tS[slot] + (kk >> 2) * 64 + (kk & 3) * 8;
          umma_f16_ts(tO[slot], pa, dv + (uint64_t)((kk * 2048) >> 4), idO, (acc || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    TileCursor cur;
    cur.init(s_tiles, n_words);
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int kt = cur.next() * kTcKeys;
      const int st = i & 1;
      const uint32_t par = (uint32_t)(i >> 1) & 1u;
      if (!__all_sync(0xffffffffu, tc_wait(&bar_k_full[st], par, a, &s_abort))) { ok = false; break; }
      tc_fence_after();
      issue_s(0, st);
      if (i > 0) {
        if (!__all_sync(0xffffffffu, tc_wait(&bar_p_full[1], (uint32_t)(i - 1) & 1u, a, &s_abort))) { ok = false; break; }
        tc_fence_after();
        issue_pv(1, st ^ 1, i > 1);
        if (lane == 0) umma_commit(&bar_v_empty[st ^ 1]);
      }
      issue_s(1, st);
      if (lane == 0) umma_commit(&bar_k_empty[st]);
      if (!__all_sync(0xffffffffu, tc_wait(&bar_v_full[st], par, a, &s_abort))) { ok = false; break; }
      if (kt + kTcKeys - 1 > i_hi) {
        // value rows past the CTA's last position may be unwritten cache (their
        // weights are 0, but 0 x NaN would not be)
        for (int rr = i_hi - kt + 1 + lane; rr < kTcKeys; rr += 32) {
#pragma unroll
          for (int rg = 0; rg < NRG; ++rg) {
            uint4* vr = reinterpret_cast<uint4*>(dsm + SM::kOffV + st * SM::kV + rg * kRegion + rr * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) vr[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_async_smem();
        __syncwarp();
      }
      if (!__all_sync(0xffffffffu, tc_wait(&bar_p_full[0], (uint32_t)i & 1u, a, &s_abort))) { ok = false; break; }
      tc_fence_after();
      issue_pv(0, st, i > 0);
    }
    if (ok && n > 0 &&
        __all_sync(0xffffffffu, tc_wait(&bar_p_full[1], (uint32_t)(n - 1) & 1u, a, &s_abort))) {
      tc_fence_after();
      issue_pv(1, (n - 1) & 1, n > 1);
      if (lane == 0) umma_commit(&bar_v_empty[(n - 1) & 1]);
    }
    if (lane == 0) {
      umma_commit(&bar_o_done);
      // every MMA this thread issued has completed before TMEM is freed
      umma_commit(&bar_fin);
      mbar_wait_bounded(&bar_fin, 0u, a.wait_ns, a.status);
    }
    __syncwarp();
  } else {
    // ---- softmax: warps 2-9 slot 0, warps 10-17 slot 1.  A query row has
    // two threads, in two warps of the same TMEM lane quarter: half h takes the
    // keys [64 h, 64 h + 64) of each tile, writes their P over the first 32 of
    // those S columns and rescales O's columns [h D/2, (h+1) D/2); the halves
    // exchange their tile maxima (and at the end their sums) through shared
    // memory under the pair's mbarrier (a bounded wait, like every other) ----
    const int sw = warp - 2;
    const int slot = sw >> 3, hf = (sw >> 2) & 1;
    const int quad = warp & 3;  // the TMEM lane quarter this warp may access
    const int row = quad * 32 + lane;
    uint64_t* pbar = &bar_pair[slot][quad];  // phase j: tile j's maxima; phase n: the sums
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tSs = tmem + slot * kTcKeys + hf * 64, tOs = tmem + (2 + slot) * kTcKeys + hf * (D / 2);
    const int t = t0 + slot * kTcRows + row;
    const bool rv = t <= t_last;
    const int pi = start + t;
    const int wlo = pi - a.W + 1;
    const int s_lo = i_lo + slot * kTcRows;          // the slot's first row position
    const int s_hi = min(i_hi, s_lo + kTcRows - 1);  // its last valid row position (< s_lo: none)
    const uint32_t* mrow = a.mask + (((size_t)b * a.NR + hh) * a.mask_rows + (rv ? t - a.mask_t0 : 0)) * a.words;
    float* xch = s_xch[slot][quad];                  // [2 tile parities][2 halves][32 lanes]
    TileCursor cur;
    cur.init(s_tiles, n_words);
    float m_used = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    auto apply_mask = [&](float (&v)[32], uint32_t bits) {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = (bits >> e) & 1u ? v[e] : -CUDART_INF_F;
    };
    // a tile every row of the slot sees whole (causal, inside sinks or window)
    // needs no mask (uniform over the slot)
    auto is_whole = [&](int kt) {
      return s_lo <= s_hi && kt + kTcKeys - 1 <= s_lo && (kt + kTcKeys - 1 < a.S || kt >= s_hi - a.W + 1);
    };
    // this row's top-p bitmask words of a tile's half (retrieval heads), loaded
    // one tile ahead of their use
    auto load_mw = [&](int kt, uint32_t (&mw)[2]) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int base = kt + hf * 64 + 32 * q;
        mw[q] = (r >= 0 && rv && kt >= 0 && base <= pi && !is_whole(kt)) ? __ldg(mrow + (base >> 5)) : 0u;
      }
    };
    int kt_next = n > 0 ? cur.next() * kTcKeys : -1;
    uint32_t mw_next[2];
    load_mw(kt_next, mw_next);
    for (int j = 0; j < n; ++j) {
      const int kt = kt_next;
      const uint32_t mw[2] = {mw_next[0], mw_next[1]};
      kt_next = j + 1 < n ? cur.next() * kTcKeys : -1;
      load_mw(kt_next, mw_next);
      const int k0 = kt + hf * 64;  // this half's first key
      // otherwise each row keeps keys <= its position that lie in the sinks,
      // its window or (retrieval heads) its top-p set: 32-key words of keep bits
      const bool whole = is_whole(kt);
      uint32_t kw[2] = {0xffffffffu, 0xffffffffu};
      bool full[2] = {true, true};  // the chunk is kept whole by every row of the warp
      if (!whole) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int base = k0 + 32 * q;
          const int nc = pi - base + 1;  // keys <= pi: bits [0, nc)
          const uint32_t causal = !rv || nc <= 0 ? 0u : nc >= 32 ? 0xffffffffu : (1u << nc) - 1u;
          const int nsk = a.S - base;    // sinks: bits [0, nsk)
          const uint32_t sink = nsk <= 0 ? 0u : nsk >= 32 ? 0xffffffffu : (1u << nsk) - 1u;
          const int nw0 = wlo - base;    // window: bits [nw0, 32)
          const uint32_t win = nw0 <= 0 ? 0xffffffffu : nw0 >= 32 ? 0u : ~((1u << nw0) - 1u);
          kw[q] = causal & (sink | win | mw[q]);
          full[q] = __all_sync(0xffffffffu, kw[q] == 0xffffffffu);
        }
      }
      // every wait's outcome is made warp-uniform: TMEM loads and stores are warp-collective
      if (!__all_sync(0xffffffffu, tc_wait(&bar_s_full[slot], (uint32_t)j & 1u, a, &s_abort))) { ok = false; break; }
      tc_fence_after();
      // One read of S: the half-row's maximum and, against the row's running
      // maximum m_used, its weights (P held in registers).  The halves then
      // exchange their maxima; a row with no maximum yet, or whose tile
      // maximum exceeds m_used by more than 2^8 (the lazy rescale threshold),
      // makes its warps (the same rows in both halves) recompute P against
      // the new maximum from S, which is still intact.
      const bool have_m = m_used != -CUDART_INF_F;
      const float mspec = have_m ? m_used : 0.f;  // a row with no maximum yet keeps only 0 weights here
      float hmax = -CUDART_INF_F, lsum0 = 0.f, lsum1 = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float v[32];
        tmem_ld32(tSs + lane_off + c * 32, v);
        tmem_wait_ld();
        if (!full[c]) apply_mask(v, kw[c]);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0 = v[2 * e], x1 = v[2 * e + 1];
          hmax = max3f(hmax, x0, x1);
          add2(x0, x1, -mspec, -mspec);
          // one weight in four on the FMA pipe, the rest on MUFU
          const float p0 = ex2f(x0), p1 = (e & 1) ? ex2_poly(x1) : ex2f(x1);
          add2(lsum0, lsum1, p0, p1);
          pk[c * 16 + e] = pack_bf16(p0, p1);
        }
      }
      float* xm = xch + (j & 1) * 64;
      xm[hf * 32 + lane] = hmax;
      mbar_arrive(pbar);  // release: the partner's wait makes xm visible
      if (!__all_sync(0xffffffffu, tc_wait(pbar, (uint32_t)j & 1u, a, &s_abort))) { ok = false; break; }
      const float tmax = fmaxf(hmax, xm[(hf ^ 1) * 32 + lane]);
      // lazy rescale: the maximum used moves only when the tile's exceeds it by > 2^8
      float m_new = m_used, f = 1.f;
      if (tmax > m_used + kRescale || (!have_m && tmax != -CUDART_INF_F)) {
        m_new = tmax;
        f = have_m ? ex2f(m_used - m_new) : 0.f;
      }
      if (!__any_sync(0xffffffffu, m_new != m_used)) {
        // P of keys [k0 + 32 c, +32) to columns [16 c, 16 c + 16)
        tmem_st16(tSs + lane_off, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tmem_st16(tSs + lane_off + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
      } else {
        // this slot's PV of the previous tile has completed (its commit precedes
        // this tile's S): O may be rescaled and P's columns written
        if (j > 0 && __any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            float o[32];
            tmem_ld32(tOs + lane_off + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 2) mul2(o[e], o[e + 1], f);
            tmem_st32(tOs + lane_off + c * 32, o);
          }
        }
        const float msub = m_new == -CUDART_INF_F ? 0.f : m_new;  // all masked so far: every weight is 0
        lsum0 = 0.f;
        lsum1 = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          // P of keys [k0 + 32 c, +32) goes to columns [16 c, 16 c + 16) of this
          // half, inside its first S chunk, already read
          float v[32];
          tmem_ld32(tSs + lane_off + c * 32, v);
          tmem_wait_ld();
          if (!full[c]) apply_mask(v, kw[c]);
          uint32_t q16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0 = v[2 * e], x1 = v[2 * e + 1];
            add2(x0, x1, -msub, -msub);
            const float p0 = ex2f(x0), p1 = (e & 1) ? ex2_poly(x1) : ex2f(x1);
            add2(lsum0, lsum1, p0, p1);
            q16[e] = pack_bf16(p0, p1);
          }
          tmem_st16(tSs + lane_off + c * 16, q16);
        }
      }
      m_used = m_new;
      l = l * f + (lsum0 + lsum1);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p_full[slot]);
    }
    // ---- epilogue: O / l -> out, each half its D/2 columns ----
    if (ok && n > 0 && __all_sync(0xffffffffu, tc_wait(&bar_o_done, 0u, a, &s_abort))) {
      tc_fence_after();
      float* xl = xch + 128;
      xl[hf * 32 + lane] = l;
      mbar_arrive(pbar);
      const bool got = __all_sync(0xffffffffu, tc_wait(pbar, (uint32_t)n & 1u, a, &s_abort));
      const float lt = got ? l + xl[(hf ^ 1) * 32 + lane] : 0.f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + (((size_t)b * a.T + (rv ? t : 0)) * a.Hq + hq) * D +
                            hf * (D / 2);
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        float o[32];
        tmem_ld32(tOs + lane_off + c * 32, o);
        tmem_wait_ld();
        if (rv && got) {
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
    for (int s = 0; s < 2; ++s) {
      mbar_wait_bounded(&bar_k_full[s], 0u, a.wait_ns, a.status);
      mbar_wait_bounded(&bar_v_full[s], 0u, a.wait_ns, a.status);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Key tiles (128 keys) in which some row of a 256-row group keeps a token: one
// bit per tile, the OR of the rows' top-p bitmask words (of each row only the
// words at or below its position hold bits).
__global__ void __launch_bounds__(256) tile_map_kernel(const __grid_constant__ TcArgs a) {
  __shared__ uint32_t s_map[kMaxTileWords];
  const int bh = blockIdx.y, b = bh / a.NR;
  const int start = a.start_pos[b];
  if (start < 0 || start + a.T > a.Lmax) return;  // uniform
  const int t0 = a.t_base + blockIdx.x * kGroupRows;
  const int t1 = min(a.t_end, t0 + kGroupRows);  // rows [t0, t1)
  const int nw = (start + t1 - 1) / 32 + 1;     // words that can hold bits
  for (int w = threadIdx.x; w < a.map_words; w += 256) s_map[w] = 0u;
  __syncthreads();
  const uint32_t* rows = a.mask + ((size_t)bh * a.mask_rows) * a.words;
  for (int wb = 0; wb < nw; wb += 256) {  // uniform trip count: the shuffles below see every lane
    const int w = wb + threadIdx.x;
    uint32_t acc = 0u;
    if (w < nw) {
      for (int t = max(t0, w * 32 - start); t < t1; ++t) acc |= __ldg(rows + (size_t)(t - a.mask_t0) * a.words + w);
    }
    // a tile is 4 words: lanes 4k .. 4k + 3
    acc |= __shfl_xor_sync(0xffffffffu, acc, 1);
    acc |= __shfl_xor_sync(0xffffffffu, acc, 2);
    const unsigned bal = __ballot_sync(0xffffffffu, acc != 0u && (threadIdx.x & 3) == 0);
    if ((threadIdx.x & 31) == 0 && bal != 0u) {
      uint32_t bits8 = 0u;
#pragma unroll
      for (int k = 0; k < 8; ++k) bits8 |= ((bal >> (4 * k)) & 1u) << k;
      const int tile0 = (wb + (threadIdx.x & ~31)) / 4;  // a multiple of 8
      atomicOr(&s_map[tile0 >> 5], bits8 << (tile0 & 31));
    }
  }
  __syncthreads();
  uint32_t* dst = a.tmap_out + ((size_t)bh * a.map_groups + a.map_g0 + blockIdx.x) * a.map_words;
  for (int w = threadIdx.x; w < a.map_words; w += 256) dst[w] = s_map[w];
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

size_t tile_map_words(const Shape& sh) { return (size_t)((sh.Lmax + kTcKeys - 1) / kTcKeys + 31) / 32; }
size_t tile_map_bytes(const Shape& sh, int T) {
  return (size_t)sh.B * sh.NR * (size_t)((T + kGroupRows - 1) / kGroupRows) * tile_map_words(sh) * sizeof(uint32_t);
}

// Query heads whose keys and values sit in the full-context layout go to the
// tcgen05 kernel (all of them unless local heads keep a ring).  With retrieval
// heads, tile_map_kernel first reduces the rows' bitmask to the key tiles each
// 256-row group keeps (t_base must be a multiple of 256).
int launch_attn_tc(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* start_pos, int T,
                   void* out, const uint32_t* mask, int t_base, int t_end, int mask_t0, int mask_rows,
                   uint32_t* tmap, unsigned long long wait_ns, cudaStream_t st) {
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
  a.tmap = tmap; a.tmap_out = tmap;
  a.map_words = (int)tile_map_words(sh);
  a.map_groups = (T + kGroupRows - 1) / kGroupRows;
  a.map_g0 = t_base / kGroupRows;
  a.wait_ns = wait_ns;
  a.kv = sh.kv;
  for (int i = 0; i < kMaxRetrieval; ++i) a.ret_rank[i] = sh.ret_rank[i];
  for (int i = 0; i < 64; ++i) a.inv_freq[i] = sh.inv_freq[i];
  // retrieval heads first: they attend the most tiles
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
  const int n_groups = (t_end - t_base + kGroupRows - 1) / kGroupRows;
  if (sh.R > 0) tile_map_kernel<<<dim3(n_groups, sh.B * sh.NR), 256, 0, st>>>(a);
  const dim3 grid(n_groups, sh.B * n);
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
