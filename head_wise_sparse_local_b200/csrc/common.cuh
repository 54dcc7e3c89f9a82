// Device helpers shared by the layer's kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "rtp.h"

namespace rtp {

// Score scale 1/sqrt(d) for the indexer widths the layer takes: d = 16 and the
// pages' ablation widths 4, 8, 32 (atlas.scime.ai summary, "Surprising
// findings"); exact for 4 and 16, rounded to fp32 for 8 and 32.
template <int IDX>
__host__ __device__ constexpr float idx_scale() {
  static_assert(IDX == 4 || IDX == 8 || IDX == 16 || IDX == 32, "indexer width");
  return IDX == 4 ? 0.5f : IDX == 8 ? 0.35355339059327376f : IDX == 16 ? 0.25f : 0.17677669529663688f;
}
constexpr int kMaxRetrieval = 64;

// ---------------------------------------------------------------------------
// element IO
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }

// Load N contiguous elements (N * sizeof(T) a multiple of 16 bytes, 16-byte
// aligned) and widen to fp32.
template <typename T, int N>
__device__ __forceinline__ void load_row(const T* __restrict__ p, float (&out)[N]) {
  static_assert((N * sizeof(T)) % 16 == 0, "row slice must be whole 16-byte vectors");
  constexpr int kVec = (N * sizeof(T)) / 16;
  const uint4* v = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    uint4 u = __ldg(v + i);
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float2 f = __bfloat1622float2(h[k]);
        out[i * 8 + 2 * k] = f.x;
        out[i * 8 + 2 * k + 1] = f.y;
      }
    } else {
      out[i * 4 + 0] = __uint_as_float(u.x);
      out[i * 4 + 1] = __uint_as_float(u.y);
      out[i * 4 + 2] = __uint_as_float(u.z);
      out[i * 4 + 3] = __uint_as_float(u.w);
    }
  }
}

// Raw 16-byte vector loads of N elements (kept packed, for software pipelining).
template <typename T, int N>
struct RawRow {
  static constexpr int kVec = (N * sizeof(T)) / 16;
  uint4 v[kVec];
  __device__ __forceinline__ void load(const T* __restrict__ p) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < kVec; ++i) v[i] = __ldg(q + i);
  }
  __device__ __forceinline__ float get(int i) const {  // i must be a compile-time index after unrolling
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(v);
      return __bfloat162float(h[i]);
    } else {
      const float* f = reinterpret_cast<const float*>(v);
      return f[i];
    }
  }
};

// ---------------------------------------------------------------------------
// score ordering for top-p
// ---------------------------------------------------------------------------
// Order-preserving 32-bit key of a (non-NaN, canonical-zero) fp32 score:
// key(a) < key(b)  <=>  a < b.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// First-level histogram bucket of a score: 2048 buckets, monotone
// non-decreasing in s.  Per sign: 16 octaves |s| in [2^-6, 2^10) with 64
// sub-buckets each; smaller magnitudes share the innermost bucket and larger
// ones the outermost.
constexpr int kNumBuckets = 2048;
constexpr int kBucketELo = 121;  // biased exponent of 2^-6
__device__ __forceinline__ int score_bucket(float s) {
  const uint32_t u = __float_as_uint(s);
  const uint32_t mag = u & 0x7fffffffu;
  const int e = int(mag >> 23);
  int t;
  if (e < kBucketELo) t = 0;
  else if (e > kBucketELo + 15) t = 1023;
  else t = (e - kBucketELo) * 64 + int((mag >> 17) & 63u);
  return (u >> 31) ? 1023 - t : 1024 + t;
}

// Softmax mass of score s relative to the row maximum m, in 2^-36 fixed point:
// x = 2^((s - m) log2(e)) * 2^36 from the hardware base-2 exponential, rounded
// to the nearest integer.  Decode and prefill use this one definition, so their
// integer sums (exact and order independent), and with them their selections,
// agree bit for bit.  x rounds to 0 below s - m = -25.65.
__device__ __forceinline__ float mass_x36(float s, float m) {
  const float t = (s - m) * 1.4426950408889634f;
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(t));
  return e * 68719476736.0f;  // 2^36
}
__device__ __forceinline__ unsigned long long mass36(float s, float m) {
  return __float2ull_rn(mass_x36(s, m));
}

// ---------------------------------------------------------------------------
// reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive warp scan of u64.
__device__ __forceinline__ unsigned long long warp_incl_scan_u64(unsigned long long v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}
__device__ __forceinline__ unsigned warp_incl_scan_u32(unsigned v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive block scan (u64 and u32 together) for blockDim.x == kThreads.
// `sm` needs 2 * (kThreads / 32) slots of each type.
template <int kThreads>
__device__ __forceinline__ void block_excl_scan2(unsigned long long a, unsigned c,
                                                 unsigned long long& a_ex, unsigned& c_ex,
                                                 unsigned long long& a_tot, unsigned& c_tot,
                                                 unsigned long long* sm_a, unsigned* sm_c) {
  constexpr int kWarps = kThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long ai = warp_incl_scan_u64(a);
  unsigned ci = warp_incl_scan_u32(c);
  if (lane == 31) { sm_a[warp] = ai; sm_c[warp] = ci; }
  __syncthreads();
  unsigned long long wa = 0, ta = 0;
  unsigned wc = 0, tc = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) { wa += sm_a[w]; wc += sm_c[w]; }
    ta += sm_a[w];
    tc += sm_c[w];
  }
  a_ex = wa + ai - a;
  c_ex = wc + ci - c;
  a_tot = ta;
  c_tot = tc;
  __syncthreads();
}

// RoPE angle pos * inv_freq (inv_freq = base^(-2k/D), computed in fp64 on the
// host), reduced to [-pi, pi] in fp64 before the fp32 sincos so that positions
// up to 2^23 keep full fp32 accuracy.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float& c, float& s) {
  const double th = (double)pos * inv_freq;
  const double two_pi = 6.283185307179586476925286766559;
  const double r = th - two_pi * rint(th * 0.15915494309189533577);  // any integer multiple works
  sincosf((float)r, &s, &c);
}

// Loads of data read once per call (the key and value streams): L2
// evict-first, so they do not push code and reused data out of L2; L1 bypass.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
template <typename V>
__device__ __forceinline__ V ld_stream(const V* ptr, uint64_t pol);
template <>
__device__ __forceinline__ uint4 ld_stream<uint4>(const uint4* ptr, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.cg.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(ptr), "l"(pol));
  return v;
}
template <>
__device__ __forceinline__ uint2 ld_stream<uint2>(const uint2* ptr, uint64_t pol) {
  uint2 v;
  asm volatile("ld.global.cg.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;" : "=r"(v.x), "=r"(v.y) : "l"(ptr), "l"(pol));
  return v;
}
template <>
__device__ __forceinline__ unsigned ld_stream<unsigned>(const unsigned* ptr, uint64_t pol) {
  unsigned v;
  asm volatile("ld.global.cg.L2::cache_hint.u32 %0, [%1], %2;" : "=r"(v) : "l"(ptr), "l"(pol));
  return v;
}

// ---------------------------------------------------------------------------
// warp-level tensor-core helpers (mma.sync m16n8k16 bf16, fp32 accumulate)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(unsigned& r0, unsigned& r1, unsigned& r2, unsigned& r3, const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void ldsm_x2(unsigned& r0, unsigned& r1, const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(a));
}
__device__ __forceinline__ void ldsm_x2_t(unsigned& r0, unsigned& r1, const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(a));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3,
                                         unsigned b0, unsigned b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ unsigned pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const unsigned*>(&v);
}

// Indexer scores on tensor cores (decode and prefill share these, so a prefill
// row and the decode step at its position compute bit-identical scores).
// S = K~ Q~^T by m16n8k16 products: the M side is 16 keys, the K side the
// indexer dims in steps of 16 (dims past d read as zero), the N side 8 query
// columns; q~ enters as a bf16 high part and a bf16 low part, all high steps
// accumulated before the low ones into one fp32 accumulator.
template <int IDX>
struct IdxMma {
  static constexpr int KS = (IDX + 15) / 16;  // k-steps of 16 dims
  static constexpr int KB = IDX * 2;          // bytes per bf16 key
  unsigned bh[KS][2], bl[KS][2];

  // B fragments from the fp32 q~ of this lane's column (lane / 4), `q`
  // pointing at its IDX values, or nullptr for a column with no query.
  __device__ __forceinline__ void set_q(const float* q, int lane) {
    const int t4 = lane & 3;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      float hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int d = ks * 16 + 2 * t4 + (e & 1) + (e >> 1) * 8;
        const float v = (q != nullptr && d < IDX) ? q[d] : 0.f;
        hi[e] = __bfloat162float(__float2bfloat16_rn(v));
        lo[e] = v - hi[e];
      }
      bh[ks][0] = pack_bf16(hi[0], hi[1]);
      bh[ks][1] = pack_bf16(hi[2], hi[3]);
      bl[ks][0] = pack_bf16(lo[0], lo[1]);
      bl[ks][1] = pack_bf16(lo[2], lo[3]);
    }
  }

  // Accumulators c[4] of the 16 keys starting at `tile` (shared memory, KB
  // bytes per key, 16-byte aligned): c[0], c[1] key lane/4, columns 2 (lane%4)
  // and 2 (lane%4) + 1; c[2], c[3] key lane/4 + 8.
  __device__ __forceinline__ void scores(const unsigned char* tile, int lane, float (&c)[4]) const {
    unsigned a[KS][4];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      if constexpr (IDX >= 16) {
        ldsm_x4(a[ks][0], a[ks][1], a[ks][2], a[ks][3],
                tile + (size_t)((lane & 7) + ((lane >> 3) & 1) * 8) * KB + ks * 32 + (lane >> 4) * 16);
      } else if constexpr (IDX == 8) {
        ldsm_x2(a[ks][0], a[ks][1], tile + (size_t)((lane & 7) + ((lane >> 3) & 1) * 8) * KB);
        a[ks][2] = 0u;
        a[ks][3] = 0u;
      } else {  // 8-byte keys: dims 2 t4, 2 t4 + 1 for t4 < 2, by plain 4-byte loads
        const int gq = lane >> 2, t4 = lane & 3;
        a[ks][0] = t4 < 2 ? *reinterpret_cast<const unsigned*>(tile + gq * KB + t4 * 4) : 0u;
        a[ks][1] = t4 < 2 ? *reinterpret_cast<const unsigned*>(tile + (gq + 8) * KB + t4 * 4) : 0u;
        a[ks][2] = 0u;
        a[ks][3] = 0u;
      }
    }
    c[0] = c[1] = c[2] = c[3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) mma_bf16(c, a[ks][0], a[ks][1], a[ks][2], a[ks][3], bh[ks][0], bh[ks][1]);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) mma_bf16(c, a[ks][0], a[ks][1], a[ks][2], a[ks][3], bl[ks][0], bl[ks][1]);
  }
};

__device__ __forceinline__ void ldsm_x4_t(unsigned& r0, unsigned& r1, unsigned& r2, unsigned& r3, const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}

// ---------------------------------------------------------------------------
// mbarriers and bulk asynchronous copies (TMA, non-tensor form)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// One thread initialises; a CTA barrier must follow before any use.
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive (the barrier's one expected arrival) and add `bytes` to the
// transaction count the current phase waits for.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// One arrival on `bar` (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

// Global -> shared bulk copy of `bytes` (a multiple of 16; both addresses
// 16-byte aligned) completing on `bar`, with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol) : "memory");
}

// 16-byte global -> shared copy (L1 bypass) with an L2 cache policy.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;"
               :: "r"(smem_u32(dst)), "l"(src), "l"(pol) : "memory");
}

// One arrival on `bar`, made once every cp.async this thread has issued so far
// has landed; it counts toward the barrier's expected arrivals.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.b32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread until the phase completes or `hint_ns`
// elapses, whichever is first: a waiting warp sleeps instead of spinning (and
// taking issue slots from the warps that work).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.b32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns) : "memory");
  return ok != 0;
}
constexpr uint32_t kWaitHintNs = 1000000;  // a waiting thread re-checks its time limit at least every 1 ms

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of `bar` to complete, for at most `limit_ns`; on
// expiry OR RTP_DEV_TIMEOUT into *status and return false (never hangs).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                                  int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait_sleep(bar, parity, kWaitHintNs)) {
    if (global_ns() - t0 > limit_ns) {
      atomicOr(status, RTP_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Programmatic dependent launch: a kernel launched with launch_pdl may start
// while its predecessor on the stream is still running.  griddep_wait() blocks
// until the predecessor grid has completed and its memory is visible;
// griddep_launch() lets the successor grid start launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

template <typename Args>
inline cudaError_t launch_pdl(void (*k)(Args), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              const Args& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, a);
}

}  // namespace rtp
