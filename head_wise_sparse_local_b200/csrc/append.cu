// rtp_append_kv: RoPE'd key, value and d-dim pre-RoPE indexer key per token.
//
// One warp per (sequence, token, KV head) row.  Lane l owns the RoPE pairs
// (k, k + D/2) for k in [l*PP, (l+1)*PP), PP = D/64, so the rotation needs no
// shuffle.  Retrieval heads also project the pre-RoPE key through W_k^(r)
// ("pre-RoPE low-dimensional projection", atlas.scime.ai summary, "Approach"):
// each lane forms partial dot products over its dims and a butterfly reduction
// gives every lane the same d sums (d = 4, 8, 16 or 32).
#include "common.cuh"
#include "internal.h"

namespace rtp {
namespace {

struct AppendArgs {
  int B, T, Hkv, D, Lmax, Lk, R;
  float rope_base;
  const void* k_pre;
  const void* v_in;
  const int* start_pos;
  const float* w_k;
  void* k;
  void* v;
  void* kidx;
  int* status;
  KvMap kv;
  int ret_rank[kMaxRetrieval];
  double inv_freq[64];
};

template <typename T, int D, int IDX>
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendArgs a) {
  // The inputs (k_pre, v, start_pos, W_k) are read and the rotated key and the
  // indexer key formed before waiting for the previous kernel on the stream;
  // only the cache stores wait (a decode step still running may read the cache).
  griddep_launch();
  constexpr int PP = D / 64;  // pairs per lane
  constexpr int H = D / 2;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long long n_rows = (long long)a.B * a.T * a.Hkv;
  if (row >= n_rows) return;
  const int h = int(row % a.Hkv);
  const int t = int((row / a.Hkv) % a.T);
  const int b = int(row / ((long long)a.Hkv * a.T));
  const int s0 = a.start_pos[b];
  const int pos = s0 + t;
  if (pos < 0 || pos >= a.Lmax) {
    if (lane == 0) atomicOr(a.status, RTP_DEV_POSITION);
    return;
  }
  // A local head in ring mode keeps the sinks and the last `ring` positions:
  // an earlier position of this call whose slot a later one takes is skipped
  // (two writes to one slot in one launch would race).
  const bool ringed = (a.kv.ring_mask >> h) & 1ull;
  if (ringed && pos >= a.kv.S && pos < s0 + a.T - a.kv.ring) return;
  const T* kp = static_cast<const T*>(a.k_pre) + row * D;
  const T* vp = static_cast<const T*>(a.v_in) + row * D;
  float x1[PP], x2[PP];
  T v1[PP], v2[PP];
#pragma unroll
  for (int i = 0; i < PP; ++i) {
    const int k = lane * PP + i;
    x1[i] = to_f32(kp[k]);
    x2[i] = to_f32(kp[k + H]);
    v1[i] = vp[k];
    v2[i] = vp[k + H];
  }
  T y1[PP], y2[PP];
#pragma unroll
  for (int i = 0; i < PP; ++i) {
    const int k = lane * PP + i;
    float c, s;
    rope_cos_sin(pos, a.inv_freq[k], c, s);
    y1[i] = from_f32<T>(x1[i] * c - x2[i] * s);
    y2[i] = from_f32<T>(x2[i] * c + x1[i] * s);
  }
  const int r = a.ret_rank[h];
  float acc[IDX];
  if (r >= 0) {  // warp-uniform
    const float* w = a.w_k + (size_t)r * IDX * D;
#pragma unroll
    for (int i = 0; i < IDX; ++i) {
      float sacc = 0.f;
#pragma unroll
      for (int p = 0; p < PP; ++p) {
        const int k = lane * PP + p;
        sacc = fmaf(__ldg(w + i * D + k), x1[p], sacc);
        sacc = fmaf(__ldg(w + i * D + k + H), x2[p], sacc);
      }
      acc[i] = sacc;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int i = 0; i < IDX; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    }
  }
  griddep_wait();
  const size_t dst = a.kv.row(b, h, pos) * D;
  T* ko = static_cast<T*>(a.k) + dst;
  T* vo = static_cast<T*>(a.v) + dst;
#pragma unroll
  for (int i = 0; i < PP; ++i) {
    const int k = lane * PP + i;
    ko[k] = y1[i];
    ko[k + H] = y2[i];
    vo[k] = v1[i];
    vo[k + H] = v2[i];
  }
  if (r >= 0) {
    T* ki = static_cast<T*>(a.kidx) + (((size_t)b * a.R + r) * a.Lk + pos) * IDX;
#pragma unroll
    for (int i = 0; i < IDX; ++i)
      if (lane == i) ki[i] = from_f32<T>(acc[i]);
  }
}

template <typename T, int D>
cudaError_t launch_append_idx(int idx, unsigned grid, cudaStream_t st, const AppendArgs& a) {
  switch (idx) {
    case 4: return launch_pdl(append_kernel<T, D, 4>, dim3(grid), dim3(256), 0, st, a);
    case 8: return launch_pdl(append_kernel<T, D, 8>, dim3(grid), dim3(256), 0, st, a);
    case 32: return launch_pdl(append_kernel<T, D, 32>, dim3(grid), dim3(256), 0, st, a);
    default: return launch_pdl(append_kernel<T, D, 16>, dim3(grid), dim3(256), 0, st, a);
  }
}

}  // namespace

int launch_append(const Shape& sh, const rtp_cache* cache, const void* k_pre, const void* v_in,
                  const int* start_pos, int T, const float* w_k, cudaStream_t st) {
  AppendArgs a;
  a.B = sh.B; a.T = T; a.Hkv = sh.Hkv; a.D = sh.D; a.Lmax = sh.Lmax; a.Lk = sh.Lk; a.R = sh.R;
  a.rope_base = sh.rope_base;
  a.k_pre = k_pre; a.v_in = v_in; a.start_pos = start_pos; a.w_k = w_k;
  a.k = cache->k; a.v = cache->v; a.kidx = cache->kidx; a.status = cache->status;
  a.kv = sh.kv;
  for (int i = 0; i < kMaxRetrieval; ++i) a.ret_rank[i] = sh.ret_rank[i];
  for (int i = 0; i < 64; ++i) a.inv_freq[i] = sh.inv_freq[i];
  const long long rows = (long long)sh.B * T * sh.Hkv;
  if (rows == 0) return RTP_OK;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  trace_begin(RTP_STAGE_APPEND, st);
  cudaError_t e;
  if (sh.dtype == RTP_BF16) {
    if (sh.D == 128) e = launch_append_idx<__nv_bfloat16, 128>(sh.idx, grid, st, a);
    else e = launch_append_idx<__nv_bfloat16, 64>(sh.idx, grid, st, a);
  } else {
    if (sh.D == 128) e = launch_append_idx<float, 128>(sh.idx, grid, st, a);
    else e = launch_append_idx<float, 64>(sh.idx, grid, st, a);
  }
  trace_end(RTP_STAGE_APPEND, st);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("append launch: ") + cudaGetErrorString(e));
    return RTP_ERR_CUDA;
  }
  return RTP_OK;
}

}  // namespace rtp
