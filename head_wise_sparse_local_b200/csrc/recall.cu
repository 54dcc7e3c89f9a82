// rtp_decode_recall: attention mass recall of a decode step's selection, a
// diagnostic the pages report for the method (atlas.scime.ai summary,
// "Experimental setup", metrics: attention mass recall).  For every sequence b
// and retrieval query head, the share of the full causal attention's softmax
// mass (over every cached position) that the attended rows carry: the top-p
// set of the bitmask rtp_decode_attn wrote, united with sinks and window.
//
// Two kernels: recall_part_kernel streams the retrieval heads' keys in chunks
// of kChunkR positions, one CTA per (chunk, sequence, retrieval q head), and
// writes (max, sum of weights, sum of attended weights) per chunk, the weights
// 2^(s - max) of the base-2 logits s = RoPE(q) . k log2(e) / sqrt(D);
// recall_merge_kernel combines a head's chunks.
#include "common.cuh"
#include "internal.h"

namespace rtp {
namespace {

constexpr int kRThreads = 256;
constexpr int kChunkR = 2048;

struct RecallArgs {
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W, words, max_seq_len, nch;
  const void* q_pre;
  const void* k;
  const int* seq_len;
  const uint32_t* mask;  // [B][NR][words]
  float* recall;         // [B][NR]
  float* part;           // [B][NR][nch][3]
  int* status;
  KvMap kv;
  int ret_head[kMaxRetrieval];
  double inv_freq[64];
};

template <typename T, int D>
__global__ void __launch_bounds__(kRThreads) recall_part_kernel(const __grid_constant__ RecallArgs a) {
  __shared__ __align__(16) float s_q[D];
  __shared__ float s_red[3][kRThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.NR, rq = bh % a.NR;
  const int r = rq / a.G, g = rq % a.G;
  const int h = a.ret_head[r];
  const int L = a.seq_len[b];
  float* out = a.part + ((size_t)bh * a.nch + chunk) * 3;
  if (L < 1 || L > a.max_seq_len) {  // uniform; the decode call flagged it
    if (tid == 0) { out[0] = -CUDART_INF_F; out[1] = 0.f; out[2] = 0.f; }
    return;
  }
  // RoPE'd query at position L - 1, scaled by log2(e)/sqrt(D)
  const float qscale = 1.4426950408889634f * rsqrtf((float)D);
  for (int k = tid; k < D / 2; k += kRThreads) {
    const T* q = static_cast<const T*>(a.q_pre) + ((size_t)b * a.Hq + h * a.G + g) * D;
    const float x1 = to_f32(q[k]), x2 = to_f32(q[k + D / 2]);
    float c, s;
    rope_cos_sin(L - 1, a.inv_freq[k], c, s);
    s_q[k] = (x1 * c - x2 * s) * qscale;
    s_q[k + D / 2] = (x2 * c + x1 * s) * qscale;
  }
  __syncthreads();
  const int j0 = chunk * kChunkR, j1 = min(L, j0 + kChunkR);
  const uint32_t* mrow = a.mask + (size_t)bh * a.words;
  const int sw0 = max(min(a.S, L), L - a.W);
  const T* kb = static_cast<const T*>(a.k) + a.kv.row(b, h, 0) * D;
  constexpr int PT = kChunkR / kRThreads;
  float sv[PT];
  bool in[PT];
  float mx = -CUDART_INF_F;
#pragma unroll
  for (int u = 0; u < PT; ++u) {
    const int j = j0 + u * kRThreads + tid;
    sv[u] = -CUDART_INF_F;
    in[u] = false;
    if (j < j1) {
      float kv[D];
      load_row<T, D>(kb + (size_t)j * D, kv);
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) acc = fmaf(s_q[d], kv[d], acc);
      sv[u] = acc;
      in[u] = j < a.S || j >= sw0 || ((__ldg(mrow + (j >> 5)) >> (j & 31)) & 1u);
      mx = fmaxf(mx, acc);
    }
  }
  mx = warp_max(mx);
  if (lane == 0) s_red[0][warp] = mx;
  __syncthreads();
  float m = s_red[0][0];
#pragma unroll
  for (int w = 1; w < kRThreads / 32; ++w) m = fmaxf(m, s_red[0][w]);
  float z = 0.f, zs = 0.f;
  if (m != -CUDART_INF_F) {
#pragma unroll
    for (int u = 0; u < PT; ++u) {
      if (sv[u] == -CUDART_INF_F) continue;
      const float e = exp2f(sv[u] - m);
      z += e;
      if (in[u]) zs += e;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    z += __shfl_xor_sync(0xffffffffu, z, o);
    zs += __shfl_xor_sync(0xffffffffu, zs, o);
  }
  __syncthreads();
  if (lane == 0) { s_red[1][warp] = z; s_red[2][warp] = zs; }
  __syncthreads();
  if (tid == 0) {
    float zt = 0.f, zst = 0.f;
#pragma unroll
    for (int w = 0; w < kRThreads / 32; ++w) { zt += s_red[1][w]; zst += s_red[2][w]; }
    out[0] = m;
    out[1] = zt;
    out[2] = zst;
  }
}

__global__ void __launch_bounds__(32) recall_merge_kernel(const __grid_constant__ RecallArgs a) {
  const int bh = blockIdx.x, lane = threadIdx.x;
  const int b = bh / a.NR;
  const int L = a.seq_len[b];
  if (L < 1 || L > a.max_seq_len) return;
  const int nch = (L + kChunkR - 1) / kChunkR;
  const float* p = a.part + (size_t)bh * a.nch * 3;
  float m = -CUDART_INF_F;
  for (int c = lane; c < nch; c += 32) m = fmaxf(m, p[c * 3]);
  m = warp_max(m);
  float z = 0.f, zs = 0.f;
  for (int c = lane; c < nch; c += 32) {
    const float mc = p[c * 3];
    if (mc == -CUDART_INF_F) continue;
    const float sc = exp2f(mc - m);
    z = fmaf(p[c * 3 + 1], sc, z);
    zs = fmaf(p[c * 3 + 2], sc, zs);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    z += __shfl_xor_sync(0xffffffffu, z, o);
    zs += __shfl_xor_sync(0xffffffffu, zs, o);
  }
  if (lane == 0) a.recall[bh] = z > 0.f ? zs / z : 0.f;
}

}  // namespace

size_t recall_workspace_bytes(const Shape& sh) {
  const size_t nch = (size_t)(sh.Lmax + kChunkR - 1) / kChunkR;
  return (size_t)sh.B * sh.NR * nch * 3 * sizeof(float);
}

int launch_recall(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* seq_len,
                  int max_seq_len, const uint32_t* sel_bitmask, float* recall, void* ws, cudaStream_t st) {
  if (sh.R == 0) return RTP_OK;
  RecallArgs a;
  a.B = sh.B; a.Hq = sh.Hq; a.Hkv = sh.Hkv; a.G = sh.G; a.D = sh.D; a.R = sh.R; a.NR = sh.NR;
  a.Lmax = sh.Lmax; a.S = sh.S; a.W = sh.W; a.words = (sh.Lmax + 31) / 32;
  a.max_seq_len = max_seq_len > 0 ? max_seq_len : sh.Lmax;
  a.nch = (a.max_seq_len + kChunkR - 1) / kChunkR;
  a.q_pre = q_pre; a.k = cache->k; a.seq_len = seq_len; a.mask = sel_bitmask; a.recall = recall;
  a.part = static_cast<float*>(ws);
  a.status = cache->status;
  a.kv = sh.kv;
  for (int i = 0; i < kMaxRetrieval; ++i) a.ret_head[i] = sh.ret_head[i];
  for (int i = 0; i < 64; ++i) a.inv_freq[i] = sh.inv_freq[i];
  const dim3 grid(a.nch, sh.B * sh.NR);
  if (sh.dtype == RTP_BF16) {
    if (sh.D == 128) recall_part_kernel<__nv_bfloat16, 128><<<grid, kRThreads, 0, st>>>(a);
    else recall_part_kernel<__nv_bfloat16, 64><<<grid, kRThreads, 0, st>>>(a);
  } else {
    if (sh.D == 128) recall_part_kernel<float, 128><<<grid, kRThreads, 0, st>>>(a);
    else recall_part_kernel<float, 64><<<grid, kRThreads, 0, st>>>(a);
  }
  recall_merge_kernel<<<sh.B * sh.NR, 32, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("recall launch: ") + cudaGetErrorString(e));
    return RTP_ERR_CUDA;
  }
  return RTP_OK;
}

}  // namespace rtp
