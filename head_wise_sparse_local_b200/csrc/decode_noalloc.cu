// rtp_decode_attn_noalloc: the decode step with its scratch in a fixed,
// library-owned device array, for callers that cannot allocate device memory.
//
// Who needs it: code that runs as a plug-in inside a host framework which owns
// the device memory pool and gives plug-ins no way to allocate; callers on a
// latency-critical path that cannot accept cudaMalloc's implicit device-wide
// synchronisation; small C callers that hold only their input and output
// buffers and have no allocator at hand.  They pass inputs and outputs exactly
// as for rtp_decode_attn; the scratch that rtp_decode_attn takes as
// `workspace` comes from g_decode_scratch below instead.
//
// Costs and rules:
//   * g_decode_scratch (RTP_NOALLOC_SCRATCH_BYTES) is reserved on every GPU
//     that loads this library, for as long as the process lives.
//   * Every call shares that one array.  It keeps whatever the previous call
//     left in it; the decode kernels clear the parts that must start at zero
//     (histograms, counters) themselves on every call.  Calls whose device work
//     overlaps (two streams, two host threads, ...) race on the array and give
//     wrong results: serialise them.
//   * The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make that
//     first call before any stream capture.
//   * Configurations whose scratch does not fit are rejected with
//     RTP_ERR_WORKSPACE before anything is enqueued.
#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace rtp {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[RTP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per
// device).  In host code the symbol names a host-side stand-in, not device
// memory, so only the address returned here may be handed to kernels.
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_error(std::string("rtp_decode_attn_noalloc: cudaGetDevice: ") + cudaGetErrorString(e));
    return RTP_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("rtp_decode_attn_noalloc: device ordinal out of range");
    return RTP_ERR_INVALID;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      set_error(std::string("rtp_decode_attn_noalloc: cudaGetSymbolAddress: ") +
                cudaGetErrorString(e));
      return RTP_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RTP_OK;
}

}  // namespace
}  // namespace rtp

using namespace rtp;

extern "C" int rtp_decode_attn_noalloc(const rtp_layer_cfg* cfg, const rtp_cache* cache,
                                       const void* q_pre, const int* seq_len, int max_seq_len,
                                       const float* w_q, void* out, uint32_t* sel_bitmask,
                                       int* sel_count, void* stream) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  const DecodeLayout lay = decode_layout(sh);
  if (lay.total > (size_t)RTP_NOALLOC_SCRATCH_BYTES) {
    set_error("rtp_decode_attn_noalloc: this configuration needs " + std::to_string(lay.total) +
              " bytes of scratch, more than the fixed " +
              std::to_string((size_t)RTP_NOALLOC_SCRATCH_BYTES) +
              "; use rtp_decode_attn with a caller workspace");
    return RTP_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  if ((rc = scratch_address(&ws)) != RTP_OK) return rc;
  return rtp_decode_attn(cfg, cache, q_pre, seq_len, max_seq_len, w_q, out, sel_bitmask, sel_count,
                         ws, (size_t)RTP_NOALLOC_SCRATCH_BYTES, stream);
}
