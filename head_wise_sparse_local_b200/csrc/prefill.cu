// rtp_prefill_attn: causal prefill chunk (work in progress).
#include "common.cuh"
#include "internal.h"

namespace rtp {

PrefillLayout prefill_layout(const Shape& sh, int T) {
  PrefillLayout l;
  (void)sh;
  (void)T;
  l.total = 256;
  return l;
}

int launch_prefill(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* start_pos,
                   int T, const float* w_q, void* out, float* sel_tau, int* sel_jcut,
                   int* sel_count, void* ws, const PrefillLayout& lay, cudaStream_t st) {
  (void)sh; (void)cache; (void)q_pre; (void)start_pos; (void)T; (void)w_q; (void)out;
  (void)sel_tau; (void)sel_jcut; (void)sel_count; (void)ws; (void)lay; (void)st;
  set_error("rtp_prefill_attn: not built yet");
  return RTP_ERR_SHAPE;
}

}  // namespace rtp
