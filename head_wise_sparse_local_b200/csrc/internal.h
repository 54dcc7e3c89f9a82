// Host-side declarations shared by the layer's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

#include "rtp.h"

namespace rtp {

void set_error(const std::string& msg);

// One-shot launch tracing (rtp_trace_stage): record the armed start event
// before, and the stop event after, a stage's kernel launch on `st`.
void trace_begin(int stage, cudaStream_t st);
void trace_end(int stage, cudaStream_t st);

struct Shape {
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W;
  float top_p, rope_base;
  int dtype;  // rtp_dtype
  int esize;  // bytes per element
  int ret_head[64];  // rank -> kv head
  int ret_rank[64];  // kv head -> rank or -1
  double inv_freq[64];  // RoPE frequencies base^(-2k/D), k < D/2, fp64 on the host
};

// Validates cfg and fills Shape; returns RTP_OK or an error (message set).
int make_shape(const rtp_layer_cfg* cfg, Shape* sh);

// Decode scratch layout (byte offsets into the workspace).
struct DecodeLayout {
  size_t logits, cmax, mask, ctl, rank_cnt, cand, pm, pl, po, total;
  int nch_score_max, n_sw_tiles, n_tiles_max;
  int n_ctl;  // u32 control words
};
DecodeLayout decode_layout(const Shape& sh);

int launch_append(const Shape& sh, const rtp_cache* cache, const void* k_pre, const void* v_in,
                  const int* start_pos, int T, const float* w_k, cudaStream_t st);

int launch_decode(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* seq_len,
                  int max_seq_len, const float* w_q, void* out, uint32_t* sel_bitmask,
                  int* sel_count, void* ws, const DecodeLayout& lay, cudaStream_t st);

struct PrefillLayout {
  size_t total;
};
PrefillLayout prefill_layout(const Shape& sh, int T);
int launch_prefill(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* start_pos,
                   int T, const float* w_q, void* out, uint32_t* sel_bitmask, float* sel_tau,
                   int* sel_jcut, int* sel_count, void* ws, const PrefillLayout& lay, cudaStream_t st);

}  // namespace rtp
