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

// Where row `pos` of KV head h of sequence b sits in the K and V buffers.
// Per sequence the heads are stored one after another, head h taking
// cap(h) rows starting at row0[h]: the whole context (Lmax rows) for
// retrieval heads, and for local heads either the whole context as well or,
// in ring mode, the S sinks followed by a ring of `ring` window rows (position
// pos >= S in slot S + (pos - S) mod ring).  Plain data, passed to kernels.
struct KvMap {
  long long rows_per_seq;
  int row0[64];
  uint64_t ring_mask;  // bit h: head h keeps sinks + a window ring
  int ring, S;
#ifdef __CUDACC__
  __host__ __device__ __forceinline__ size_t row(int b, int h, int pos) const {
    int slot = pos;
    if ((ring_mask >> h) & 1ull) slot = pos < S ? pos : S + (pos - S) % ring;
    return (size_t)b * (size_t)rows_per_seq + (size_t)row0[h] + (size_t)slot;
  }
#endif
};

struct Shape {
  int B, Hq, Hkv, G, D, R, NR, Lmax, S, W;
  int ring;          // window rows a local head keeps in ring mode (0: whole context)
  int top_k;         // > 0: retrieval heads keep a fixed k tokens (static top-k) instead of top-p
  int idx;           // indexer width d (4, 8, 16 or 32)
  int Lk;            // indexer-key rows per (sequence, retrieval head) block of the kidx cache
  KvMap kv;
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
  size_t logits, cmax, mask, cand, sw_scratch, sel_scratch, total;
  int nch_score_max;
};
DecodeLayout decode_layout(const Shape& sh);

// Test hook behind rtp_debug_wait_expiry: the next decode call on this host
// thread waits on copy barriers that expect bytes that never come, giving up
// after `polls` x 100 ns.
void arm_wait_expiry(int polls);

int launch_append(const Shape& sh, const rtp_cache* cache, const void* k_pre, const void* v_in,
                  const int* start_pos, int T, const float* w_k, cudaStream_t st);

int launch_decode(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* seq_len,
                  int max_seq_len, const float* w_q, void* out, uint32_t* sel_bitmask,
                  int* sel_count, void* ws, const DecodeLayout& lay, cudaStream_t st);

size_t recall_workspace_bytes(const Shape& sh);
int launch_recall(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* seq_len,
                  int max_seq_len, const uint32_t* sel_bitmask, float* recall, void* ws, cudaStream_t st);

struct PrefillLayout {
  size_t total;
  size_t tmap;     // offset of the attention's key-tile map
  int block_rows;  // query rows per selection + attention pass (a multiple of 256 unless the whole chunk)
};
size_t tile_map_bytes(const Shape& sh, int T);
PrefillLayout prefill_layout(const Shape& sh, int T);
int launch_attn_tc(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* start_pos, int T,
                   void* out, const uint32_t* mask, int t_base, int t_end, int mask_t0, int mask_rows,
                   uint32_t* tmap, unsigned long long wait_ns, cudaStream_t st);
int launch_prefill(const Shape& sh, const rtp_cache* cache, const void* q_pre, const int* start_pos,
                   int T, const float* w_q, void* out, uint32_t* sel_bitmask, float* sel_tau,
                   int* sel_jcut, int* sel_count, void* ws, const PrefillLayout& lay, cudaStream_t st);

}  // namespace rtp
