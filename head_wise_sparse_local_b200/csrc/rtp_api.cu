// C ABI of the layer (include/rtp.h): argument validation, buffer sizes and
// dispatch to the kernels.  No allocation, no synchronisation, no state beyond
// a thread-local error message.
#include <cstdint>
#include <cstring>
#include <string>

#include <cmath>
#include "internal.h"

namespace rtp {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

struct TraceSlot {
  cudaEvent_t start = nullptr, stop = nullptr;
  bool started = false;
};
static thread_local TraceSlot g_trace[RTP_STAGE_COUNT];

void trace_begin(int stage, cudaStream_t st) {
  TraceSlot& t = g_trace[stage];
  if (!t.start || t.started) return;
  cudaEventRecord(t.start, st);
  t.started = true;
}

void trace_end(int stage, cudaStream_t st) {
  TraceSlot& t = g_trace[stage];
  if (!t.started) return;
  cudaEventRecord(t.stop, st);
  t = TraceSlot();
}

static int fail(int code, const std::string& msg) {
  set_error(msg);
  return code;
}

int make_shape(const rtp_layer_cfg* cfg, Shape* sh) {
  if (!cfg) return fail(RTP_ERR_INVALID, "cfg is NULL");
  if (cfg->dtype != RTP_BF16 && cfg->dtype != RTP_FP32)
    return fail(RTP_ERR_DTYPE, "dtype must be RTP_BF16 or RTP_FP32");
  if (cfg->batch < 1 || cfg->n_q_heads < 1 || cfg->n_kv_heads < 1)
    return fail(RTP_ERR_SHAPE, "batch and head counts must be >= 1");
  if (cfg->n_kv_heads > 64) return fail(RTP_ERR_SHAPE, "at most 64 KV heads");
  if (cfg->n_q_heads % cfg->n_kv_heads != 0)
    return fail(RTP_ERR_SHAPE, "n_q_heads must be a multiple of n_kv_heads");
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(RTP_ERR_SHAPE, "group size n_q_heads/n_kv_heads must be 1, 2, 4 or 8");
  if (cfg->head_dim != 64 && cfg->head_dim != 128)
    return fail(RTP_ERR_SHAPE, "head_dim must be 64 or 128");
  if (cfg->idx_dim != 4 && cfg->idx_dim != 8 && cfg->idx_dim != 16 && cfg->idx_dim != 32)
    return fail(RTP_ERR_SHAPE, "idx_dim must be 4, 8, 16 or 32");
  if (cfg->max_ctx < 1 || cfg->max_ctx > (1 << 23))
    return fail(RTP_ERR_SHAPE, "max_ctx must be in [1, 2^23]");
  if (cfg->n_sink < 0) return fail(RTP_ERR_INVALID, "n_sink must be >= 0");
  if (cfg->window < 1) return fail(RTP_ERR_INVALID, "window must be >= 1");
  if (!(cfg->top_p > 0.0f) || !(cfg->top_p <= 1.0f))
    return fail(RTP_ERR_INVALID, "top_p must be in (0, 1]");
  if (!(cfg->rope_base > 1.0f)) return fail(RTP_ERR_INVALID, "rope_base must be > 1");
  if (cfg->n_kv_heads < 64 && (cfg->retrieval_mask >> cfg->n_kv_heads) != 0ull)
    return fail(RTP_ERR_SHAPE, "retrieval_mask names a KV head >= n_kv_heads");
  sh->B = cfg->batch;
  sh->Hq = cfg->n_q_heads;
  sh->Hkv = cfg->n_kv_heads;
  sh->G = G;
  sh->D = cfg->head_dim;
  sh->Lmax = cfg->max_ctx;
  sh->S = cfg->n_sink;
  sh->W = cfg->window;
  sh->top_p = cfg->top_p;
  sh->rope_base = cfg->rope_base;
  sh->dtype = cfg->dtype;
  sh->esize = cfg->dtype == RTP_BF16 ? 2 : 4;
  sh->idx = cfg->idx_dim;
  // an indexer-key block of (sequence, retrieval head) starts on a 16-byte
  // boundary: 8-byte rows (bf16, d = 4) take an even number of rows
  sh->Lk = sh->idx * sh->esize < 16 ? (sh->Lmax + 1) & ~1 : sh->Lmax;
  int r = 0;
  for (int h = 0; h < 64; ++h) {
    sh->ret_rank[h] = -1;
    sh->ret_head[h] = -1;
  }
  for (int h = 0; h < sh->Hkv; ++h) {
    if ((cfg->retrieval_mask >> h) & 1ull) {
      sh->ret_rank[h] = r;
      sh->ret_head[r] = h;
      ++r;
    }
  }
  sh->R = r;
  sh->NR = r * G;
  if (cfg->local_cap < 0) return fail(RTP_ERR_INVALID, "local_cap must be >= 0");
  if (cfg->top_k < 0) return fail(RTP_ERR_INVALID, "top_k must be >= 0");
  sh->top_k = cfg->top_k;
  if (cfg->local_cap > 0 && cfg->local_cap < cfg->window)
    return fail(RTP_ERR_SHAPE, "local_cap must be 0 or at least the window");
  // ring mode only when it actually saves rows
  sh->ring = (cfg->local_cap > 0 && (long long)sh->S + cfg->local_cap < (long long)sh->Lmax) ? cfg->local_cap : 0;
  sh->kv.ring = sh->ring > 0 ? sh->ring : 1;
  sh->kv.S = sh->S;
  sh->kv.ring_mask = 0ull;
  long long rows = 0;
  for (int h = 0; h < 64; ++h) sh->kv.row0[h] = 0;
  for (int h = 0; h < sh->Hkv; ++h) {
    sh->kv.row0[h] = (int)rows;
    const bool ring = sh->ring > 0 && sh->ret_rank[h] < 0;
    if (ring) sh->kv.ring_mask |= 1ull << h;
    rows += ring ? (long long)sh->S + sh->ring : sh->Lmax;
  }
  if (rows > INT32_MAX) return fail(RTP_ERR_SHAPE, "cache rows per sequence exceed 2^31");
  sh->kv.rows_per_seq = rows;
  for (int k = 0; k < 64; ++k)
    sh->inv_freq[k] = k < sh->D / 2 ? std::pow((double)sh->rope_base, -2.0 * k / (double)sh->D) : 0.0;
  return RTP_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_cache(const Shape& sh, const rtp_cache* c) {
  if (!c) return fail(RTP_ERR_INVALID, "cache is NULL");
  if (!c->k || !c->v || !c->status) return fail(RTP_ERR_INVALID, "cache k/v/status is NULL");
  if (sh.R > 0 && !c->kidx) return fail(RTP_ERR_INVALID, "cache kidx is NULL with retrieval heads");
  if (!aligned16(c->k) || !aligned16(c->v) || (c->kidx && !aligned16(c->kidx)))
    return fail(RTP_ERR_INVALID, "cache buffers must be 16-byte aligned");
  return RTP_OK;
}

}  // namespace rtp

using namespace rtp;

extern "C" {

const char* rtp_last_error(void) { return g_last_error.c_str(); }

const char* rtp_version(void) { return "rtp 0.1 sm_100a"; }

int rtp_trace_stage(int stage, void* start_event, void* stop_event) {
  if (stage < 0 || stage >= RTP_STAGE_COUNT) return fail(RTP_ERR_INVALID, "unknown stage");
  TraceSlot& t = g_trace[stage];
  t = TraceSlot();
  if (start_event && stop_event) {
    t.start = static_cast<cudaEvent_t>(start_event);
    t.stop = static_cast<cudaEvent_t>(stop_event);
  }
  return RTP_OK;
}

int rtp_debug_wait_expiry(int polls) {
  arm_wait_expiry(polls > 0 ? polls : 0);
  return RTP_OK;
}

int rtp_cache_bytes(const rtp_layer_cfg* cfg, size_t* k_bytes, size_t* v_bytes,
                    size_t* kidx_bytes) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  const size_t kv = (size_t)sh.B * (size_t)sh.kv.rows_per_seq * sh.D * sh.esize;
  if (k_bytes) *k_bytes = kv;
  if (v_bytes) *v_bytes = kv;
  if (kidx_bytes) *kidx_bytes = (size_t)sh.B * sh.R * sh.Lk * sh.idx * sh.esize;
  return RTP_OK;
}

int rtp_decode_workspace_bytes(const rtp_layer_cfg* cfg, size_t* bytes) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  if (!bytes) return fail(RTP_ERR_INVALID, "bytes is NULL");
  *bytes = decode_layout(sh).total;
  return RTP_OK;
}

int rtp_prefill_workspace_bytes(const rtp_layer_cfg* cfg, int T, size_t* bytes) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  if (!bytes) return fail(RTP_ERR_INVALID, "bytes is NULL");
  if (T < 1 || T > sh.Lmax) return fail(RTP_ERR_SHAPE, "T must be in [1, max_ctx]");
  *bytes = prefill_layout(sh, T).total;
  return RTP_OK;
}

int rtp_append_kv(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* k_pre,
                  const void* v_in, const int* start_pos, int T, const float* w_k,
                  void* stream) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  if ((rc = check_cache(sh, cache)) != RTP_OK) return rc;
  if (T < 0 || T > sh.Lmax) return fail(RTP_ERR_SHAPE, "T must be in [0, max_ctx]");
  if (T == 0) return RTP_OK;
  if (!k_pre || !v_in || !start_pos) return fail(RTP_ERR_INVALID, "k_pre/v_in/start_pos is NULL");
  if (sh.R > 0 && !w_k) return fail(RTP_ERR_INVALID, "w_k is NULL with retrieval heads");
  return launch_append(sh, cache, k_pre, v_in, start_pos, T, w_k, (cudaStream_t)stream);
}

int rtp_decode_attn(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* q_pre,
                    const int* seq_len, int max_seq_len, const float* w_q, void* out,
                    uint32_t* sel_bitmask, int* sel_count, void* workspace,
                    size_t workspace_bytes, void* stream) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  if ((rc = check_cache(sh, cache)) != RTP_OK) return rc;
  if (!q_pre || !seq_len || !out) return fail(RTP_ERR_INVALID, "q_pre/seq_len/out is NULL");
  if (sh.R > 0 && !w_q) return fail(RTP_ERR_INVALID, "w_q is NULL with retrieval heads");
  if (max_seq_len < 0 || max_seq_len > sh.Lmax)
    return fail(RTP_ERR_SHAPE, "max_seq_len must be in [0, max_ctx]");
  if (!aligned16(q_pre) || (w_q && !aligned16(w_q)))
    return fail(RTP_ERR_INVALID, "q_pre and w_q must be 16-byte aligned");
  const DecodeLayout lay = decode_layout(sh);
  if (!workspace) return fail(RTP_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(RTP_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (workspace_bytes < lay.total)
    return fail(RTP_ERR_WORKSPACE, "workspace smaller than rtp_decode_workspace_bytes");
  return launch_decode(sh, cache, q_pre, seq_len, max_seq_len, w_q, out, sel_bitmask, sel_count,
                       workspace, lay, (cudaStream_t)stream);
}

int rtp_decode_recall(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* q_pre,
                      const int* seq_len, int max_seq_len, const uint32_t* sel_bitmask,
                      float* recall, void* workspace, size_t workspace_bytes, void* stream) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  if ((rc = check_cache(sh, cache)) != RTP_OK) return rc;
  if (max_seq_len < 0 || max_seq_len > sh.Lmax)
    return fail(RTP_ERR_SHAPE, "max_seq_len must be in [0, max_ctx]");
  if (sh.R == 0) return RTP_OK;
  if (!q_pre || !seq_len || !sel_bitmask || !recall)
    return fail(RTP_ERR_INVALID, "q_pre/seq_len/sel_bitmask/recall is NULL");
  if (!workspace) return fail(RTP_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(RTP_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (workspace_bytes < recall_workspace_bytes(sh))
    return fail(RTP_ERR_WORKSPACE, "workspace too small for rtp_decode_recall");
  return launch_recall(sh, cache, q_pre, seq_len, max_seq_len, sel_bitmask, recall, workspace,
                       (cudaStream_t)stream);
}

int rtp_prefill_attn(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* q_pre,
                     const int* start_pos, int T, const float* w_q, void* out,
                     uint32_t* sel_bitmask, float* sel_tau, int* sel_jcut, int* sel_count,
                     void* workspace, size_t workspace_bytes, void* stream) {
  Shape sh;
  int rc = make_shape(cfg, &sh);
  if (rc != RTP_OK) return rc;
  if ((rc = check_cache(sh, cache)) != RTP_OK) return rc;
  if (T < 1 || T > sh.Lmax) return fail(RTP_ERR_SHAPE, "T must be in [1, max_ctx]");
  if (sh.top_k > 0)
    return fail(RTP_ERR_SHAPE, "static top-k (cfg top_k > 0) is a decode-only variant; prefill selects by top-p");
  if (sh.ring > 0 && (long long)T + sh.W - 1 > sh.ring)
    return fail(RTP_ERR_SHAPE, "ring mode: a prefill chunk needs local_cap >= T + window - 1");
  if (!q_pre || !start_pos || !out) return fail(RTP_ERR_INVALID, "q_pre/start_pos/out is NULL");
  if (sh.R > 0 && !w_q) return fail(RTP_ERR_INVALID, "w_q is NULL with retrieval heads");
  if (!aligned16(q_pre) || (w_q && !aligned16(w_q)))
    return fail(RTP_ERR_INVALID, "q_pre and w_q must be 16-byte aligned");
  const PrefillLayout lay = prefill_layout(sh, T);
  if (!workspace) return fail(RTP_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(RTP_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (workspace_bytes < lay.total)
    return fail(RTP_ERR_WORKSPACE, "workspace smaller than rtp_prefill_workspace_bytes");
  return launch_prefill(sh, cache, q_pre, start_pos, T, w_q, out, sel_bitmask, sel_tau, sel_jcut,
                        sel_count, workspace, lay, (cudaStream_t)stream);
}

}  // extern "C"
