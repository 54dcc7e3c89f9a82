/*
 * rtp.h -- C ABI of the B200 (sm_100a) head-wise sparse attention layer.
 *
 * The layer is the one described for RTPurbo in "Full Attention Strikes Back:
 * Transferring Full Attention into Sparse within Hundred Training Steps"
 * (arXiv 2605.16928): only a few KV heads ("retrieval heads") keep the whole
 * context; the others ("local heads") attend to attention sinks plus a sliding
 * window (atlas.scime.ai summary, "Approach").  Retrieval heads choose tokens
 * with a 16-dimensional pre-RoPE indexer (abstract, observation (2)) and keep
 * a query-dependent top-p set instead of a fixed top-k (abstract, observation
 * (3); atlas "Approach": "query-adaptive top-p threshold"), then run exact
 * attention over the kept rows.
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless the comment says "host".  The caller
 *     owns all memory; the library never allocates, frees or keeps a pointer
 *     after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work is enqueued on it; nothing synchronises.
 *   - The return value is an rtp_status.  Errors that the host can see (null
 *     pointers, bad shapes, small workspace, a failed launch) return at once
 *     with nothing enqueued and a message in rtp_last_error().
 *   - Errors only the device can see (a sequence length or a position outside
 *     the cache) never trap: the kernels skip the offending sequence/row and
 *     OR an RTP_DEV_* bit into *cache->status, which the caller reads back
 *     when it wants (it is never cleared by the library).
 *   - Device buffers must be 16-byte aligned (torch and cudaMalloc allocations
 *     are); a misaligned pointer returns RTP_ERR_INVALID.
 *   - Layouts are dense row-major in the order written, e.g. K [B][Hkv][Lmax][D]
 *     means element (b, h, j, d) sits at ((b*Hkv + h)*Lmax + j)*D + d.
 *   - Element type of q, k, v, out and of the caches is cfg->dtype (bf16 or
 *     fp32); the indexer projections are always fp32; accumulation is fp32.
 */
#ifndef RTP_H_
#define RTP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host-visible status codes. */
typedef enum rtp_status {
  RTP_OK = 0,
  RTP_ERR_INVALID = 1,   /* null pointer or scalar argument out of range */
  RTP_ERR_SHAPE = 2,     /* unsupported head_dim / group size / sizes */
  RTP_ERR_DTYPE = 3,     /* dtype not RTP_BF16 or RTP_FP32 */
  RTP_ERR_WORKSPACE = 4, /* workspace NULL, too small or not 256-byte aligned */
  RTP_ERR_CUDA = 5       /* a CUDA runtime call or kernel launch failed */
} rtp_status;

/* Device-side status bits OR-ed into *cache->status. */
#define RTP_DEV_SEQ_LEN  0x1  /* decode: seq_len[b] < 1 or > max_seq_len; sequence b skipped */
#define RTP_DEV_POSITION 0x2  /* append/prefill: a position outside [0, max_ctx); rows skipped */
#define RTP_DEV_TIMEOUT  0x4  /* decode or prefill: a bounded in-kernel wait gave up; that call's output is invalid */

typedef enum rtp_dtype { RTP_BF16 = 0, RTP_FP32 = 1 } rtp_dtype;

/* One attention layer.
 *   batch         B, sequences per call
 *   n_q_heads     Hq;  n_kv_heads Hkv;  G = Hq / Hkv query heads share a KV head
 *                 (GQA; q head hq reads KV head hq / G).  Supported G: 1, 2, 4, 8.
 *   head_dim      D: 64 or 128
 *   idx_dim       d, the indexer width: 16 (abstract, observation (2)), or 4, 8
 *                 or 32 for the pages' indexer-dimension ablation
 *                 (atlas.scime.ai summary, "Surprising findings": dimension 4).
 *                 Scores are q~ . k~ / sqrt(d), with 1/sqrt(d) rounded to fp32.
 *   max_ctx       Lmax, cache capacity per sequence (positions [0, Lmax));
 *                 at most 2^23
 *   n_sink        S >= 0: positions [0, S) are always attended (sinks)
 *   window        W >= 1: the last W positions up to and including the query
 *                 position are always attended (sliding window)
 *   top_p         p in (0, 1]: retrieval heads keep the smallest set of tokens
 *                 whose indexer softmax mass reaches p (>= p), ties to the lower
 *                 token index; p = 1 keeps every token
 *   rope_base     rotary base (10000 for Qwen3); rotate-half convention
 *   retrieval_mask bit h set => KV head h is a retrieval head.  Retrieval
 *                 heads are ranked r = 0..R-1 in increasing h; R <= 64
 *   dtype         rtp_dtype of q, k, v, out and the caches
 *   local_cap     0: every KV head keeps the whole context in the cache.
 *                 > 0 (ring mode, at least `window`): local heads keep only
 *                 the S sinks and a ring of local_cap window rows, so the cache
 *                 holds the full context only for retrieval heads (abstract:
 *                 the full KV cache is kept for retrieval heads only).  A
 *                 prefill chunk of T tokens then needs local_cap >= T + W - 1.
 *                 Ignored (whole context kept) when S + local_cap >= max_ctx.
 *   top_k         0: top-p selection.  k > 0: static top-k, the pages' fixed-
 *                 budget baseline (atlas.scime.ai summary, "Key results" and
 *                 "Baselines": static top-k): retrieval query heads keep the k
 *                 highest indexer scores (ties to the lower index; every token
 *                 when k >= the context), united with sinks and window as for
 *                 top-p.  Decode only: rtp_prefill_attn returns RTP_ERR_SHAPE.
 */
typedef struct rtp_layer_cfg {
  int batch;
  int n_q_heads;
  int n_kv_heads;
  int head_dim;
  int idx_dim;
  int max_ctx;
  int n_sink;
  int window;
  float top_p;
  float rope_base;
  uint64_t retrieval_mask;
  int dtype;
  int local_cap;
  int top_k;
} rtp_layer_cfg;

/* The layer's cache (device memory owned by the caller; sizes from
 * rtp_cache_bytes):
 *   k       [B][Hkv][Lmax][D]  keys after RoPE at their own position
 *   v       [B][Hkv][Lmax][D]  values
 *           In ring mode (cfg->local_cap > 0) k and v are [B][rows][D]: per
 *           sequence the KV heads follow one another in order h = 0..Hkv-1,
 *           a retrieval head taking Lmax rows (position j in row j) and a local
 *           head S + local_cap rows (position j < S in row j, position j >= S
 *           in row S + (j - S) mod local_cap).
 *   kidx    [B][R][Lk][d]      d-dim indexer keys k~ = W_k k_pre, one row per
 *                              token for each retrieval KV head (pre-RoPE);
 *                              Lk = Lmax, except Lmax rounded up to even when a
 *                              row is 8 bytes (bf16, d = 4), so that every
 *                              (b, r) block starts on a 16-byte boundary
 *   status  one int of device-side error bits (see RTP_DEV_*), zeroed by the
 *           caller before first use
 */
typedef struct rtp_cache {
  void* k;
  void* v;
  void* kidx;
  int* status;
} rtp_cache;

/* Host.  Bytes of each cache buffer for cfg.  Any output pointer may be NULL. */
int rtp_cache_bytes(const rtp_layer_cfg* cfg, size_t* k_bytes, size_t* v_bytes,
                    size_t* kidx_bytes);

/* Host.  Scratch bytes rtp_decode_attn needs for cfg (any max_seq_len <= max_ctx). */
int rtp_decode_workspace_bytes(const rtp_layer_cfg* cfg, size_t* bytes);

/* Host.  Scratch bytes rtp_prefill_attn needs for cfg and chunk length T. */
int rtp_prefill_workspace_bytes(const rtp_layer_cfg* cfg, int T, size_t* bytes);

/* Append T tokens per sequence to the cache.
 *
 * For every sequence b, token t and KV head h, at position pos = start_pos[b] + t:
 *   k[b][h][pos] = RoPE(k_pre[b][t][h], pos)            (stored in dtype)
 *   v[b][h][pos] = v_in[b][t][h]
 *   kidx[b][r][pos] = W_k^(r) k_pre[b][t][h]              (retrieval head h of rank r;
 *                                                         fp32 accumulation, stored in dtype)
 * The indexer key is taken BEFORE RoPE, as the pages' "pre-RoPE" projection
 * says (atlas.scime.ai summary, "Approach" and its one-line summary).
 *
 *   k_pre, v_in  [B][T][Hkv][D] dtype, device
 *   start_pos    [B] int32, device
 *   w_k          [R][d][D] fp32, device (may be NULL when R = 0)
 * Rows with pos outside [0, max_ctx) are skipped and set RTP_DEV_POSITION.
 */
int rtp_append_kv(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* k_pre,
                  const void* v_in, const int* start_pos, int T, const float* w_k,
                  void* stream);

/* One decode step: the query of sequence b sits at position seq_len[b] - 1 (the
 * token just appended with rtp_append_kv) and sees positions [0, seq_len[b]).
 *
 * Local KV heads: exact attention over sinks [0, S) and window
 * [seq_len-W, seq_len) (atlas.scime.ai summary, "Approach").
 * Retrieval KV heads, for each of their G query heads separately:
 *   q~ = W_q^(r) q_pre (fp32), s_j = q~ . kidx_j / sqrt(d) for every cached j
 *   (fp32; for a bf16 layer on tensor cores from q~'s bf16 high and low parts,
 *   the fp32 score to about 2^-17 of the score),
 *   P = softmax(s); keep the smallest set, ordered by (P desc, j asc), whose
 *   mass reaches top_p (abstract, observations (2)-(3)); attend exactly over
 *   that set united with the sinks and the window.
 * Attention: softmax(RoPE(q, pos) . k_j / sqrt(D)) over the attended rows.
 *
 *   q_pre        [B][Hq][D] dtype, device, pre-RoPE queries
 *   seq_len      [B] int32, device, 1 <= seq_len[b] <= max_seq_len
 *   max_seq_len  host int, an upper bound on seq_len (sizes the grid);
 *                0 means cfg->max_ctx
 *   w_q          [R][d][D] fp32, device
 *   out          [B][Hq][D] dtype, device
 *   sel_bitmask  optional (NULL to skip) [B][R*G][ceil(max_ctx/32)] uint32: bit
 *                j of head (b, r*G+g) is set iff token j is in that query head's
 *                top-p set (before the sinks/window union).  Words covering
 *                positions >= max_seq_len are not written.
 *   sel_count    optional [B][R*G] int32: size of each top-p set
 *   workspace    >= rtp_decode_workspace_bytes, 256-byte aligned, device; its
 *                contents need no initialisation and are clobbered
 * A sequence with an invalid seq_len is skipped (its out rows untouched) and
 * sets RTP_DEV_SEQ_LEN.
 * q_pre, w_q and seq_len are read before the kernels wait for the work already
 * on the stream (only the cache reads wait): they must not be written by a
 * kernel that may still be running when this call's kernels start, such as an
 * earlier kernel launched with programmatic dependent launch.
 * The bounded waits inside the call (on the asynchronous copies of the
 * indexer keys, of the scores and of the sink/window rows) give up after about
 * 0.4 s; the call's output is then invalid and RTP_DEV_TIMEOUT is set.
 */
int rtp_decode_attn(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* q_pre,
                    const int* seq_len, int max_seq_len, const float* w_q, void* out,
                    uint32_t* sel_bitmask, int* sel_count, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Attention mass recall of a decode step's retrieval heads, a diagnostic the
 * method is evaluated by (atlas.scime.ai summary, "Experimental setup",
 * metrics): for each sequence b and retrieval query head r*G+g, the share of
 * the full causal attention's softmax mass, softmax(RoPE(q, L-1) . k_j /
 * sqrt(D)) over every j in [0, L), L = seq_len[b], that the rows the decode
 * step attended carry: the top-p set of sel_bitmask united with the sinks
 * [0, S) and the window [L-W, L).  fp32 arithmetic; a full-attention pass
 * over the retrieval heads' keys, so it costs about a dense decode step.
 *
 *   q_pre, seq_len, max_seq_len  as for the rtp_decode_attn call that wrote
 *                sel_bitmask (same cache contents)
 *   sel_bitmask  [B][R*G][ceil(max_ctx/32)] uint32, device, as rtp_decode_attn
 *                writes it
 *   recall       [B][R*G] float, device, in [0, 1]
 *   workspace    device, 256-byte aligned, contents clobbered; a workspace of
 *                rtp_decode_workspace_bytes bytes is always large enough
 * A sequence with an invalid seq_len is skipped (its recall entries untouched).
 * With no retrieval heads the call does nothing.
 */
int rtp_decode_recall(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* q_pre,
                      const int* seq_len, int max_seq_len, const uint32_t* sel_bitmask,
                      float* recall, void* workspace, size_t workspace_bytes, void* stream);

/* Size of the fixed device scratch array behind rtp_decode_attn_noalloc. */
#define RTP_NOALLOC_SCRATCH_BYTES (32u << 20)

/* rtp_decode_attn without a caller workspace, for callers that cannot
 * allocate device memory: plug-ins inside a host framework that owns the
 * device memory pool, latency-critical callers that cannot accept
 * cudaMalloc's implicit synchronisation, plain C callers holding only their
 * input and output buffers.  (The paper has no counterpart; this is an
 * interface convenience.)
 *
 * Arguments, results and errors are those of rtp_decode_attn minus
 * `workspace`/`workspace_bytes`: the scratch lives in one library-owned
 * device array of RTP_NOALLOC_SCRATCH_BYTES (32 MiB), reserved on every GPU
 * that loads the library until the process exits.  The call allocates
 * nothing.
 *   - Configurations needing more scratch than that (rtp_decode_workspace_bytes
 *     > RTP_NOALLOC_SCRATCH_BYTES) return RTP_ERR_WORKSPACE, nothing enqueued.
 *   - All calls share the array and it keeps the last call's contents; the
 *     kernels clear what must start at zero.  Calls whose device work
 *     overlaps (several streams or threads) race on it: serialise them.
 *   - The first call on each device looks up the array's device address with
 *     that device current and caches it; make that first call before any
 *     stream capture.  The cached address is not looked up again: do not use
 *     this entry point after a cudaDeviceReset in the same process.
 */
int rtp_decode_attn_noalloc(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* q_pre,
                            const int* seq_len, int max_seq_len, const float* w_q, void* out,
                            uint32_t* sel_bitmask, int* sel_count, void* stream);

/* One causal prefill chunk: query row t of sequence b sits at position
 * i = start_pos[b] + t and sees positions [0, i].  The chunk's keys and values
 * must already be in the cache (rtp_append_kv with the same start_pos and T).
 * Per row the layer computes exactly what rtp_decode_attn computes for a
 * query at position i (top-p over the indexer scores of [0, i] for retrieval
 * query heads; sinks and window [i-W+1, i] for every head).  The indexer
 * scores are computed on tensor cores from q~ split into a bf16 high part and
 * a bf16 low part accumulated in fp32 (the fp32 score to about 2^-17 of the
 * score), with exactly the arithmetic rtp_decode_attn uses for a bf16 layer:
 * a row's top-p set equals the decode step's at that position, bit for bit.
 * The attention itself runs on tensor cores in bf16 with fp32 accumulation
 * (atlas.scime.ai summary, "Approach"; abstract, observations (2)-(3)).
 * cfg->dtype must be RTP_BF16.
 *
 *   q_pre        [B][T][Hq][D] bf16, device
 *   start_pos    [B] int32, device; 0 <= start_pos[b] and start_pos[b] + T <= max_ctx
 *                (else the sequence is skipped and RTP_DEV_POSITION is set)
 *   w_q          [R][d][D] fp32, device
 *   out          [B][T][Hq][D] bf16, device
 *   sel_bitmask  optional [B][R*G][T][ceil(max_ctx/32)] uint32: row (b, r*G+g, t)
 *                has bit j set iff token j is in that row's top-p set; words
 *                past position i of the row are not written
 *   sel_tau      optional [B][R*G][T] float: score of the last kept token
 *                (-inf when p = 1 keeps every token)
 *   sel_jcut     optional [B][R*G][T] int32: tokens with score == sel_tau are kept
 *                iff their index <= sel_jcut (so membership is
 *                s_j > tau || (s_j == tau && j <= jcut))
 *   sel_count    optional [B][R*G][T] int32: size of the row's top-p set
 *   workspace    >= rtp_prefill_workspace_bytes(cfg, T), 256-byte aligned.  It
 *                holds a per-row top-p bitmask for a block of rows at a time;
 *                the block is sized so the workspace stays under 1 GiB, and
 *                longer chunks run block by block.
 * Ring mode (cfg->local_cap > 0) needs local_cap >= T + W - 1, else
 * RTP_ERR_SHAPE.
 */
int rtp_prefill_attn(const rtp_layer_cfg* cfg, const rtp_cache* cache, const void* q_pre,
                     const int* start_pos, int T, const float* w_q, void* out,
                     uint32_t* sel_bitmask, float* sel_tau, int* sel_jcut, int* sel_count,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Kernel stages, for rtp_trace_stage. */
typedef enum rtp_stage {
  RTP_STAGE_APPEND = 0,         /* rtp_append_kv: RoPE + cache + indexer-key store */
  RTP_STAGE_DECODE_SCORE = 1,   /* decode: indexer scores over the d-dim key cache */
  RTP_STAGE_DECODE_SELECT = 2,  /* decode: exact top-p selection, bitmask, kept-row attention */
  RTP_STAGE_DECODE_LOCAL = 3,   /* decode: sink/window attention of every KV head (beside the selection), final merge */
  RTP_STAGE_PREFILL_INDEX = 4,  /* prefill: per-row exact top-p selection */
  RTP_STAGE_PREFILL_ATTN = 5,   /* prefill: masked causal attention */
  RTP_STAGE_COUNT = 6
} rtp_stage;

/* Host.  Optional instrumentation (no work is skipped or added).  Arms a
 * one-shot trace: the next kernel of `stage` launched by an rtp_* call on this
 * host thread is bracketed by cudaEventRecord(start_event) and
 * cudaEventRecord(stop_event) on its launch stream.  Events are cudaEvent_t
 * passed as void*, created and owned by the caller (with timing enabled to
 * read cudaEventElapsedTime).  A stage launched several times by one call
 * (prefill chunks longer than one row block) records around its first launch.
 * NULL events disarm the stage.  Returns RTP_ERR_INVALID for an unknown stage. */
int rtp_trace_stage(int stage, void* start_event, void* stop_event);

/* Host.  Test hook for the bounded waits of rtp_decode_attn (no counterpart
 * in the paper).  Arms the next rtp_decode_attn call on this host thread to
 * wait for completion flags that never reach the awaited value, giving up
 * after `polls` polls (about 100 ns each): the call then sets RTP_DEV_TIMEOUT,
 * its output is invalid, and the GPU stays usable.  polls <= 0 disarms.
 * Returns RTP_OK. */
int rtp_debug_wait_expiry(int polls);

/* Host.  Message for the last non-OK return on this thread ("" if none). */
const char* rtp_last_error(void);

/* Host.  Library version string. */
const char* rtp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RTP_H_ */
