/*
 * bytecross.h -- C ABI of the B200 (sm_100a) decode-step library libbytecross.so
 *
 * One batch-1 decode step of a Llama-style GQA transformer in the four modes
 * of "Where Activation Sparsity and KV-Cache Sparsity Cross in LLM Decoding"
 * (ByteCross README, "Timing and quality on a GPU"): dense, activation-sparse
 * projections ("proj"; all seven projections), attention-scored KV selection
 * ("sel") and both.  A keep ratio of 1.0 disables a branch.  Every mode reads
 * its cache through the same split-K attention kernel (README, "Overview":
 * "One attention kernel for every mode").
 *
 * Keep ratios are passed as double and every keep count is
 * ceil(ratio * n - 1e-9) evaluated in double.  (A float ratio would not do:
 * 0.3f is 0.300000012, which keeps 385 instead of 384 of 1280 pages.)
 *
 * Conventions shared by every entry point
 *  - Ownership: the caller owns every device buffer (weights, KV pool,
 *    metadata pool, workspace, outputs) and the CUDA stream.  The library owns
 *    only the opaque host handle bc_model.  It never allocates device memory.
 *  - Asynchrony: calls that take a stream enqueue work on it and return
 *    without waiting, except where stated.  Launch errors are returned, never
 *    thrown; a sticky CUDA error maps to BC_ECUDA.  Nothing aborts.
 *  - Errors: every function returns a bc_status; bc_last_error() gives a
 *    thread-local message for the last failure.
 *  - Types: "bf16" is IEEE bfloat16 (uint16 bit patterns); "f32" is float.
 *    All matrices are row-major and densely packed.
 *  - Device: sm_100a only.
 */
#ifndef BYTECROSS_H
#define BYTECROSS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BC_API __attribute__((visibility("default")))

typedef enum {
  BC_OK = 0,
  BC_EINVAL = 1,     /* bad argument: null pointer, bad size, ratio outside (0,1], page mismatch */
  BC_ENOMEM = 2,     /* caller-supplied buffer smaller than the size query asks for */
  BC_ECAPACITY = 3,  /* KV pool full (append past max_ctx) */
  BC_ECUDA = 4,      /* a CUDA launch or call failed (message in bc_last_error) */
  BC_ETIMEOUT = 5    /* a bounded device-side wait gave up (reserved; no kernel spins today) */
} bc_status;

/* Decode modes (ByteCross README, "Timing and quality on a GPU": dense,
 * proj, sel, both; BC_SNAP is the once-after-prefill selection; BC_MASKED is
 * the masked dense baseline of the README's FAQ, "A KV method reports a
 * speedup above its byte bound"). */
typedef enum { BC_DENSE = 0, BC_ACT = 1, BC_KV = 2, BC_BOTH = 3, BC_SNAP = 4, BC_MASKED = 5 } bc_mode;

/* Model dimensions: the Hugging Face config fields the README's byte account
 * reads ("Quick start"), plus KV capacity and page size.
 * Requirements checked by bc_model_create: n_heads*head_dim == hidden (README
 * FAQ, "Which models does the byte account cover?"), head_dim in {64, 128},
 * n_heads/n_kv_heads in 1..8, page == 16, hidden and intermediate multiples
 * of 256. */
typedef struct {
  int n_layers, hidden, intermediate, n_heads, n_kv_heads, head_dim, vocab;
  int max_ctx;        /* KV capacity in tokens */
  int page;           /* tokens per KV page; must be 16 */
  float rms_eps;      /* RMSNorm epsilon */
  float rope_theta;   /* rotary base */
} bc_config;

/* Device pointers to the weights, all bf16, layers stacked on the leading axis.
 * Projection matrices are input-channel-major (W^T, one contiguous row per
 * input channel) so that an activation-selected channel is one contiguous
 * row stream.
 *   embed      [vocab][hidden]
 *   lm_head    [vocab][hidden]             output-major (dense in every mode)
 *   final_norm [hidden]
 *   attn_norm  [L][hidden],  mlp_norm [L][hidden]
 *   wqkv_t     [L][hidden][(Hq + 2 Hkv) hd]  q cols, then k cols, then v cols
 *   wo_t       [L][Hq hd][hidden]
 *   wgu_t      [L][hidden][2 intermediate]   gate cols first, then up
 *   wd_t       [L][intermediate][hidden]
 * The library reads them only; they must stay alive while the model exists. */
typedef struct {
  const void *embed, *lm_head, *final_norm;
  const void *attn_norm, *mlp_norm;
  const void *wqkv_t, *wo_t, *wgu_t, *wd_t;
} bc_weights;

typedef struct bc_model bc_model;

/* ------------------------------------------------------------------ sizes */

/* Bytes of the paged KV pool: bf16 [L][Hkv][Pmax][2][page][hd], keys then
 * values of each page adjacent (one 8 KiB block per page at hd=128),
 * Pmax = ceil(max_ctx / page).  0 on a bad config. */
BC_API size_t bc_kv_pool_bytes(const bc_config* cfg);

/* Bytes of the page key-bound pool: bf16 [L][Hkv][Pmax][2][hd], the
 * channelwise min then max of each page's valid keys.  0 on a bad config. */
BC_API size_t bc_meta_pool_bytes(const bc_config* cfg);

/* Bytes of the scratch workspace (activations, per-layer traces, split-K
 * partials, counters).  0 on a bad config. */
BC_API size_t bc_workspace_bytes(const bc_config* cfg);

/* ------------------------------------------------------------------ model */

/* Validates cfg and records the caller's buffers.  Host-only apart from one
 * cudaMemsetAsync of the workspace counters on `stream` (a cudaStream_t; NULL
 * is the legacy default stream).  kv_pool, meta_pool and workspace must be
 * 256-byte aligned device buffers of at least the queried sizes.  The KV
 * length starts at 0.  Errors: BC_EINVAL (bad config or null pointer),
 * BC_ENOMEM (ws_bytes too small), BC_ECUDA. */
BC_API bc_status bc_model_create(const bc_config* cfg, const bc_weights* w,
                                 void* kv_pool, void* meta_pool,
                                 void* workspace, size_t ws_bytes,
                                 void* stream, bc_model** out);

BC_API bc_status bc_model_destroy(bc_model* m);

/* Stream used by later calls on this model. */
BC_API bc_status bc_set_stream(bc_model* m, void* stream);

/* Decode steps through CUDA graphs (enable != 0, the default) or through
 * direct launches.  With graphs on, the first step of a configuration
 * (mode, rp, rkv, sinks, recent) launches directly; the next one captures the
 * step on a private stream of the library (created on first use) into a
 * graph, and every later step of that configuration updates the few kernel
 * nodes that depend on the position, token, page counts and logits buffer
 * and launches the graph on the model's stream.  Results are identical
 * either way (the same kernels with the same arguments).  Host-only. */
BC_API bc_status bc_set_graphs(bc_model* m, int enable);

/* Number of cached tokens. */
BC_API int bc_kv_length(const bc_model* m);

/* Number of kernels this model has launched since bc_model_create
 * (decode steps and appends). */
BC_API long long bc_launch_count(const bc_model* m);

/* Truncates the cache to its first n_ctx tokens (0 <= n_ctx <= length).
 * Host-only: later appends recompute the bounds of the page they land in
 * from its valid keys, so nothing on the device needs clearing.  Voids a
 * once-after-prefill selection. */
BC_API bc_status bc_kv_reset(bc_model* m, int n_ctx);

/* Appends n_tokens (>= 0) keys and values to every layer and kv head.
 * k, v: device bf16 [L][Hkv][n_tokens][hd], keys already rotated (they stand
 * for what a dense prefill wrote).  Writes the pages and recomputes the key
 * bounds of every page touched.  Voids a once-after-prefill selection.
 * Async on the model's stream.
 * Errors: BC_ECAPACITY if length + n_tokens > max_ctx; BC_EINVAL; BC_ECUDA. */
BC_API bc_status bc_kv_append(bc_model* m, const void* k, const void* v, int n_tokens);

/* Once-after-prefill page selection over the n = bc_kv_length(m) cached
 * tokens: the pages' own KV mode (ByteCross README, "Timing and quality on a
 * GPU": an attention-scored selection made once after prefill, in the
 * manner of SnapKV).  A window of n_obs observation queries per query head
 * (the last prompt positions' queries, rotated) votes with its softmax
 * attention over all n tokens (scale 1/sqrt(hd)); the score of a page of kv
 * head h is the attention mass its valid tokens receive from the n_obs*G
 * observation queries of h's group.  With P = ceil(n/page) pages, the same
 * rule as the KV branch keeps K = clamp(ceil(rkv*P - 1e-9), |F|, P) pages:
 * the forced first `sinks` and last `recent` pages and the best scored
 * others (descending, ties: lower page).  The kept lists are frozen: every
 * later BC_SNAP step attends over them plus every page begun after the
 * selection, with no per-step scoring.
 *   q_obs  device f32 [L][n_obs][Hq][hd], read during the call's kernels.
 *   n_obs  1 <= n_obs and n_obs*G <= 128.
 * Runs four kernels per layer on the model's stream (not captured in the
 * step graphs); the selection is voided by bc_kv_append and bc_kv_reset.
 * With hd = 128 and n_obs*G <= 64 the logits run on the tcgen05 tensor
 * cores (tensor-memory accumulators, keys brought by tensor copies), other
 * shapes on mma.sync.  Returns after the stream has drained, having read
 * the scorer's status word (its bounded waits).
 * Traces: BC_TRACE_SNAP_SCORES, BC_TRACE_SNAP_PAGES.
 * Errors: BC_EINVAL (no tokens, bad sizes or ratios), BC_ECUDA (also when a
 * bounded wait of the scorer gave up). */
BC_API bc_status bc_kv_snap_select(bc_model* m, const float* q_obs, int n_obs, double rkv, int sinks,
                                   int recent);

/* One decode step at position n = bc_kv_length(m) for input token `token`:
 * embedding row, then per layer RMSNorm -> [act: top-k |x| select] -> q/k/v
 * GEMV -> rotary -> append k, v (bf16) at position n and refresh the page's
 * key bounds -> [kv: page scores, page select] -> split-K attention over the
 * kept pages' n+1 tokens -> combine -> [act: select] -> o GEMV + residual ->
 * RMSNorm -> [act: select] -> gate/up GEMV -> SwiGLU -> [act: select] ->
 * down GEMV + residual; then final RMSNorm and the dense LM head.
 *
 *   mode    BC_DENSE, BC_ACT, BC_KV, BC_BOTH, or BC_SNAP: dense projections and
 *           attention over the pages a bc_kv_snap_select kept plus every
 *           page begun since (BC_EINVAL without a valid selection; rp, rkv,
 *           sinks and recent are then not used), or BC_MASKED: dense
 *           projections and the KV window (the first `sinks` and the last
 *           `recent` pages) computed the way the README's masked dense
 *           baseline does it: attention over every cached page with an
 *           additive mask (0 on the window's pages, -inf elsewhere), which
 *           reads every KV byte (rp and rkv are not used)
 *   rp      projection keep ratio in (0,1]; per projection input of width
 *           d_in the k = ceil(rp*d_in - 1e-9) channels of largest |x| are
 *           read (ties: lower index).  Ignored unless mode is ACT or BOTH.
 *   rkv     KV keep ratio in (0,1], in pages: with P pages after the append,
 *           K = clamp(ceil(rkv*P - 1e-9), |F|, P) pages are read, where the
 *           forced set F is the first `sinks` pages and the last `recent`
 *           pages; the other K - |F| are the best by page score (descending,
 *           ties: lower page).  The page score of kv head h is
 *           max over its query heads of sum_c max(q_c*kmin_c, q_c*kmax_c).
 *           Ignored unless mode is KV or BOTH.
 *   sinks   >= 0 pages; recent >= 1 pages (the page being written is always
 *           kept); page must equal cfg.page.
 *   logits  device f32 [vocab], written.
 * Async on the model's stream; the KV length becomes n + 1.
 * Errors: BC_EINVAL, BC_ECAPACITY (n + 1 > max_ctx), BC_ECUDA. */
BC_API bc_status bc_decode_step(bc_model* m, int token, bc_mode mode, double rp, double rkv,
                                int sinks, int recent, int page, float* logits);

/* The same step for callers holding host memory: logits_host is a host
 * f32 [vocab] buffer (pinned memory is fastest).  Enqueues the step, copies
 * the logits device -> host and waits for the stream.  Uses the workspace's
 * logits slot as the device-side destination. */
BC_API bc_status bc_decode_step_host(bc_model* m, int token, bc_mode mode, double rp, double rkv,
                                     int sinks, int recent, int page, float* logits_host);

/* ------------------------------------------------------------------ traces */

/* Per-layer intermediates the last decode step left in the workspace, for
 * parity checks.  *ptr receives a device pointer into the workspace, *count
 * the number of valid elements (f32 unless noted; 0 when the step did not
 * produce it).  The ranked vectors are exactly what the activation select
 * ranked by magnitude; they exist only after an ACT or BOTH step.
 *   BC_TRACE_XN        x * g, RMSNorm input times gain, ranked for q/k/v [hidden]
 *                      (the norm's positive scale does not change the ranking)
 *   BC_TRACE_SEL_QKV   int32 selected channels, ascending       [k]
 *   BC_TRACE_Q         rotated queries                          [Hq hd]
 *   BC_TRACE_ATTN      attention output (ranked for o)          [Hq hd]
 *   BC_TRACE_SEL_O     int32                                    [k]
 *   BC_TRACE_XN2       x * g ranked for gate/up                 [hidden]
 *   BC_TRACE_SEL_GU    int32                                    [k]
 *   BC_TRACE_H         silu(gate)*up ranked for down            [intermediate]
 *   BC_TRACE_SEL_D     int32                                    [k]
 *   BC_TRACE_X         residual stream after the layer          [hidden]
 *   BC_TRACE_PAGE_SCORES f32 [Hkv][stride] (count = P, stride = Pmax)
 *   BC_TRACE_PAGES     int32 [Hkv][stride] kept pages ascending (count = K)
 *   BC_TRACE_QKV       raw q/k/v GEMV output before rotation    [(Hq+2Hkv) hd]
 *   BC_TRACE_SNAP_SCORES f32 [Hkv][stride] page scores of the last
 *                      once-after-prefill selection (count = its P)
 *   BC_TRACE_SNAP_PAGES int32 [Hkv][stride] its kept pages, ascending
 *                      (count = its K) */
typedef enum {
  BC_TRACE_XN = 0, BC_TRACE_SEL_QKV, BC_TRACE_Q, BC_TRACE_ATTN, BC_TRACE_SEL_O,
  BC_TRACE_XN2, BC_TRACE_SEL_GU, BC_TRACE_H, BC_TRACE_SEL_D, BC_TRACE_X,
  BC_TRACE_PAGE_SCORES, BC_TRACE_PAGES, BC_TRACE_QKV, BC_TRACE_SNAP_SCORES, BC_TRACE_SNAP_PAGES,
  BC_TRACE_COUNT
} bc_trace_kind;

BC_API bc_status bc_trace(const bc_model* m, int layer, bc_trace_kind kind,
                          const void** ptr, int* count, int* stride);

/* ------------------------------------------------------------------ single kernels */

/* Column-gathered GEMV, the projection kernel of every mode:
 *   y[j] = sum over c in S of x[c] * W[c][j],   j in [0, d_out)
 * W: device bf16 [d_in][d_out] (input-channel-major); x: device f32 [d_in];
 * idx: device int32 [k] ascending channel list, or NULL for all d_in
 * channels (then k must equal d_in); y: device f32 [d_out], overwritten.
 * scratch: device buffer of bc_gemv_scratch_bytes(d_out) bytes (split-K
 * partial sums and ticket counters; zero it before the first call: every
 * call leaves the counters at zero).  d_out must be a multiple of 256.
 * stream: cudaStream_t.  Deterministic: the split-K partials are summed in a
 * fixed order. */
BC_API size_t bc_gemv_scratch_bytes(int d_out);
BC_API bc_status bc_gemv(const void* W, int d_in, int d_out, const float* x, const int* idx, int k,
                         float* y, void* scratch, size_t scratch_bytes, void* stream);

/* Column-gathered GEMV that allocates nothing: the same computation and
 * arguments as bc_gemv without the scratch buffer.  The paper has no
 * counterpart; this is for callers that cannot allocate device memory, such
 * as an operator inside another framework whose allocator owns the device
 * memory and hands the operator only its inputs and outputs, or a serving
 * path that must not call cudaMalloc (it can synchronise the device).
 * The split-K scratch lives in a file-scope __device__ array of
 * 8 MiB + 1 KiB, held on every GPU that loads the library until exit; d_out
 * above bc_gemv_noalloc_max_dout() (32768) is rejected with BC_EINVAL.  The
 * first call on a device, with that device current, looks the array's
 * address up; make it before any stream capture.  Every call clears the
 * tickets it needs and shares the array with every other call: calls that
 * overlap on the GPU race and must be serialised by the caller.  Allocates
 * no device memory (no cudaMalloc, cudaFree or allocating library call). */
BC_API int bc_gemv_noalloc_max_dout(void);
BC_API bc_status bc_gemv_noalloc(const void* W, int d_in, int d_out, const float* x, const int* idx, int k,
                                 float* y, void* stream);

/* Batched column-gathered GEMV over the union of the sequences' kept
 * channels, the projection of a batched decode step (README, "Usage: The byte
 * account": crossover_batch, where a batch reads the union of its kept
 * projection weights once).  Each sequence keeps its own channels, so
 *   y[b][j] = sum over c in S_b of x[b][c] * W[c][j],   b in [0, batch)
 * is what bc_gemv gives for sequence b alone, while the rows of the union
 * U = S_0 u ... u S_{batch-1} are read once for the whole batch.
 * W: device bf16 [d_in][d_out] (input-channel-major); x: device f32
 * [batch][d_in]; idx: device int32 [batch][k], row b the channels S_b
 * (any order; duplicates and values outside [0, d_in) are ignored), or NULL
 * for all d_in channels (then k must equal d_in); y: device f32
 * [batch][d_out], overwritten; n_union: device int32 [1] that receives |U|,
 * or NULL.  scratch: device buffer of bc_gemv_batch_scratch_bytes(d_in,
 * d_out, batch) bytes (union list and split partials; no zeroing
 * needed).  1 <= batch <= 8, 1 <= k <= d_in <= 16384, d_out a multiple of
 * 256.  stream: cudaStream_t.  Deterministic: the partial sums
 * of a column are added in a fixed order.  Invalid sizes: BC_EINVAL; small
 * scratch: BC_ENOMEM; nothing is launched then. */
BC_API size_t bc_gemv_batch_scratch_bytes(int d_in, int d_out, int batch);
BC_API bc_status bc_gemv_batch(const void* W, int d_in, int d_out, const float* x, const int* idx, int k,
                               int batch, float* y, int* n_union, void* scratch, size_t scratch_bytes,
                               void* stream);

/* Exact top-k selection: writes to idx (device int32 [k]) the k indices of
 * largest |v| (v: device f32 [n]), ascending; ties go to the lower index.
 * 1 <= k <= n <= 16384. */
BC_API bc_status bc_select_topk(const float* v, int n, int k, int* idx, void* stream);

/* Split-K flash-decode attention of one layer over a page list, the
 * attention kernel of every mode (README, "Overview").
 *   q      device f32 [Hkv*G][hd] rotated queries (G query heads per kv head);
 *          q, kv and out 16-byte aligned (else BC_EINVAL)
 *   kv     device bf16 pages of one layer, [Hkv][Pmax][2][16][hd]
 *   pages  device int32 [Hkv][Pmax] kept pages per kv head (first n_pages of
 *          each row used, ascending), or NULL for pages 0..n_pages-1
 *   n_tok  valid tokens; the page n_tok/16 is partial
 *   out    device f32 [Hkv*G][hd]
 *   scratch  bc_attention_scratch_bytes(Hkv*G, hd) bytes: split partials and
 *            one ticket counter per kv head; zero it before the first call
 *            (every call leaves the counters at zero) */
BC_API size_t bc_attention_scratch_bytes(int n_q_heads, int head_dim);
BC_API bc_status bc_attention(const float* q, const void* kv, int n_kv_heads, int group, int head_dim,
                              int Pmax, const int* pages, int n_pages, int n_tok,
                              float* out, void* scratch, size_t scratch_bytes, void* stream);

/* ------------------------------------------------------------------ batched decode step */

/* A batched decode step: `batch` sequences (1..8) share one model's weights
 * and decode in lock step (ByteCross README, "Usage: The byte account":
 * crossover_batch, where a batch reads the union of its sequences' kept
 * projection weights once per step).  Each sequence has its own KV cache,
 * page bounds, activations and selections, and all hold the same number of
 * tokens.  Per layer every sequence keeps its own channels (its own top-k of
 * |x| at every projection input, as at batch 1) and its own pages; each
 * projection reads the union of the batch's kept rows once (the
 * bc_gemv_batch kernels), the selections, page scores and attention run per
 * sequence in batched grids, and the LM head reads its weights once for the
 * whole batch.  Sequence b's result equals its batch-1 step up to fp32
 * summation order.
 *   kv_pools    device, batch * bc_kv_pool_bytes(cfg) bytes: sequence b's
 *               pool starts at byte b * bc_kv_pool_bytes(cfg)
 *   meta_pools  device, batch * bc_meta_pool_bytes(cfg) bytes, likewise
 *   workspace   device, bc_batch_workspace_bytes(cfg, batch) bytes
 * All three 256-byte aligned; the caller owns them and the stream.  cfg must
 * also have a q/k/v width ((n_heads + 2 n_kv_heads) head_dim) that is a
 * multiple of 128, and batch * hidden floats must fit one CTA's shared
 * memory (the LM head holds every sequence's normed state: 227 KB on B200,
 * so batch 8 up to hidden 7168).  Errors as for bc_model_create. */
typedef struct bc_batch bc_batch;
BC_API size_t bc_batch_workspace_bytes(const bc_config* cfg, int batch);
BC_API bc_status bc_batch_create(const bc_config* cfg, const bc_weights* w, int batch, void* kv_pools,
                                 void* meta_pools, void* workspace, size_t ws_bytes, void* stream,
                                 bc_batch** out);
BC_API bc_status bc_batch_destroy(bc_batch* b);
/* CUDA graphs on (default) or off for later steps, as bc_set_graphs. */
BC_API bc_status bc_batch_set_graphs(bc_batch* b, int enable);
/* Tokens cached per sequence (the same for all). */
BC_API int bc_batch_length(const bc_batch* b);
/* Kernels launched since bc_batch_create. */
BC_API long long bc_batch_launch_count(const bc_batch* b);
/* Truncates every sequence's cache to n_ctx tokens, as bc_kv_reset. */
BC_API bc_status bc_batch_reset(bc_batch* b, int n_ctx);
/* Appends n_tokens keys and values to every sequence: k, v device bf16
 * [batch][L][Hkv][n_tokens][hd], keys already rotated.  As bc_kv_append. */
BC_API bc_status bc_batch_append(bc_batch* b, const void* k, const void* v, int n_tokens);
/* One decode step of every sequence at position n = bc_batch_length(b):
 * tokens host int [batch]; mode BC_DENSE, BC_ACT, BC_KV or BC_BOTH with rp,
 * rkv, sinks, recent and page as for bc_decode_step; logits device f32
 * [batch][vocab].  Async on the batch's stream; the length becomes n + 1.
 * Errors: BC_EINVAL (bad mode, ratio, token), BC_ECAPACITY, BC_ECUDA. */
BC_API bc_status bc_batch_step(bc_batch* b, const int* tokens, bc_mode mode, double rp, double rkv, int sinks,
                               int recent, int page, float* logits);
/* Per-sequence traces of the last batched step, as bc_trace, for sequence
 * seq: BC_TRACE_XN, SEL_QKV, Q, ATTN, SEL_O, XN2, SEL_GU, H, SEL_D, X,
 * PAGE_SCORES, PAGES and QKV (others: BC_EINVAL). */
BC_API bc_status bc_batch_trace(const bc_batch* b, int seq, int layer, bc_trace_kind kind, const void** ptr,
                                int* count, int* stride);

/* ------------------------------------------------------------------ byte account */

/* Bytes of one decode step.  Paper form: the pages' byte account (README,
 * "Usage: The byte account": Equations 1-5, reconstructed so that every
 * printed value is reproduced).  Implementation form: the bytes this
 * library's step at context n_ctx (n_ctx tokens cached, token n_ctx
 * appended) must move in `mode`.  For BC_SNAP: the step right after a
 * once-after-prefill selection made at n_ctx with rkv, sinks and recent
 * (its kept pages plus a page the token opens; no bounds read); its paper
 * form is the KV branch's.  BC_MASKED reads what a dense step reads (every
 * KV byte; the mask saves none), and its paper form saves nothing. */
typedef struct {
  /* paper form */
  double weight_bytes;        /* W = 2 L P_l, the seven projections */
  double head_bytes;          /* H = 2 V d */
  double kv_bytes_per_token;  /* 2 L 2 Hkv hd */
  double dense_bytes;         /* B = W + H + n kv_tok */
  double saved_bytes;         /* dB = (1-rp) W + (1-rkv) n kv_tok for the mode's ratios */
  double bound;               /* B / (B - dB) */
  double n_star;              /* Equation 5: (1-rp) P_l / ((1-rkv) 2 Hkv hd) tokens */
  double n_star_ff;           /* the same with only gate/up/down sparsified */
  /* implementation form */
  double impl_weight_bytes;   /* selected weight rows of all projections */
  double impl_head_bytes;     /* dense LM head */
  double impl_kv_read_bytes;  /* keys and values of the kept pages' valid tokens */
  double impl_meta_read_bytes;/* page key bounds read by the scorer */
  double impl_kv_write_bytes; /* appended k, v and the rewritten page bounds */
  double impl_other_bytes;    /* norm gains, embedding row, logits, page re-read for bounds */
  double impl_total_bytes;
  long long pages_total;      /* P per (layer, kv head) after the append */
  long long pages_kept;       /* K per (layer, kv head) */
} bc_bytes;

BC_API bc_status bc_byte_account(const bc_config* cfg, bc_mode mode, double rp, double rkv,
                                 long long n_ctx, int sinks, int recent, int page, bc_bytes* out);

/* Batch crossover (README, "Usage: The byte account", crossover_batch): the
 * context, in tokens, at which the projection branch of a batch of `batch`
 * sequences -- which reads the union of its sequences' kept weight rows,
 * a fraction union_keep of them -- saves as many bytes as the KV branch at
 * keep rkv, which saves per sequence:
 *   n* = (1 - union_keep) P_l / (batch (1 - rkv) 2 Hkv hd)
 * (P_l as for bc_byte_account's n_star).  Host only.  BC_EINVAL unless
 * 0 < union_keep <= 1, 0 < rkv < 1 and batch >= 1. */
BC_API bc_status bc_crossover_batch(const bc_config* cfg, double union_keep, double rkv, int batch,
                                    double* n_star);

/* ------------------------------------------------------------------ errors */

BC_API const char* bc_last_error(void);
BC_API const char* bc_status_string(bc_status s);

#ifdef __cplusplus
}
#endif
#endif /* BYTECROSS_H */
