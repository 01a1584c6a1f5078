// C ABI of libbytecross: model handle, workspace layout, the decode-step
// launch sequence, single-kernel entry points and the byte account.
#include "../../include/bytecross.h"
#include "common.cuh"
#include "kernels.h"

#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>
#include <algorithm>
#include <string>
#include <vector>

using namespace bc;

// ------------------------------------------------------------------ errors
static thread_local std::string g_err;

static bc_status fail(bc_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static bc_status fail(bc_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

static bc_status cuda_fail(cudaError_t e, const char* where) {
  return fail(BC_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define BC_CUDA(call, where)                              \
  do {                                                    \
    cudaError_t e_ = (call);                              \
    if (e_ != cudaSuccess) return cuda_fail(e_, where);   \
  } while (0)

extern "C" const char* bc_last_error(void) { return g_err.c_str(); }

void bc::set_error(const char* msg) { g_err = msg; }

extern "C" const char* bc_status_string(bc_status s) {
  switch (s) {
    case BC_OK: return "ok";
    case BC_EINVAL: return "invalid argument";
    case BC_ENOMEM: return "buffer too small";
    case BC_ECAPACITY: return "KV capacity exceeded";
    case BC_ECUDA: return "CUDA error";
    case BC_ETIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

// ------------------------------------------------------------------ config and layout
static bool check_config(const bc_config* c, std::string* why) {
  if (!c) { *why = "null config"; return false; }
  if (c->n_layers < 1 || c->hidden < 1 || c->intermediate < 1 || c->vocab < 1 || c->max_ctx < 1) {
    *why = "dimensions must be positive"; return false;
  }
  if (c->head_dim != 64 && c->head_dim != 128) { *why = "head_dim must be 64 or 128"; return false; }
  if (c->n_kv_heads < 1 || c->n_heads % c->n_kv_heads != 0 || c->n_heads / c->n_kv_heads > 8) {
    *why = "n_heads must be 1..8 times n_kv_heads"; return false;
  }
  if (c->n_heads * c->head_dim != c->hidden) { *why = "n_heads * head_dim must equal hidden"; return false; }
  if (c->page != kPage) { *why = "page must be 16"; return false; }
  if (c->hidden % kColTile || c->intermediate % kColTile) {
    *why = "hidden and intermediate must be multiples of 256"; return false;
  }
  if (c->intermediate > kMaxSelect || c->hidden > kMaxSelect) { *why = "hidden/intermediate above 16384"; return false; }
  if ((c->max_ctx + kPage - 1) / kPage > kMaxSelect) { *why = "max_ctx above 262144"; return false; }
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) { *why = "rms_eps > 0 and rope_theta > 1 required"; return false; }
  return true;
}

struct Layout {
  size_t x, xf, logits, xn, qkv, q, attn, xn2, gu, h, xo;    // f32 (per-layer ones are [L][..])
  size_t sel_qkv, sel_o, sel_gu, sel_d;                         // int32 [L][..]
  size_t pscore, pages;                                         // [L][Hkv][Pmax]
  size_t snap_scores, snap_pages;                               // [L][Hkv][Pmax]
  size_t snap_part, snap_stats;                                 // float2 [Hkv][chunks][Q], [Hkv][Q]
  size_t snap_pp;                                               // float2 [Hkv][Pmax][64] (one layer)
  size_t part_o, part_ml, gemv_part, counters;
  size_t total;
  int nqkv, hq, Pmax, max_dout;
};

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Ticket counters: 4 GEMV sites x column tiles, then attention and page
// select per kv head.  Zeroed at create; every kernel leaves its own at zero.
static size_t counter_bytes(const bc_config* c, const Layout& y) {
  return 4 * (4 * (size_t)(y.max_dout / 128) + 2 * (size_t)c->n_kv_heads);
}

static Layout make_layout(const bc_config* c) {
  Layout y;
  const size_t L = c->n_layers, d = c->hidden, f = c->intermediate;
  y.hq = c->n_heads * c->head_dim;
  y.nqkv = (c->n_heads + 2 * c->n_kv_heads) * c->head_dim;
  y.Pmax = (c->max_ctx + kPage - 1) / kPage;
  y.max_dout = (int)std::max<size_t>(std::max<size_t>(y.nqkv, d), 2 * f);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  y.x = take(4 * d);
  y.xf = take(4 * d);
  y.logits = take(4 * (size_t)c->vocab);
  y.xn = take(4 * L * d);
  y.qkv = take(4 * L * y.nqkv);
  y.q = take(4 * L * y.hq);
  y.attn = take(4 * L * y.hq);
  y.xn2 = take(4 * L * d);
  y.gu = take(4 * L * 2 * f);
  y.h = take(4 * L * f);
  y.xo = take(4 * L * d);
  y.sel_qkv = take(4 * L * d);
  y.sel_o = take(4 * L * y.hq);
  y.sel_gu = take(4 * L * d);
  y.sel_d = take(4 * L * f);
  y.pscore = take(4 * L * c->n_kv_heads * (size_t)y.Pmax);
  y.pages = take(4 * L * c->n_kv_heads * (size_t)y.Pmax);
  y.snap_scores = take(4 * L * c->n_kv_heads * (size_t)y.Pmax);
  y.snap_pages = take(4 * L * c->n_kv_heads * (size_t)y.Pmax);
  y.snap_part = take(8 * (size_t)c->n_kv_heads * snap_chunks(c->max_ctx) * kSnapMaxQ);
  y.snap_stats = take(8 * (size_t)c->n_kv_heads * kSnapMaxQ);
  y.snap_pp = c->head_dim == 128 ? take(8 * (size_t)c->n_kv_heads * y.Pmax * 64) : o;
  y.part_o = take(4 * (size_t)c->n_heads * kMaxSplits * c->head_dim);
  y.part_ml = take(4 * (size_t)c->n_heads * kMaxSplits * 2);
  y.gemv_part = take(4 * (size_t)kGemvMaxContrib * y.max_dout);
  y.counters = take(counter_bytes(c, y));
  y.total = o;
  return y;
}

extern "C" size_t bc_kv_pool_bytes(const bc_config* c) {
  std::string why;
  if (!check_config(c, &why)) return 0;
  const size_t Pmax = (c->max_ctx + kPage - 1) / kPage;
  return (size_t)c->n_layers * c->n_kv_heads * Pmax * 2 * kPage * c->head_dim * 2;
}

extern "C" size_t bc_meta_pool_bytes(const bc_config* c) {
  std::string why;
  if (!check_config(c, &why)) return 0;
  const size_t Pmax = (c->max_ctx + kPage - 1) / kPage;
  return (size_t)c->n_layers * c->n_kv_heads * Pmax * 2 * c->head_dim * 2;
}

extern "C" size_t bc_workspace_bytes(const bc_config* c) {
  std::string why;
  if (!check_config(c, &why)) return 0;
  return make_layout(c).total;
}

// ------------------------------------------------------------------ model
struct bc_model {
  bc_config cfg;
  bc_weights w;
  __nv_bfloat16* kv;
  __nv_bfloat16* meta;
  char* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  Layout lay;
  int n;               // cached tokens
  int sms;
  long long launches;  // kernels launched so far
  // what the last step left in the traces
  int last_k[4];       // kept channels per site (0 = no selection)
  int last_P, last_K;  // pages after the append, kept pages (0 = no selection)
  bool last_act;       // the last step ranked activations (XN, XN2, H traces valid)
  // CUDA graphs of the step, one per step configuration
  bool use_graphs;
  // the once-after-prefill selection: valid until the cache is appended to
  // in bulk or reset; P and K at the selection
  bool snap_valid;
  int snap_P, snap_K;
  cudaStream_t cap_stream;                 // private stream the steps are captured on
  std::vector<struct StepGraph*> graphs;
};

// A kernel node of a captured step whose arguments change from step to step.
enum NodeKind { NK_QKV = 0, NK_SEL_EMBED, NK_PAGES, NK_PAGE_SEL, NK_ATTN, NK_LMHEAD };
struct NodeRec {
  cudaGraphNode_t node;
  int kind, layer;
  cudaKernelNodeParams kp;   // function and launch shape read back from the graph
  union {
    GemvArgs g;
    SelectArgs s;
    PageArgs p;
    AttnArgs a;
    LmHeadArgs lm;
  } args;
};

// A captured decode step for one (mode, rp, rkv, sinks, recent).
struct StepGraph {
  bc_mode mode;
  int psel;              // page-select variant of the captured page counts (kv modes)
  double rp, rkv;
  int sinks, recent;
  cudaGraph_t graph;
  cudaGraphExec_t exec;
  std::vector<NodeRec> nodes;
  long long launches;
};

static void destroy_graph(StepGraph* g) {
  if (!g) return;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
}

template <typename T>
static T* at(const bc_model* m, size_t off) { return reinterpret_cast<T*>(m->ws + off); }

static int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

extern "C" bc_status bc_model_create(const bc_config* cfg, const bc_weights* w, void* kv_pool,
                                     void* meta_pool, void* workspace, size_t ws_bytes,
                                     void* stream, bc_model** out) {
  std::string why;
  if (!out) return fail(BC_EINVAL, "out is null");
  *out = nullptr;
  if (!check_config(cfg, &why)) return fail(BC_EINVAL, "bad config: %s", why.c_str());
  if (!w || !w->embed || !w->lm_head || !w->final_norm || !w->attn_norm || !w->mlp_norm ||
      !w->wqkv_t || !w->wo_t || !w->wgu_t || !w->wd_t)
    return fail(BC_EINVAL, "null weight pointer");
  if (!kv_pool || !meta_pool || !workspace) return fail(BC_EINVAL, "null pool or workspace");
  if (((uintptr_t)kv_pool | (uintptr_t)meta_pool | (uintptr_t)workspace) & 255)
    return fail(BC_EINVAL, "pools and workspace must be 256-byte aligned");
  Layout lay = make_layout(cfg);
  if (ws_bytes < lay.total)
    return fail(BC_ENOMEM, "workspace has %zu bytes, needs %zu", ws_bytes, lay.total);
  bc_model* m = new bc_model();
  m->cfg = *cfg;
  m->w = *w;
  m->kv = static_cast<__nv_bfloat16*>(kv_pool);
  m->meta = static_cast<__nv_bfloat16*>(meta_pool);
  m->ws = static_cast<char*>(workspace);
  m->ws_bytes = ws_bytes;
  m->stream = static_cast<cudaStream_t>(stream);
  m->lay = lay;
  m->n = 0;
  m->sms = device_sms();
  m->launches = 0;
  memset(m->last_k, 0, sizeof m->last_k);
  m->last_P = m->last_K = 0;
  m->last_act = false;
  m->use_graphs = true;
  m->snap_valid = false;
  m->snap_P = m->snap_K = 0;
  m->cap_stream = nullptr;
  cudaError_t e = cudaMemsetAsync(m->ws + lay.counters, 0, counter_bytes(cfg, lay), m->stream);
  if (e != cudaSuccess) {
    delete m;
    return cuda_fail(e, "bc_model_create: clearing counters");
  }
  *out = m;
  return BC_OK;
}

extern "C" bc_status bc_model_destroy(bc_model* m) {
  if (!m) return BC_OK;
  for (StepGraph* g : m->graphs) destroy_graph(g);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  delete m;
  return BC_OK;
}

extern "C" bc_status bc_set_graphs(bc_model* m, int enable) {
  if (!m) return fail(BC_EINVAL, "null model");
  m->use_graphs = enable != 0;
  return BC_OK;
}

extern "C" bc_status bc_set_stream(bc_model* m, void* stream) {
  if (!m) return fail(BC_EINVAL, "null model");
  m->stream = static_cast<cudaStream_t>(stream);
  return BC_OK;
}

extern "C" int bc_kv_length(const bc_model* m) { return m ? m->n : -1; }

extern "C" long long bc_launch_count(const bc_model* m) { return m ? m->launches : -1; }

extern "C" bc_status bc_kv_reset(bc_model* m, int n_ctx) {
  if (!m) return fail(BC_EINVAL, "null model");
  if (n_ctx < 0 || n_ctx > m->n) return fail(BC_EINVAL, "reset to %d outside [0, %d]", n_ctx, m->n);
  m->n = n_ctx;
  m->snap_valid = false;
  return BC_OK;
}

extern "C" bc_status bc_kv_snap_select(bc_model* m, const float* q_obs, int n_obs, double rkv, int sinks,
                                       int recent) {
  if (!m || !q_obs) return fail(BC_EINVAL, "null argument");
  const bc_config& c = m->cfg;
  const Layout& y = m->lay;
  const int G = c.n_heads / c.n_kv_heads, Hkv = c.n_kv_heads, L = c.n_layers;
  if (n_obs < 1 || n_obs * G > kSnapMaxQ)
    return fail(BC_EINVAL, "n_obs %d outside [1, %d]", n_obs, kSnapMaxQ / G);
  if (!(rkv > 0.0 && rkv <= 1.0)) return fail(BC_EINVAL, "rkv %g outside (0, 1]", rkv);
  if (sinks < 0 || recent < 1) return fail(BC_EINVAL, "sinks must be >= 0 and recent >= 1");
  if (m->n < 1) return fail(BC_EINVAL, "the cache holds no tokens");
  const int n = m->n, P = (n + kPage - 1) / kPage, Pmax = y.Pmax;
  const int sink_end = std::min(sinks, P), rec_begin = std::max(P - recent, 0);
  const int n_forced = sink_end + (P - std::max(rec_begin, sink_end));
  const int K = std::max(n_forced, (int)std::min<double>(P, ceil(rkv * P - 1e-9)));
  const size_t kv_layer = (size_t)Hkv * Pmax * 2 * kPage * c.head_dim;
  m->snap_valid = false;
  for (int l = 0; l < L; ++l) {
    SnapArgs sa;
    sa.q_obs = q_obs + (size_t)l * n_obs * c.n_heads * c.head_dim;
    sa.kv = m->kv + l * kv_layer;
    sa.Hkv = Hkv;
    sa.G = G;
    sa.hd = c.head_dim;
    sa.Pmax = Pmax;
    sa.n_obs = n_obs;
    sa.n_tok = n;
    sa.part = at<float2>(m, y.snap_part);
    sa.stats = at<float2>(m, y.snap_stats);
    sa.scores = at<float>(m, y.snap_scores) + (size_t)l * Hkv * Pmax;
    sa.pp = c.head_dim == 128 ? at<float2>(m, y.snap_pp) : nullptr;
    BC_CUDA(launch_snap_scores(sa, m->stream, true), "snap page scores");
    PageArgs pa{nullptr, nullptr, Hkv, G, c.head_dim, Pmax, P, K, sinks, recent, 0, sa.scores,
                at<int>(m, y.snap_pages) + (size_t)l * Hkv * Pmax, nullptr};
    BC_CUDA(launch_page_select(pa, m->stream, true), "snap page select");
  }
  m->launches += 4LL * L;
  unsigned status = 0;
  BC_CUDA(snap_status(&status, m->stream), "snap status");
  if (status) return fail(BC_ECUDA, "snap scorer: a bounded wait gave up (status %u)", status);
  m->snap_valid = true;
  m->snap_P = P;
  m->snap_K = K;
  return BC_OK;
}

extern "C" bc_status bc_kv_append(bc_model* m, const void* k, const void* v, int n_tokens) {
  if (!m) return fail(BC_EINVAL, "null model");
  if (n_tokens < 0) return fail(BC_EINVAL, "n_tokens < 0");
  if (n_tokens == 0) return BC_OK;
  if (!k || !v) return fail(BC_EINVAL, "null k or v");
  if ((long long)m->n + n_tokens > m->cfg.max_ctx)
    return fail(BC_ECAPACITY, "append of %d tokens to %d exceeds max_ctx %d", n_tokens, m->n, m->cfg.max_ctx);
  KvAppendArgs a;
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.n_new = n_tokens;
  a.n0 = m->n;
  a.L = m->cfg.n_layers;
  a.Hkv = m->cfg.n_kv_heads;
  a.hd = m->cfg.head_dim;
  a.Pmax = m->lay.Pmax;
  a.pool = m->kv;
  a.meta = m->meta;
  BC_CUDA(launch_kv_append(a, m->stream, true), "bc_kv_append");
  m->launches += 2;
  m->n += n_tokens;
  m->snap_valid = false;
  return BC_OK;
}

static int keep_count(double ratio, int n) {
  const double v = ceil(ratio * n - 1e-9);
  return (int)std::max(1.0, std::min((double)n, v));
}

static bc_status check_step(const bc_model* m, bc_mode mode, double rp, double rkv, int sinks,
                            int recent, int page) {
  if (!m) return fail(BC_EINVAL, "null model");
  if (mode < BC_DENSE || mode > BC_MASKED) return fail(BC_EINVAL, "bad mode %d", (int)mode);
  if (mode == BC_SNAP && !m->snap_valid)
    return fail(BC_EINVAL, "snap mode needs a selection (bc_kv_snap_select) since the last append or reset");
  if (page != m->cfg.page) return fail(BC_EINVAL, "page %d differs from the model's %d", page, m->cfg.page);
  if (!(rp > 0.0 && rp <= 1.0)) return fail(BC_EINVAL, "rp %g outside (0, 1]", rp);
  if (!(rkv > 0.0 && rkv <= 1.0)) return fail(BC_EINVAL, "rkv %g outside (0, 1]", rkv);
  if (sinks < 0 || recent < 1) return fail(BC_EINVAL, "sinks must be >= 0 and recent >= 1");
  if (m->n + 1 > m->cfg.max_ctx) return fail(BC_ECAPACITY, "KV cache full (%d tokens)", m->n);
  return BC_OK;
}

static cudaError_t step_select(bc_model* m, int prep, int n, int k, const float* x,
                               const __nv_bfloat16* gain, const __nv_bfloat16* emb, float* x_init,
                               float* vout, int* idx, SelectArgs* out_args) {
  SelectArgs s;
  memset(&s, 0, sizeof s);
  s.prep = prep;
  s.n = n;
  s.k = k;
  s.x = x;
  s.gain = gain;
  s.embed_row = emb;
  s.x_init = x_init;
  s.vout = vout;
  s.idx = idx;
  if (out_args) *out_args = s;
  return launch_select(s, m->stream, true);
}

static unsigned* gemv_counters(bc_model* m, int site) {
  return at<unsigned>(m, m->lay.counters) + site * (m->lay.max_dout / 128);
}

static cudaError_t step_gemv(bc_model* m, int site, const __nv_bfloat16* W, int d_in, int d_out, int prep,
                             const float* x, const __nv_bfloat16* gain, const __nv_bfloat16* emb,
                             float* x_init, const int* idx, int k, int epi, float* y, float* y_copy,
                             const QkvEpilogue* qe, GemvArgs* out_args) {
  GemvArgs g;
  memset(&g, 0, sizeof g);
  g.W = W;
  g.d_in = d_in;
  g.d_out = d_out;
  g.prep = prep;
  g.x = x;
  g.gain = gain;
  g.eps = m->cfg.rms_eps;
  g.embed_row = emb;
  g.x_init = x_init;
  g.idx = idx;
  g.k = k;
  gemv_plan(k, d_out, m->sms, &g.TW, &g.S, &g.C);
  g.max_rows = (k + g.S * g.C - 1) / (g.S * g.C);
  g.partial = at<float>(m, m->lay.gemv_part);
  g.counters = gemv_counters(m, site);
  g.epi = epi;
  g.y = y;
  g.y_copy = y_copy;
  if (qe) g.qkv = *qe;
  if (out_args) *out_args = g;
  return launch_gemv(g, m->stream, true);
}

// The kernel node the last launch added to a stream being captured.
static cudaGraphNode_t captured_node(cudaStream_t st) {
  cudaStreamCaptureStatus status;
  const cudaGraphNode_t* deps = nullptr;
  size_t n = 0;
  if (cudaStreamGetCaptureInfo(st, &status, nullptr, nullptr, &deps, &n) != cudaSuccess) return nullptr;
  return (status == cudaStreamCaptureStatusActive && n == 1) ? deps[0] : nullptr;
}

template <typename A>
static bool record(std::vector<NodeRec>* rec, cudaStream_t st, int kind, int layer, const A& args) {
  if (!rec) return true;
  NodeRec r;
  memset(&r, 0, sizeof r);
  r.node = captured_node(st);
  if (!r.node) return false;
  r.kind = kind;
  r.layer = layer;
  memcpy(&r.args, &args, sizeof(A));
  rec->push_back(r);
  return true;
}

// Per-step values every mode derives from the position.
struct StepShape {
  int pos, n_tok, P, K, splits, pps;
  int list_len, tail0;      // attention page list: listed entries, then pages tail0, tail0+1, ...
  int mask_on, mask_sink_end, mask_rec_begin;   // BC_MASKED: the window's pages unmasked
  int k_qkv, k_o, k_gu, k_d;
};

static StepShape step_shape(const bc_model* m, bc_mode mode, double rp, double rkv, int sinks, int recent) {
  const bc_config& c = m->cfg;
  const bool act = mode == BC_ACT || mode == BC_BOTH;
  const bool kvs = mode == BC_KV || mode == BC_BOTH;
  StepShape sh;
  sh.pos = m->n;
  sh.n_tok = sh.pos + 1;
  sh.P = (sh.n_tok + kPage - 1) / kPage;
  sh.K = sh.P;
  sh.list_len = 0;
  sh.tail0 = 0;
  sh.mask_on = mode == BC_MASKED;
  sh.mask_sink_end = std::min(sinks, sh.P);
  sh.mask_rec_begin = std::max(sh.P - recent, 0);
  if (mode == BC_SNAP) {
    sh.K = m->snap_K + std::max(0, sh.P - m->snap_P);
    sh.list_len = m->snap_K;
    sh.tail0 = m->snap_P;
  }
  if (kvs) {
    const int sink_end = std::min(sinks, sh.P), rec_begin = std::max(sh.P - recent, 0);
    const int n_forced = sink_end + (sh.P - std::max(rec_begin, sink_end));
    const int want = (int)std::min<double>(sh.P, ceil(rkv * sh.P - 1e-9));
    sh.K = std::max(n_forced, want);
    sh.list_len = sh.K;
  }
  attn_plan(sh.K, c.n_kv_heads, m->sms, &sh.splits, &sh.pps);
  sh.k_qkv = act ? keep_count(rp, c.hidden) : c.hidden;
  sh.k_o = act ? keep_count(rp, m->lay.hq) : m->lay.hq;
  sh.k_gu = act ? keep_count(rp, c.hidden) : c.hidden;
  sh.k_d = act ? keep_count(rp, c.intermediate) : c.intermediate;
  return sh;
}

static void commit_step(bc_model* m, bc_mode mode, const StepShape& sh, long long launches) {
  const bool act = mode == BC_ACT || mode == BC_BOTH;
  const bool kvs = mode == BC_KV || mode == BC_BOTH;
  m->launches += launches;
  m->n = sh.n_tok;
  m->last_k[0] = act ? sh.k_qkv : 0;
  m->last_k[1] = act ? sh.k_o : 0;
  m->last_k[2] = act ? sh.k_gu : 0;
  m->last_k[3] = act ? sh.k_d : 0;
  m->last_act = act;
  m->last_P = sh.P;
  m->last_K = kvs ? sh.K : 0;
}

// Enqueues one decode step on m->stream (launching, or recording into a
// capture when rec is given).  Returns the number of kernels in *launches.
static bc_status enqueue_step(bc_model* m, int token, bc_mode mode, double rp, double rkv, int sinks,
                              int recent, float* logits, std::vector<NodeRec>* rec, long long* n_launch) {
  const bc_config& c = m->cfg;
  const Layout& y = m->lay;
  const bool act = mode == BC_ACT || mode == BC_BOTH;
  const bool kvs = mode == BC_KV || mode == BC_BOTH;
  const int L = c.n_layers, d = c.hidden, f = c.intermediate, hd = c.head_dim;
  const int Hq = c.n_heads, Hkv = c.n_kv_heads, G = Hq / Hkv;
  const int hq = y.hq, nqkv = y.nqkv, Pmax = y.Pmax;
  const StepShape sh = step_shape(m, mode, rp, rkv, sinks, recent);
  const int pos = sh.pos, n_tok = sh.n_tok, P = sh.P, K = sh.K;
  const int k_qkv = sh.k_qkv, k_o = sh.k_o, k_gu = sh.k_gu, k_d = sh.k_d;
  cudaStream_t st = m->stream;

  const __nv_bfloat16* emb = static_cast<const __nv_bfloat16*>(m->w.embed) + (size_t)token * d;
  const __nv_bfloat16* attn_norm = static_cast<const __nv_bfloat16*>(m->w.attn_norm);
  const __nv_bfloat16* mlp_norm = static_cast<const __nv_bfloat16*>(m->w.mlp_norm);
  const __nv_bfloat16* wqkv = static_cast<const __nv_bfloat16*>(m->w.wqkv_t);
  const __nv_bfloat16* wo = static_cast<const __nv_bfloat16*>(m->w.wo_t);
  const __nv_bfloat16* wgu = static_cast<const __nv_bfloat16*>(m->w.wgu_t);
  const __nv_bfloat16* wd = static_cast<const __nv_bfloat16*>(m->w.wd_t);
  float* x = at<float>(m, y.x);
  const size_t kv_layer = (size_t)Hkv * Pmax * 2 * kPage * hd;
  const size_t meta_layer = (size_t)Hkv * Pmax * 2 * hd;
  unsigned* att_counters = gemv_counters(m, 4);
  unsigned* page_counters = att_counters + Hkv;

  const int splits = sh.splits, pps = sh.pps;
  long long launches = 0;

  for (int l = 0; l < L; ++l) {
    float* xn = at<float>(m, y.xn) + (size_t)l * d;
    float* qkv = at<float>(m, y.qkv) + (size_t)l * nqkv;
    float* q = at<float>(m, y.q) + (size_t)l * hq;
    float* attn = at<float>(m, y.attn) + (size_t)l * hq;
    float* xn2 = at<float>(m, y.xn2) + (size_t)l * d;
    float* gu = at<float>(m, y.gu) + (size_t)l * 2 * f;
    float* hmid = at<float>(m, y.h) + (size_t)l * f;
    float* xo = at<float>(m, y.xo) + (size_t)l * d;
    int* s_qkv = at<int>(m, y.sel_qkv) + (size_t)l * d;
    int* s_o = at<int>(m, y.sel_o) + (size_t)l * hq;
    int* s_gu = at<int>(m, y.sel_gu) + (size_t)l * d;
    int* s_d = at<int>(m, y.sel_d) + (size_t)l * f;
    float* pscore = at<float>(m, y.pscore) + (size_t)l * Hkv * Pmax;
    int* pages = at<int>(m, y.pages) + (size_t)l * Hkv * Pmax;
    __nv_bfloat16* kvl = m->kv + l * kv_layer;
    __nv_bfloat16* metal = m->meta + l * meta_layer;
    const __nv_bfloat16* g_attn = attn_norm + (size_t)l * d;
    const __nv_bfloat16* g_mlp = mlp_norm + (size_t)l * d;
    const bool first = l == 0;

    // attention block: [select] -> q/k/v GEMV (RMSNorm folded in; rotary,
    // append and page bounds in the epilogue) -> [page scores + select] ->
    // split-K attention with fused combine
    // gate/up with the SwiGLU epilogue (h = silu(gate) * up written by the
    // GEMV) when its column tiles pair whole channels; otherwise the down
    // projection forms h from gate and up while staging
    int tw_gu = 0, s_gu_ = 0, c_gu_ = 0;
    gemv_plan(k_gu, 2 * f, m->sms, &tw_gu, &s_gu_, &c_gu_);
    const bool sw = f % (tw_gu / 2) == 0;
    float* d_in_vec = sw ? hmid : gu;
    if (act) {
      SelectArgs sa;
      BC_CUDA(step_select(m, first ? SP_EMBED_NORM : SP_NORM, d, k_qkv, x, g_attn, emb, x, xn, s_qkv, &sa),
              "select qkv");
      if (first && !record(rec, st, NK_SEL_EMBED, l, sa)) return fail(BC_ECUDA, "capture: no node");
      ++launches;
    }
    QkvEpilogue qe;
    qe.Hq = Hq;
    qe.Hkv = Hkv;
    qe.hd = hd;
    qe.pos = pos;
    qe.Pmax = Pmax;
    qe.rope_theta = c.rope_theta;
    qe.q_out = q;
    qe.kv_layer = kvl;
    qe.meta_layer = metal;
    GemvArgs ga;
    BC_CUDA(step_gemv(m, 0, wqkv + (size_t)l * d * nqkv, d, nqkv, first ? GP_EMBED_NORM : GP_NORM, x, g_attn,
                      emb, x, act ? s_qkv : nullptr, k_qkv, EPI_QKV, qkv, nullptr, &qe, &ga), "gemv qkv");
    if (!record(rec, st, NK_QKV, l, ga)) return fail(BC_ECUDA, "capture: no node");
    ++launches;
    if (kvs) {
      PageArgs pa{q, metal, Hkv, G, hd, Pmax, P, K, sinks, recent, page_rounds(P, hd, Hkv, m->sms),
                  pscore, pages, page_counters};
      BC_CUDA(launch_page_scores(pa, st, true), "page scores");
      if (!record(rec, st, NK_PAGES, l, pa)) return fail(BC_ECUDA, "capture: no node");
      BC_CUDA(launch_page_select(pa, st, true), "page select");
      if (!record(rec, st, NK_PAGE_SEL, l, pa)) return fail(BC_ECUDA, "capture: no node");
      launches += 2;
    }
    AttnArgs aa;
    memset(&aa, 0, sizeof aa);
    aa.q = q;
    aa.kv = kvl;
    aa.pages = kvs ? pages : mode == BC_SNAP ? at<int>(m, y.snap_pages) + (size_t)l * Hkv * Pmax : nullptr;
    aa.list_len = sh.list_len;
    aa.tail0 = sh.tail0;
    aa.Hkv = Hkv;
    aa.G = G;
    aa.hd = hd;
    aa.Pmax = Pmax;
    aa.n_pages = K;
    aa.n_tok = n_tok;
    aa.splits = splits;
    aa.pages_per_split = pps;
    aa.mask_on = sh.mask_on;
    aa.mask_sink_end = sh.mask_sink_end;
    aa.mask_rec_begin = sh.mask_rec_begin;
    aa.part_o = at<float>(m, y.part_o);
    aa.part_ml = at<float>(m, y.part_ml);
    aa.counters = att_counters;
    aa.out = attn;
    BC_CUDA(launch_attention(aa, st, true), "attention");
    if (!record(rec, st, NK_ATTN, l, aa)) return fail(BC_ECUDA, "capture: no node");
    ++launches;
    if (act) {
      BC_CUDA(step_select(m, SP_NONE, hq, k_o, attn, nullptr, nullptr, nullptr, nullptr, s_o, nullptr),
              "select o");
      ++launches;
    }
    BC_CUDA(step_gemv(m, 1, wo + (size_t)l * hq * d, hq, d, GP_NONE, attn, nullptr, nullptr, nullptr,
                      act ? s_o : nullptr, k_o, EPI_RESID, x, nullptr, nullptr, nullptr), "gemv o");
    ++launches;
    // feed-forward block: [select] -> gate/up GEMV (RMSNorm folded in) ->
    // [select] -> down GEMV (SwiGLU folded in) + residual
    if (act) {
      BC_CUDA(step_select(m, SP_NORM, d, k_gu, x, g_mlp, nullptr, nullptr, xn2, s_gu, nullptr),
              "select gate/up");
      ++launches;
    }
    BC_CUDA(step_gemv(m, 2, wgu + (size_t)l * d * 2 * f, d, 2 * f, GP_NORM, x, g_mlp, nullptr, nullptr,
                      act ? s_gu : nullptr, k_gu, sw ? EPI_SWIGLU : EPI_STORE, d_in_vec, nullptr, nullptr,
                      nullptr), "gemv gate/up");
    ++launches;
    if (act) {
      BC_CUDA(step_select(m, sw ? SP_NONE : SP_SWIGLU, f, k_d, d_in_vec, nullptr, nullptr, nullptr,
                          sw ? nullptr : hmid, s_d, nullptr),
              "select down");
      ++launches;
    }
    BC_CUDA(step_gemv(m, 3, wd + (size_t)l * f * d, f, d, sw ? GP_NONE : GP_SWIGLU, d_in_vec, nullptr, nullptr,
                      nullptr, act ? s_d : nullptr, k_d, EPI_RESID, x, xo, nullptr, nullptr), "gemv down");
    ++launches;
  }
  LmHeadArgs lm{static_cast<const __nv_bfloat16*>(m->w.lm_head), c.vocab, d, x,
                static_cast<const __nv_bfloat16*>(m->w.final_norm), c.rms_eps, logits};
  BC_CUDA(launch_lmhead(lm, m->sms, st, true), "lm head");
  if (!record(rec, st, NK_LMHEAD, 0, lm)) return fail(BC_ECUDA, "capture: no node");
  ++launches;
  *n_launch = launches;
  return BC_OK;
}

// Captures the step for this configuration on the private stream.
static bc_status capture_step(bc_model* m, int token, bc_mode mode, double rp, double rkv, int sinks,
                              int recent, float* logits, StepGraph** out) {
  if (!m->cap_stream) BC_CUDA(cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking), "capture stream");
  StepGraph* g = new StepGraph();
  g->mode = mode;
  g->psel = 0;
  g->rp = rp;
  g->rkv = rkv;
  g->sinks = sinks;
  g->recent = recent;
  g->graph = nullptr;
  g->exec = nullptr;
  cudaStream_t user = m->stream;
  m->stream = m->cap_stream;
  cudaError_t e = cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal);
  bc_status s = BC_OK;
  if (e == cudaSuccess) s = enqueue_step(m, token, mode, rp, rkv, sinks, recent, logits, &g->nodes, &g->launches);
  cudaError_t e2 = cudaStreamEndCapture(m->cap_stream, &g->graph);
  m->stream = user;
  if (e != cudaSuccess || s != BC_OK || e2 != cudaSuccess) {
    destroy_graph(g);
    cudaGetLastError();
    return fail(BC_ECUDA, "capturing the step failed (%s)", cudaGetErrorString(e != cudaSuccess ? e : e2));
  }
  e = cudaGraphInstantiate(&g->exec, g->graph, 0);
  for (size_t i = 0; e == cudaSuccess && i < g->nodes.size(); ++i)
    e = cudaGraphKernelNodeGetParams(g->nodes[i].node, &g->nodes[i].kp);
  if (e != cudaSuccess) {
    destroy_graph(g);
    return cuda_fail(e, "instantiating the step graph");
  }
  *out = g;
  return BC_OK;
}

// Points the recorded nodes at this step's position, token, page counts and
// logits buffer, then launches the graph on the model's stream.
static cudaError_t launch_step_graph(bc_model* m, StepGraph* g, int token, const StepShape& sh, float* logits) {
  const bc_config& c = m->cfg;
  const __nv_bfloat16* emb = static_cast<const __nv_bfloat16*>(m->w.embed) + (size_t)token * c.hidden;
  for (NodeRec& r : g->nodes) {
    cudaKernelNodeParams kp = r.kp;
    void* argp = &r.args;
    switch (r.kind) {
      case NK_QKV:
        r.args.g.qkv.pos = sh.pos;
        if (r.args.g.prep == GP_EMBED_NORM) r.args.g.embed_row = emb;
        break;
      case NK_SEL_EMBED:
        r.args.s.embed_row = emb;
        break;
      case NK_PAGES:
        r.args.p.P = sh.P;
        r.args.p.K = sh.K;
        r.args.p.rounds = page_rounds(sh.P, c.head_dim, c.n_kv_heads, m->sms);
        kp.gridDim = pages_grid(r.args.p);
        break;
      case NK_PAGE_SEL:
        r.args.p.P = sh.P;
        r.args.p.K = sh.K;
        break;
      case NK_ATTN:
        r.args.a.n_pages = sh.K;
        r.args.a.list_len = sh.list_len;
        r.args.a.tail0 = sh.tail0;
        r.args.a.n_tok = sh.n_tok;
        r.args.a.splits = sh.splits;
        r.args.a.pages_per_split = sh.pps;
        r.args.a.mask_sink_end = sh.mask_sink_end;
        r.args.a.mask_rec_begin = sh.mask_rec_begin;
        kp.gridDim = dim3(sh.splits, c.n_kv_heads);
        break;
      case NK_LMHEAD:
        r.args.lm.logits = logits;
        break;
    }
    kp.kernelParams = &argp;
    kp.extra = nullptr;
    cudaError_t e = cudaGraphExecKernelNodeSetParams(g->exec, r.node, &kp);
    if (e != cudaSuccess) return e;
  }
  return cudaGraphLaunch(g->exec, m->stream);
}

static bc_status run_step(bc_model* m, int token, bc_mode mode, double rp, double rkv, int sinks, int recent,
                          float* logits) {
  const StepShape sh = step_shape(m, mode, rp, rkv, sinks, recent);
  if (m->use_graphs) {
    StepGraph* g = nullptr;
    const bool kvs = mode == BC_KV || mode == BC_BOTH;
    const int psel = kvs ? page_select_variant(sh.P) : 0;
    for (StepGraph* c : m->graphs)
      if (c->mode == mode && c->psel == psel && c->rp == rp && c->rkv == rkv && c->sinks == sinks &&
          c->recent == recent)
        g = c;
    if (g) {
      cudaError_t e = launch_step_graph(m, g, token, sh, logits);
      if (e == cudaSuccess) {
        commit_step(m, mode, sh, g->launches);
        return BC_OK;
      }
      // an update the graph refused: drop it, run directly, capture again next time
      cudaGetLastError();
      m->graphs.erase(std::find(m->graphs.begin(), m->graphs.end(), g));
      destroy_graph(g);
    } else if (m->launches > 0) {
      // the kernels' attributes are set up by an earlier direct step: capture now
      if (capture_step(m, token, mode, rp, rkv, sinks, recent, logits, &g) == BC_OK) {
        g->psel = psel;
        m->graphs.push_back(g);
        if (launch_step_graph(m, g, token, sh, logits) == cudaSuccess) {
          commit_step(m, mode, sh, g->launches);
          return BC_OK;
        }
        cudaGetLastError();
        m->graphs.pop_back();
        destroy_graph(g);
      }
    }
  }
  long long launches = 0;
  bc_status s = enqueue_step(m, token, mode, rp, rkv, sinks, recent, logits, nullptr, &launches);
  if (s == BC_OK) commit_step(m, mode, sh, launches);
  return s;
}

extern "C" bc_status bc_decode_step(bc_model* m, int token, bc_mode mode, double rp, double rkv,
                                    int sinks, int recent, int page, float* logits) {
  bc_status s = check_step(m, mode, rp, rkv, sinks, recent, page);
  if (s != BC_OK) return s;
  if (!logits) return fail(BC_EINVAL, "null logits");
  if (token < 0 || token >= m->cfg.vocab) return fail(BC_EINVAL, "token %d outside the vocabulary", token);
  return run_step(m, token, mode, rp, rkv, sinks, recent, logits);
}

extern "C" bc_status bc_decode_step_host(bc_model* m, int token, bc_mode mode, double rp, double rkv,
                                         int sinks, int recent, int page, float* logits_host) {
  bc_status s = check_step(m, mode, rp, rkv, sinks, recent, page);
  if (s != BC_OK) return s;
  if (!logits_host) return fail(BC_EINVAL, "null logits");
  if (token < 0 || token >= m->cfg.vocab) return fail(BC_EINVAL, "token %d outside the vocabulary", token);
  float* dev = at<float>(m, m->lay.logits);
  s = run_step(m, token, mode, rp, rkv, sinks, recent, dev);
  if (s != BC_OK) return s;
  BC_CUDA(cudaMemcpyAsync(logits_host, dev, sizeof(float) * m->cfg.vocab, cudaMemcpyDeviceToHost, m->stream),
          "bc_decode_step_host: copy logits");
  BC_CUDA(cudaStreamSynchronize(m->stream), "bc_decode_step_host: sync");
  return BC_OK;
}

extern "C" bc_status bc_trace(const bc_model* m, int layer, bc_trace_kind kind, const void** ptr,
                              int* count, int* stride) {
  if (!m || !ptr || !count) return fail(BC_EINVAL, "null argument");
  const bc_config& c = m->cfg;
  const Layout& y = m->lay;
  if (layer < 0 || layer >= c.n_layers) return fail(BC_EINVAL, "layer %d out of range", layer);
  const int d = c.hidden, f = c.intermediate, hq = y.hq;
  size_t off = 0;
  int n = 0, st = 0;
  switch (kind) {
    case BC_TRACE_XN: off = y.xn + 4ull * layer * d; n = m->last_act ? d : 0; break;
    case BC_TRACE_SEL_QKV: off = y.sel_qkv + 4ull * layer * d; n = m->last_k[0]; break;
    case BC_TRACE_Q: off = y.q + 4ull * layer * hq; n = hq; break;
    case BC_TRACE_ATTN: off = y.attn + 4ull * layer * hq; n = hq; break;
    case BC_TRACE_SEL_O: off = y.sel_o + 4ull * layer * hq; n = m->last_k[1]; break;
    case BC_TRACE_XN2: off = y.xn2 + 4ull * layer * d; n = m->last_act ? d : 0; break;
    case BC_TRACE_SEL_GU: off = y.sel_gu + 4ull * layer * d; n = m->last_k[2]; break;
    case BC_TRACE_H: off = y.h + 4ull * layer * f; n = m->last_act ? f : 0; break;
    case BC_TRACE_SEL_D: off = y.sel_d + 4ull * layer * f; n = m->last_k[3]; break;
    case BC_TRACE_X: off = y.xo + 4ull * layer * d; n = d; break;
    case BC_TRACE_PAGE_SCORES:
      off = y.pscore + 4ull * layer * c.n_kv_heads * y.Pmax; n = m->last_K ? m->last_P : 0; st = y.Pmax; break;
    case BC_TRACE_PAGES:
      off = y.pages + 4ull * layer * c.n_kv_heads * y.Pmax; n = m->last_K; st = y.Pmax; break;
    case BC_TRACE_QKV: off = y.qkv + 4ull * layer * y.nqkv; n = y.nqkv; break;
    case BC_TRACE_SNAP_SCORES:
      off = y.snap_scores + 4ull * layer * c.n_kv_heads * y.Pmax; n = m->snap_valid ? m->snap_P : 0; st = y.Pmax;
      break;
    case BC_TRACE_SNAP_PAGES:
      off = y.snap_pages + 4ull * layer * c.n_kv_heads * y.Pmax; n = m->snap_valid ? m->snap_K : 0; st = y.Pmax;
      break;
    default: return fail(BC_EINVAL, "bad trace kind %d", (int)kind);
  }
  *ptr = m->ws + off;
  *count = n;
  if (stride) *stride = st;
  return BC_OK;
}

// ------------------------------------------------------------------ single kernels
extern "C" size_t bc_gemv_scratch_bytes(int d_out) {
  if (d_out <= 0 || d_out % kColTile) return 0;
  return align256(4ull * kGemvMaxContrib * d_out) + align256(4ull * (d_out / 128));
}

extern "C" bc_status bc_gemv(const void* W, int d_in, int d_out, const float* x, const int* idx, int k,
                             float* y, void* scratch, size_t scratch_bytes, void* stream) {
  if (!W || !x || !y || !scratch) return fail(BC_EINVAL, "null pointer");
  if (d_in <= 0 || d_out <= 0 || d_out % kColTile) return fail(BC_EINVAL, "d_out must be a positive multiple of 256");
  if (k < 1 || k > d_in || (!idx && k != d_in)) return fail(BC_EINVAL, "k must be in [1, d_in] (= d_in without idx)");
  if (scratch_bytes < bc_gemv_scratch_bytes(d_out)) return fail(BC_ENOMEM, "scratch too small");
  GemvArgs g;
  memset(&g, 0, sizeof g);
  g.W = static_cast<const __nv_bfloat16*>(W);
  g.d_in = d_in;
  g.d_out = d_out;
  g.prep = GP_NONE;
  g.x = x;
  g.idx = idx;
  g.k = k;
  gemv_plan(k, d_out, device_sms(), &g.TW, &g.S, &g.C);
  g.max_rows = (k + g.S * g.C - 1) / (g.S * g.C);
  g.partial = static_cast<float*>(scratch);
  g.counters = reinterpret_cast<unsigned*>(static_cast<char*>(scratch) + align256(4ull * kGemvMaxContrib * d_out));
  g.epi = EPI_STORE;
  g.y = y;
  BC_CUDA(launch_gemv(g, static_cast<cudaStream_t>(stream), true), "bc_gemv");
  return BC_OK;
}

extern "C" size_t bc_gemv_batch_scratch_bytes(int d_in, int d_out, int batch) {
  if (d_in < 1 || d_in > kMaxSelect || d_out < kColTile || d_out % kColTile || batch < 1 || batch > kBatchMax)
    return 0;
  return gemv_batch_scratch(d_in, d_out, batch);
}

extern "C" bc_status bc_gemv_batch(const void* W, int d_in, int d_out, const float* x, const int* idx, int k,
                                   int batch, float* y, int* n_union, void* scratch, size_t scratch_bytes,
                                   void* stream) {
  if (!W || !x || !y || !scratch) return fail(BC_EINVAL, "null pointer");
  if (batch < 1 || batch > kBatchMax) return fail(BC_EINVAL, "batch %d outside [1, %d]", batch, kBatchMax);
  if (d_in < 1 || d_in > kMaxSelect) return fail(BC_EINVAL, "d_in %d outside [1, %d]", d_in, kMaxSelect);
  if (d_out < kColTile || d_out % kColTile) return fail(BC_EINVAL, "d_out must be a positive multiple of 256");
  if (k < 1 || k > d_in || (!idx && k != d_in)) return fail(BC_EINVAL, "k must be in [1, d_in] (= d_in without idx)");
  if (scratch_bytes < gemv_batch_scratch(d_in, d_out, batch)) return fail(BC_ENOMEM, "scratch too small");
  BatchGemvArgs a;
  memset(&a, 0, sizeof a);
  a.W = static_cast<const __nv_bfloat16*>(W);
  a.d_in = d_in;
  a.d_out = d_out;
  a.k = k;
  a.B = batch;
  a.x = x;
  a.idx = idx;
  a.y = y;
  a.S = gemv_batch_splits(d_in, d_out, k, batch, device_sms());
  gemv_batch_bind(&a, scratch, n_union);
  BC_CUDA(launch_gemv_batch(a, static_cast<cudaStream_t>(stream), true), "bc_gemv_batch");
  return BC_OK;
}

extern "C" bc_status bc_select_topk(const float* v, int n, int k, int* idx, void* stream) {
  if (!v || !idx) return fail(BC_EINVAL, "null pointer");
  if (n < 1 || n > kMaxSelect || k < 1 || k > n) return fail(BC_EINVAL, "need 1 <= k <= n <= 16384");
  SelectArgs s;
  memset(&s, 0, sizeof s);
  s.prep = SP_NONE;
  s.n = n;
  s.k = k;
  s.x = v;
  s.idx = idx;
  BC_CUDA(launch_select(s, static_cast<cudaStream_t>(stream), true), "bc_select_topk");
  return BC_OK;
}

extern "C" size_t bc_attention_scratch_bytes(int n_q_heads, int head_dim) {
  if (n_q_heads <= 0 || head_dim <= 0) return 0;
  return align256(4ull * n_q_heads * kMaxSplits * head_dim) + align256(4ull * n_q_heads * kMaxSplits * 2) +
         align256(4ull * n_q_heads);
}

extern "C" bc_status bc_attention(const float* q, const void* kv, int n_kv_heads, int group, int head_dim,
                                  int Pmax, const int* pages, int n_pages, int n_tok, float* out,
                                  void* scratch, size_t scratch_bytes, void* stream) {
  if (!q || !kv || !out || !scratch) return fail(BC_EINVAL, "null pointer");
  if (((uintptr_t)q | (uintptr_t)kv | (uintptr_t)out) & 15) return fail(BC_EINVAL, "q, kv and out must be 16-byte aligned");
  if (head_dim != 64 && head_dim != 128) return fail(BC_EINVAL, "head_dim must be 64 or 128");
  if (n_kv_heads < 1 || group < 1 || group > 8) return fail(BC_EINVAL, "bad head counts");
  if (n_tok < 1 || n_pages < 1 || Pmax < n_pages || (n_tok + kPage - 1) / kPage > Pmax)
    return fail(BC_EINVAL, "bad page counts");
  if (!pages && n_pages != (n_tok + kPage - 1) / kPage) return fail(BC_EINVAL, "without a page list n_pages must cover n_tok");
  const int nq = n_kv_heads * group;
  if (scratch_bytes < bc_attention_scratch_bytes(nq, head_dim)) return fail(BC_ENOMEM, "scratch too small");
  AttnArgs a;
  memset(&a, 0, sizeof a);
  a.q = q;
  a.kv = static_cast<const __nv_bfloat16*>(kv);
  a.pages = pages;
  a.Hkv = n_kv_heads;
  a.G = group;
  a.hd = head_dim;
  a.Pmax = Pmax;
  a.n_pages = n_pages;
  a.n_tok = n_tok;
  a.list_len = n_pages;
  a.tail0 = 0;
  attn_plan(n_pages, n_kv_heads, device_sms(), &a.splits, &a.pages_per_split);
  char* sc = static_cast<char*>(scratch);
  const size_t o_bytes = align256(4ull * nq * kMaxSplits * head_dim);
  const size_t ml_bytes = align256(4ull * nq * kMaxSplits * 2);
  a.part_o = reinterpret_cast<float*>(sc);
  a.part_ml = reinterpret_cast<float*>(sc + o_bytes);
  a.counters = reinterpret_cast<unsigned*>(sc + o_bytes + ml_bytes);
  a.out = out;
  BC_CUDA(launch_attention(a, static_cast<cudaStream_t>(stream), true), "bc_attention");
  return BC_OK;
}
