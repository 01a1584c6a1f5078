// Batched decode step: `batch` sequences (1..8) of equal length share one
// pass over the weights.  The ByteCross README ("Usage: The byte account",
// crossover_batch) prices a batch as reading the union of its sequences'
// kept projection weights once per step; this is that step.
//
// Every sequence keeps its own channels (its own top-k of |x| at every
// projection input, as at batch 1) and its own KV pages; per layer:
//
//   prep (x*g and the RMSNorm scale of every sequence, or the embedding rows)
//   -> [act: select per sequence] -> projection over the union of the kept
//   rows (the bc_gemv_batch kernels: union, GEMV, split reduce) -> epilogue
//   per sequence (norm scale, rotary, bf16 KV append and page bounds; or the
//   residual add; or SwiGLU) -> [kv: page scores and page select per
//   sequence] -> split-K attention per sequence -> ... -> the LM head, whose
//   weights are read once for the whole batch.
//
// The per-sequence kernels are the batch-1 kernels launched over a batch grid
// dimension, each sequence offset by a fixed stride (the sequences' caches,
// bounds and activations are laid out back to back).  The step is captured
// in a CUDA graph per configuration, like the batch-1 step.
#include "../../include/bytecross.h"
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>
#include <algorithm>
#include <string>
#include <vector>

namespace bc {

// ------------------------------------------------------------------ kernels

struct BatchPrepArgs {
  int prep;                        // GP_NORM or GP_EMBED_NORM
  int d;
  const float* x;                  // [B][d] residual streams (NORM)
  const __nv_bfloat16* gain;       // [d]
  const __nv_bfloat16* embed;      // [vocab][d] (EMBED_NORM)
  int tokens[kBatchMax];           // EMBED_NORM: the sequences' tokens
  float eps;
  float* x_init;                   // EMBED_NORM: [B][d] residual streams initialised
  float* v;                        // [B][d] out: x * g
  float* scale;                    // [B] out: 1 / sqrt(mean(x^2) + eps)
};

constexpr int kPrepThreads = 256;

// One CTA per sequence: the projection input x*g and the norm's scale (the
// scale factors out of the projection and is applied by the epilogue).
__global__ void __launch_bounds__(kPrepThreads) k_batch_prep(BatchPrepArgs a) {
  __shared__ float s_red[kPrepThreads / 32];
  const int b = blockIdx.x, tid = threadIdx.x, d = a.d;
  pdl_wait();
  pdl_trigger();
  const float* xb = a.x + (size_t)b * d;
  const __nv_bfloat16* eb = a.embed + (size_t)a.tokens[b] * d;
  float* vb = a.v + (size_t)b * d;
  float ss = 0.f;
  for (int c = tid; c < d; c += kPrepThreads) {
    float xv;
    if (a.prep == GP_EMBED_NORM) {
      xv = bf16f(eb[c]);
      a.x_init[(size_t)b * d + c] = xv;
    } else {
      xv = xb[c];
    }
    ss = fmaf(xv, xv, ss);
    vb[c] = xv * bf16f(a.gain[c]);
  }
  const float tot = block_sum<kPrepThreads>(ss, s_red);
  if (tid == 0) a.scale[b] = 1.0f / sqrtf(tot / (float)d + a.eps);
}

struct BatchEpiArgs {
  int epi;                         // EPI_QKV, EPI_RESID or EPI_SWIGLU
  int d_out;                       // columns of y per sequence
  const float* y;                  // [B][d_out] projection outputs (unscaled)
  const float* scale;              // [B] norm scales, or nullptr (1)
  float* x;                        // RESID: [B][d_out] += y; SWIGLU: h [B][d_out / 2]
  float* x_copy;                   // RESID: [B][d_out] copy of the updated x, or nullptr
  float* raw;                      // QKV: [B][d_out] scaled, unrotated outputs, or nullptr
  QkvEpilogue qkv;                 // QKV: sequence 0's queries, pages and bounds
  long long q_stride, kv_stride, meta_stride;   // QKV: sequence strides (elements)
};

constexpr int kEpiCols = 128;      // columns per CTA: a multiple of every head size

// CTA (column tile, sequence).
__global__ void __launch_bounds__(kEpiCols) k_batch_epi(BatchEpiArgs a) {
  __shared__ float s_v[kColTile];
  const int b = blockIdx.y, tid = threadIdx.x;
  const int col0 = blockIdx.x * kEpiCols, col = col0 + tid;
  pdl_wait();
  pdl_trigger();
  const float s = a.scale ? a.scale[b] : 1.0f;
  const float* yb = a.y + (size_t)b * a.d_out;
  if (a.epi == EPI_QKV) {
    const float v = yb[col] * s;                 // d_out is a multiple of kEpiCols
    if (a.raw) a.raw[(size_t)b * a.d_out + col] = v;
    QkvEpilogue e = a.qkv;
    e.q_out += b * a.q_stride;
    e.kv_layer += b * a.kv_stride;
    e.meta_layer += b * a.meta_stride;
    qkv_epilogue<kEpiCols>(e, col0, v, s_v, qkv_prologue(e, col));
  } else if (a.epi == EPI_RESID) {
    if (col < a.d_out) {
      float* xb = a.x + (size_t)b * a.d_out;
      const float nx = xb[col] + yb[col];
      xb[col] = nx;
      if (a.x_copy) a.x_copy[(size_t)b * a.d_out + col] = nx;
    }
  } else {
    const int f = a.d_out / 2;
    if (col < f) {
      const float g = yb[col] * s, u = yb[f + col] * s;
      a.x[(size_t)b * f + col] = g / (1.0f + expf(-g)) * u;
    }
  }
}

struct BatchLmArgs {
  const __nv_bfloat16* W;          // [V][d]
  int V, d;
  const float* x;                  // [NB][d] residual streams
  const __nv_bfloat16* gain;       // final RMSNorm gain [d]
  float eps;
  float* logits;                   // [NB][V]
};

constexpr int kLmbThreads = 512;

// The LM head of the whole batch: every weight row is read once and dotted
// with the NB sequences' x*g (in shared memory); each sequence's final norm
// scale multiplies its dot products.  A warp streams two rows at a time.
template <int NB>
__global__ void __launch_bounds__(kLmbThreads) k_lmhead_batch(BatchLmArgs a) {
  extern __shared__ __align__(16) float s_x[];   // [NB][d]
  __shared__ float s_red[kLmbThreads / 32];
  __shared__ float s_scale[NB];
  const int tid = threadIdx.x, lane = tid & 31;
  pdl_wait();
  pdl_trigger();
  for (int b = 0; b < NB; ++b) {
    float ss = 0.f;
    for (int i = tid; i < a.d; i += kLmbThreads) {
      const float xv = a.x[(size_t)b * a.d + i];
      ss = fmaf(xv, xv, ss);
      s_x[b * a.d + i] = xv * bf16f(a.gain[i]);
    }
    const float tot = block_sum<kLmbThreads>(ss, s_red);
    if (tid == 0) s_scale[b] = 1.0f / sqrtf(tot / (float)a.d + a.eps);
  }
  __syncthreads();
  const int warps = gridDim.x * (kLmbThreads / 32);
  const int gw = blockIdx.x * (kLmbThreads / 32) + (tid >> 5);
  const int vecs = a.d / 8;
  for (int r = gw * 2; r < a.V; r += warps * 2) {
    const bool two = r + 1 < a.V;
    const __nv_bfloat16* w0 = a.W + (size_t)r * a.d;
    const __nv_bfloat16* w1 = w0 + a.d;
    float s0[NB], s1[NB];
    #pragma unroll
    for (int b = 0; b < NB; ++b) s0[b] = s1[b] = 0.f;
    for (int v = lane; v < vecs; v += 32 * 4) {
      uint4 x0[4], x1[4];
      #pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int vv = v + 32 * u;
        x0[u] = vv < vecs ? ld_stream(w0 + vv * 8) : make_uint4(0, 0, 0, 0);
        x1[u] = (two && vv < vecs) ? ld_stream(w1 + vv * 8) : make_uint4(0, 0, 0, 0);
      }
      #pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int vv = v + 32 * u;
        if (vv >= vecs) break;
        const float w0f[8] = {bf16_lo(x0[u].x), bf16_hi(x0[u].x), bf16_lo(x0[u].y), bf16_hi(x0[u].y),
                              bf16_lo(x0[u].z), bf16_hi(x0[u].z), bf16_lo(x0[u].w), bf16_hi(x0[u].w)};
        const float w1f[8] = {bf16_lo(x1[u].x), bf16_hi(x1[u].x), bf16_lo(x1[u].y), bf16_hi(x1[u].y),
                              bf16_lo(x1[u].z), bf16_hi(x1[u].z), bf16_lo(x1[u].w), bf16_hi(x1[u].w)};
        #pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float4 xa = *reinterpret_cast<const float4*>(&s_x[b * a.d + vv * 8]);
          const float4 xb = *reinterpret_cast<const float4*>(&s_x[b * a.d + vv * 8 + 4]);
          const float xs[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
          #pragma unroll
          for (int j = 0; j < 8; ++j) {
            s0[b] = fmaf(xs[j], w0f[j], s0[b]);
            s1[b] = fmaf(xs[j], w1f[j], s1[b]);
          }
        }
      }
    }
    #pragma unroll
    for (int b = 0; b < NB; ++b) {
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        s0[b] += __shfl_xor_sync(0xffffffffu, s0[b], o);
        s1[b] += __shfl_xor_sync(0xffffffffu, s1[b], o);
      }
    }
    if (lane == 0) {
      #pragma unroll
      for (int b = 0; b < NB; ++b) {
        a.logits[(size_t)b * a.V + r] = s0[b] * s_scale[b];
        if (two) a.logits[(size_t)b * a.V + r + 1] = s1[b] * s_scale[b];
      }
    }
  }
}

static cudaLaunchConfig_t batch_cfg(dim3 g, dim3 blk, size_t smem, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = g;
  cfg.blockDim = blk;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Largest dynamic shared memory a CTA of the batched LM head may take: the
// device's opt-in limit less a margin for the kernel's static arrays.
static int lm_smem_limit() {
  static int limit = -1;
  if (limit < 0) {
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      optin = 227 * 1024;
    cudaGetLastError();
    limit = optin - 1024;
  }
  return limit;
}

template <int NB>
static cudaError_t launch_lm_nb(const BatchLmArgs& a, int sms, cudaStream_t st) {
  static bool attr_done = false;
  const size_t smem = (size_t)NB * a.d * sizeof(float);
  if (smem > (size_t)lm_smem_limit()) return cudaErrorInvalidValue;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_lmhead_batch<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         std::min(lm_smem_limit(), (int)(NB * kMaxSelect * sizeof(float))));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int rows_per_cta = 2 * (kLmbThreads / 32);
  const int ctas = std::min(2 * sms, (a.V + rows_per_cta - 1) / rows_per_cta);
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t c = batch_cfg(dim3(ctas), dim3(kLmbThreads), smem, st, attr);
  return cudaLaunchKernelEx(&c, k_lmhead_batch<NB>, a);
}

static cudaError_t launch_lm_batch(const BatchLmArgs& a, int nb, int sms, cudaStream_t st) {
  switch (nb) {
    case 1: return launch_lm_nb<1>(a, sms, st);
    case 2: return launch_lm_nb<2>(a, sms, st);
    case 3: return launch_lm_nb<3>(a, sms, st);
    case 4: return launch_lm_nb<4>(a, sms, st);
    case 5: return launch_lm_nb<5>(a, sms, st);
    case 6: return launch_lm_nb<6>(a, sms, st);
    case 7: return launch_lm_nb<7>(a, sms, st);
    default: return launch_lm_nb<8>(a, sms, st);
  }
}

}  // namespace bc

using namespace bc;

// ------------------------------------------------------------------ host side

static bc_status bfail(bc_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static bc_status bfail(bc_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  set_error(buf);
  return s;
}

#define BC_BCUDA(call, where)                                                     \
  do {                                                                            \
    cudaError_t e_ = (call);                                                      \
    if (e_ != cudaSuccess) return bfail(BC_ECUDA, "%s: %s", where, cudaGetErrorString(e_)); \
  } while (0)

static size_t b_align(size_t x) { return (x + 255) & ~(size_t)255; }

namespace {

struct BatchLayout {
  size_t x, v_qkv, v_gu, scale, y, q, attn, h, xo, raw;    // f32
  size_t sel;                                                // int32 [L][4][B * max(d, f)]
  size_t pscore, pages;                                      // [L][B][Hkv][Pmax]
  size_t part_o, part_ml, counters;
  size_t gscratch;
  size_t total;
  int nqkv, hq, Pmax, sel_stride;
};

BatchLayout batch_layout(const bc_config* c, int B) {
  BatchLayout y;
  const size_t L = c->n_layers, d = c->hidden, f = c->intermediate;
  y.hq = c->n_heads * c->head_dim;
  y.nqkv = (c->n_heads + 2 * c->n_kv_heads) * c->head_dim;
  y.Pmax = (c->max_ctx + kPage - 1) / kPage;
  y.sel_stride = (int)(B * std::max(d, f));
  const size_t max_dout = std::max<size_t>(std::max<size_t>(y.nqkv, d), 2 * f);
  const size_t nq = c->n_heads;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = b_align(o + bytes); return at; };
  y.x = take(4 * B * d);
  y.v_qkv = take(4 * L * B * d);
  y.v_gu = take(4 * L * B * d);
  y.scale = take(4 * B);
  y.y = take(4 * B * max_dout);
  y.q = take(4 * L * B * y.hq);
  y.attn = take(4 * L * B * y.hq);
  y.h = take(4 * L * B * f);
  y.xo = take(4 * L * B * d);
  y.raw = take(4 * L * B * y.nqkv);
  y.sel = take(4 * L * 4 * (size_t)y.sel_stride);
  y.pscore = take(4 * L * B * c->n_kv_heads * (size_t)y.Pmax);
  y.pages = take(4 * L * B * c->n_kv_heads * (size_t)y.Pmax);
  y.part_o = take(4 * (size_t)B * nq * kMaxSplits * c->head_dim);
  y.part_ml = take(4 * (size_t)B * nq * kMaxSplits * 2);
  y.counters = take(4 * (size_t)B * c->n_kv_heads);
  y.gscratch = take(gemv_batch_scratch((int)std::max(d, f), (int)max_dout, B));
  y.total = o;
  return y;
}

bool batch_config_ok(const bc_config* c, int B, std::string* why) {
  if (!c) { *why = "null config"; return false; }
  if (B < 1 || B > kBatchMax) { *why = "batch must be 1..8"; return false; }
  if (c->n_layers < 1 || c->hidden < 1 || c->intermediate < 1 || c->vocab < 1 || c->max_ctx < 1) {
    *why = "dimensions must be positive"; return false;
  }
  if (c->head_dim != 64 && c->head_dim != 128) { *why = "head_dim must be 64 or 128"; return false; }
  if (c->n_kv_heads < 1 || c->n_heads % c->n_kv_heads != 0 || c->n_heads / c->n_kv_heads > 8) {
    *why = "n_heads must be 1..8 times n_kv_heads"; return false;
  }
  if (c->n_heads * c->head_dim != c->hidden) { *why = "n_heads * head_dim must equal hidden"; return false; }
  if (c->page != kPage) { *why = "page must be 16"; return false; }
  if (c->hidden % kColTile || c->intermediate % kColTile) { *why = "hidden and intermediate must be multiples of 256"; return false; }
  if (((c->n_heads + 2 * c->n_kv_heads) * c->head_dim) % kEpiCols) { *why = "q/k/v width must be a multiple of 128"; return false; }
  if (c->intermediate > kMaxSelect || c->hidden > kMaxSelect) { *why = "hidden/intermediate above 16384"; return false; }
  if ((c->max_ctx + kPage - 1) / kPage > kMaxSelect) { *why = "max_ctx above 262144"; return false; }
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) { *why = "rms_eps > 0 and rope_theta > 1 required"; return false; }
  return true;
}

size_t kv_seq_elems(const bc_config* c) {
  const size_t Pmax = (c->max_ctx + kPage - 1) / kPage;
  return (size_t)c->n_layers * c->n_kv_heads * Pmax * 2 * kPage * c->head_dim;
}
size_t meta_seq_elems(const bc_config* c) {
  const size_t Pmax = (c->max_ctx + kPage - 1) / kPage;
  return (size_t)c->n_layers * c->n_kv_heads * Pmax * 2 * c->head_dim;
}

enum BatchNodeKind { BN_PREP0 = 0, BN_EPI_QKV, BN_PAGES, BN_PSEL, BN_ATTN, BN_LM };
struct BatchNode {
  cudaGraphNode_t node;
  int kind;
  cudaKernelNodeParams kp;
  union {
    BatchPrepArgs prep;
    BatchEpiArgs epi;
    PageArgs p;
    AttnArgs a;
    BatchLmArgs lm;
  } args;
};

struct BatchGraph {
  bc_mode mode;
  int psel;
  double rp, rkv;
  int sinks, recent;
  cudaGraph_t graph;
  cudaGraphExec_t exec;
  std::vector<BatchNode> nodes;
  long long launches;
};

void destroy_bgraph(BatchGraph* g) {
  if (!g) return;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
}

struct BatchShape {
  int pos, n_tok, P, K, splits, pps;
  int k_qkv, k_o, k_gu, k_d;
};

int b_keep(double ratio, int n) {
  const double v = ceil(ratio * n - 1e-9);
  return (int)std::max(1.0, std::min((double)n, v));
}

}  // namespace

struct bc_batch {
  bc_config cfg;
  bc_weights w;
  int B;
  __nv_bfloat16* kv;
  __nv_bfloat16* meta;
  size_t kv_seq, meta_seq;         // elements per sequence
  char* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  BatchLayout lay;
  int n;
  int sms;
  long long launches;
  int last_k[4], last_P, last_K;
  bool last_act, last_kv;
  bool use_graphs;
  cudaStream_t cap_stream;
  std::vector<BatchGraph*> graphs;
};

template <typename T>
static T* bat(const bc_batch* m, size_t off) { return reinterpret_cast<T*>(m->ws + off); }

static int b_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

extern "C" size_t bc_batch_workspace_bytes(const bc_config* cfg, int batch) {
  std::string why;
  if (!batch_config_ok(cfg, batch, &why)) return 0;
  return batch_layout(cfg, batch).total;
}

extern "C" bc_status bc_batch_create(const bc_config* cfg, const bc_weights* w, int batch, void* kv_pools,
                                     void* meta_pools, void* workspace, size_t ws_bytes, void* stream,
                                     bc_batch** out) {
  std::string why;
  if (!out) return bfail(BC_EINVAL, "out is null");
  *out = nullptr;
  if (!batch_config_ok(cfg, batch, &why)) return bfail(BC_EINVAL, "bad batch config: %s", why.c_str());
  if (!w || !w->embed || !w->lm_head || !w->final_norm || !w->attn_norm || !w->mlp_norm || !w->wqkv_t ||
      !w->wo_t || !w->wgu_t || !w->wd_t)
    return bfail(BC_EINVAL, "null weight pointer");
  if (!kv_pools || !meta_pools || !workspace) return bfail(BC_EINVAL, "null pools or workspace");
  if (((uintptr_t)kv_pools | (uintptr_t)meta_pools | (uintptr_t)workspace) & 255)
    return bfail(BC_EINVAL, "pools and workspace must be 256-byte aligned");
  if ((size_t)batch * cfg->hidden * sizeof(float) > (size_t)lm_smem_limit())
    return bfail(BC_EINVAL, "batch * hidden floats (%zu bytes) exceed the shared memory of one CTA (%d)",
                 (size_t)batch * cfg->hidden * sizeof(float), lm_smem_limit());
  BatchLayout lay = batch_layout(cfg, batch);
  if (ws_bytes < lay.total) return bfail(BC_ENOMEM, "workspace has %zu bytes, needs %zu", ws_bytes, lay.total);
  bc_batch* m = new bc_batch();
  m->cfg = *cfg;
  m->w = *w;
  m->B = batch;
  m->kv = static_cast<__nv_bfloat16*>(kv_pools);
  m->meta = static_cast<__nv_bfloat16*>(meta_pools);
  m->kv_seq = kv_seq_elems(cfg);
  m->meta_seq = meta_seq_elems(cfg);
  m->ws = static_cast<char*>(workspace);
  m->ws_bytes = ws_bytes;
  m->stream = static_cast<cudaStream_t>(stream);
  m->lay = lay;
  m->n = 0;
  m->sms = b_sms();
  m->launches = 0;
  memset(m->last_k, 0, sizeof m->last_k);
  m->last_P = m->last_K = 0;
  m->last_act = m->last_kv = false;
  m->use_graphs = true;
  m->cap_stream = nullptr;
  cudaError_t e = cudaMemsetAsync(m->ws + lay.counters, 0, 4ull * batch * cfg->n_kv_heads, m->stream);
  if (e != cudaSuccess) {
    delete m;
    return bfail(BC_ECUDA, "bc_batch_create: clearing counters: %s", cudaGetErrorString(e));
  }
  *out = m;
  return BC_OK;
}

extern "C" bc_status bc_batch_destroy(bc_batch* m) {
  if (!m) return BC_OK;
  for (BatchGraph* g : m->graphs) destroy_bgraph(g);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  delete m;
  return BC_OK;
}

extern "C" bc_status bc_batch_set_graphs(bc_batch* m, int enable) {
  if (!m) return bfail(BC_EINVAL, "null batch");
  m->use_graphs = enable != 0;
  return BC_OK;
}

extern "C" int bc_batch_length(const bc_batch* m) { return m ? m->n : -1; }

extern "C" long long bc_batch_launch_count(const bc_batch* m) { return m ? m->launches : -1; }

extern "C" bc_status bc_batch_reset(bc_batch* m, int n_ctx) {
  if (!m) return bfail(BC_EINVAL, "null batch");
  if (n_ctx < 0 || n_ctx > m->n) return bfail(BC_EINVAL, "reset to %d outside [0, %d]", n_ctx, m->n);
  m->n = n_ctx;
  return BC_OK;
}

extern "C" bc_status bc_batch_append(bc_batch* m, const void* k, const void* v, int n_tokens) {
  if (!m) return bfail(BC_EINVAL, "null batch");
  if (n_tokens < 0) return bfail(BC_EINVAL, "n_tokens < 0");
  if (n_tokens == 0) return BC_OK;
  if (!k || !v) return bfail(BC_EINVAL, "null k or v");
  if ((long long)m->n + n_tokens > m->cfg.max_ctx)
    return bfail(BC_ECAPACITY, "append of %d tokens to %d exceeds max_ctx %d", n_tokens, m->n, m->cfg.max_ctx);
  // the batch's pools are the sequences' pools back to back: one append over
  // batch * n_layers layers
  KvAppendArgs a;
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.n_new = n_tokens;
  a.n0 = m->n;
  a.L = m->B * m->cfg.n_layers;
  a.Hkv = m->cfg.n_kv_heads;
  a.hd = m->cfg.head_dim;
  a.Pmax = m->lay.Pmax;
  a.pool = m->kv;
  a.meta = m->meta;
  BC_BCUDA(launch_kv_append(a, m->stream, true), "bc_batch_append");
  m->launches += 2;
  m->n += n_tokens;
  return BC_OK;
}

static BatchShape batch_shape(const bc_batch* m, bc_mode mode, double rp, double rkv, int sinks, int recent) {
  const bc_config& c = m->cfg;
  const bool act = mode == BC_ACT || mode == BC_BOTH;
  const bool kvs = mode == BC_KV || mode == BC_BOTH;
  BatchShape sh;
  sh.pos = m->n;
  sh.n_tok = sh.pos + 1;
  sh.P = (sh.n_tok + kPage - 1) / kPage;
  sh.K = sh.P;
  if (kvs) {
    const int sink_end = std::min(sinks, sh.P), rec_begin = std::max(sh.P - recent, 0);
    const int n_forced = sink_end + (sh.P - std::max(rec_begin, sink_end));
    const int want = (int)std::min<double>(sh.P, ceil(rkv * sh.P - 1e-9));
    sh.K = std::max(n_forced, want);
  }
  // the batch's B * Hkv kv heads share the machine
  attn_plan(sh.K, c.n_kv_heads * m->B, m->sms, &sh.splits, &sh.pps);
  sh.k_qkv = act ? b_keep(rp, c.hidden) : c.hidden;
  sh.k_o = act ? b_keep(rp, m->lay.hq) : m->lay.hq;
  sh.k_gu = act ? b_keep(rp, c.hidden) : c.hidden;
  sh.k_d = act ? b_keep(rp, c.intermediate) : c.intermediate;
  return sh;
}

static cudaGraphNode_t b_captured_node(cudaStream_t st) {
  cudaStreamCaptureStatus status;
  const cudaGraphNode_t* deps = nullptr;
  size_t n = 0;
  if (cudaStreamGetCaptureInfo(st, &status, nullptr, nullptr, &deps, &n) != cudaSuccess) return nullptr;
  return (status == cudaStreamCaptureStatusActive && n == 1) ? deps[0] : nullptr;
}

template <typename A>
static bool b_record(std::vector<BatchNode>* rec, cudaStream_t st, int kind, const A& args) {
  if (!rec) return true;
  BatchNode r;
  memset(&r, 0, sizeof r);
  r.node = b_captured_node(st);
  if (!r.node) return false;
  r.kind = kind;
  memcpy(&r.args, &args, sizeof(A));
  rec->push_back(r);
  return true;
}

// The projection of one site for the whole batch: union of the kept rows,
// the GEMV over it, the split reduce (bc_gemv_batch's kernels).
static cudaError_t batch_projection(bc_batch* m, const __nv_bfloat16* W, int d_in, int d_out, const float* x,
                                    const int* idx, int k, float* y, long long* launches) {
  BatchGemvArgs g;
  memset(&g, 0, sizeof g);
  g.W = W;
  g.d_in = d_in;
  g.d_out = d_out;
  g.k = k;
  g.B = m->B;
  g.x = x;
  g.idx = idx;
  g.y = y;
  g.S = gemv_batch_splits(d_in, d_out, k, m->B, m->sms);
  gemv_batch_bind(&g, m->ws + m->lay.gscratch, nullptr);
  *launches += g.S > 1 ? 3 : 2;
  return launch_gemv_batch(g, m->stream, true);
}

static bc_status enqueue_batch(bc_batch* m, const int* tokens, bc_mode mode, double rp, double rkv, int sinks,
                               int recent, float* logits, std::vector<BatchNode>* rec, long long* n_launch) {
  const bc_config& c = m->cfg;
  const BatchLayout& y = m->lay;
  const bool act = mode == BC_ACT || mode == BC_BOTH;
  const bool kvs = mode == BC_KV || mode == BC_BOTH;
  const int B = m->B, L = c.n_layers, d = c.hidden, f = c.intermediate, hd = c.head_dim;
  const int Hq = c.n_heads, Hkv = c.n_kv_heads, G = Hq / Hkv;
  const int hq = y.hq, nqkv = y.nqkv, Pmax = y.Pmax;
  const BatchShape sh = batch_shape(m, mode, rp, rkv, sinks, recent);
  cudaStream_t st = m->stream;
  long long launches = 0;
  cudaLaunchAttribute attr[1];

  const __nv_bfloat16* attn_norm = static_cast<const __nv_bfloat16*>(m->w.attn_norm);
  const __nv_bfloat16* mlp_norm = static_cast<const __nv_bfloat16*>(m->w.mlp_norm);
  const __nv_bfloat16* wqkv = static_cast<const __nv_bfloat16*>(m->w.wqkv_t);
  const __nv_bfloat16* wo = static_cast<const __nv_bfloat16*>(m->w.wo_t);
  const __nv_bfloat16* wgu = static_cast<const __nv_bfloat16*>(m->w.wgu_t);
  const __nv_bfloat16* wd = static_cast<const __nv_bfloat16*>(m->w.wd_t);
  float* X = bat<float>(m, y.x);
  float* S = bat<float>(m, y.scale);
  float* Y = bat<float>(m, y.y);
  const size_t kv_layer = (size_t)Hkv * Pmax * 2 * kPage * hd;
  const size_t meta_layer = (size_t)Hkv * Pmax * 2 * hd;
  unsigned* counters = bat<unsigned>(m, y.counters);

  for (int l = 0; l < L; ++l) {
    float* Vq = bat<float>(m, y.v_qkv) + (size_t)l * B * d;
    float* Vg = bat<float>(m, y.v_gu) + (size_t)l * B * d;
    float* Q = bat<float>(m, y.q) + (size_t)l * B * hq;
    float* A = bat<float>(m, y.attn) + (size_t)l * B * hq;
    float* Hm = bat<float>(m, y.h) + (size_t)l * B * f;
    float* XO = bat<float>(m, y.xo) + (size_t)l * B * d;
    float* RAW = bat<float>(m, y.raw) + (size_t)l * B * nqkv;
    int* sel = bat<int>(m, y.sel) + (size_t)l * 4 * y.sel_stride;
    float* PS = bat<float>(m, y.pscore) + (size_t)l * B * Hkv * Pmax;
    int* PG = bat<int>(m, y.pages) + (size_t)l * B * Hkv * Pmax;

    // ---- attention block
    BatchPrepArgs pr;
    memset(&pr, 0, sizeof pr);
    pr.prep = l == 0 ? GP_EMBED_NORM : GP_NORM;
    pr.d = d;
    pr.x = X;
    pr.gain = attn_norm + (size_t)l * d;
    pr.embed = static_cast<const __nv_bfloat16*>(m->w.embed);
    for (int b = 0; b < B; ++b) pr.tokens[b] = tokens[b];
    pr.eps = c.rms_eps;
    pr.x_init = X;
    pr.v = Vq;
    pr.scale = S;
    {
      cudaLaunchConfig_t cfg = batch_cfg(dim3(B), dim3(kPrepThreads), 0, st, attr);
      BC_BCUDA(cudaLaunchKernelEx(&cfg, k_batch_prep, pr), "batch prep");
      if (l == 0 && !b_record(rec, st, BN_PREP0, pr)) return bfail(BC_ECUDA, "capture: no node");
      ++launches;
    }
    int* s_qkv = sel;
    if (act) {
      SelectArgs sa;
      memset(&sa, 0, sizeof sa);
      sa.prep = SP_NONE;
      sa.n = d;
      sa.k = sh.k_qkv;
      sa.x = Vq;
      sa.idx = s_qkv;
      sa.x_stride = d;
      sa.idx_stride = sh.k_qkv;
      BC_BCUDA(launch_select(sa, st, true, B), "batch select qkv");
      ++launches;
    }
    BC_BCUDA(batch_projection(m, wqkv + (size_t)l * d * nqkv, d, nqkv, Vq, act ? s_qkv : nullptr, sh.k_qkv, Y,
                              &launches), "batch projection qkv");
    BatchEpiArgs ea;
    memset(&ea, 0, sizeof ea);
    ea.epi = EPI_QKV;
    ea.d_out = nqkv;
    ea.y = Y;
    ea.scale = S;
    ea.raw = RAW;
    ea.qkv.Hq = Hq;
    ea.qkv.Hkv = Hkv;
    ea.qkv.hd = hd;
    ea.qkv.pos = sh.pos;
    ea.qkv.Pmax = Pmax;
    ea.qkv.rope_theta = c.rope_theta;
    ea.qkv.q_out = Q;
    ea.qkv.kv_layer = m->kv + l * kv_layer;
    ea.qkv.meta_layer = m->meta + l * meta_layer;
    ea.q_stride = hq;
    ea.kv_stride = (long long)m->kv_seq;
    ea.meta_stride = (long long)m->meta_seq;
    {
      cudaLaunchConfig_t cfg = batch_cfg(dim3(nqkv / kEpiCols, B), dim3(kEpiCols), 0, st, attr);
      BC_BCUDA(cudaLaunchKernelEx(&cfg, k_batch_epi, ea), "batch epilogue qkv");
      if (!b_record(rec, st, BN_EPI_QKV, ea)) return bfail(BC_ECUDA, "capture: no node");
      ++launches;
    }
    if (kvs) {
      PageArgs pa;
      memset(&pa, 0, sizeof pa);
      pa.q = Q;
      pa.meta = m->meta + l * meta_layer;
      pa.Hkv = Hkv;
      pa.G = G;
      pa.hd = hd;
      pa.Pmax = Pmax;
      pa.P = sh.P;
      pa.K = sh.K;
      pa.sinks = sinks;
      pa.recent = recent;
      pa.rounds = page_rounds(sh.P, hd, Hkv * B, m->sms);
      pa.scores = PS;
      pa.pages = PG;
      pa.q_stride = hq;
      pa.meta_stride = (long long)m->meta_seq;
      pa.sp_stride = (long long)Hkv * Pmax;
      BC_BCUDA(launch_page_scores(pa, st, true, B), "batch page scores");
      if (!b_record(rec, st, BN_PAGES, pa)) return bfail(BC_ECUDA, "capture: no node");
      BC_BCUDA(launch_page_select(pa, st, true, B), "batch page select");
      if (!b_record(rec, st, BN_PSEL, pa)) return bfail(BC_ECUDA, "capture: no node");
      launches += 2;
    }
    AttnArgs aa;
    memset(&aa, 0, sizeof aa);
    aa.q = Q;
    aa.kv = m->kv + l * kv_layer;
    aa.pages = kvs ? PG : nullptr;
    aa.Hkv = Hkv;
    aa.G = G;
    aa.hd = hd;
    aa.Pmax = Pmax;
    aa.n_pages = sh.K;
    aa.n_tok = sh.n_tok;
    aa.list_len = kvs ? sh.K : 0;
    aa.tail0 = 0;
    aa.splits = sh.splits;
    aa.pages_per_split = sh.pps;
    aa.part_o = bat<float>(m, y.part_o);
    aa.part_ml = bat<float>(m, y.part_ml);
    aa.counters = counters;
    aa.out = A;
    aa.q_stride = hq;
    aa.kv_stride = (long long)m->kv_seq;
    aa.list_stride = (long long)Hkv * Pmax;
    aa.part_stride = (long long)Hq * kMaxSplits;
    aa.out_stride = hq;
    aa.counters_stride = Hkv;
    BC_BCUDA(launch_attention(aa, st, true, B), "batch attention");
    if (!b_record(rec, st, BN_ATTN, aa)) return bfail(BC_ECUDA, "capture: no node");
    ++launches;

    // ---- o projection + residual
    int* s_o = sel + y.sel_stride;
    if (act) {
      SelectArgs sa;
      memset(&sa, 0, sizeof sa);
      sa.prep = SP_NONE;
      sa.n = hq;
      sa.k = sh.k_o;
      sa.x = A;
      sa.idx = s_o;
      sa.x_stride = hq;
      sa.idx_stride = sh.k_o;
      BC_BCUDA(launch_select(sa, st, true, B), "batch select o");
      ++launches;
    }
    BC_BCUDA(batch_projection(m, wo + (size_t)l * hq * d, hq, d, A, act ? s_o : nullptr, sh.k_o, Y, &launches),
             "batch projection o");
    memset(&ea, 0, sizeof ea);
    ea.epi = EPI_RESID;
    ea.d_out = d;
    ea.y = Y;
    ea.x = X;
    {
      cudaLaunchConfig_t cfg = batch_cfg(dim3((d + kEpiCols - 1) / kEpiCols, B), dim3(kEpiCols), 0, st, attr);
      BC_BCUDA(cudaLaunchKernelEx(&cfg, k_batch_epi, ea), "batch epilogue o");
      ++launches;
    }

    // ---- feed-forward block
    pr.prep = GP_NORM;
    pr.gain = mlp_norm + (size_t)l * d;
    pr.v = Vg;
    {
      cudaLaunchConfig_t cfg = batch_cfg(dim3(B), dim3(kPrepThreads), 0, st, attr);
      BC_BCUDA(cudaLaunchKernelEx(&cfg, k_batch_prep, pr), "batch prep mlp");
      ++launches;
    }
    int* s_gu = sel + 2 * (size_t)y.sel_stride;
    if (act) {
      SelectArgs sa;
      memset(&sa, 0, sizeof sa);
      sa.prep = SP_NONE;
      sa.n = d;
      sa.k = sh.k_gu;
      sa.x = Vg;
      sa.idx = s_gu;
      sa.x_stride = d;
      sa.idx_stride = sh.k_gu;
      BC_BCUDA(launch_select(sa, st, true, B), "batch select gate/up");
      ++launches;
    }
    BC_BCUDA(batch_projection(m, wgu + (size_t)l * d * 2 * f, d, 2 * f, Vg, act ? s_gu : nullptr, sh.k_gu, Y,
                              &launches), "batch projection gate/up");
    memset(&ea, 0, sizeof ea);
    ea.epi = EPI_SWIGLU;
    ea.d_out = 2 * f;
    ea.y = Y;
    ea.scale = S;
    ea.x = Hm;
    {
      cudaLaunchConfig_t cfg = batch_cfg(dim3((f + kEpiCols - 1) / kEpiCols, B), dim3(kEpiCols), 0, st, attr);
      BC_BCUDA(cudaLaunchKernelEx(&cfg, k_batch_epi, ea), "batch epilogue swiglu");
      ++launches;
    }
    int* s_d = sel + 3 * (size_t)y.sel_stride;
    if (act) {
      SelectArgs sa;
      memset(&sa, 0, sizeof sa);
      sa.prep = SP_NONE;
      sa.n = f;
      sa.k = sh.k_d;
      sa.x = Hm;
      sa.idx = s_d;
      sa.x_stride = f;
      sa.idx_stride = sh.k_d;
      BC_BCUDA(launch_select(sa, st, true, B), "batch select down");
      ++launches;
    }
    BC_BCUDA(batch_projection(m, wd + (size_t)l * f * d, f, d, Hm, act ? s_d : nullptr, sh.k_d, Y, &launches),
             "batch projection down");
    memset(&ea, 0, sizeof ea);
    ea.epi = EPI_RESID;
    ea.d_out = d;
    ea.y = Y;
    ea.x = X;
    ea.x_copy = XO;
    {
      cudaLaunchConfig_t cfg = batch_cfg(dim3((d + kEpiCols - 1) / kEpiCols, B), dim3(kEpiCols), 0, st, attr);
      BC_BCUDA(cudaLaunchKernelEx(&cfg, k_batch_epi, ea), "batch epilogue down");
      ++launches;
    }
  }
  BatchLmArgs lm{static_cast<const __nv_bfloat16*>(m->w.lm_head), c.vocab, d, X,
                 static_cast<const __nv_bfloat16*>(m->w.final_norm), c.rms_eps, logits};
  BC_BCUDA(launch_lm_batch(lm, B, m->sms, st), "batch lm head");
  if (!b_record(rec, st, BN_LM, lm)) return bfail(BC_ECUDA, "capture: no node");
  ++launches;
  *n_launch = launches;
  return BC_OK;
}

static bc_status capture_batch(bc_batch* m, const int* tokens, bc_mode mode, double rp, double rkv, int sinks,
                               int recent, float* logits, BatchGraph** out) {
  if (!m->cap_stream) BC_BCUDA(cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking), "capture stream");
  BatchGraph* g = new BatchGraph();
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
  if (e == cudaSuccess) s = enqueue_batch(m, tokens, mode, rp, rkv, sinks, recent, logits, &g->nodes, &g->launches);
  cudaError_t e2 = cudaStreamEndCapture(m->cap_stream, &g->graph);
  m->stream = user;
  if (e != cudaSuccess || s != BC_OK || e2 != cudaSuccess) {
    destroy_bgraph(g);
    cudaGetLastError();
    return bfail(BC_ECUDA, "capturing the batch step failed (%s)", cudaGetErrorString(e != cudaSuccess ? e : e2));
  }
  e = cudaGraphInstantiate(&g->exec, g->graph, 0);
  for (size_t i = 0; e == cudaSuccess && i < g->nodes.size(); ++i)
    e = cudaGraphKernelNodeGetParams(g->nodes[i].node, &g->nodes[i].kp);
  if (e != cudaSuccess) {
    destroy_bgraph(g);
    return bfail(BC_ECUDA, "instantiating the batch step graph: %s", cudaGetErrorString(e));
  }
  *out = g;
  return BC_OK;
}

static cudaError_t launch_batch_graph(bc_batch* m, BatchGraph* g, const int* tokens, const BatchShape& sh,
                                      float* logits) {
  const bc_config& c = m->cfg;
  for (BatchNode& r : g->nodes) {
    cudaKernelNodeParams kp = r.kp;
    void* argp = &r.args;
    switch (r.kind) {
      case BN_PREP0:
        for (int b = 0; b < m->B; ++b) r.args.prep.tokens[b] = tokens[b];
        break;
      case BN_EPI_QKV:
        r.args.epi.qkv.pos = sh.pos;
        break;
      case BN_PAGES:
        r.args.p.P = sh.P;
        r.args.p.K = sh.K;
        r.args.p.rounds = page_rounds(sh.P, c.head_dim, c.n_kv_heads * m->B, m->sms);
        kp.gridDim = pages_grid(r.args.p);
        kp.gridDim.z = m->B;
        break;
      case BN_PSEL:
        r.args.p.P = sh.P;
        r.args.p.K = sh.K;
        break;
      case BN_ATTN:
        r.args.a.n_pages = sh.K;
        r.args.a.list_len = r.args.a.pages ? sh.K : 0;
        r.args.a.n_tok = sh.n_tok;
        r.args.a.splits = sh.splits;
        r.args.a.pages_per_split = sh.pps;
        kp.gridDim = dim3(sh.splits, c.n_kv_heads, m->B);
        break;
      case BN_LM:
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

static void commit_batch(bc_batch* m, bc_mode mode, const BatchShape& sh, long long launches) {
  const bool act = mode == BC_ACT || mode == BC_BOTH;
  const bool kvs = mode == BC_KV || mode == BC_BOTH;
  m->launches += launches;
  m->n = sh.n_tok;
  m->last_k[0] = act ? sh.k_qkv : 0;
  m->last_k[1] = act ? sh.k_o : 0;
  m->last_k[2] = act ? sh.k_gu : 0;
  m->last_k[3] = act ? sh.k_d : 0;
  m->last_act = act;
  m->last_kv = kvs;
  m->last_P = sh.P;
  m->last_K = kvs ? sh.K : 0;
}

extern "C" bc_status bc_batch_step(bc_batch* m, const int* tokens, bc_mode mode, double rp, double rkv, int sinks,
                                   int recent, int page, float* logits) {
  if (!m || !tokens || !logits) return bfail(BC_EINVAL, "null argument");
  if (mode < BC_DENSE || mode > BC_BOTH) return bfail(BC_EINVAL, "batched steps take modes dense, act, kv, both");
  if (page != m->cfg.page) return bfail(BC_EINVAL, "page %d differs from the model's %d", page, m->cfg.page);
  if (!(rp > 0.0 && rp <= 1.0)) return bfail(BC_EINVAL, "rp %g outside (0, 1]", rp);
  if (!(rkv > 0.0 && rkv <= 1.0)) return bfail(BC_EINVAL, "rkv %g outside (0, 1]", rkv);
  if (sinks < 0 || recent < 1) return bfail(BC_EINVAL, "sinks must be >= 0 and recent >= 1");
  if (m->n + 1 > m->cfg.max_ctx) return bfail(BC_ECAPACITY, "KV cache full (%d tokens)", m->n);
  for (int b = 0; b < m->B; ++b)
    if (tokens[b] < 0 || tokens[b] >= m->cfg.vocab) return bfail(BC_EINVAL, "token %d outside the vocabulary", tokens[b]);
  const BatchShape sh = batch_shape(m, mode, rp, rkv, sinks, recent);
  if (m->use_graphs) {
    const bool kvs = mode == BC_KV || mode == BC_BOTH;
    const int psel = kvs ? page_select_variant(sh.P) : 0;
    BatchGraph* g = nullptr;
    for (BatchGraph* cg_ : m->graphs)
      if (cg_->mode == mode && cg_->psel == psel && cg_->rp == rp && cg_->rkv == rkv && cg_->sinks == sinks &&
          cg_->recent == recent)
        g = cg_;
    if (g) {
      cudaError_t e = launch_batch_graph(m, g, tokens, sh, logits);
      if (e == cudaSuccess) {
        commit_batch(m, mode, sh, g->launches);
        return BC_OK;
      }
      cudaGetLastError();
      m->graphs.erase(std::find(m->graphs.begin(), m->graphs.end(), g));
      destroy_bgraph(g);
    } else if (m->launches > 0) {
      if (capture_batch(m, tokens, mode, rp, rkv, sinks, recent, logits, &g) == BC_OK) {
        g->psel = psel;
        m->graphs.push_back(g);
        if (launch_batch_graph(m, g, tokens, sh, logits) == cudaSuccess) {
          commit_batch(m, mode, sh, g->launches);
          return BC_OK;
        }
        cudaGetLastError();
        m->graphs.pop_back();
        destroy_bgraph(g);
      }
    }
  }
  long long launches = 0;
  bc_status s = enqueue_batch(m, tokens, mode, rp, rkv, sinks, recent, logits, nullptr, &launches);
  if (s == BC_OK) commit_batch(m, mode, sh, launches);
  return s;
}

extern "C" bc_status bc_batch_trace(const bc_batch* m, int seq, int layer, bc_trace_kind kind, const void** ptr,
                                    int* count, int* stride) {
  if (!m || !ptr || !count) return bfail(BC_EINVAL, "null argument");
  const bc_config& c = m->cfg;
  const BatchLayout& y = m->lay;
  if (seq < 0 || seq >= m->B) return bfail(BC_EINVAL, "sequence %d out of range", seq);
  if (layer < 0 || layer >= c.n_layers) return bfail(BC_EINVAL, "layer %d out of range", layer);
  const size_t B = m->B, b = seq, l = layer, d = c.hidden, f = c.intermediate, hq = y.hq;
  const size_t sp = (size_t)c.n_kv_heads * y.Pmax;
  const size_t sel = y.sel + 4 * l * 4 * (size_t)y.sel_stride;
  size_t off = 0;
  int n = 0, st = 0;
  switch (kind) {
    case BC_TRACE_XN: off = y.v_qkv + 4 * (l * B + b) * d; n = m->last_act ? (int)d : 0; break;
    case BC_TRACE_SEL_QKV: off = sel + 4 * b * m->last_k[0]; n = m->last_k[0]; break;
    case BC_TRACE_Q: off = y.q + 4 * (l * B + b) * hq; n = (int)hq; break;
    case BC_TRACE_ATTN: off = y.attn + 4 * (l * B + b) * hq; n = (int)hq; break;
    case BC_TRACE_SEL_O: off = sel + 4 * ((size_t)y.sel_stride + b * m->last_k[1]); n = m->last_k[1]; break;
    case BC_TRACE_XN2: off = y.v_gu + 4 * (l * B + b) * d; n = m->last_act ? (int)d : 0; break;
    case BC_TRACE_SEL_GU: off = sel + 4 * (2 * (size_t)y.sel_stride + b * m->last_k[2]); n = m->last_k[2]; break;
    case BC_TRACE_H: off = y.h + 4 * (l * B + b) * f; n = m->last_act ? (int)f : 0; break;
    case BC_TRACE_SEL_D: off = sel + 4 * (3 * (size_t)y.sel_stride + b * m->last_k[3]); n = m->last_k[3]; break;
    case BC_TRACE_X: off = y.xo + 4 * (l * B + b) * d; n = (int)d; break;
    case BC_TRACE_PAGE_SCORES: off = y.pscore + 4 * (l * B + b) * sp; n = m->last_K ? m->last_P : 0; st = y.Pmax; break;
    case BC_TRACE_PAGES: off = y.pages + 4 * (l * B + b) * sp; n = m->last_K; st = y.Pmax; break;
    case BC_TRACE_QKV: off = y.raw + 4 * (l * B + b) * y.nqkv; n = y.nqkv; break;
    default: return bfail(BC_EINVAL, "trace kind %d is not kept for batches", (int)kind);
  }
  *ptr = m->ws + off;
  *count = n;
  if (stride) *stride = st;
  return BC_OK;
}
