// Host-side launchers of the decode-step kernels (internal to libbytecross).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace bc {

// Records the message bc_last_error() returns on this thread.
void set_error(const char* msg);

// ------------------------------------------------------------------ GEMV
enum GemvEpi { EPI_STORE = 0, EPI_RESID = 1, EPI_QKV = 2, EPI_SWIGLU = 3 };
// How the GEMV input v is formed from x while staging (see gemv.cu).
enum GemvPrep { GP_NONE = 0, GP_NORM = 1, GP_EMBED_NORM = 2, GP_SWIGLU = 3 };

constexpr int kGemvMaxContrib = 64;   // clusters contributing to one column tile
constexpr int kGemvMaxPer = 4096;     // listed rows per CTA (shared-memory staging)

struct QkvEpilogue {
  int Hq, Hkv, hd, pos, Pmax;
  float rope_theta;
  float* q_out;              // [Hq*hd] rotated queries
  __nv_bfloat16* kv_layer;   // this layer's pages [Hkv][Pmax][2][16][hd]
  __nv_bfloat16* meta_layer; // this layer's key bounds [Hkv][Pmax][2][hd]
};

struct GemvArgs {
  const __nv_bfloat16* W;    // [d_in][d_out]
  int d_in, d_out;
  int prep;
  const float* x;            // NONE: v; NORM: residual stream; SWIGLU: [gate | up] (2 d_in)
  const __nv_bfloat16* gain; // NORM / EMBED_NORM
  float eps;
  const __nv_bfloat16* embed_row;  // EMBED_NORM
  float* x_init;             // EMBED_NORM: residual stream written by CTA 0
  const int* idx;            // [k] ascending, or nullptr for all rows
  int k;
  int TW;                    // columns per tile: 256 or 128
  int S, C;                  // CTAs per cluster, clusters per column tile
  int max_rows;              // rows of the longest run: ceil(k / (S*C))
  float* partial;            // [d_out/TW][kGemvMaxContrib][TW] (C > 1 only)
  unsigned* counters;        // [d_out / TW], zero between launches
  int epi;
  float* y;                  // STORE: y = r; RESID: y += r; QKV: y = r (raw); SWIGLU: h [d_out/2]
  float* y_copy;             // RESID: optional copy of the updated y
  QkvEpilogue qkv;
};

// Shape of a GEMV of k listed rows and d_out columns on `sms` SMs: TW
// columns per tile, S CTAs per cluster, C clusters per tile.
void gemv_plan(int k, int d_out, int sms, int* TW, int* S, int* C);
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------ activation select
enum SelPrep { SP_NONE = 0, SP_NORM = 1, SP_EMBED_NORM = 2, SP_SWIGLU = 3 };

struct SelectArgs {
  int prep;
  int n;                          // vector length (<= kMaxSelect)
  int k;                          // kept count
  const float* x;                 // NONE: scored vector; NORM: x; SWIGLU: [gate | up] (2n)
  const __nv_bfloat16* gain;      // NORM / EMBED_NORM
  const __nv_bfloat16* embed_row; // EMBED_NORM: the token's embedding row
  float* x_init;                  // EMBED_NORM: residual stream initialised here
  float* vout;                    // the ranked vector (trace), or nullptr
  int* idx;                       // [k] ascending
  // batched launch (nb vectors, one per sequence): vector b is read from
  // x + b*x_stride and ranked into idx + b*idx_stride (SP_NONE only)
  long long x_stride, idx_stride;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st, bool pdl, int nb = 1);

// ------------------------------------------------------------------ KV pages
// Page scores (grid-wide), then the page select (one CTA, or above 8192
// pages one cluster, per kv head).
struct PageArgs {
  const float* q;                 // rotated queries [Hkv*G][hd]
  const __nv_bfloat16* meta;      // layer key bounds [Hkv][Pmax][2][hd]
  int Hkv, G, hd, Pmax, P, K, sinks, recent;
  int rounds;                     // scorer: rounds of pages per CTA (page_rounds)
  float* scores;                  // [Hkv][Pmax]
  int* pages;                     // [Hkv][Pmax], first K ascending
  unsigned* counters;             // unused (kept for the workspace layout)
  // batched launch (nb sequences of equal length): sequence b's queries,
  // bounds, scores and pages are at q + b*q_stride, meta + b*meta_stride,
  // scores / pages + b*sp_stride (elements)
  long long q_stride, meta_stride, sp_stride;
};
cudaError_t launch_page_scores(const PageArgs& a, cudaStream_t st, bool pdl, int nb = 1);
cudaError_t launch_page_select(const PageArgs& a, cudaStream_t st, bool pdl, int nb = 1);
// Which page-select kernel P pages take: keys per thread of the one-CTA
// kernel (2, 4 or 8), or 0 for the cluster.  A captured step serves only
// page counts of its own variant.
int page_select_variant(int P);
// Launch shape of the page scorer for P pages (graph node updates).
int page_rounds(int P, int hd, int Hkv, int sms);
dim3 pages_grid(const PageArgs& a);

// ------------------------------------------------------------------ once-after-prefill page scores
constexpr int kSnapMaxQ = 128;    // observation queries per kv head (n_obs * G)
struct SnapArgs {
  const float* q_obs;             // this layer's observation queries [n_obs][Hq][hd], post-rotary
  const __nv_bfloat16* kv;        // this layer's pages [Hkv][Pmax][2][16][hd]
  int Hkv, G, hd, Pmax, n_obs, n_tok;
  float2* part;                   // [Hkv][snap_chunks(n_tok)][Q] per-chunk (max, sum), base 2
  float2* stats;                  // [Hkv][Q] (max, sum) over all n_tok tokens
  float* scores;                  // [Hkv][Pmax] page scores (attention mass)
  float2* pp;                     // tcgen05 scorer: [Hkv][Pmax][Q] each page's (max, sum) per query
};
int snap_chunks(int n_tok);
// head_dim 128 with at most 64 observation queries per kv head (and pp set)
// runs in one pass over the keys on the tcgen05 tensor cores, other shapes in
// two passes on mma.sync
cudaError_t launch_snap_scores(const SnapArgs& a, cudaStream_t st, bool pdl);
// Synchronises the stream and reads the tcgen05 scorer's status word: 0, or
// the bits of the waits that gave up (a lost copy or MMA completion).
cudaError_t snap_status(unsigned* status, cudaStream_t st);

// ------------------------------------------------------------------ attention
struct AttnArgs {
  const float* q;                 // [Hkv*G][hd]
  const __nv_bfloat16* kv;        // layer pages [Hkv][Pmax][2][16][hd]
  const int* pages;               // [Hkv][Pmax] or nullptr (pages 0..n_pages-1)
  int Hkv, G, hd, Pmax, n_pages, n_tok;
  int list_len, tail0;            // entries >= list_len are pages tail0, tail0+1, ... (not listed)
  int splits, pages_per_split;
  // additive page mask (the masked dense baseline): with mask_on, a page p
  // of the list adds 0 to its logits when p < mask_sink_end or
  // p >= mask_rec_begin and -inf otherwise; its bytes are read either way
  int mask_on, mask_sink_end, mask_rec_begin;
  float* part_o;                  // [Hkv*G][kMaxSplits][hd]
  float* part_ml;                 // [Hkv*G][kMaxSplits][2]
  unsigned* counters;             // [Hkv], zero between launches
  float* out;                     // [Hkv*G][hd]
  // batched launch (nb sequences of equal length): sequence b's tensors are
  // offset by b times these strides (elements)
  long long q_stride, kv_stride, list_stride, part_stride, out_stride;
  int counters_stride;
};
void attn_plan(int n_pages, int Hkv, int sms, int* splits, int* pps);
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st, bool pdl, int nb = 1);

// ------------------------------------------------------------------ KV append (bulk)
struct KvAppendArgs {
  const __nv_bfloat16* k;         // [L][Hkv][n_new][hd]
  const __nv_bfloat16* v;
  int n_new, n0, L, Hkv, hd, Pmax;
  __nv_bfloat16* pool;            // [L][Hkv][Pmax][2][16][hd]
  __nv_bfloat16* meta;            // [L][Hkv][Pmax][2][hd]
};
cudaError_t launch_kv_append(const KvAppendArgs& a, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------ LM head
struct LmHeadArgs {
  const __nv_bfloat16* W;         // [V][d]
  int V, d;
  const float* x;                 // residual stream [d]
  const __nv_bfloat16* gain;      // final RMSNorm gain [d]
  float eps;
  float* logits;                  // [V]
};
cudaError_t launch_lmhead(const LmHeadArgs& a, int sms, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------ batched projection over a union
constexpr int kBatchMax = 8;        // sequences per batched projection
constexpr int kBatchMaxSplit = 32;  // row runs per column tile
struct BatchGemvArgs {
  const __nv_bfloat16* W;         // [d_in][d_out]
  int d_in, d_out, k, B;
  const float* x;                 // [B][d_in]
  const int* idx;                 // [B][k] kept channels per sequence, or nullptr for all (k == d_in)
  int* ulist;                     // [d_in] union U, ascending (first |U| entries): channel | sequence bits << 16
  int* n_union;                   // |U|
  float* partial;                 // [S][B][d_out] (S > 1 only)
  int S;                          // row runs per column tile
  float* y;                       // [B][d_out]
};
int gemv_batch_splits(int d_in, int d_out, int k, int B, int sms);
size_t gemv_batch_scratch(int d_in, int d_out, int B);
// Carves ulist / n_union / partial out of scratch (n_union stays in
// scratch unless given).
void gemv_batch_bind(BatchGemvArgs* a, void* scratch, int* n_union);
cudaError_t launch_gemv_batch(const BatchGemvArgs& a, cudaStream_t st, bool pdl);

}  // namespace bc
