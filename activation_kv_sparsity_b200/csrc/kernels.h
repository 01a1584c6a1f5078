// Host-side launchers of the decode-step kernels (internal to libbytecross).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace bc {

// Records the message bc_last_error() returns on this thread.
void set_error(const char* msg);

// ------------------------------------------------------------------ GEMV
enum GemvEpi { EPI_STORE = 0, EPI_RESID = 1, EPI_QKV = 2 };

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
  const float* x;            // [d_in]
  const int* idx;            // [k] ascending, or nullptr for all rows
  int k;
  int chunk, n_chunks;       // rows per split, number of splits
  float* partial;            // [n_chunks][d_out]
  unsigned* counters;        // [d_out / 256], zero between launches
  int epi;
  float* y;                  // STORE: y = r; RESID: y += r; QKV: y = r (raw)
  float* y_copy;             // RESID: optional copy of the updated y
  QkvEpilogue qkv;
};

// Grid shape for a GEMV of k rows and d_out columns on `sms` SMs.
void gemv_plan(int k, int d_out, int sms, int max_chunks, int* chunk, int* n_chunks);
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st, bool pdl);
constexpr int kGemvMaxChunks = 64;
constexpr int kGemvMaxChunkRows = 2048;

// ------------------------------------------------------------------ selection / elementwise prep
enum Prep { PREP_NONE = 0, PREP_NORM = 1, PREP_EMBED_NORM = 2, PREP_SWIGLU = 3 };

struct SelectArgs {
  int prep;
  int n;                          // vector length
  int k;                          // kept count (used when do_select)
  int do_select;
  const float* v;                 // NONE: scored vector; NORM: x; SWIGLU: [gate | up] (2n)
  const __nv_bfloat16* gain;      // NORM / EMBED_NORM
  float eps;
  const __nv_bfloat16* embed_row; // EMBED_NORM: the token's embedding row
  float* x_out;                   // EMBED_NORM: residual stream initialised here
  float* out;                     // NORM / SWIGLU output vector (the GEMV input)
  int* idx;                       // [k] ascending
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------ KV pages
struct PageScoreArgs {
  const float* q;                 // rotated queries [Hkv*G][hd]
  const __nv_bfloat16* meta;      // layer key bounds [Hkv][Pmax][2][hd]
  int Hkv, G, hd, Pmax, P;
  float* scores;                  // [Hkv][Pmax]
};
cudaError_t launch_page_scores(const PageScoreArgs& a, cudaStream_t st, bool pdl);

struct PageSelectArgs {
  const float* scores;            // [Hkv][Pmax]
  int Hkv, Pmax, P, K, sinks, recent;
  int* pages;                     // [Hkv][Pmax], first K ascending
};
cudaError_t launch_page_select(const PageSelectArgs& a, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------ attention
struct AttnArgs {
  const float* q;                 // [Hkv*G][hd]
  const __nv_bfloat16* kv;        // layer pages [Hkv][Pmax][2][16][hd]
  const int* pages;               // [Hkv][Pmax] or nullptr (pages 0..n_pages-1)
  int Hkv, G, hd, Pmax, n_pages, n_tok;
  int splits, pages_per_split;
  float* part_o;                  // [Hkv*G][kMaxSplits][hd]
  float* part_ml;                 // [Hkv*G][kMaxSplits][2]
  float* out;                     // [Hkv*G][hd]
};
void attn_plan(int n_pages, int Hkv, int sms, int* splits, int* pps);
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st, bool pdl);

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
  const float* xf;                // [d]
  float* logits;                  // [V]
};
cudaError_t launch_lmhead(const LmHeadArgs& a, int sms, cudaStream_t st, bool pdl);

}  // namespace bc
