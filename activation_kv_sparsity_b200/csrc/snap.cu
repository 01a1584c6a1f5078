// Once-after-prefill page scores: the pages' own KV mode (ByteCross README,
// "Timing and quality on a GPU": an attention-scored selection made once
// after prefill, in the manner of SnapKV, listed on the mlsanity page).
//
// A window of observation queries per query head (the last prompt
// positions' queries, post-rotary) votes for the cached tokens with its
// softmax attention over the whole prefix, scale 1/sqrt(hd).  A page's score
// is the attention mass its valid tokens receive from every observation
// query of the kv head's group:
//
//   score_p = sum_q sum_{t in p} exp(s_qt - M_q) / L_q,
//   M_q = max_t s_qt,  L_q = sum_t exp(s_qt - M_q)   (t over all n tokens).
//
// Three kernels per layer: per-chunk (max, sum) of every query, their merge,
// and the page masses (logits recomputed).  A CTA takes a chunk of 8 pages
// (128 tokens) of one kv head and a tile of up to 64 queries; each thread
// computes a 4-token x 8-query block of logits from keys and queries staged
// in shared memory dimension-major (one 16-byte read of keys and two of
// queries per dimension, conflict-free).  Base-2 logits throughout.  This
// runs once per selection, not per decode step; it is CUDA-core fp32 work
// (about 1 FMA per query, key element and pass).
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace bc {

constexpr int kSnapThreads = 256;
constexpr int kSnapTok = 8 * kPage;           // tokens per chunk
constexpr int kSnapQTile = 64;                // queries per tile

template <int HD>
struct SnapSmem {
  alignas(16) float k[HD][kSnapTok];         // keys of the chunk, dimension-major
  alignas(16) float q[HD][kSnapQTile];       // the query tile, dimension-major
  float mass[8][kSnapTok];                   // pass 1: token mass per query group
};

// PASS 0: per-chunk (max, sum) of every query.  PASS 1: page masses.
template <int HD, int PASS>
__global__ void __launch_bounds__(kSnapThreads) k_snap(SnapArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SnapSmem<HD>& sm = *reinterpret_cast<SnapSmem<HD>*>(smem_raw);
  const int chunk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int tt = tid & 31, qq = tid >> 5;      // tokens 4*tt .. +4, queries 8*qq .. +8 of the tile
  const int Q = a.n_obs * a.G;
  const int t0 = chunk * kSnapTok;
  const float scale = 1.4426950408889634f * rsqrtf((float)HD);
  pdl_wait();
  pdl_trigger();

  // keys of the chunk's tokens (pages are consecutive), converted to fp32
  const __nv_bfloat16* head = a.kv + (size_t)h * a.Pmax * 2 * kPage * HD;
  constexpr int DC = HD / 8;
  for (int idx = tid; idx < kSnapTok * DC; idx += kSnapThreads) {
    const int t = idx % kSnapTok, dc = idx / kSnapTok;
    const int tok = t0 + t;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (tok < a.n_tok) {
      const int page = tok / kPage, slot = tok % kPage;
      w = *reinterpret_cast<const uint4*>(head + ((size_t)page * 2 * kPage + slot) * HD + dc * 8);
    }
    sm.k[dc * 8 + 0][t] = bf16_lo(w.x); sm.k[dc * 8 + 1][t] = bf16_hi(w.x);
    sm.k[dc * 8 + 2][t] = bf16_lo(w.y); sm.k[dc * 8 + 3][t] = bf16_hi(w.y);
    sm.k[dc * 8 + 4][t] = bf16_lo(w.z); sm.k[dc * 8 + 5][t] = bf16_hi(w.z);
    sm.k[dc * 8 + 6][t] = bf16_lo(w.w); sm.k[dc * 8 + 7][t] = bf16_hi(w.w);
  }
  float tokmass[4] = {0.f, 0.f, 0.f, 0.f};
  for (int q0 = 0; q0 < Q; q0 += kSnapQTile) {
    __syncthreads();                           // keys staged; the previous tile's queries consumed
    // query tile: query qi = j*G + g is observation j of head h*G + g;
    // consecutive threads take consecutive queries of one dimension, so the
    // dimension-major stores are conflict-free
    for (int idx = tid; idx < kSnapQTile * HD; idx += kSnapThreads) {
      const int ql = idx % kSnapQTile, d = idx / kSnapQTile, qi = q0 + ql;
      float v = 0.f;
      if (qi < Q) {
        const int j = qi / a.G, g = qi % a.G;
        v = a.q_obs[((size_t)j * a.Hkv * a.G + h * a.G + g) * HD + d] * scale;
      }
      sm.q[d][ql] = v;
    }
    __syncthreads();
    float acc[4][8];
    #pragma unroll
    for (int i = 0; i < 4; ++i)
      #pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    #pragma unroll 4
    for (int d = 0; d < HD; ++d) {
      const float4 kv = *reinterpret_cast<const float4*>(&sm.k[d][4 * tt]);
      const float4 qa = *reinterpret_cast<const float4*>(&sm.q[d][8 * qq]);
      const float4 qb = *reinterpret_cast<const float4*>(&sm.q[d][8 * qq + 4]);
      const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
      const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
      #pragma unroll
      for (int i = 0; i < 4; ++i)
        #pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(kk[i], qv[j], acc[i][j]);
    }
    bool tvalid[4];
    #pragma unroll
    for (int i = 0; i < 4; ++i) tvalid[i] = t0 + 4 * tt + i < a.n_tok;
    #pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int qi = q0 + 8 * qq + j;
      if (PASS == 0) {
        // this warp covers all 128 tokens of the chunk for its 8 queries
        float m = -INFINITY;
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          if (tvalid[i]) m = fmaxf(m, acc[i][j]);
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          if (tvalid[i]) l += exp2f(acc[i][j] - m);
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (tt == 0 && qi < Q) a.part[((size_t)h * gridDim.x + chunk) * Q + qi] = make_float2(m, l);
      } else if (qi < Q) {
        const float2 st = a.stats[(size_t)h * Q + qi];
        const float inv = 1.0f / st.y;
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          if (tvalid[i]) tokmass[i] += exp2f(acc[i][j] - st.x) * inv;
      }
    }
  }
  if (PASS == 1) {
    // sum the 8 query groups, then the 16 tokens of each page
    #pragma unroll
    for (int i = 0; i < 4; ++i) sm.mass[qq][4 * tt + i] = tokmass[i];
    __syncthreads();
    if (tid < kSnapTok) {
      float v = 0.f;
      #pragma unroll
      for (int w = 0; w < 8; ++w) v += sm.mass[w][tid];
      #pragma unroll
      for (int o = kPage / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, kPage);
      const int page = (t0 + tid) / kPage;
      if ((tid % kPage) == 0 && page * kPage < a.n_tok) a.scores[(size_t)h * a.Pmax + page] = v;
    }
  }
}

// Merges the chunks' (max, sum) of every query: one thread per (kv head, query).
__global__ void k_snap_merge(SnapArgs a, int chunks) {
  const int Q = a.n_obs * a.G;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (e >= a.Hkv * Q) return;
  const int h = e / Q, qi = e % Q;
  float M = -INFINITY;
  for (int c = 0; c < chunks; ++c) M = fmaxf(M, a.part[((size_t)h * chunks + c) * Q + qi].x);
  float L = 0.f;
  for (int c = 0; c < chunks; ++c) {
    const float2 p = a.part[((size_t)h * chunks + c) * Q + qi];
    if (p.x != -INFINITY) L += p.y * exp2f(p.x - M);
  }
  a.stats[(size_t)h * Q + qi] = make_float2(M, L);
}

int snap_chunks(int n_tok) { return (n_tok + kSnapTok - 1) / kSnapTok; }

template <int HD>
static cudaError_t launch_hd(const SnapArgs& a, cudaStream_t st, bool pdl) {
  const size_t smem = sizeof(SnapSmem<HD>);
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_snap<HD, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_snap<HD, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int chunks = snap_chunks(a.n_tok);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(chunks, a.Hkv);
  cfg.blockDim = dim3(kSnapThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_snap<HD, 0>, a);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c2 = cfg;
  const int Q = a.n_obs * a.G;
  c2.gridDim = dim3((a.Hkv * Q + 127) / 128);
  c2.blockDim = dim3(128);
  c2.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&c2, k_snap_merge, a, chunks);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k_snap<HD, 1>, a);
}

cudaError_t launch_snap_scores(const SnapArgs& a, cudaStream_t st, bool pdl) {
  if (a.n_tok < 1 || a.n_obs < 1 || a.n_obs * a.G > kSnapMaxQ) return cudaErrorInvalidValue;
  if (a.hd == 128) return launch_hd<128>(a, st, pdl);
  if (a.hd == 64) return launch_hd<64>(a, st, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace bc
