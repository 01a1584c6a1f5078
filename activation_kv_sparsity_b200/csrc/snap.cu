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
// and the page masses (logits recomputed).  The logits are a dense
// contraction (queries x keys x hd), so they run on the tensor cores with the
// attention kernel's operand layout: mma m16n8k16 with 8 observation queries
// per A block (rows 0-7 their bf16 "hi" parts, rows 8-15 the residues, so the
// sum of both keeps about 16 bits of the fp32 query) and 8 keys per B block.
// A CTA takes a chunk of 32 pages of one kv head; each of its 4 warps takes
// every 4th page, with the next page's keys in flight (lane (g, t) loads dims
// u*32 + t*8 .. +8 of key rows g and g+8, and the contraction dims are
// permuted alike in the query fragments).  The query fragments of all blocks
// are staged once per CTA in shared memory, one 16-byte read per lane, block
// and k16 step; each key fragment feeds 4 query blocks in turn, so a warp has
// 8 independent accumulator chains in flight.  Base-2 logits throughout.  It runs once per selection, not
// per decode step.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace bc {

constexpr int kSnapWarps = 4;
constexpr int kSnapPages = 32;                // pages per chunk (CTA)
constexpr int kSnapTok = kSnapPages * kPage;  // tokens per chunk
constexpr int kSnapBlocks = kSnapMaxQ / 8;    // query blocks of 8
constexpr int kSnapGrp = 4;                   // blocks per key-fragment pass: 8 independent mma chains

// PASS 0: per-chunk (max, sum) of every query.  PASS 1: page masses.
template <int HD, int PASS>
__global__ void __launch_bounds__(kSnapWarps * 32, 2) k_snap(SnapArgs a) {
  constexpr int KSTEPS = HD / 16;
  constexpr int U4 = HD / 32;                 // 16-byte vectors per lane and key row
  constexpr int PAGE_ELEMS = 2 * kPage * HD;
  extern __shared__ __align__(16) uint4 s_qa[];   // [blocks][KSTEPS][32 lanes]
  __shared__ float s_m[kSnapWarps][kSnapMaxQ], s_l[kSnapWarps][kSnapMaxQ];
  const int chunk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int Q = a.n_obs * a.G;
  const int NB = ((Q + 8 * kSnapGrp - 1) / (8 * kSnapGrp)) * kSnapGrp;   // blocks, zero-padded
  const float qscale = 1.4426950408889634f * rsqrtf((float)HD);
  pdl_wait();
  pdl_trigger();

  // query fragments: block b holds queries 8b .. 8b+7 (query qi = j*G + gg is
  // observation j of head h*G + gg); lane (g, t) of k-step s takes dims
  // (s/2)*32 + 4*(s%2) + t*8 + 0..3 of query 8b + g
  for (int e = tid; e < NB * KSTEPS * 32; e += kSnapWarps * 32) {
    const int ln = e % 32, s = (e / 32) % KSTEPS, blk = e / (32 * KSTEPS);
    const int qi = 8 * blk + (ln >> 2), tt = ln & 3;
    const int d0 = (s / 2) * 32 + 4 * (s % 2) + tt * 8;
    float q[4] = {0.f, 0.f, 0.f, 0.f};
    if (qi < Q) {
      const int j = qi / a.G, gg = qi % a.G;
      const float* qp = a.q_obs + ((size_t)j * a.Hkv * a.G + h * a.G + gg) * HD + d0;
      #pragma unroll
      for (int c = 0; c < 4; ++c) q[c] = qp[c] * qscale;
    }
    uint4 f;
    split2(q[0], q[1], f.x, f.y);
    split2(q[2], q[3], f.z, f.w);
    s_qa[e] = f;
  }
  __syncthreads();

  // per lane: query g of every block, running (max, sum) or its (M, 1/L)
  float m_run[kSnapBlocks], l_run[kSnapBlocks];
  #pragma unroll
  for (int b = 0; b < kSnapBlocks; ++b) {
    m_run[b] = -INFINITY;
    l_run[b] = 0.f;
    if (PASS == 1 && b < NB && 8 * b + g < Q) {
      const float2 st = a.stats[(size_t)h * Q + 8 * b + g];
      m_run[b] = st.x;
      l_run[b] = 1.0f / st.y;
    }
  }
  const __nv_bfloat16* head = a.kv + (size_t)h * a.Pmax * PAGE_ELEMS;
  const int p0 = chunk * kSnapPages;
  const int p_end = min(p0 + kSnapPages, (a.n_tok + kPage - 1) / kPage);
  auto load = [&](int page, uint4* k0, uint4* k1) {
    const __nv_bfloat16* pk = head + (size_t)page * PAGE_ELEMS + t * 8;
    #pragma unroll
    for (int u = 0; u < U4; ++u) {
      k0[u] = ld_stream(pk + g * HD + 32 * u);
      k1[u] = ld_stream(pk + (g + 8) * HD + 32 * u);
    }
  };
  auto process = [&](int page, const uint4* k0, const uint4* k1) {
    const uint32_t* kr0 = reinterpret_cast<const uint32_t*>(k0);
    const uint32_t* kr1 = reinterpret_cast<const uint32_t*>(k1);
    const int valid = min(kPage, a.n_tok - page * kPage);
    const int tok[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
    float mass = 0.f;
    #pragma unroll
    for (int b0 = 0; b0 < kSnapBlocks; b0 += kSnapGrp) {
      if (b0 >= NB) break;
      float c[kSnapGrp][2][4];
      #pragma unroll
      for (int i = 0; i < kSnapGrp; ++i)
        #pragma unroll
        for (int r = 0; r < 4; ++r) c[i][0][r] = c[i][1][r] = 0.f;
      #pragma unroll
      for (int s = 0; s < KSTEPS; ++s)
        #pragma unroll
        for (int i = 0; i < kSnapGrp; ++i) {
          const uint4 f = s_qa[((b0 + i) * KSTEPS + s) * 32 + lane];
          const uint32_t qa[4] = {f.x, f.y, f.z, f.w};
          mma16816(c[i][0], qa, kr0[2 * s], kr0[2 * s + 1]);
          mma16816(c[i][1], qa, kr1[2 * s], kr1[2 * s + 1]);
        }
      #pragma unroll
      for (int i = 0; i < kSnapGrp; ++i) {
        const int b = b0 + i;
        const float sc[4] = {c[i][0][0] + c[i][0][2], c[i][0][1] + c[i][0][3],
                             c[i][1][0] + c[i][1][2], c[i][1][1] + c[i][1][3]};
        if (PASS == 0) {
          float mx = -INFINITY;
          #pragma unroll
          for (int j = 0; j < 4; ++j)
            if (tok[j] < valid) mx = fmaxf(mx, sc[j]);
          const float m_new = fmaxf(m_run[b], mx);
          float add = 0.f;
          #pragma unroll
          for (int j = 0; j < 4; ++j)
            if (tok[j] < valid) add += exp2f(sc[j] - m_new);
          l_run[b] = (m_run[b] == -INFINITY ? 0.f : l_run[b] * exp2f(m_run[b] - m_new)) + add;
          m_run[b] = m_new;
        } else if (8 * b + g < Q) {
          #pragma unroll
          for (int j = 0; j < 4; ++j)
            if (tok[j] < valid) mass += exp2f(sc[j] - m_run[b]) * l_run[b];
        }
      }
    }
    if (PASS == 1) {
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) mass += __shfl_xor_sync(0xffffffffu, mass, o);
      if (lane == 0) a.scores[(size_t)h * a.Pmax + page] = mass;
    }
  };
  uint4 ka0[U4], ka1[U4], kb0[U4], kb1[U4];
  int p = p0 + warp;
  if (p < p_end) load(p, ka0, ka1);
  while (p < p_end) {
    int q = p + kSnapWarps;
    if (q < p_end) load(q, kb0, kb1);
    process(p, ka0, ka1);
    p = q;
    if (p >= p_end) break;
    q = p + kSnapWarps;
    if (q < p_end) load(q, ka0, ka1);
    process(p, kb0, kb1);
    p = q;
  }
  if (PASS == 0) {
    // the quad's lanes hold the same query: merge them, then the warps
    #pragma unroll
    for (int b = 0; b < kSnapBlocks; ++b) {
      if (b >= NB) break;
      float m = m_run[b], l = l_run[b];
      #pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
        const float mm = fmaxf(m, m2);
        l = (m == -INFINITY ? 0.f : l * exp2f(m - mm)) + (m2 == -INFINITY ? 0.f : l2 * exp2f(m2 - mm));
        m = mm;
      }
      if (t == 0) {
        s_m[warp][8 * b + g] = m;
        s_l[warp][8 * b + g] = l;
      }
    }
    __syncthreads();
    for (int qi = tid; qi < Q; qi += kSnapWarps * 32) {
      float M = -INFINITY;
      #pragma unroll
      for (int w = 0; w < kSnapWarps; ++w) M = fmaxf(M, s_m[w][qi]);
      float L = 0.f;
      #pragma unroll
      for (int w = 0; w < kSnapWarps; ++w)
        if (s_m[w][qi] != -INFINITY) L += s_l[w][qi] * exp2f(s_m[w][qi] - M);
      a.part[((size_t)h * gridDim.x + chunk) * Q + qi] = make_float2(M, L);
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
  constexpr int KSTEPS = HD / 16;
  const int Q = a.n_obs * a.G;
  const int NB = ((Q + 8 * kSnapGrp - 1) / (8 * kSnapGrp)) * kSnapGrp;
  const size_t smem = (size_t)NB * KSTEPS * 32 * sizeof(uint4);
  static bool attr_done = false;
  if (!attr_done) {
    const int max_smem = kSnapBlocks * KSTEPS * 32 * (int)sizeof(uint4);
    cudaError_t e = cudaFuncSetAttribute(k_snap<HD, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_snap<HD, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int chunks = snap_chunks(a.n_tok);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(chunks, a.Hkv);
  cfg.blockDim = dim3(kSnapWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_snap<HD, 0>, a);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c2 = cfg;
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
