// Split-K flash-decode attention over a page list: the one attention kernel
// of every mode.  The ByteCross README ("Overview": "One attention kernel for
// every mode"; FAQ: a masked dense baseline inflates KV speedups about
// fivefold) insists that dense and sparse modes read the cache through the
// same split-K kernel; here dense mode is simply the full page list.
//
// Layout: the pages of one (layer, kv head) are 2*16*hd bf16 each, the 16
// keys then the 16 values (8 KiB at hd = 128).  CTA (split, kv head) walks a
// contiguous slice of the page list; its 4 warps take every 4th page.
//
// Per page a warp runs the two products on the tensor cores with
// mma.m16n8k16 (bf16 in, fp32 accumulate).  The A operand rows 0..7 carry the
// G <= 8 query heads of the group rounded to bf16 ("hi"), rows 8..15 the
// rounding residues ("lo"), so S = S_hi + S_lo keeps about 16 significant
// bits of the fp32 query; the softmax weights P are split the same way for
// P*V.  Keys are loaded straight into B fragments: lane (g, t) reads dims
// u*32 + t*8 .. +8 (u = 0..hd/32-1) of key rows g and g+8, so the four lanes
// of a row read 64 contiguous bytes per instruction, and the contraction
// dims are permuted consistently in A and B, which leaves the dot products
// unchanged.  Value fragments are transposed in registers with movmatrix;
// each lane ends with its head row's output over the same dims.
//
// A listed slice may end in an implicit run: entries from list_len on are
// the pages tail0, tail0 + 1, ... (the pages begun after a once-after-prefill
// selection).
//
// With mask_on the kernel is the masked dense baseline of the README's FAQ
// ("A KV method reports a speedup above its byte bound"): it reads every
// page of the list and adds an additive mask, 0 on the window's pages (the
// sinks and the recent pages) and -inf elsewhere, to the logits.  Masked
// pages cost their bytes and contribute nothing.
//
// Partials (m, l, o) per (query head, split) use base-2 logits.  The last
// CTA of each kv head to finish (an atomic ticket, no spinning) merges them:
// o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, summing in split order.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>
#include <type_traits>

namespace bc {

constexpr int kAttnWarps = 4;

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <int HD>
__global__ void __launch_bounds__(kAttnWarps * 32, 2) k_attn(AttnArgs a) {
  constexpr int KSTEPS = HD / 16;   // k16 steps of q.k
  constexpr int NBLK = HD / 8;      // n8 blocks of p.v
  constexpr int DPL = HD / 4;       // dims per lane
  constexpr int U4 = DPL / 8;       // 16-byte vectors per lane and row
  constexpr int PAGE_ELEMS = 2 * kPage * HD;

  __shared__ float s_o[kAttnWarps][8][HD];
  __shared__ float s_m[kAttnWarps][8], s_l[kAttnWarps][8];

  if (blockIdx.z) {                               // batched launch: sequence blockIdx.z
    const long long b = blockIdx.z;
    a.q += b * a.q_stride;
    a.kv += b * a.kv_stride;
    if (a.pages) a.pages += b * a.list_stride;
    a.part_o += b * a.part_stride * HD;
    a.part_ml += b * a.part_stride * 2;
    a.counters += b * a.counters_stride;
    a.out += b * a.out_stride;
  }
  const int split = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = a.G;

  // The cached pages do not depend on the previous kernel (it only appends
  // to the last page, and L2 keeps that coherent): with the implicit page
  // list, pull each warp's first two pages into L2 before waiting for it.
  if (!a.pages && lane == 0) {
    const int i0 = split * a.pages_per_split + warp;
    const int i_end0 = min(a.n_pages, (split + 1) * a.pages_per_split);
    for (int i = i0; i < i_end0 && i < i0 + 2 * kAttnWarps; i += kAttnWarps)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                   :: "l"(a.kv + ((size_t)h * a.Pmax + i) * PAGE_ELEMS), "r"(PAGE_ELEMS * 2) : "memory");
  }
  pdl_wait();
  pdl_trigger();

  // This lane's query values: k-step s contracts dims (s/2)*32 + t*8 +
  // 4*(s%2) + 0..3.  They are loaded here and turned into A fragments only
  // after the first page's loads are issued, so the two latencies overlap.
  const float qscale = 1.4426950408889634f * rsqrtf((float)HD);
  float4 qraw[KSTEPS];
  {
    const float* qrow = a.q + (size_t)(h * G + g) * HD + t * 8;
    #pragma unroll
    for (int s = 0; s < KSTEPS; ++s)
      qraw[s] = g < G ? *reinterpret_cast<const float4*>(qrow + (s / 2) * 32 + 4 * (s % 2))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  uint32_t qa[KSTEPS][4];

  float o[NBLK][4];
  #pragma unroll
  for (int b = 0; b < NBLK; ++b) o[b][0] = o[b][1] = o[b][2] = o[b][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  const int i_begin = split * a.pages_per_split;
  const int i_end = min(a.n_pages, i_begin + a.pages_per_split);
  const __nv_bfloat16* head_base = a.kv + (size_t)h * a.Pmax * PAGE_ELEMS;
  const int* plist = a.pages ? a.pages + (size_t)h * a.Pmax : nullptr;

  // one page: keys then values of 16 tokens, lane (g, t) holds 32 dims of
  // token rows g and g+8
  // lane (g, t) takes dims u*32 + t*8 .. +8 of its rows: the four lanes of a
  // row cover 64 contiguous bytes per load, whole 32-byte sectors
  auto load_page = [&](int page, uint4* k0, uint4* k1, uint4* v0, uint4* v1) {
    const __nv_bfloat16* pk = head_base + (size_t)page * PAGE_ELEMS + t * 8;
    const __nv_bfloat16* pv = pk + kPage * HD;
    #pragma unroll
    for (int u = 0; u < U4; ++u) {
      k0[u] = ld_stream(pk + g * HD + 32 * u);
      k1[u] = ld_stream(pk + (g + 8) * HD + 32 * u);
      v0[u] = ld_stream(pv + g * HD + 32 * u);
      v1[u] = ld_stream(pv + (g + 8) * HD + 32 * u);
    }
  };
  auto process_page = [&](int page, uint4* k0, uint4* k1, uint4* v0, uint4* v1) {
    const bool masked = a.mask_on && page >= a.mask_sink_end && page < a.mask_rec_begin;
    const int valid = masked ? 0 : min(kPage, a.n_tok - page * kPage);
    if (g >= valid) {
      #pragma unroll
      for (int u = 0; u < U4; ++u) v0[u] = make_uint4(0, 0, 0, 0);
    }
    if (g + 8 >= valid) {
      #pragma unroll
      for (int u = 0; u < U4; ++u) v1[u] = make_uint4(0, 0, 0, 0);
    }
    const uint32_t* kr0 = reinterpret_cast<const uint32_t*>(k0);
    const uint32_t* kr1 = reinterpret_cast<const uint32_t*>(k1);
    const uint32_t* vr0 = reinterpret_cast<const uint32_t*>(v0);
    const uint32_t* vr1 = reinterpret_cast<const uint32_t*>(v1);

    // logits of tokens 0-7 (c0) and 8-15 (c1): rows g = hi, g+8 = lo
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
    for (int s = 0; s < KSTEPS; ++s) {
      mma16816(c0, qa[s], kr0[2 * s], kr0[2 * s + 1]);
      mma16816(c1, qa[s], kr1[2 * s], kr1[2 * s + 1]);
    }
    float sc[4] = {c0[0] + c0[2], c0[1] + c0[3], c1[0] + c1[2], c1[1] + c1[3]};
    const int tok[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
    #pragma unroll
    for (int j = 0; j < 4; ++j)
      if (tok[j] >= valid) sc[j] = -INFINITY;
    float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    // no valid logit yet (only masked pages so far): scale by 2^0, not 2^(-inf + inf)
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = exp2f(m_run - m_use);
    float p[4];
    #pragma unroll
    for (int j = 0; j < 4; ++j) p[j] = exp2f(sc[j] - m_use);
    l_run = l_run * alpha + (p[0] + p[1]) + (p[2] + p[3]);
    m_run = m_new;
    #pragma unroll
    for (int b = 0; b < NBLK; ++b) {
      o[b][0] *= alpha; o[b][1] *= alpha; o[b][2] *= alpha; o[b][3] *= alpha;
    }
    uint32_t pa[4];
    split2(p[0], p[1], pa[0], pa[1]);
    split2(p[2], p[3], pa[2], pa[3]);
    #pragma unroll
    for (int b = 0; b < NBLK; ++b) {
      const uint32_t b0 = transpose8x8(vr0[b]);
      const uint32_t b1 = transpose8x8(vr1[b]);
      mma16816(o[b], pa, b0, b1);
    }
  };
  // The warp's page numbers: iteration jj handles list entry
  // i_begin + warp + kAttnWarps * jj.  A listed slice is held in two
  // 32-entry register windows (lane l holds entries base + l and
  // base + 32 + l), read by shuffles, so no page load waits on an index
  // load; the window moves on by 32 entries long before they are needed.
  auto entry = [&](int jj) {
    const int i = i_begin + warp + kAttnWarps * jj;
    return i < i_end ? (i < a.list_len ? plist[i] : a.tail0 + (i - a.list_len)) : 0;
  };
  int win0 = 0, win1 = 0, base = 0;
  if (plist) {
    win0 = entry(lane);
    win1 = entry(32 + lane);
  }
  auto page_of = [&](int jj) {
    if (!plist) return i_begin + warp + kAttnWarps * jj;
    const int rel = jj - base;                       // warp-uniform, 0 <= rel < 64
    return __shfl_sync(0xffffffffu, rel < 32 ? win0 : win1, rel & 31);
  };
  auto advance = [&](int jj) {                       // before looking up jj + 2
    if (plist && jj + 2 - base >= 64) {
      base += 32;
      win0 = win1;
      win1 = entry(base + 32 + lane);
    }
  };
  const int n_it = i_begin + warp < i_end ? (i_end - i_begin - warp + kAttnWarps - 1) / kAttnWarps : 0;
  auto prefetch = [&](int jj) {
    if (jj < n_it) {
      const int page = page_of(jj);
      if (lane == 0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                     :: "l"(head_base + (size_t)page * PAGE_ELEMS), "r"(PAGE_ELEMS * 2) : "memory");
    }
  };

  // ping-pong over two register buffers: the next page is in flight while
  // this one is processed, and the page two steps ahead is pulled into L2
  uint4 ka0[U4], ka1[U4], va0[U4], va1[U4];
  uint4 kb0[U4], kb1[U4], vb0[U4], vb1[U4];
  int pa_cur = 0, pb_cur = 0;
  if (n_it > 0) {
    pa_cur = page_of(0);
    load_page(pa_cur, ka0, ka1, va0, va1);
  }
  // A fragments of the queries, pre-scaled to base-2 logits
  #pragma unroll
  for (int s = 0; s < KSTEPS; ++s) {
    split2(qraw[s].x * qscale, qraw[s].y * qscale, qa[s][0], qa[s][1]);
    split2(qraw[s].z * qscale, qraw[s].w * qscale, qa[s][2], qa[s][3]);
  }
  for (int jj = 0; jj < n_it;) {
    advance(jj);
    prefetch(jj + 2);
    if (jj + 1 < n_it) {
      pb_cur = page_of(jj + 1);
      load_page(pb_cur, kb0, kb1, vb0, vb1);
    }
    process_page(pa_cur, ka0, ka1, va0, va1);
    if (++jj >= n_it) break;
    advance(jj);
    prefetch(jj + 2);
    if (jj + 1 < n_it) {
      pa_cur = page_of(jj + 1);
      load_page(pa_cur, ka0, ka1, va0, va1);
    }
    process_page(pb_cur, kb0, kb1, vb0, vb1);
    ++jj;
  }

  // this warp's state for head row g (lanes of a quad share it)
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  if (g < G) {
    #pragma unroll
    for (int b = 0; b < NBLK; ++b) {         // block b holds dims (b/4)*32 + t*8 + 2*(b%4) + 0..1
      const int dd = (b / 4) * 32 + t * 8 + 2 * (b % 4);
      s_o[warp][g][dd] = o[b][0] + o[b][2];
      s_o[warp][g][dd + 1] = o[b][1] + o[b][3];
    }
    if (t == 0) {
      s_m[warp][g] = m_run;
      s_l[warp][g] = l_run;
    }
  }
  __syncthreads();
  // merge the warps: thread handles (head, dim) pairs
  for (int e = threadIdx.x; e < G * HD; e += kAttnWarps * 32) {
    const int hh = e / HD, d = e % HD;
    float M = -INFINITY;
    #pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w][hh]);
    float L = 0.f, acc = 0.f;
    #pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      const float sc = (s_m[w][hh] == -INFINITY) ? 0.f : exp2f(s_m[w][hh] - M);
      L += sc * s_l[w][hh];
      acc += sc * s_o[w][hh][d];
    }
    const int qh = h * G + hh;
    a.part_o[((size_t)qh * kMaxSplits + split) * HD + d] = acc;
    if (d == 0) {
      a.part_ml[((size_t)qh * kMaxSplits + split) * 2] = M;
      a.part_ml[((size_t)qh * kMaxSplits + split) * 2 + 1] = L;
    }
  }

  // The last split CTA of this kv head to finish merges the partials.  The
  // barrier orders the CTA's partial stores before thread 0's release
  // increment of the ticket; the last CTA's acquire orders its reads after
  // every other CTA's stores.
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned prev;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(prev) : "l"(a.counters + h) : "memory");
    s_last = prev == (unsigned)(a.splits - 1);
  }
  __syncthreads();
  if (!s_last) return;
  if (threadIdx.x == 0) a.counters[h] = 0u;
  // One warp per query head of the group; lane l owns dims DPL2*l .. +DPL2.
  // Each lane issues the splits' (m, l) and its own slice of their outputs
  // together (up to kComb splits in flight), so the merge costs one round
  // trip to L2 per kComb splits: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
  constexpr int DPL2 = HD / 32;
  constexpr int kComb = 40;
  using vec_t = typename std::conditional<DPL2 == 4, float4, float2>::type;
  for (int hh = warp; hh < G; hh += kAttnWarps) {
    const int qh = h * G + hh;
    const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + (size_t)qh * kMaxSplits;
    const vec_t* po = reinterpret_cast<const vec_t*>(a.part_o + (size_t)qh * kMaxSplits * HD) + lane;
    float acc[DPL2];
    #pragma unroll
    for (int d = 0; d < DPL2; ++d) acc[d] = 0.f;
    float M = -INFINITY, L = 0.f;
    for (int sp0 = 0; sp0 < a.splits; sp0 += kComb) {
      const int nsp = min(kComb, a.splits - sp0);
      vec_t ov[kComb];
      #pragma unroll
      for (int u = 0; u < kComb; ++u)
        if (u < nsp) ov[u] = __ldcg(po + (size_t)(sp0 + u) * (HD / DPL2));
      // (m, l) of splits sp0 + lane and sp0 + 32 + lane
      float2 m0 = make_float2(-INFINITY, 0.f), m1 = m0;
      if (lane < nsp) m0 = __ldcg(ml + sp0 + lane);
      if (32 + lane < nsp) m1 = __ldcg(ml + sp0 + 32 + lane);
      float cm = fmaxf(m0.x, m1.x);
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
      const float M_new = fmaxf(M, cm);
      const float base2 = M_new == -INFINITY ? 0.f : M_new;
      const float w0 = m0.x == -INFINITY ? 0.f : exp2f(m0.x - base2);
      const float w1 = m1.x == -INFINITY ? 0.f : exp2f(m1.x - base2);
      float cl = w0 * m0.y + w1 * m1.y;
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) cl += __shfl_xor_sync(0xffffffffu, cl, o);
      const float scale = M == -INFINITY ? 0.f : exp2f(M - base2);
      L = L * scale + cl;
      #pragma unroll
      for (int d = 0; d < DPL2; ++d) acc[d] *= scale;
      #pragma unroll
      for (int u = 0; u < kComb; ++u) {
        if (u < nsp) {
          const float w = __shfl_sync(0xffffffffu, u < 32 ? w0 : w1, u & 31);
          const float* ovf = reinterpret_cast<const float*>(&ov[u]);
          #pragma unroll
          for (int d = 0; d < DPL2; ++d) acc[d] = fmaf(w, ovf[d], acc[d]);
        }
      }
      M = M_new;
    }
    const float inv = 1.0f / L;
    float* dst = a.out + (size_t)qh * HD + lane * DPL2;
    #pragma unroll
    for (int d = 0; d < DPL2; ++d) dst[d] = acc[d] * inv;
  }
}

void attn_plan(int n_pages, int Hkv, int sms, int* splits, int* pps) {
  const int target = 2 * sms;                   // two resident CTAs per SM (register bound)
  int s = std::max(1, (target + Hkv - 1) / Hkv);
  s = std::min(s, kMaxSplits);
  // at least one page per warp: short lists use fewer, fuller splits
  s = std::min(s, std::max(1, n_pages / kAttnWarps));
  int per = (n_pages + s - 1) / s;
  per = std::max(per, 1);
  *pps = per;
  *splits = std::max(1, (n_pages + per - 1) / per);
}

template <typename K>
static cudaError_t launch_k(K kern, dim3 grid, dim3 block, cudaStream_t st, bool pdl, const AttnArgs& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st, bool pdl, int nb) {
  if (a.hd == 128) return launch_k(k_attn<128>, dim3(a.splits, a.Hkv, nb), dim3(kAttnWarps * 32), st, pdl, a);
  if (a.hd == 64) return launch_k(k_attn<64>, dim3(a.splits, a.Hkv, nb), dim3(kAttnWarps * 32), st, pdl, a);
  return cudaErrorInvalidValue;
}

}  // namespace bc
