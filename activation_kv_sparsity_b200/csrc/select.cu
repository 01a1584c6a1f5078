// Selection kernels of the two sparse branches.
//
// * Activation select (projection branch; ByteCross README, "Timing and
//   quality on a GPU": the projection branch sparsifies the inputs of all
//   seven projections, in the manner of TEAL's magnitude sparsity): keep the
//   k = ceil(rp*d_in) input channels of largest |v|, ties to the lower index.
//   The CTA forms v itself from the previous step's output: x*g for the two
//   RMSNorm sites (the norm's positive scale does not change the ranking, and
//   the GEMV applies it), the attention output, or silu(gate)*up.
// * Page scores (KV branch; the README's "attention-scored selection", with
//   the page key bound of Quest, listed among the paper's closest ancestors
//   on its mlsanity page): s_p = max over the group's query heads of
//   sum_c max(q_c*kmin_pc, q_c*kmax_pc).
// * Page select, per kv head (one CTA up to 8192 pages, else a cluster):
//   forced sinks and recent pages plus the best-scored others (README, "What
//   it does in one picture": sinks, part of the history and the recent
//   entries).
//
// Exact top-k over 32-bit order keys: an interval search that splits the
// candidates' key range into 256 bins per pass, then a placement pass in
// index order, so ties at the cut go to the lower indices and the list comes
// out ascending.  One CTA ranks a vector of up to 8192 elements, or a kv
// head's scores of up to 8192 pages, with its keys in registers (topk.cuh);
// the cluster version below spreads a longer vector, or more pages, over the
// CTAs of a cluster and combines the passes of their slices through
// distributed shared memory.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

#include <cooperative_groups.h>

namespace cg = cooperative_groups;

namespace bc {

// ------------------------------------------------------------------ activation select
// Above 8192 elements a cluster of kSelCluster CTAs (one per SM) ranks one vector: CTA r owns the
// r-th contiguous slice of it.  The key range, every pass's histogram and the
// final placement offsets are combined through distributed shared memory
// between hardware cluster barriers, so each CTA ends with the same cut and
// writes the kept indices of its own slice at their global positions.
constexpr int kSelCluster = 8;
constexpr int kSelClThreads = 512;
constexpr int kSelSlice = kMaxSelect / kSelCluster;   // largest slice

struct SelClusterSmem {
  int hist[2][256];
  alignas(16) int ghist[256];
  int red[32];
  uint32_t rmin[32], rmax[32];
  uint32_t lo, hi;
  int gt_tot, eq_tot;
};

// Ranks the candidates of a vector split over the cluster: this CTA holds the
// keys of [s0, s0 + ns) in s_key, and lo/hi, the min and max candidate key it
// saw.  Writes the forced elements and the `need` best candidates (ties to
// the lower index) of the whole vector, ascending, to out.  Every CTA of the
// cluster calls it with its slice; all threads of each CTA take part.
template <typename StateF>
__device__ void cluster_topk(const uint32_t* s_key, int s0, int ns, int need, StateF state, uint32_t lo,
                             uint32_t hi, int* out, SelClusterSmem& sm, cg::cluster_group& cl) {
  const int tid = threadIdx.x;
  for (int b = tid; b < 2 * 256; b += kSelClThreads) (&sm.hist[0][0])[b] = 0;
  block_minmax<kSelClThreads>(lo, hi, sm.rmin, sm.rmax);
  if (tid == 0) {
    sm.lo = lo;
    sm.hi = hi;
  }
  cl.sync();
  lo = 0xFFFFFFFFu;
  hi = 0u;
  for (int q = 0; q < kSelCluster; ++q) {
    lo = min(lo, *cl.map_shared_rank(&sm.lo, q));
    hi = max(hi, *cl.map_shared_rank(&sm.hi, q));
  }
  uint32_t base = lo, span_m1 = hi - lo;
  int rem = need;
  if (need <= 0) span_m1 = 0;

  // interval passes: local histograms of the slices, summed across the cluster
  #pragma unroll 1
  for (int pass = 0; pass < 5 && span_m1 > 0; ++pass) {
    int* H = sm.hist[pass & 1];
    const int sh = max(0, 24 - __clz(span_m1));
    for (int j = tid; j < ns; j += kSelClThreads) {
      if (state(s0 + j) != ST_CAND) continue;
      const uint32_t kk = s_key[j];
      if (kk >= base && kk - base <= span_m1) atomicAdd(&H[(kk - base) >> sh], 1);
    }
    cl.sync();   // every slice's histogram is complete; the other buffer is free
    if (tid < 256) {
      int g = 0;
      #pragma unroll
      for (int q = 0; q < kSelCluster; ++q) g += cl.map_shared_rank(H, q)[tid];
      sm.ghist[tid] = g;
      sm.hist[(pass + 1) & 1][tid] = 0;
    }
    __syncthreads();
    // every warp finds the boundary bin itself (the next pass writes ghist
    // only after the next cluster barrier, which every warp reaches after
    // reading it)
    int bin, above, cnt;
    warp_find_bin(sm.ghist, rem, bin, above, cnt);
    const uint32_t b_lo = (uint32_t)bin << sh;
    rem -= above;
    base += b_lo;
    span_m1 = min((1u << sh) - 1u, span_m1 - b_lo);
    if (cnt == rem) break;                        // the whole bin is kept
  }

  // placement: forced elements, keys above the interval, and the first
  // `rem` candidates (by index) inside it
  const uint32_t top = base + span_m1;
  const int per = (ns + kSelClThreads - 1) / kSelClThreads;
  const int b0 = min(ns, tid * per), b1 = min(ns, b0 + per);
  int gt = 0, eq = 0;
  for (int j = b0; j < b1; ++j) {
    const uint8_t st = state(s0 + j);
    if (st == ST_FORCED) {
      ++gt;
    } else if (st == ST_CAND && need > 0) {
      const uint32_t kk = s_key[j];
      gt += kk > top;
      eq += kk >= base && kk <= top;
    }
  }
  int total;
  const int excl = block_excl_scan<kSelClThreads>((gt << 16) | eq, sm.red, &total);
  if (tid == 0) {
    sm.gt_tot = total >> 16;
    sm.eq_tot = total & 0xFFFF;
  }
  cl.sync();
  int gt_before = 0, eq_before = 0;
  for (int q = 0; q < (int)cl.block_rank(); ++q) {
    gt_before += *cl.map_shared_rank(&sm.gt_tot, q);
    eq_before += *cl.map_shared_rank(&sm.eq_tot, q);
  }
  int er = eq_before + (excl & 0xFFFF);
  int pos = gt_before + (excl >> 16) + min(er, rem);
  for (int j = b0; j < b1; ++j) {
    const uint8_t st = state(s0 + j);
    bool keep = st == ST_FORCED;
    if (st == ST_CAND && need > 0) {
      const uint32_t kk = s_key[j];
      if (kk > top) {
        keep = true;
      } else if (kk >= base) {
        keep = er < rem;
        ++er;
      }
    }
    if (keep) out[pos++] = s0 + j;
  }
  cl.sync();   // peers may still be reading this CTA's totals
}

__global__ void __launch_bounds__(kSelClThreads, 1) k_select(SelectArgs a) {
  a.x += blockIdx.y * a.x_stride;                 // batched launch: vector blockIdx.y
  a.idx += blockIdx.y * a.idx_stride;
  __shared__ uint32_t s_key[kSelSlice];
  __shared__ SelClusterSmem sm;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int tid = threadIdx.x;
  const int n = a.n;
  const int s0 = (int)(((long long)n * rank) / kSelCluster);
  const int ns = (int)(((long long)n * (rank + 1)) / kSelCluster) - s0;
  pdl_wait();
  pdl_trigger();

  // the slice's keys, with 8 elements per thread per round of loads
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int j0 = 0; j0 < ns; j0 += 8 * kSelClThreads) {
    float a0[8], a1[8];
    #pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * kSelClThreads + tid, i = s0 + j;
      a0[u] = 0.f;
      a1[u] = 0.f;
      if (j < ns) {
        switch (a.prep) {
          case SP_NORM: a0[u] = a.x[i]; a1[u] = bf16f(a.gain[i]); break;
          case SP_EMBED_NORM: a0[u] = bf16f(a.embed_row[i]); a1[u] = bf16f(a.gain[i]); break;
          case SP_SWIGLU: a0[u] = a.x[i]; a1[u] = a.x[n + i]; break;
          default: a0[u] = a.x[i];
        }
      }
    }
    #pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * kSelClThreads + tid, i = s0 + j;
      if (j >= ns) break;
      float v;
      switch (a.prep) {
        case SP_NORM: v = a0[u] * a1[u]; break;
        case SP_EMBED_NORM: a.x_init[i] = a0[u]; v = a0[u] * a1[u]; break;
        case SP_SWIGLU: v = a0[u] / (1.0f + expf(-a0[u])) * a1[u]; break;
        default: v = a0[u];
      }
      if (a.vout) a.vout[i] = v;
      const uint32_t kk = __float_as_uint(fabsf(v));
      s_key[j] = kk;
      lo = min(lo, kk);
      hi = max(hi, kk);
    }
  }
  cluster_topk(s_key, s0, ns, a.k, [](int) { return (uint8_t)ST_CAND; }, lo, hi, a.idx, sm, cl);
}

// Vectors up to kSelOneCta elements: one CTA ranks the whole vector with its
// keys in registers (a cluster's barriers cost more than they save at this
// size).  Warp w loads the elements (w*KPT + c)*32 + lane, c < KPT: rows of
// 32 consecutive elements, all KPT rows in flight together.  (256 threads
// with 16 keys each ran faster alone but slower inside the step: 7.5 against
// 5.8 us per selection.)
constexpr int kSelOneCta = 8192;
constexpr int kSelThreads1 = 1024;

template <int KPT>
__global__ void __launch_bounds__(kSelThreads1, 1) k_select_cta(SelectArgs a) {
  a.x += blockIdx.x * a.x_stride;                 // batched launch: vector blockIdx.x
  a.idx += blockIdx.x * a.idx_stride;
  __shared__ RegTopkSmem<kSelThreads1> sm;
  const int tid = threadIdx.x, n = a.n;
  const int ibase = (tid >> 5) * KPT * 32 + (tid & 31);
  pdl_wait();
  pdl_trigger();
  float a0[KPT], a1[KPT];
  #pragma unroll
  for (int c = 0; c < KPT; ++c) {
    const int i = ibase + 32 * c;
    a0[c] = 0.f;
    a1[c] = 0.f;
    if (i < n) {
      switch (a.prep) {
        case SP_NORM: a0[c] = a.x[i]; a1[c] = bf16f(a.gain[i]); break;
        case SP_EMBED_NORM: a0[c] = bf16f(a.embed_row[i]); a1[c] = bf16f(a.gain[i]); break;
        case SP_SWIGLU: a0[c] = a.x[i]; a1[c] = a.x[n + i]; break;
        default: a0[c] = a.x[i];
      }
    }
  }
  uint32_t kr[KPT];
  #pragma unroll
  for (int c = 0; c < KPT; ++c) {
    const int i = ibase + 32 * c;
    float v;
    switch (a.prep) {
      case SP_NORM: v = a0[c] * a1[c]; break;
      case SP_EMBED_NORM: v = a0[c] * a1[c]; break;
      case SP_SWIGLU: v = a0[c] / (1.0f + expf(-a0[c])) * a1[c]; break;
      default: v = a0[c];
    }
    if (i < n) {
      if (a.prep == SP_EMBED_NORM) a.x_init[i] = a0[c];
      if (a.vout) a.vout[i] = v;
    }
    kr[c] = __float_as_uint(fabsf(v));
  }
  reg_topk<kSelThreads1, KPT>(kr, n, a.k, [](int) { return (uint8_t)ST_CAND; }, a.idx, sm);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st, bool pdl, int nb) {
  cudaLaunchConfig_t cfg = {};
  if (a.n <= kSelOneCta) {
    cfg.gridDim = dim3(nb);
    cfg.blockDim = dim3(kSelThreads1);
    cfg.stream = st;
    cudaLaunchAttribute attr1[1];
    attr1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr1[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr1;
    cfg.numAttrs = pdl ? 1 : 0;
    if (a.n <= kSelThreads1 * 4) return cudaLaunchKernelEx(&cfg, k_select_cta<4>, a);
    return cudaLaunchKernelEx(&cfg, k_select_cta<8>, a);
  }
  cfg.gridDim = dim3(kSelCluster, nb);
  cfg.blockDim = dim3(kSelClThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSelCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_select, a);
}

// ------------------------------------------------------------------ page scores + select
// A group of hd/8 lanes scores one page: each lane holds 8 channels of the
// group's queries and reads 16 bytes of kmin and 16 bytes of kmax.  A CTA
// walks `rounds` rounds of 64 pages (at hd = 128); the next round's bounds
// are in flight while the current round is scored.
constexpr int kPageThreads = 256;

// The page bound of one page for the group's query heads: the max over
// heads of sum_c max(q_c * kmin_c, q_c * kmax_c) = sum_c q_c * (q_c >= 0 ?
// kmax_c : kmin_c).  The LPP lanes of a page each hold 8 channels (mn/mx:
// their 8 bf16 bounds) and sum them for every head; a transpose-reduce then
// halves the heads a lane carries at each of the first log2(GMAX) butterfly
// steps (it keeps one half and sends the other), so all GMAX sums complete
// in about GMAX + log2(LPP / GMAX) shuffles instead of GMAX * log2(LPP),
// and a last butterfly takes the max over the heads.  Every lane of the page
// returns the page's score.  Heads g >= G count as -inf.
template <int LPP, int GMAX>
__device__ __forceinline__ float page_bound_score(const float (&qv)[GMAX][8], int G, const uint4& mn,
                                                  const uint4& mx) {
  static_assert(GMAX <= LPP, "one head per lane after the transpose");
  const uint32_t mnw[4] = {mn.x, mn.y, mn.z, mn.w};
  const uint32_t mxw[4] = {mx.x, mx.y, mx.z, mx.w};
  float lo[8], hi[8];
  #pragma unroll
  for (int j = 0; j < 4; ++j) {
    lo[2 * j] = bf16_lo(mnw[j]);
    lo[2 * j + 1] = bf16_hi(mnw[j]);
    hi[2 * j] = bf16_lo(mxw[j]);
    hi[2 * j + 1] = bf16_hi(mxw[j]);
  }
  float v[GMAX];
  #pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    float t = 0.f;
    #pragma unroll
    for (int c = 0; c < 8; ++c) t = fmaf(qv[g][c], qv[g][c] >= 0.f ? hi[c] : lo[c], t);
    v[g] = t;
  }
  const int lane = threadIdx.x & 31;
  // transpose-reduce: at offset o = LPP/2, LPP/4, ... a lane keeps the lower
  // or upper half of its heads (by the lane bit o) and adds its partner's
  // copy of that half
  int head = 0;
  #pragma unroll
  for (int n = GMAX, o = LPP / 2; n > 1; n >>= 1, o >>= 1) {
    const bool upper = (lane & o) != 0;
    #pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = upper ? v[j] : v[j + n / 2];
      const float keep = upper ? v[j + n / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
    head = 2 * head + (upper ? 1 : 0);
  }
  float s = v[0];
  #pragma unroll
  for (int o = LPP / (2 * GMAX); o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  // head now names the sum this lane holds; max over the heads
  s = head < G ? s : -INFINITY;
  #pragma unroll
  for (int o = LPP / GMAX; o < LPP; o <<= 1) s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, o));
  return s;
}

template <int HD>
__host__ __device__ constexpr int pages_per_round() {
  return (kPageThreads / 32) * (32 / (HD / 8)) * 4;
}

template <int HD, int GMAX>
__global__ void __launch_bounds__(kPageThreads, GMAX <= 4 ? 2 : 1) k_pages(PageArgs a) {
  a.q += blockIdx.z * a.q_stride;                 // batched launch: sequence blockIdx.z
  a.meta += blockIdx.z * a.meta_stride;
  a.scores += blockIdx.z * a.sp_stride;
  constexpr int LPP = HD / 8;          // lanes per page
  constexpr int PPW = 32 / LPP;        // pages per warp step
  constexpr int STEPS = 4;             // warp steps per round
  constexpr int PPR = pages_per_round<HD>();
  const int h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPP, cl = lane % LPP;
  const __nv_bfloat16* mbase = a.meta + (size_t)h * a.Pmax * 2 * HD;
  float* scores = a.scores + (size_t)h * a.Pmax;
  const int p_cta = blockIdx.x * a.rounds * PPR;
  auto page_of = [&](int round, int it) { return p_cta + round * PPR + (it * (kPageThreads / 32) + warp) * PPW + sub; };
  auto load_one = [&](int p, uint4& mn, uint4& mx) {
    const __nv_bfloat16* mp = mbase + (size_t)p * 2 * HD + cl * 8;
    mn = ld_stream(mp);
    mx = ld_stream(mp + HD);
  };
  auto load_round = [&](int round, uint4* mn, uint4* mx, int p_end) {
    #pragma unroll
    for (int it = 0; it < STEPS; ++it) {
      const int p = page_of(round, it);
      mn[it] = make_uint4(0, 0, 0, 0);
      mx[it] = mn[it];
      if (round < a.rounds && p < p_end) load_one(p, mn[it], mx[it]);
    }
  };
  // The bounds do not depend on the previous kernel except those of the last
  // page, which the q/k/v epilogue rewrites as it appends: load the first
  // round's others before waiting for it.
  uint4 mna[STEPS], mxa[STEPS], mnb[STEPS], mxb[STEPS];
  load_round(0, mna, mxa, a.P - 1);
  pdl_wait();
  pdl_trigger();
  #pragma unroll
  for (int it = 0; it < STEPS; ++it)
    if (a.rounds > 0 && page_of(0, it) == a.P - 1) load_one(a.P - 1, mna[it], mxa[it]);
  float qv[GMAX][8];   // [head][channel]
  #pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    float4 q0 = make_float4(0.f, 0.f, 0.f, 0.f), q1 = q0;
    if (g < a.G) {
      const float4* qp = reinterpret_cast<const float4*>(a.q + (size_t)(h * a.G + g) * HD + cl * 8);
      q0 = qp[0];
      q1 = qp[1];
    }
    qv[g][0] = q0.x; qv[g][1] = q0.y; qv[g][2] = q0.z; qv[g][3] = q0.w;
    qv[g][4] = q1.x; qv[g][5] = q1.y; qv[g][6] = q1.z; qv[g][7] = q1.w;
  }
  auto score_round = [&](int round, const uint4* mn, const uint4* mx) {
    #pragma unroll
    for (int it = 0; it < STEPS; ++it) {
      const int p = page_of(round, it);
      const float best = page_bound_score<LPP, GMAX>(qv, a.G, mn[it], mx[it]);
      if (p < a.P && cl == 0) scores[p] = best;
    }
  };
  for (int r = 0; r < a.rounds; r += 2) {
    load_round(r + 1, mnb, mxb, a.P);
    score_round(r, mna, mxa);
    if (r + 1 >= a.rounds) break;
    load_round(r + 2, mna, mxa, a.P);
    score_round(r + 1, mnb, mxb);
  }
}

// Page select above 8192 pages: one cluster per kv head; CTA r ranks the
// r-th slice of the head's page scores.  Forced pages (sinks, recent) are
// kept and not ranked.  (One 1024-thread CTA with 16 keys a thread measured
// slower.)
__global__ void __launch_bounds__(kSelClThreads, 1) k_page_select(PageArgs a) {
  a.scores += blockIdx.z * a.sp_stride;           // batched launch: sequence blockIdx.z
  a.pages += blockIdx.z * a.sp_stride;
  __shared__ uint32_t s_key[kSelSlice];
  __shared__ SelClusterSmem sm;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int h = blockIdx.y, tid = threadIdx.x;
  const int P = a.P;
  const int s0 = (int)(((long long)P * rank) / kSelCluster);
  const int ns = (int)(((long long)P * (rank + 1)) / kSelCluster) - s0;
  pdl_wait();
  pdl_trigger();
  const int sink_end = min(a.sinks, P), rec_begin = max(P - a.recent, 0);
  const int n_forced = sink_end + (P - max(rec_begin, sink_end));
  const float* scores = a.scores + (size_t)h * a.Pmax;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  #pragma unroll 4
  for (int j = tid; j < ns; j += kSelClThreads) {
    const int i = s0 + j;
    const uint32_t kk = float_order_key(scores[i]);
    s_key[j] = kk;
    if (i >= sink_end && i < rec_begin) {
      lo = min(lo, kk);
      hi = max(hi, kk);
    }
  }
  cluster_topk(
      s_key, s0, ns, a.K - n_forced,
      [&](int i) { return (uint8_t)((i < sink_end || i >= rec_begin) ? ST_FORCED : ST_CAND); }, lo, hi,
      a.pages + (size_t)h * a.Pmax, sm, cl);
}

// Page select up to 8192 pages, one CTA per kv head: the head's P scores as
// register keys (KPT per thread, P <= 1024*KPT), forced pages kept.
template <int KPT>
__global__ void __launch_bounds__(kSelThreads1, 1) k_page_select_cta(PageArgs a) {
  a.scores += blockIdx.y * a.sp_stride;           // batched launch: sequence blockIdx.y
  a.pages += blockIdx.y * a.sp_stride;
  __shared__ RegTopkSmem<kSelThreads1> sm;
  const int h = blockIdx.x, tid = threadIdx.x, P = a.P;
  const int ibase = (tid >> 5) * KPT * 32 + (tid & 31);
  pdl_wait();
  pdl_trigger();
  const float* scores = a.scores + (size_t)h * a.Pmax;
  float v[KPT];
  #pragma unroll
  for (int c = 0; c < KPT; ++c) v[c] = ibase + 32 * c < P ? scores[ibase + 32 * c] : 0.f;
  uint32_t kr[KPT];
  #pragma unroll
  for (int c = 0; c < KPT; ++c) kr[c] = float_order_key(v[c]);
  const int sink_end = min(a.sinks, P), rec_begin = max(P - a.recent, 0);
  const int n_forced = sink_end + (P - max(rec_begin, sink_end));
  reg_topk<kSelThreads1, KPT>(
      kr, P, a.K - n_forced,
      [&](int i) { return (uint8_t)((i < sink_end || i >= rec_begin) ? ST_FORCED : ST_CAND); },
      a.pages + (size_t)h * a.Pmax, sm);
}

int page_rounds(int P, int hd, int Hkv, int sms) {
  const int ppr = hd == 128 ? pages_per_round<128>() : pages_per_round<64>();
  const int units = Hkv * ((P + ppr - 1) / ppr);          // rounds of work in all
  const int r = (units + 2 * sms - 1) / (2 * sms);        // about two CTAs per SM
  return r < 1 ? 1 : (r > 8 ? 8 : r);
}

dim3 pages_grid(const PageArgs& a) {
  const int ppc = (a.hd == 128 ? pages_per_round<128>() : pages_per_round<64>()) * a.rounds;
  return dim3((a.P + ppc - 1) / ppc, a.Hkv);
}

cudaError_t launch_page_scores(const PageArgs& a, cudaStream_t st, bool pdl, int nb) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = pages_grid(a);
  cfg.gridDim.z = nb;
  cfg.blockDim = dim3(kPageThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const bool g4 = a.G <= 4;
  if (a.hd == 128) return g4 ? cudaLaunchKernelEx(&cfg, k_pages<128, 4>, a) : cudaLaunchKernelEx(&cfg, k_pages<128, 8>, a);
  if (a.hd == 64) return g4 ? cudaLaunchKernelEx(&cfg, k_pages<64, 4>, a) : cudaLaunchKernelEx(&cfg, k_pages<64, 8>, a);
  return cudaErrorInvalidValue;
}

int page_select_variant(int P) {
  if (P <= kSelThreads1 * 2) return 2;
  if (P <= kSelThreads1 * 4) return 4;
  if (P <= kSelThreads1 * 8) return 8;
  return 0;
}

cudaError_t launch_page_select(const PageArgs& a, cudaStream_t st, bool pdl, int nb) {
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const int variant = page_select_variant(a.P);
  if (variant) {
    cfg.gridDim = dim3(a.Hkv, nb);
    cfg.blockDim = dim3(kSelThreads1);
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (variant == 2) return cudaLaunchKernelEx(&cfg, k_page_select_cta<2>, a);
    if (variant == 4) return cudaLaunchKernelEx(&cfg, k_page_select_cta<4>, a);
    return cudaLaunchKernelEx(&cfg, k_page_select_cta<8>, a);
  }
  cfg.gridDim = dim3(kSelCluster, a.Hkv, nb);
  cfg.blockDim = dim3(kSelClThreads);
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = kSelCluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = pdl ? attr : attr + 1;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_page_select, a);
}

}  // namespace bc
