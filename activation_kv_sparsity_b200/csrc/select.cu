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
// * Page select, run by the last scoring CTA of each kv head to finish:
//   forced sinks and recent pages plus the best-scored others (README, "What
//   it does in one picture": sinks, part of the history and the recent
//   entries).
//
// Exact top-k over 32-bit order keys: an interval search that splits the
// candidates' key range into 256 bins per pass.  Only the first pass sweeps
// every key; the keys of the boundary bin are gathered into shared memory and
// the remaining passes (at most four) run on them.  A single block scan over
// packed (above-cut, at-cut) counts in index order then places every kept
// index: ties at the cut go to the lower indices, and the list comes out
// ascending.
#include "common.cuh"
#include "kernels.h"

namespace bc {

enum : uint8_t { ST_OUT = 0, ST_CAND = 1, ST_FORCED = 2 };

constexpr int kCandCap = 2048;   // boundary-bin candidates kept in shared memory

template <int NT>
struct TopkSmem {
  int hist[256];
  int red[32];
  uint32_t rmin[32], rmax[32];
  uint32_t cand_key[kCandCap];
  int cand_n;
  uint32_t bin;
  int above, cnt;
};

// One pass of the interval search over `m` keys: counts them into at most 256
// equal power-of-two-wide bins of [base, base + span_m1] and finds the bin
// where the count from the top reaches rem.  Narrows the interval to that bin, lowers rem by the keys
// above it and returns the bin's count.  All NT threads call it.
template <int NT, typename KeyAt>
__device__ int interval_pass(int m, KeyAt key_at, uint32_t& base, uint32_t& span_m1, int& rem,
                             TopkSmem<NT>& sm) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // power-of-two bin width: the smallest 2^sh with (span_m1 >> sh) < 256
  const int sh = max(0, 24 - __clz(span_m1));
  const uint32_t width = 1u << sh;
  for (int i = tid; i < m; i += NT) {
    uint32_t kk;
    if (!key_at(i, kk)) continue;
    if (kk >= base && kk - base <= span_m1) atomicAdd(&sm.hist[(kk - base) >> sh], 1);
  }
  __syncthreads();
  if (warp == 0) {
    int c[8], sum = 0;
    #pragma unroll
    for (int j = 0; j < 8; ++j) {                 // lane owns bins 255-8*lane .. 248-8*lane
      c[j] = sm.hist[255 - 8 * lane - j];
      sum += c[j];
    }
    int incl = sum;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int above = incl - sum;
    #pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (above < rem && above + c[j] >= rem) {
        sm.bin = (uint32_t)(255 - 8 * lane - j);
        sm.above = above;
        sm.cnt = c[j];
      }
      above += c[j];
    }
  }
  __syncthreads();
  const uint32_t b_lo = sm.bin * width;
  rem -= sm.above;
  const int cnt = sm.cnt;
  base += b_lo;
  span_m1 = min(width - 1u, span_m1 - b_lo);
  for (int j = tid; j < 256; j += NT) sm.hist[j] = 0;
  __syncthreads();
  return cnt;
}

// Writes the forced elements and the `need` best candidates (by key, higher
// first; ties to the lower index) of [0, n) to out, ascending.  All NT
// threads must call it, each with the min and max key of the candidates it
// saw (lo/hi; the block combines them), and sm.hist zeroed.
//
// The search keeps an interval [base, base + span_m1] of key values that
// holds the cut: candidates above it are kept, below it dropped.  A pass
// splits the interval into 256 equal bins and keeps the bin where the count
// from the top reaches `need`, so the interval shrinks 256-fold per pass
// until one key value is left or the bin is kept whole.  Starting from the
// candidates' [min, max] spreads keys over the bins however their exponents
// cluster.  Only the first pass sweeps all n keys: the boundary bin's keys
// are then gathered into shared memory and the later passes run on them.
template <int NT, typename KeyF, typename StateF>
__device__ void radix_topk(int n, int need, KeyF key, StateF state, int* out, TopkSmem<NT>& sm,
                           uint32_t lo, uint32_t hi) {
  static_assert(NT >= 256 && NT % 32 == 0 && NT <= 1024, "block shape");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t base = 0, span_m1 = 0xFFFFFFFFu;
  int rem = need;
  if (need > 0) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      sm.rmin[warp] = lo;
      sm.rmax[warp] = hi;
    }
    if (tid == 0) sm.cand_n = 0;
    __syncthreads();
    lo = 0xFFFFFFFFu;
    hi = 0u;
    #pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
      lo = min(lo, sm.rmin[w]);
      hi = max(hi, sm.rmax[w]);
    }
    base = lo;
    span_m1 = hi - lo;
    auto full = [&](int i, uint32_t& kk) {
      if (state(i) != ST_CAND) return false;
      kk = key(i);
      return true;
    };
    int cnt = span_m1 > 0 ? interval_pass<NT>(n, full, base, span_m1, rem, sm) : 0;
    if (span_m1 > 0 && cnt != rem) {
      if (cnt <= kCandCap) {
        // gather the boundary bin's keys, then narrow on them alone
        for (int i = tid; i < n; i += NT) {
          if (state(i) != ST_CAND) continue;
          const uint32_t kk = key(i);
          if (kk >= base && kk - base <= span_m1) sm.cand_key[atomicAdd(&sm.cand_n, 1)] = kk;
        }
        __syncthreads();
        const int m = sm.cand_n;
        auto small = [&](int i, uint32_t& kk) {
          kk = sm.cand_key[i];
          return true;
        };
        #pragma unroll 1
        for (int pass = 0; pass < 4 && span_m1 > 0; ++pass)
          if (interval_pass<NT>(m, small, base, span_m1, rem, sm) == rem) break;
      } else {
        #pragma unroll 1
        for (int pass = 0; pass < 4 && span_m1 > 0; ++pass)
          if (interval_pass<NT>(n, full, base, span_m1, rem, sm) == rem) break;
      }
    }
  }
  // keep: key above the interval, or inside it among the first `rem` by index
  const uint32_t top = base + span_m1;            // inclusive upper end
  const int per = (n + NT - 1) / NT;
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  int gt = 0, eq = 0;
  for (int i = b0; i < b1; ++i) {
    const uint8_t st = state(i);
    if (st == ST_FORCED) {
      ++gt;
    } else if (st == ST_CAND && need > 0) {
      const uint32_t kk = key(i);
      gt += kk > top;
      eq += kk >= base && kk <= top;
    }
  }
  int total;
  const int excl = block_excl_scan<NT>((gt << 16) | eq, sm.red, &total);
  int er = excl & 0xFFFF;
  int pos = (excl >> 16) + min(er, rem);
  for (int i = b0; i < b1; ++i) {
    const uint8_t st = state(i);
    bool keep = st == ST_FORCED;
    if (st == ST_CAND && need > 0) {
      const uint32_t kk = key(i);
      if (kk > top) {
        keep = true;
      } else if (kk >= base) {
        keep = er < rem;
        ++er;
      }
    }
    if (keep) out[pos++] = i;
  }
}

// ------------------------------------------------------------------ activation select
constexpr int kSelThreads2 = 1024;

__global__ void __launch_bounds__(kSelThreads2, 1) k_select(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t s_key[];
  __shared__ TopkSmem<kSelThreads2> sm;
  const int tid = threadIdx.x, n = a.n;
  pdl_wait();
  pdl_trigger();
  // prep: 8 elements per thread per round, their loads in flight together
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int j = tid; j < 256; j += kSelThreads2) sm.hist[j] = 0;
  for (int i0 = 0; i0 < n; i0 += 8 * kSelThreads2) {
    float a0[8], a1[8];
    #pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kSelThreads2 + tid;
      a0[u] = 0.f;
      a1[u] = 0.f;
      if (i < n) {
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
      const int i = i0 + u * kSelThreads2 + tid;
      if (i >= n) break;
      float v;
      switch (a.prep) {
        case SP_NORM: v = a0[u] * a1[u]; break;
        case SP_EMBED_NORM: a.x_init[i] = a0[u]; v = a0[u] * a1[u]; break;
        case SP_SWIGLU: v = a0[u] / (1.0f + expf(-a0[u])) * a1[u]; break;
        default: v = a0[u];
      }
      if (a.vout) a.vout[i] = v;
      const uint32_t kk = __float_as_uint(fabsf(v));
      s_key[i] = kk;
      lo = min(lo, kk);
      hi = max(hi, kk);
    }
  }
  __syncthreads();
  radix_topk<kSelThreads2>(
      n, a.k, [&](int i) { return s_key[i]; }, [](int) { return (uint8_t)ST_CAND; }, a.idx, sm, lo, hi);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)kMaxSelect * sizeof(uint32_t);
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kSelThreads2);
  cfg.dynamicSmemBytes = (size_t)a.n * sizeof(uint32_t);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_select, a);
}

// ------------------------------------------------------------------ page scores + select
// A group of hd/8 lanes scores one page: each lane holds 8 channels of the
// group's G queries and reads 16 bytes of kmin and 16 bytes of kmax.
constexpr int kPageThreads = 256;

template <int HD>
__global__ void __launch_bounds__(kPageThreads) k_pages(PageArgs a) {
  constexpr int LPP = HD / 8;          // lanes per page
  constexpr int PPW = 32 / LPP;        // pages per warp step
  constexpr int PAGES_PER_CTA = (kPageThreads / 32) * PPW * 4;
  __shared__ TopkSmem<kPageThreads> sm;
  __shared__ int s_last;
  const int h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPP, cl = lane % LPP;
  pdl_wait();
  pdl_trigger();
  float qv[8][8];   // [head][channel], G <= 8
  #pragma unroll
  for (int g = 0; g < 8; ++g)
    #pragma unroll
    for (int j = 0; j < 8; ++j)
      qv[g][j] = (g < a.G) ? a.q[(size_t)(h * a.G + g) * HD + cl * 8 + j] : 0.f;
  const int p_begin = blockIdx.x * PAGES_PER_CTA;
  const int p_end = min(a.P, p_begin + PAGES_PER_CTA);
  const __nv_bfloat16* mbase = a.meta + (size_t)h * a.Pmax * 2 * HD;
  float* scores = a.scores + (size_t)h * a.Pmax;
  // warp-uniform loop: every lane takes part in the shuffles
  for (int pb = p_begin + warp * PPW; pb < p_end; pb += (kPageThreads / 32) * PPW) {
    const int p = pb + sub;
    const bool valid = p < p_end;
    uint4 mn = make_uint4(0, 0, 0, 0), mx = make_uint4(0, 0, 0, 0);
    if (valid) {
      const __nv_bfloat16* mp = mbase + (size_t)p * 2 * HD + cl * 8;
      mn = ld_stream(mp);
      mx = ld_stream(mp + HD);
    }
    const uint32_t mnw[4] = {mn.x, mn.y, mn.z, mn.w}, mxw[4] = {mx.x, mx.y, mx.z, mx.w};
    float best = -INFINITY;
    #pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (g >= a.G) break;
      float s = 0.f;
      #pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo0 = bf16_lo(mnw[j]), lo1 = bf16_hi(mnw[j]);
        const float hi0 = bf16_lo(mxw[j]), hi1 = bf16_hi(mxw[j]);
        s += fmaxf(qv[g][2 * j] * lo0, qv[g][2 * j] * hi0);
        s += fmaxf(qv[g][2 * j + 1] * lo1, qv[g][2 * j + 1] * hi1);
      }
      #pragma unroll
      for (int o = LPP / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o, LPP);
      best = fmaxf(best, s);
    }
    if (valid && cl == 0) scores[p] = best;
  }
  // the last CTA of this kv head to finish selects its pages
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.counters[h], 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) a.counters[h] = 0u;
  const int P = a.P;
  extern __shared__ __align__(16) uint32_t s_key[];
  const int sink_end = min(a.sinks, P), rec_begin = max(P - a.recent, 0);
  const int n_forced = sink_end + (P - max(rec_begin, sink_end));
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int j = tid; j < 256; j += kPageThreads) sm.hist[j] = 0;
  #pragma unroll 8
  for (int i = tid; i < P; i += kPageThreads) {
    const uint32_t kk = float_order_key(ld_cg(&scores[i]));
    s_key[i] = kk;
    if (i >= sink_end && i < rec_begin) {
      lo = min(lo, kk);
      hi = max(hi, kk);
    }
  }
  __syncthreads();
  radix_topk<kPageThreads>(
      P, a.K - n_forced, [&](int i) { return s_key[i]; },
      [&](int i) { return (uint8_t)((i < sink_end || i >= rec_begin) ? ST_FORCED : ST_CAND); },
      a.pages + (size_t)h * a.Pmax, sm, lo, hi);
}

dim3 pages_grid(const PageArgs& a) {
  const int ppc = (kPageThreads / 32) * (32 / (a.hd / 8)) * 4;
  return dim3((a.P + ppc - 1) / ppc, a.Hkv);
}

size_t pages_smem(const PageArgs& a) { return (size_t)a.P * sizeof(uint32_t); }

cudaError_t launch_pages(const PageArgs& a, cudaStream_t st, bool pdl) {
  static bool attr_done = false;
  if (!attr_done) {
    const int smem = kMaxSelect * (int)sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(k_pages<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_pages<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = pages_grid(a);
  cfg.blockDim = dim3(kPageThreads);
  cfg.dynamicSmemBytes = pages_smem(a);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (a.hd == 128) return cudaLaunchKernelEx(&cfg, k_pages<128>, a);
  if (a.hd == 64) return cudaLaunchKernelEx(&cfg, k_pages<64>, a);
  return cudaErrorInvalidValue;
}

}  // namespace bc
