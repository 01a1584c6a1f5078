// Selection kernels of the two sparse branches.
//
// * Activation select (projection branch; ByteCross README, "Timing and
//   quality on a GPU": the projection branch sparsifies the inputs of all
//   seven projections, in the manner of TEAL's magnitude sparsity): keep the
//   k = ceil(rp*d_in) input channels of largest |x|, ties to the lower index.
//   The same CTA first produces the vector it ranks: RMSNorm (optionally
//   starting from the token's embedding row) or SwiGLU, so that dense mode
//   runs the same kernel with the ranking switched off.
// * Page scorer (KV branch; the README's "attention-scored selection", with
//   the page key bound of Quest, listed among the paper's closest ancestors
//   on its mlsanity page): s_p = max over the group's query heads of
//   sum_c max(q_c*kmin_pc, q_c*kmax_pc).
// * Page select: forced sinks and recent pages plus the best-scored others
//   (README, "What it does in one picture": sinks, part of the history and
//   the recent entries).
//
// Exact top-k: MSB-first radix select over 32-bit order keys in three passes
// (11, 11 and 10 bits) finds the key T of the last kept element and how many
// elements equal to T are kept; two block scans in index order then resolve
// ties to the lower index and write the kept indices ascending.
#include "common.cuh"
#include "kernels.h"

namespace bc {

// State of an element for the ranking.
enum : uint8_t { ST_OUT = 0, ST_CAND = 1, ST_FORCED = 2 };

// Ranks the candidates of s_key/s_state[0..n) and writes the kept indices
// (forced ones included) ascending to idx.  need = kept candidates.
// All kSelThreads threads must call it.  s_hist holds 2048 ints.
__device__ void topk_write(const uint32_t* s_key, const uint8_t* s_state, int n, int need,
                           int* s_hist, int* s_red, int* idx) {
  const int tid = threadIdx.x;
  __shared__ uint32_t s_digit;
  __shared__ int s_above;
  uint32_t prefix = 0, pmask = 0;
  int rem = need;
  if (need > 0) {
    #pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nb = pass == 2 ? 1024 : 2048;
      for (int b = tid; b < 2048; b += kSelThreads) s_hist[b] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kSelThreads) {
        const uint32_t key = s_key[i];
        if (s_state[i] == ST_CAND && (key & pmask) == prefix)
          atomicAdd(&s_hist[(key >> shift) & (nb - 1)], 1);
      }
      __syncthreads();
      // thread t owns digits nb-1-2t and nb-2-2t (descending order)
      const int d0 = nb - 1 - 2 * tid, d1 = nb - 2 - 2 * tid;
      const int c0 = d0 >= 0 ? s_hist[d0] : 0;
      const int c1 = d1 >= 0 ? s_hist[d1] : 0;
      int total;
      const int above0 = block_excl_scan<kSelThreads>(c0 + c1, s_red, &total);
      if (d0 >= 0 && above0 < rem && above0 + c0 >= rem) {
        s_digit = (uint32_t)d0;
        s_above = above0;
      } else if (d1 >= 0 && above0 + c0 < rem && above0 + c0 + c1 >= rem) {
        s_digit = (uint32_t)d1;
        s_above = above0 + c0;
      }
      __syncthreads();
      prefix |= s_digit << shift;
      pmask |= (uint32_t)(nb - 1) << shift;
      rem -= s_above;
      __syncthreads();
    }
  }
  const uint32_t T = prefix;   // key of the last kept candidate
  // contiguous ownership for index-order scans
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  int ties = 0;
  if (need > 0)
    for (int i = b0; i < b1; ++i) ties += (s_state[i] == ST_CAND && s_key[i] == T);
  int tot;
  int tie_rank = block_excl_scan<kSelThreads>(ties, s_red, &tot);
  int kept = 0;
  {
    int tr = tie_rank;
    for (int i = b0; i < b1; ++i) {
      const uint8_t st = s_state[i];
      bool keep = st == ST_FORCED;
      if (st == ST_CAND && need > 0) {
        const uint32_t key = s_key[i];
        keep = key > T || (key == T && tr < rem);
        tr += (key == T);
      }
      kept += keep;
    }
  }
  int pos = block_excl_scan<kSelThreads>(kept, s_red, &tot);
  {
    int tr = tie_rank;
    for (int i = b0; i < b1; ++i) {
      const uint8_t st = s_state[i];
      bool keep = st == ST_FORCED;
      if (st == ST_CAND && need > 0) {
        const uint32_t key = s_key[i];
        keep = key > T || (key == T && tr < rem);
        tr += (key == T);
      }
      if (keep) idx[pos++] = i;
    }
  }
}

// One CTA: prepare the vector (norm / swiglu / as is) and optionally rank it.
__global__ void __launch_bounds__(kSelThreads, 1) k_select(SelectArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* s_key = reinterpret_cast<uint32_t*>(smem);
  uint8_t* s_state = reinterpret_cast<uint8_t*>(smem + sizeof(uint32_t) * kMaxSelect);
  __shared__ int s_hist[2048];
  __shared__ int s_red[32];
  __shared__ float s_redf[32];
  const int tid = threadIdx.x, n = a.n;

  pdl_wait();
  pdl_trigger();
  float scale = 1.f;
  if (a.prep == PREP_NORM || a.prep == PREP_EMBED_NORM) {
    float ss = 0.f;
    for (int i = tid; i < n; i += kSelThreads) {
      float xv;
      if (a.prep == PREP_EMBED_NORM) {
        xv = bf16f(a.embed_row[i]);
        a.x_out[i] = xv;
      } else {
        xv = a.v[i];
      }
      ss = fmaf(xv, xv, ss);
    }
    ss = block_sum<kSelThreads>(ss, s_redf);
    scale = 1.0f / sqrtf(ss / (float)n + a.eps);
  }
  for (int i = tid; i < n; i += kSelThreads) {
    float o;
    if (a.prep == PREP_NORM) {
      o = a.v[i] * scale * bf16f(a.gain[i]);
    } else if (a.prep == PREP_EMBED_NORM) {
      o = bf16f(a.embed_row[i]) * scale * bf16f(a.gain[i]);
    } else if (a.prep == PREP_SWIGLU) {
      const float g = a.v[i], u = a.v[n + i];
      o = g / (1.0f + expf(-g)) * u;
    } else {
      o = a.v[i];
    }
    if (a.out) a.out[i] = o;
    if (a.do_select) {
      s_key[i] = __float_as_uint(fabsf(o));
      s_state[i] = ST_CAND;
    }
  }
  if (!a.do_select) return;
  __syncthreads();
  topk_write(s_key, s_state, n, a.k, s_hist, s_red, a.idx);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)kMaxSelect * (sizeof(uint32_t) + sizeof(uint8_t));
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = a.do_select ? smem : 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_select, a);
}

// ------------------------------------------------------------------ page scores
// A group of hd/8 lanes scores one page: each lane holds 8 channels of the
// group's G queries and reads 16 bytes of kmin and 16 bytes of kmax.
template <int HD>
__global__ void __launch_bounds__(256) k_page_scores(PageScoreArgs a) {
  constexpr int LPP = HD / 8;          // lanes per page
  constexpr int PPW = 32 / LPP;        // pages per warp step
  const int h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPP, cl = lane % LPP;
  pdl_wait();
  pdl_trigger();
  float qv[8][8];   // [head][channel], G <= 8
  #pragma unroll
  for (int g = 0; g < 8; ++g)
    #pragma unroll
    for (int j = 0; j < 8; ++j)
      qv[g][j] = (g < a.G) ? a.q[(size_t)(h * a.G + g) * HD + cl * 8 + j] : 0.f;
  const int pages_per_cta = 8 * PPW * 4;
  const int p_begin = blockIdx.x * pages_per_cta;
  const int p_end = min(a.P, p_begin + pages_per_cta);
  const __nv_bfloat16* mbase = a.meta + (size_t)h * a.Pmax * 2 * HD;
  // warp-uniform loop: every lane takes part in the shuffles
  for (int pb = p_begin + warp * PPW; pb < p_end; pb += 8 * PPW) {
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
    if (valid && cl == 0) a.scores[(size_t)h * a.Pmax + p] = best;
  }
}

cudaError_t launch_page_scores(const PageScoreArgs& a, cudaStream_t st, bool pdl) {
  const int ppw = 32 / (a.hd / 8);
  const int pages_per_cta = 8 * ppw * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.P + pages_per_cta - 1) / pages_per_cta, a.Hkv);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (a.hd == 128) return cudaLaunchKernelEx(&cfg, k_page_scores<128>, a);
  if (a.hd == 64) return cudaLaunchKernelEx(&cfg, k_page_scores<64>, a);
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ page select
__global__ void __launch_bounds__(kSelThreads, 1) k_page_select(PageSelectArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* s_key = reinterpret_cast<uint32_t*>(smem);
  uint8_t* s_state = reinterpret_cast<uint8_t*>(smem + sizeof(uint32_t) * kMaxSelect);
  __shared__ int s_hist[2048];
  __shared__ int s_red[32];
  const int h = blockIdx.x, tid = threadIdx.x, P = a.P;
  pdl_wait();
  pdl_trigger();
  const int sink_end = min(a.sinks, P), rec_begin = max(P - a.recent, 0);
  int forced = 0;
  for (int p = tid; p < P; p += kSelThreads) {
    const bool f = p < sink_end || p >= rec_begin;
    s_state[p] = f ? ST_FORCED : ST_CAND;
    s_key[p] = float_order_key(a.scores[(size_t)h * a.Pmax + p]);
    forced += f;
  }
  __syncthreads();
  const int n_forced = sink_end + (P - max(rec_begin, sink_end));
  topk_write(s_key, s_state, P, a.K - n_forced, s_hist, s_red, a.pages + (size_t)h * a.Pmax);
  (void)forced;
}

cudaError_t launch_page_select(const PageSelectArgs& a, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)kMaxSelect * (sizeof(uint32_t) + sizeof(uint8_t));
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_page_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.Hkv);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_page_select, a);
}

}  // namespace bc
