// Exact top-k inside one CTA, shared by the selection kernels and the GEMV
// that ranks its own input.
//
// Keys are 32-bit order keys.  The cut is found by an interval search that
// splits the candidates' key range into 256 bins per pass.  Only the first
// pass sweeps every key; the keys of the boundary bin are gathered into
// shared memory and the remaining passes (at most four) run on them.
// Placement then walks the vector in index order, a warp per contiguous
// segment and 32 elements per ballot: an element is kept when it is forced,
// its key lies above the cut interval, or it is among the first `rem` keys
// inside the interval by index.  Its slot in the ascending output is the
// number of kept elements before it, so ties at the cut go to the lower
// indices and the list comes out ascending.
#pragma once

#include "common.cuh"

namespace bc {

enum : uint8_t { ST_OUT = 0, ST_CAND = 1, ST_FORCED = 2 };

constexpr int kCandCap = 2048;   // boundary-bin candidates kept in shared memory

template <int NT>
struct TopkSmem {
  int hist[256];
  int red[32];
  int wtot[2][32];
  uint32_t rmin[32], rmax[32];
  uint32_t cand_key[kCandCap];
  int cand_n;
  uint32_t bin;
  int above, cnt;
};

// One pass of the interval search over `m` keys: counts them into at most 256
// equal power-of-two-wide bins of [base, base + span_m1] and finds the bin
// where the count from the top reaches rem.  Narrows the interval to that
// bin, lowers rem by the keys above it and returns the bin's count.  All NT
// threads call it.
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

// The cut of the `need` best candidates (by key, higher first) of [0, n):
// on return every candidate key above [base, base + span_m1] is kept, every
// one below it dropped, and the first `rem` inside it (by index) are kept.
// All NT threads call it, each with the min and max key of the candidates it
// saw (lo/hi; the block combines them), and sm.hist zeroed.
//
// Starting from the candidates' [min, max] spreads keys over the bins however
// their exponents cluster; each pass shrinks the interval 256-fold until one
// key value is left or the boundary bin is kept whole.
template <int NT, typename KeyF, typename StateF>
__device__ void topk_cut(int n, int need, KeyF key, StateF state, TopkSmem<NT>& sm, uint32_t lo, uint32_t hi,
                         uint32_t& base, uint32_t& span_m1, int& rem) {
  static_assert(NT >= 256 && NT % 32 == 0 && NT <= 1024, "block shape");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  base = 0;
  span_m1 = 0xFFFFFFFFu;
  rem = need;
  if (need <= 0) return;
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
  const int cnt = span_m1 > 0 ? interval_pass<NT>(n, full, base, span_m1, rem, sm) : 0;
  if (span_m1 == 0 || cnt == rem) return;
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

// Places the kept elements of [0, n) given the cut: emit(slot, index) is
// called once per kept element, slot = its rank in the ascending list.  Warp
// w walks the w-th contiguous segment of the vector 32 elements at a time.
// All NT threads call it.
template <int NT, typename KeyF, typename StateF, typename EmitF>
__device__ void topk_place(int n, int need, uint32_t base, uint32_t span_m1, int rem, KeyF key, StateF state,
                           EmitF emit, TopkSmem<NT>& sm) {
  constexpr int NW = NT / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t top = base + span_m1;            // inclusive upper end
  const int seg = ((n + NW * 32 - 1) / (NW * 32)) * 32;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  auto flags = [&](int i, bool& gt, bool& eq) {
    gt = false;
    eq = false;
    if (i >= s1) return;
    const uint8_t st = state(i);
    if (st == ST_FORCED) {
      gt = true;
    } else if (st == ST_CAND && need > 0) {
      const uint32_t kk = key(i);
      gt = kk > top;
      eq = kk >= base && kk <= top;
    }
  };
  int gt_w = 0, eq_w = 0;
  for (int c = s0; c < s1; c += 32) {
    bool g, e;
    flags(c + lane, g, e);
    gt_w += __popc(__ballot_sync(0xffffffffu, g));
    eq_w += __popc(__ballot_sync(0xffffffffu, e));
  }
  if (lane == 0) {
    sm.wtot[0][warp] = gt_w;
    sm.wtot[1][warp] = eq_w;
  }
  __syncthreads();
  int gt_b = 0, eq_b = 0;
  for (int w = 0; w < warp; ++w) {
    gt_b += sm.wtot[0][w];
    eq_b += sm.wtot[1][w];
  }
  const unsigned lt = (1u << lane) - 1u;
  for (int c = s0; c < s1; c += 32) {
    bool g, e;
    flags(c + lane, g, e);
    const unsigned gm = __ballot_sync(0xffffffffu, g), em = __ballot_sync(0xffffffffu, e);
    const int gb = gt_b + __popc(gm & lt), eb = eq_b + __popc(em & lt);
    if (g || (e && eb < rem)) emit(gb + min(eb, rem), c + lane);
    gt_b += __popc(gm);
    eq_b += __popc(em);
  }
}

// Writes the forced elements and the `need` best candidates of [0, n) (ties
// to the lower index) to out, ascending.
template <int NT, typename KeyF, typename StateF>
__device__ void radix_topk(int n, int need, KeyF key, StateF state, int* out, TopkSmem<NT>& sm,
                           uint32_t lo, uint32_t hi) {
  uint32_t base, span_m1;
  int rem;
  topk_cut<NT>(n, need, key, state, sm, lo, hi, base, span_m1, rem);
  topk_place<NT>(n, need, base, span_m1, rem, key, state, [&](int slot, int i) { out[slot] = i; }, sm);
}

}  // namespace bc
