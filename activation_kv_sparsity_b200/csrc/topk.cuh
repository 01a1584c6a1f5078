// Exact top-k of one vector inside one CTA, keys held in registers.
//
// Keys are 32-bit order keys.  Warp w owns the KPT*32 consecutive elements
// from w*KPT*32; lane l holds in kr[c] the key of element (w*KPT + c)*32 + l,
// so every load, ballot and store below is one coalesced row of 32 elements.
//
// The cut is found by an interval search: a pass counts the keys inside the
// current interval [base, base + span] into 256 equal power-of-two-wide
// bins and keeps the bin where the count from the top reaches the number
// still needed; the interval shrinks 256-fold per pass, starting from the
// keys' [min, max], until one key value is left or the boundary bin is kept
// whole.  A pass costs one barrier: every warp reads the finished histogram
// and finds the bin itself, and three histograms rotate so that the one
// being cleared is never the one being counted into or read.
//
// Placement walks the elements in index order: an element is kept when its
// key lies above the interval, or it is among the first `rem` keys inside it
// by index; its slot in the ascending output is the number of kept elements
// before it (ballots within a warp, a masked sum across warps), so ties at
// the cut go to the lower indices and the list comes out ascending.
#pragma once

#include "common.cuh"

namespace bc {

enum : uint8_t { ST_OUT = 0, ST_CAND = 1, ST_FORCED = 2 };

// Block-wide min of lo and max of hi, returned to every thread (one barrier;
// warp reductions in hardware).
template <int NT>
__device__ __forceinline__ void block_minmax(uint32_t& lo, uint32_t& hi, uint32_t* rmin, uint32_t* rmax) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    rmin[warp] = lo;
    rmax[warp] = hi;
  }
  __syncthreads();
  lo = __reduce_min_sync(0xffffffffu, lane < NT / 32 ? rmin[lane] : 0xFFFFFFFFu);
  hi = __reduce_max_sync(0xffffffffu, lane < NT / 32 ? rmax[lane] : 0u);
}

// Within one warp: the bin of a 256-bin histogram H (16-byte aligned) where
// the count from the top reaches rem (1 <= rem <= total), the count above
// that bin and the bin's own count, returned to every lane.  Lane l reads
// its 8 bins 255-8l .. 248-8l as two 16-byte loads: the warp's loads are
// conflict-free, which matters because every warp of the block runs this.
__device__ __forceinline__ void warp_find_bin(const int* H, int rem, int& bin, int& above, int& cnt) {
  const int lane = threadIdx.x & 31;
  const int4* H4 = reinterpret_cast<const int4*>(H) + 2 * (31 - lane);
  const int4 v0 = H4[0], v1 = H4[1];             // bins 248-8l .. 251-8l, 252-8l .. 255-8l
  const int c[8] = {v1.w, v1.z, v1.y, v1.x, v0.w, v0.z, v0.y, v0.x};
  int sum = 0;
  #pragma unroll
  for (int j = 0; j < 8; ++j) sum += c[j];
  int incl = sum;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int a = incl - sum, b = -1, ab = 0, cb = 0;
  #pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (a < rem && a + c[j] >= rem) {
      b = 255 - 8 * lane - j;
      ab = a;
      cb = c[j];
    }
    a += c[j];
  }
  const unsigned who = __ballot_sync(0xffffffffu, b >= 0);
  const int src = who ? __ffs(who) - 1 : 0;
  bin = __shfl_sync(0xffffffffu, b, src);
  above = __shfl_sync(0xffffffffu, ab, src);
  cnt = __shfl_sync(0xffffffffu, cb, src);
}

template <int NT>
struct RegTopkSmem {
  alignas(16) int hist[3][256];
  uint32_t rmin[32], rmax[32];
  int wtot[2][32];
};

// Writes the forced elements and the `need` candidates of largest key of
// [0, n) (ties to the lower index) to out, ascending.  n <= NT*KPT; kr as
// described above (entries of elements >= n are ignored); state(i) is
// ST_CAND, ST_FORCED (kept, not ranked) or ST_OUT.  All NT threads call it.
template <int NT, int KPT, typename StateF>
__device__ void reg_topk(const uint32_t (&kr)[KPT], int n, int need, StateF state, int* out,
                         RegTopkSmem<NT>& sm) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ibase = warp * KPT * 32 + lane;
  // the state of key c (recomputed where needed: fewer live registers)
  auto st = [&](int c) { return ibase + 32 * c < n ? state(ibase + 32 * c) : (uint8_t)ST_OUT; };
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  #pragma unroll
  for (int c = 0; c < KPT; ++c)
    if (st(c) == ST_CAND) {
      lo = min(lo, kr[c]);
      hi = max(hi, kr[c]);
    }
  for (int j = tid; j < 2 * 256; j += NT) (&sm.hist[0][0])[j] = 0;
  block_minmax<NT>(lo, hi, sm.rmin, sm.rmax);      // its barrier also orders the clearing
  uint32_t base = lo, span = hi - lo;
  int rem = need;
  if (need <= 0) span = 0;
  #pragma unroll 1
  for (int pass = 0; pass < 5 && span > 0; ++pass) {
    int* H = sm.hist[pass % 3];
    const int sh = max(0, 24 - __clz(span));
    #pragma unroll
    for (int c = 0; c < KPT; ++c) {
      const uint32_t kk = kr[c];
      if (st(c) == ST_CAND && kk >= base && kk - base <= span) atomicAdd(&H[(kk - base) >> sh], 1);
    }
    __syncthreads();
    int bin, above, cnt;
    warp_find_bin(H, rem, bin, above, cnt);
    // the histogram of the previous pass: every warp read it before this
    // pass's barrier, and the pass after next counts into it
    int* Z = sm.hist[(pass + 2) % 3];
    for (int j = tid; j < 256; j += NT) Z[j] = 0;
    const uint32_t b_lo = (uint32_t)bin << sh;
    rem -= above;
    base += b_lo;
    span = min((1u << sh) - 1u, span - b_lo);
    if (cnt == rem) break;                          // the whole bin is kept
  }
  // placement: kept above the interval (gt) or inside it (eq), per row of 32
  const uint32_t top = base + span;
  auto rows = [&](int c, unsigned& gm, unsigned& em) {
    const uint8_t s = st(c);
    const bool in = need > 0 && s == ST_CAND;
    const uint32_t kk = kr[c];
    gm = __ballot_sync(0xffffffffu, s == ST_FORCED || (in && kk > top));
    em = __ballot_sync(0xffffffffu, in && kk >= base && kk <= top);
  };
  int gt_w = 0, eq_w = 0;
  #pragma unroll
  for (int c = 0; c < KPT; ++c) {
    unsigned gm, em;
    rows(c, gm, em);
    gt_w += __popc(gm);
    eq_w += __popc(em);
  }
  if (lane == 0) {
    sm.wtot[0][warp] = gt_w;
    sm.wtot[1][warp] = eq_w;
  }
  __syncthreads();
  // the warps before this one
  int gt_b = (int)__reduce_add_sync(0xffffffffu, lane < warp ? (unsigned)sm.wtot[0][lane] : 0u);
  int eq_b = (int)__reduce_add_sync(0xffffffffu, lane < warp ? (unsigned)sm.wtot[1][lane] : 0u);
  const unsigned lt = (1u << lane) - 1u, me = 1u << lane;
  #pragma unroll
  for (int c = 0; c < KPT; ++c) {
    unsigned gm, em;
    rows(c, gm, em);
    const int gb = gt_b + __popc(gm & lt), eb = eq_b + __popc(em & lt);
    if ((gm & me) || ((em & me) && eb < rem)) out[gb + min(eb, rem)] = ibase + 32 * c;
    gt_b += __popc(gm);
    eq_b += __popc(em);
  }
}

}  // namespace bc
