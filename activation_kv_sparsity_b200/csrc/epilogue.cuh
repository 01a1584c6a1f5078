// The q/k/v epilogue shared by the batch-1 GEMV and the batched step.
#pragma once

#include "common.cuh"
#include "kernels.h"

#include <math.h>

namespace bc {

// What the epilogue of one column needs that does not depend on the GEMV:
// the rotation (cos, sin) of a q or k column, and for a k column the bounds
// of the page's earlier keys (already in the pool).  Computed by the GEMV
// before it waits for its input, so the double-precision angle and the loads
// overlap the weight stream.
struct QkvPre {
  float c, s;          // rotation of this column's pair
  float mn, mx;        // k columns: min / max over the page's earlier slots (+-inf if none)
};

__device__ __forceinline__ QkvPre qkv_prologue(const QkvEpilogue& e, int col) {
  QkvPre p{1.f, 0.f, INFINITY, -INFINITY};
  const int hd = e.hd, half = hd >> 1;
  const int i = col % hd;
  const int qcols = e.Hq * hd, kcols = e.Hkv * hd;
  if (col >= qcols + kcols) return p;
  const int j = (i < half) ? i : i - half;
  // angle pos * theta^(-2j/hd) in double, then the rotation in fp32
  const double inv = exp(-(2.0 * j / hd) * log((double)e.rope_theta));
  double sn, cs;
  sincos((double)e.pos * inv, &sn, &cs);
  p.c = (float)cs;
  p.s = (float)sn;
  if (col >= qcols) {
    const int head = (col - qcols) / hd;
    const int page = e.pos / kPage, slot = e.pos % kPage;
    const __nv_bfloat16* pg = e.kv_layer + ((size_t)head * e.Pmax + page) * (2 * kPage * hd);
    #pragma unroll
    for (int t = 0; t < kPage - 1; ++t) {
      if (t < slot) {
        const float kt = __bfloat162float(pg[t * hd + i]);
        p.mn = fminf(p.mn, kt);
        p.mx = fmaxf(p.mx, kt);
      }
    }
  }
  return p;
}

// Rotary embedding, bf16 append and key-bound refresh for one TW-column tile
// of the q/k/v output (v = this thread's column, pre its qkv_prologue).
// Heads never straddle a tile (TW is a multiple of hd).  All threads pass
// the one barrier; threads past the tile's width do nothing else.
template <int TW>
__device__ void qkv_epilogue(const QkvEpilogue& e, int col0, float v, float* s_v, const QkvPre& pre) {
  const int tid = threadIdx.x;
  const int col = col0 + tid;
  if (tid < TW) s_v[tid] = v;
  __syncthreads();
  if (tid >= TW) return;
  const int hd = e.hd, half = hd >> 1;
  const int i = col % hd;
  const int qcols = e.Hq * hd, kcols = e.Hkv * hd;
  const bool is_v = col >= qcols + kcols;
  float out = v;
  if (!is_v) {
    const int partner = (i < half) ? tid + half : tid - half;
    const float x1 = (i < half) ? v : s_v[partner];
    const float x2 = (i < half) ? s_v[partner] : v;
    out = (i < half) ? (x1 * pre.c - x2 * pre.s) : (x2 * pre.c + x1 * pre.s);
  }
  if (col < qcols) {
    e.q_out[col] = out;
  } else {
    const int head = is_v ? (col - qcols - kcols) / hd : (col - qcols) / hd;
    const int page = e.pos / kPage, slot = e.pos % kPage;
    __nv_bfloat16* pg = e.kv_layer + ((size_t)head * e.Pmax + page) * (2 * kPage * hd);
    const __nv_bfloat16 b = __float2bfloat16_rn(out);
    if (is_v) {
      pg[kPage * hd + slot * hd + i] = b;
    } else {
      pg[slot * hd + i] = b;
      // bounds over the page's valid keys: the earlier slots, then this one
      const float kb = __bfloat162float(b);
      __nv_bfloat16* mt = e.meta_layer + ((size_t)head * e.Pmax + page) * (2 * hd);
      mt[i] = __float2bfloat16_rn(fminf(pre.mn, kb));
      mt[hd + i] = __float2bfloat16_rn(fmaxf(pre.mx, kb));
    }
  }
}

}  // namespace bc
