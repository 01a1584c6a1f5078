// The q/k/v epilogue shared by the batch-1 GEMV and the batched step.
#pragma once

#include "common.cuh"
#include "kernels.h"

#include <math.h>

namespace bc {

// Rotary embedding, bf16 append and key-bound refresh for one TW-column tile
// of the q/k/v output (v = this thread's column).  Heads never straddle a
// tile (TW is a multiple of hd).  All threads pass the one barrier; threads
// past the tile's width do nothing else.
template <int TW>
__device__ void qkv_epilogue(const QkvEpilogue& e, int col0, float v, float* s_v) {
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
    const int j = (i < half) ? i : i - half;
    const int partner = (i < half) ? tid + half : tid - half;
    // angle pos * theta^(-2j/hd) in double, then the rotation in fp32
    const double inv = exp(-(2.0 * j / hd) * log((double)e.rope_theta));
    double sn, cs;
    sincos((double)e.pos * inv, &sn, &cs);
    const float c = (float)cs, s = (float)sn;
    const float x1 = (i < half) ? v : s_v[partner];
    const float x2 = (i < half) ? s_v[partner] : v;
    out = (i < half) ? (x1 * c - x2 * s) : (x2 * c + x1 * s);
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
      // bounds over the page's valid keys: earlier slots from the pool, this one
      float mn = __bfloat162float(b), mx = mn;
      #pragma unroll
      for (int t = 0; t < kPage - 1; ++t) {
        if (t < slot) {
          const float kt = __bfloat162float(pg[t * hd + i]);
          mn = fminf(mn, kt);
          mx = fmaxf(mx, kt);
        }
      }
      __nv_bfloat16* mt = e.meta_layer + ((size_t)head * e.Pmax + page) * (2 * hd);
      mt[i] = __float2bfloat16_rn(mn);
      mt[hd + i] = __float2bfloat16_rn(mx);
    }
  }
}

}  // namespace bc
