// Bulk KV append (the synthetic stand-in for a dense prefill) and the dense
// LM head.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace bc {

// ------------------------------------------------------------------ bulk append
// Copies n_new tokens of keys and values into their pages, 16 bytes a thread.
__global__ void __launch_bounds__(256) k_kv_copy(KvAppendArgs a) {
  const int lh = blockIdx.y;                       // layer * Hkv + head
  const int vec_per_tok = a.hd / 8;
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (e >= (long long)a.n_new * vec_per_tok) return;
  const int tok = (int)(e / vec_per_tok), part = (int)(e % vec_per_tok);
  const int pos = a.n0 + tok, page = pos / kPage, slot = pos % kPage;
  const size_t src = ((size_t)lh * a.n_new + tok) * a.hd + part * 8;
  const size_t dst = (((size_t)lh * a.Pmax + page) * 2 * kPage + slot) * a.hd + part * 8;
  *reinterpret_cast<uint4*>(a.pool + dst) = *reinterpret_cast<const uint4*>(a.k + src);
  *reinterpret_cast<uint4*>(a.pool + dst + kPage * a.hd) = *reinterpret_cast<const uint4*>(a.v + src);
}

// Recomputes the key bounds of every page the append touched.
__global__ void k_kv_bounds(KvAppendArgs a) {
  const int lh = blockIdx.y;
  const int page = a.n0 / kPage + blockIdx.x;
  const int c = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int n_tok = a.n0 + a.n_new;
  const int valid = min(kPage, n_tok - page * kPage);
  const __nv_bfloat16* pk = a.pool + ((size_t)lh * a.Pmax + page) * 2 * kPage * a.hd;
  float mn = INFINITY, mx = -INFINITY;
  for (int t = 0; t < valid; ++t) {
    const float v = __bfloat162float(pk[t * a.hd + c]);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  __nv_bfloat16* mt = a.meta + ((size_t)lh * a.Pmax + page) * 2 * a.hd;
  mt[c] = __float2bfloat16_rn(mn);
  mt[a.hd + c] = __float2bfloat16_rn(mx);
}

static cudaLaunchConfig_t make_cfg(dim3 g, dim3 b, size_t smem, cudaStream_t st, bool pdl,
                                   cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = g;
  cfg.blockDim = b;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cfg;
}

cudaError_t launch_kv_append(const KvAppendArgs& a, cudaStream_t st, bool pdl) {
  if (a.n_new <= 0) return cudaSuccess;
  cudaLaunchAttribute attr[1];
  const long long vecs = (long long)a.n_new * (a.hd / 8);
  cudaLaunchConfig_t c1 = make_cfg(dim3((unsigned)((vecs + 255) / 256), a.L * a.Hkv), dim3(256), 0, st, pdl, attr);
  cudaError_t e = cudaLaunchKernelEx(&c1, k_kv_copy, a);
  if (e != cudaSuccess) return e;
  const int p0 = a.n0 / kPage, p1 = (a.n0 + a.n_new - 1) / kPage;
  cudaLaunchConfig_t c2 = make_cfg(dim3(p1 - p0 + 1, a.L * a.Hkv), dim3(a.hd), 0, st, pdl, attr);
  return cudaLaunchKernelEx(&c2, k_kv_bounds, a);
}

// ------------------------------------------------------------------ LM head
// logits[r] = s * W[r] . (x * g) with s = 1/sqrt(mean(x^2) + eps): the final
// RMSNorm folded in (its scale factors out of every dot product).  W is
// output-major [V][d].  Each warp streams two rows at a time, 16 bytes per
// lane per step; x*g sits in shared memory.
constexpr int kLmThreads = 256;

__global__ void __launch_bounds__(kLmThreads) k_lmhead(LmHeadArgs a) {
  extern __shared__ __align__(16) float s_x[];
  __shared__ float s_red[kLmThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31;
  pdl_wait();
  pdl_trigger();
  float ss = 0.f;
  for (int i = tid; i < a.d; i += kLmThreads) {
    const float xv = a.x[i];
    ss = fmaf(xv, xv, ss);
    s_x[i] = xv * bf16f(a.gain[i]);
  }
  const float scale = 1.0f / sqrtf(block_sum<kLmThreads>(ss, s_red) / (float)a.d + a.eps);
  const int warps = gridDim.x * (kLmThreads / 32);
  const int gw = blockIdx.x * (kLmThreads / 32) + (tid >> 5);
  const int vecs = a.d / 8;            // 16-byte vectors per row
  for (int r = gw * 2; r < a.V; r += warps * 2) {
    const bool two = r + 1 < a.V;
    const __nv_bfloat16* w0 = a.W + (size_t)r * a.d;
    const __nv_bfloat16* w1 = w0 + a.d;
    float s0 = 0.f, s1 = 0.f;
    for (int v = lane; v < vecs; v += 32 * 4) {
      uint4 x0[4], x1[4];
      #pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int vv = v + 32 * u;
        x0[u] = vv < vecs ? ld_stream(w0 + vv * 8) : make_uint4(0, 0, 0, 0);
        x1[u] = (two && vv < vecs) ? ld_stream(w1 + vv * 8) : make_uint4(0, 0, 0, 0);
      }
      #pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int vv = v + 32 * u;
        if (vv >= vecs) break;
        const float4 xa = *reinterpret_cast<const float4*>(&s_x[vv * 8]);
        const float4 xb = *reinterpret_cast<const float4*>(&s_x[vv * 8 + 4]);
        s0 = fmaf(xa.x, bf16_lo(x0[u].x), s0); s0 = fmaf(xa.y, bf16_hi(x0[u].x), s0);
        s0 = fmaf(xa.z, bf16_lo(x0[u].y), s0); s0 = fmaf(xa.w, bf16_hi(x0[u].y), s0);
        s0 = fmaf(xb.x, bf16_lo(x0[u].z), s0); s0 = fmaf(xb.y, bf16_hi(x0[u].z), s0);
        s0 = fmaf(xb.z, bf16_lo(x0[u].w), s0); s0 = fmaf(xb.w, bf16_hi(x0[u].w), s0);
        s1 = fmaf(xa.x, bf16_lo(x1[u].x), s1); s1 = fmaf(xa.y, bf16_hi(x1[u].x), s1);
        s1 = fmaf(xa.z, bf16_lo(x1[u].y), s1); s1 = fmaf(xa.w, bf16_hi(x1[u].y), s1);
        s1 = fmaf(xb.x, bf16_lo(x1[u].z), s1); s1 = fmaf(xb.y, bf16_hi(x1[u].z), s1);
        s1 = fmaf(xb.z, bf16_lo(x1[u].w), s1); s1 = fmaf(xb.w, bf16_hi(x1[u].w), s1);
      }
    }
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, o);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if (lane == 0) {
      a.logits[r] = s0 * scale;
      if (two) a.logits[r + 1] = s1 * scale;
    }
  }
}

cudaError_t launch_lmhead(const LmHeadArgs& a, int sms, cudaStream_t st, bool pdl) {
  cudaLaunchAttribute attr[1];
  const size_t smem = (size_t)a.d * sizeof(float);
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_lmhead, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int rows_per_cta = 2 * (kLmThreads / 32);
  const int ctas = std::min(4 * sms, (a.V + rows_per_cta - 1) / rows_per_cta);
  cudaLaunchConfig_t c = make_cfg(dim3(ctas), dim3(kLmThreads), smem, st, pdl, attr);
  return cudaLaunchKernelEx(&c, k_lmhead, a);
}

}  // namespace bc
