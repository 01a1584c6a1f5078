// Device helpers shared by the decode-step kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace bc {

constexpr int kPage = 16;          // tokens per KV page
constexpr int kColTile = 256;      // GEMV output columns per CTA tile (8 per lane)
constexpr int kSelThreads = 1024;  // threads of a selection CTA
constexpr int kMaxSelect = 16384;  // largest vector a selection CTA ranks
constexpr int kMaxSplits = 128;    // split-K attention partials per head

// ---------------------------------------------------------------- programmatic dependent launch
// Every kernel waits for its predecessor grid before touching memory that
// grid wrote, and lets its dependent launch early.  Waiting unconditionally
// at the start keeps the dependency transitive along the whole chain.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- bf16
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ float bf16f(__nv_bfloat16 b) { return __bfloat162float(b); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// D += A * B on the tensor cores, m16n8k16, bf16 inputs, fp32 accumulate
// (A row-major 16x16 in four registers, B column-major 16x8 in two).
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// hi/lo bf16 split of two floats: hi = (bf16(x0), bf16(x1)), lo = residues.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
  hi = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
  lo = pack_bf16x2(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
}

// Streaming 16-byte load of data read once per step (weights, KV pages).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// ---------------------------------------------------------------- mbarriers
// Spin limit of an mbarrier wait (each try_wait also suspends in hardware for
// a while): far beyond any copy's or MMA's latency, so reaching it means an
// error, which the caller records before giving up.
constexpr int kMbarSpinLimit = 1 << 22;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Waits until the barrier's phase of the given parity has completed; false
// after kMbarSpinLimit tries.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (int i = 0; i < kMbarSpinLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// L2-coherent load of data another CTA of the same grid wrote.
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }

// Monotone map of a float to uint32: a > b  <=>  key(a) > key(b).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- block reductions
template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (w == 0) {
    t = (l < NT / 32) ? red[l] : 0.f;
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (l == 0) red[0] = t;
  }
  __syncthreads();
  t = red[0];
  __syncthreads();
  return t;
}

// Exclusive prefix sum over the block (thread order) of one int per thread.
// Returns the exclusive prefix; *total receives the block total.
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* red, int* total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  int x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (l >= o) x += y;
  }
  if (l == 31) red[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = (l < NT / 32) ? red[l] : 0;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (l >= o) t += y;
    }
    if (l < NT / 32) red[l] = t;   // inclusive warp totals
  }
  __syncthreads();
  const int before = (w > 0) ? red[w - 1] : 0;
  *total = red[NT / 32 - 1];
  __syncthreads();
  return before + x - v;
}

}  // namespace bc
