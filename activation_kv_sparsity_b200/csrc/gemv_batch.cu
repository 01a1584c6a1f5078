// Batched column-gathered GEMV over the union of the sequences' kept
// channels: the projection kernel of a batched decode step.
//
// Every sequence b keeps its own channel list S_b (its own top-k of |x_b|,
// as in the batch-1 step), so its projection is unchanged,
//
//   y[b][j] = sum over c in S_b of x[b][c] * W[c][j],
//
// while the batch reads each row of the union U = S_0 u ... u S_{B-1} once
// and applies it to all B inputs, masked to their own lists (ByteCross README,
// "Usage: The byte account": crossover_batch, where a batch reads the union
// of its kept projection weights once per step).
//
// Three launches, chained by programmatic dependent launch:
//   k_union         one CTA: marks every listed channel with its sequences'
//                   bits in shared memory and compacts the marked channels
//                   (ascending) into the union list, each entry the channel
//                   with its sequences' bits; |U| to device memory.
//   k_gemv_batch<B> a column tile of 256 outputs (8 per lane: one 16-byte
//                   load of a row segment) and a contiguous run of at most
//                   1024 union rows per CTA, cut from the device-side |U|
//                   (the grid is planned for the largest union,
//                   min(d_in, B*k), and to fill whole waves of 2 CTAs per
//                   SM).  The run's channel ids and inputs (0 where a
//                   sequence did not keep the row) are gathered into shared
//                   memory first, so a row's weight load waits on no global
//                   load; 8 warps, 16 row segments per lane in flight
//                   (8 for B > 4), B x 8 accumulators per lane; warps reduced
//                   in shared memory; a tile split over several runs writes
//                   one partial per run.
//   k_batch_reduce  sums the runs' partials in run order (deterministic);
//                   skipped when one run covers a tile.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace bc {

constexpr int kUnionThreads = 1024;
constexpr int kBatchWarps = 8;
constexpr int kBatchThreads = kBatchWarps * 32;
constexpr int kBatchRunCap = 1024;              // union rows per CTA run (staged in shared memory)
constexpr int kBatchCols = kBatchThreads;       // columns per tile: 8 per lane, one per thread in the reduction

__global__ void __launch_bounds__(kUnionThreads) k_union(BatchGemvArgs a) {
  extern __shared__ uint32_t s_mark[];          // [d_in]: bit b = kept by sequence b
  __shared__ int s_red[32];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const uint32_t all = (1u << a.B) - 1u;
  for (int c = tid; c < a.d_in; c += kUnionThreads) s_mark[c] = a.idx ? 0u : all;
  __syncthreads();
  if (a.idx) {
    // four independent list loads per thread in flight, then their marks
    const int total = a.B * a.k;
    for (int e0 = tid; e0 < total; e0 += 4 * kUnionThreads) {
      int c[4];
      #pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * kUnionThreads;
        c[u] = e < total ? a.idx[e] : -1;
      }
      #pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c[u] >= 0 && c[u] < a.d_in) atomicOr(&s_mark[c[u]], 1u << ((e0 + u * kUnionThreads) / a.k));
    }
    __syncthreads();
  }
  // thread t owns the contiguous channels [t*per, (t+1)*per): the union
  // comes out ascending; an entry packs the channel (low 16 bits) with its
  // sequences' bits (bits 16-23)
  const int per = (a.d_in + kUnionThreads - 1) / kUnionThreads;
  const int c0 = min(a.d_in, tid * per), c1 = min(a.d_in, c0 + per);
  int cnt = 0;
  for (int c = c0; c < c1; ++c) cnt += s_mark[c] != 0u;
  int total;
  int off = block_excl_scan<kUnionThreads>(cnt, s_red, &total);
  for (int c = c0; c < c1; ++c) {
    const uint32_t m = s_mark[c];
    if (m) a.ulist[off++] = (int)((uint32_t)c | (m << 16));
  }
  if (tid == 0) *a.n_union = total;
}

__device__ __forceinline__ void fma8b(float* acc, float xv, const uint4& w) {
  acc[0] = fmaf(xv, bf16_lo(w.x), acc[0]);
  acc[1] = fmaf(xv, bf16_hi(w.x), acc[1]);
  acc[2] = fmaf(xv, bf16_lo(w.y), acc[2]);
  acc[3] = fmaf(xv, bf16_hi(w.y), acc[3]);
  acc[4] = fmaf(xv, bf16_lo(w.z), acc[4]);
  acc[5] = fmaf(xv, bf16_hi(w.z), acc[5]);
  acc[6] = fmaf(xv, bf16_lo(w.w), acc[6]);
  acc[7] = fmaf(xv, bf16_hi(w.w), acc[7]);
}

// The B inputs of one union row from shared memory (rows start 4*B-byte
// aligned; every lane reads the same address: a broadcast).
template <int B>
__device__ __forceinline__ void load_inputs(const float* p, float* v) {
  if constexpr (B % 4 == 0) {
    #pragma unroll
    for (int i = 0; i < B; i += 4) {
      const float4 f = *reinterpret_cast<const float4*>(p + i);
      v[i] = f.x; v[i + 1] = f.y; v[i + 2] = f.z; v[i + 3] = f.w;
    }
  } else if constexpr (B % 2 == 0) {
    #pragma unroll
    for (int i = 0; i < B; i += 2) {
      const float2 f = *reinterpret_cast<const float2*>(p + i);
      v[i] = f.x; v[i + 1] = f.y;
    }
  } else {
    #pragma unroll
    for (int i = 0; i < B; ++i) v[i] = p[i];
  }
}

template <int B>
__global__ void __launch_bounds__(kBatchThreads, 2) k_gemv_batch(BatchGemvArgs a) {
  constexpr int KR = B > 4 ? 8 : 16;            // row segments per lane in flight
  __shared__ __align__(16) float s_red[kBatchWarps][kBatchCols];
  extern __shared__ __align__(16) unsigned char s_dyn[];
  int* s_id = reinterpret_cast<int*>(s_dyn);                          // [kBatchRunCap]
  float* s_x = reinterpret_cast<float*>(s_dyn + 4 * kBatchRunCap);    // [kBatchRunCap][B]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, run = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int n = *a.n_union;
  const int r0 = (int)((long long)run * n / a.S), r1 = (int)((long long)(run + 1) * n / a.S);
  const int len = r1 - r0;                      // <= kBatchRunCap: S is planned for it
  // the run's channel ids and masked inputs, gathered once per CTA
  #pragma unroll 4
  for (int i = tid; i < len * B; i += kBatchThreads) {
    const int row = i / B, b = i - row * B;
    const uint32_t e = (uint32_t)__ldg(a.ulist + r0 + row);
    const int c = (int)(e & 0xFFFFu);
    if (b == 0) s_id[row] = c;
    s_x[i] = ((e >> (16 + b)) & 1u) ? __ldg(a.x + (size_t)b * a.d_in + c) : 0.f;
  }
  __syncthreads();
  const __nv_bfloat16* Wc = a.W + (size_t)tile * kBatchCols + lane * 8;
  float acc[B][8];
  #pragma unroll
  for (int b = 0; b < B; ++b)
    #pragma unroll
    for (int j = 0; j < 8; ++j) acc[b][j] = 0.f;
  for (int r = warp; r < len; r += kBatchWarps * KR) {
    // all KR loads before the first FMA (rows past the run re-read its last
    // row and are not accumulated)
    uint4 w[KR];
    #pragma unroll
    for (int i = 0; i < KR; ++i) w[i] = ld_stream(Wc + (size_t)s_id[min(r + i * kBatchWarps, len - 1)] * a.d_out);
    #pragma unroll
    for (int i = 0; i < KR; ++i) {
      const int ri = r + i * kBatchWarps;
      if (ri < len) {
        float xv[B];
        load_inputs<B>(s_x + ri * B, xv);
        #pragma unroll
        for (int b = 0; b < B; ++b) fma8b(acc[b], xv[b], w[i]);
      }
    }
  }
  float* out = a.S == 1 ? a.y : a.partial + (size_t)run * B * a.d_out;
  #pragma unroll
  for (int b = 0; b < B; ++b) {
    float4* dst = reinterpret_cast<float4*>(&s_red[warp][lane * 8]);
    dst[0] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
    dst[1] = make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
    __syncthreads();
    float v = 0.f;
    #pragma unroll
    for (int w = 0; w < kBatchWarps; ++w) v += s_red[w][tid];
    out[(size_t)b * a.d_out + (size_t)tile * kBatchCols + tid] = v;
    __syncthreads();
  }
}

__global__ void k_batch_reduce(BatchGemvArgs a) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int n = a.B * a.d_out;
  if (e >= n) return;
  // four runs' partials in flight at a time, added in run order
  const float* p = a.partial + e;
  float v = 0.f;
  int s = 0;
  for (; s + 4 <= a.S; s += 4) {
    const float p0 = p[(size_t)s * n], p1 = p[(size_t)(s + 1) * n];
    const float p2 = p[(size_t)(s + 2) * n], p3 = p[(size_t)(s + 3) * n];
    v += p0;
    v += p1;
    v += p2;
    v += p3;
  }
  for (; s < a.S; ++s) v += p[(size_t)s * n];
  a.y[e] = v;
}

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

// Row runs per column tile: enough that a run fits the shared-memory stage,
// then the fewest that fill the 2-CTAs-per-SM slots to 90% in their last
// wave (or the best fill up to the cap).
int gemv_batch_splits(int d_in, int d_out, int k, int B, int sms) {
  const int tiles = d_out / kBatchCols;
  const int rows = std::min(d_in, B * k);
  const int s_min = std::max(1, (rows + kBatchRunCap - 1) / kBatchRunCap);
  const double slots = 2.0 * sms;
  int best = s_min;
  double best_fill = 0;
  for (int S = s_min; S <= kBatchMaxSplit; ++S) {
    const double waves = tiles * (double)S / slots;
    const double fill = waves / std::ceil(waves);
    if (fill >= 0.9) return S;
    if (fill > best_fill + 1e-9) {
      best_fill = fill;
      best = S;
    }
  }
  return best;
}

size_t gemv_batch_scratch(int d_in, int d_out, int B) {
  return al256(4ull * d_in) + 256 + al256(4ull * kBatchMaxSplit * B * d_out);
}

void gemv_batch_bind(BatchGemvArgs* a, void* scratch, int* n_union) {
  char* p = static_cast<char*>(scratch);
  a->ulist = reinterpret_cast<int*>(p);
  p += al256(4ull * a->d_in);
  a->n_union = n_union ? n_union : reinterpret_cast<int*>(p);
  p += 256;
  a->partial = reinterpret_cast<float*>(p);
}

template <int B>
static cudaError_t launch_b(const cudaLaunchConfig_t& base, const BatchGemvArgs& a) {
  cudaLaunchConfig_t c = base;
  c.gridDim = dim3(a.d_out / kBatchCols, a.S);
  c.blockDim = dim3(kBatchThreads);
  c.dynamicSmemBytes = (size_t)kBatchRunCap * (4 + 4 * B);
  return cudaLaunchKernelEx(&c, k_gemv_batch<B>, a);
}

cudaError_t launch_gemv_batch(const BatchGemvArgs& a, cudaStream_t st, bool pdl) {
  if (a.B < 1 || a.B > kBatchMax || a.d_in < 1 || a.d_in > kMaxSelect || a.k < 1 || a.k > a.d_in ||
      a.d_out < kBatchCols || a.d_out % kBatchCols || a.S < 1 || a.S > kBatchMaxSplit ||
      (std::min(a.d_in, a.B * a.k) + a.S - 1) / a.S > kBatchRunCap)
    return cudaErrorInvalidValue;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_union, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kMaxSelect * (int)sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kUnionThreads);
  cfg.dynamicSmemBytes = (size_t)a.d_in * sizeof(uint32_t);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_union, a);
  if (e != cudaSuccess) return e;
  switch (a.B) {
    case 1: e = launch_b<1>(cfg, a); break;
    case 2: e = launch_b<2>(cfg, a); break;
    case 3: e = launch_b<3>(cfg, a); break;
    case 4: e = launch_b<4>(cfg, a); break;
    case 5: e = launch_b<5>(cfg, a); break;
    case 6: e = launch_b<6>(cfg, a); break;
    case 7: e = launch_b<7>(cfg, a); break;
    default: e = launch_b<8>(cfg, a); break;
  }
  if (e != cudaSuccess || a.S == 1) return e;
  cudaLaunchConfig_t r = cfg;
  r.gridDim = dim3((a.B * a.d_out + 255) / 256);
  r.blockDim = dim3(256);
  r.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&r, k_batch_reduce, a);
}

}  // namespace bc
