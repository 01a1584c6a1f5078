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
// From 7 sequences k_gemv_batch_tc<B> replaces k_gemv_batch<B>: the same
// runs and outputs with the multiplies on the tensor cores (below).
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

// ------------------------------------------------------------------ tensor-core variant
// The same projection with the multiplies on the tensor cores (mma.sync
// m16n8k16, bf16 in, fp32 accumulate): output columns are M, the batch
// (padded to 8) is N, the union rows are K.  Row segments of 32 union rows
// (512 bytes each, padded to 528 so that an 8-row ldmatrix touches every
// bank once) stream through a 4-stage shared-memory ring by 16-byte
// cp.async, one commit group (and one barrier) per stage; ldmatrix.trans
// turns a 16 x 16 block of a stage (rows c, columns j) into the A fragment
// W^T.  The inputs, split
// into three bf16 parts (about 24 bits of the fp32 value), are the B
// fragments: three MMAs per block.  Warp w owns output columns 32w .. 32w+31
// (two 16-column blocks) of the tile for every row, so no reduction across
// warps is needed.  With B x 8 FMAs per 16 weight bytes the CUDA-core
// version is bound by its FMAs at large B; here the bytes set the time.
constexpr int kTcbStages = 4;
constexpr int kTcbRows = 32;                                // rows per stage: two MMA k-blocks of 16
constexpr int kTcbRowBytes = kBatchCols * 2 + 16;           // a 512-byte row segment + 16 bytes of pad
constexpr int kTcbStageBytes = kTcbRows * kTcbRowBytes;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// Three bf16 parts of two floats (hi, mid, lo), each pair packed low/high.
__device__ __forceinline__ void split3(float x0, float x1, uint32_t (&p)[3]) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
  const float r0 = x0 - __bfloat162float(h0), r1 = x1 - __bfloat162float(h1);
  const __nv_bfloat16 m0 = __float2bfloat16_rn(r0), m1 = __float2bfloat16_rn(r1);
  p[0] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
  p[1] = (uint32_t)__bfloat16_as_ushort(m0) | ((uint32_t)__bfloat16_as_ushort(m1) << 16);
  p[2] = pack_bf16x2(r0 - __bfloat162float(m0), r1 - __bfloat162float(m1));
}

__host__ __device__ constexpr size_t tcb_ring_offset(int B) {
  return ((size_t)kBatchRunCap * (4 + 4 * B) + 127) & ~(size_t)127;
}

template <int B>
__global__ void __launch_bounds__(kBatchThreads, 2) k_gemv_batch_tc(BatchGemvArgs a) {
  extern __shared__ __align__(16) unsigned char s_dyn[];
  int* s_id = reinterpret_cast<int*>(s_dyn);                          // [kBatchRunCap]
  float* s_x = reinterpret_cast<float*>(s_dyn + 4 * kBatchRunCap);    // [kBatchRunCap][B]
  const uint32_t ring = smem_addr(s_dyn + tcb_ring_offset(B));        // [stages][16 rows][528 B]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, run = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int n = *a.n_union;
  const int r0 = (int)((long long)run * n / a.S), r1 = (int)((long long)(run + 1) * n / a.S);
  const int len = r1 - r0;                      // <= kBatchRunCap: S is planned for it
  #pragma unroll 4
  for (int i = tid; i < len * B; i += kBatchThreads) {
    const int row = i / B, b = i - row * B;
    const uint32_t e = (uint32_t)__ldg(a.ulist + r0 + row);
    const int c = (int)(e & 0xFFFFu);
    if (b == 0) s_id[row] = c;
    s_x[i] = ((e >> (16 + b)) & 1u) ? __ldg(a.x + (size_t)b * a.d_in + c) : 0.f;
  }
  __syncthreads();
  const int nblk = (len + kTcbRows - 1) / kTcbRows;
  const __nv_bfloat16* Wt = a.W + (size_t)tile * kBatchCols;
  // a stage is 32 rows x 32 chunks of 16 bytes: thread t copies chunks t + 256h, h < 4
  auto issue = [&](int blk) {
    if (blk < nblk) {
      const uint32_t dst = ring + (uint32_t)((blk % kTcbStages) * kTcbStageBytes);
      #pragma unroll
      for (int h = 0; h < kTcbRows * 32 / kBatchThreads; ++h) {
        const int q = tid + h * kBatchThreads, row = q >> 5, part = q & 31;
        const int r = blk * kTcbRows + row;
        const bool ok = r < len;                  // rows past the run are zero-filled
        const __nv_bfloat16* src = Wt + (size_t)s_id[ok ? r : 0] * a.d_out + part * 8;
        cp_async16(dst + row * kTcbRowBytes + part * 16, src, ok ? 16 : 0);
      }
    }
    cp_async_commit();                            // one group per stage, empty past the run
  };
  #pragma unroll
  for (int s = 0; s < kTcbStages - 1; ++s) issue(s);
  float d[2][4];
  #pragma unroll
  for (int mb = 0; mb < 2; ++mb)
    #pragma unroll
    for (int j = 0; j < 4; ++j) d[mb][j] = 0.f;
  const int g = lane >> 2, t = lane & 3;
  // ldmatrix row address of this lane: matrix q = lane / 8 (k half q / 2,
  // column half q % 2), row lane % 8
  const int lq = lane >> 3, lr = lane & 7;
  const uint32_t lane_off = (uint32_t)(((lq >> 1) * 8 + lr) * kTcbRowBytes + ((lq & 1) * 8 + warp * 32) * 2);
  for (int blk = 0; blk < nblk; ++blk) {
    cp_async_wait<kTcbStages - 2>();              // this thread's copies of blk have landed
    __syncthreads();                              // everyone's; every warp is done with blk - 1
    issue(blk + kTcbStages - 1);                  // into blk - 1's slot
    const uint32_t st = ring + (uint32_t)((blk % kTcbStages) * kTcbStageBytes);
    #pragma unroll
    for (int kb = 0; kb < kTcbRows / 16; ++kb) {
      // B fragments: input g (the batch) at rows 2t, 2t+1 and 2t+8, 2t+9 of the k-block
      float xv[4] = {0.f, 0.f, 0.f, 0.f};
      if (g < B) {
        const int rb = blk * kTcbRows + kb * 16;
        const int rr[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          if (rb + rr[i] < len) xv[i] = s_x[(rb + rr[i]) * B + g];
      }
      uint32_t b0[3], b1[3];
      split3(xv[0], xv[1], b0);
      split3(xv[2], xv[3], b1);
      #pragma unroll
      for (int mb = 0; mb < 2; ++mb) {
        uint32_t A[4];
        ldmatrix_x4_trans(A, st + kb * 16 * kTcbRowBytes + lane_off + mb * 32);
        #pragma unroll
        for (int p = 0; p < 3; ++p) mma16816(d[mb], A, b0[p], b1[p]);
      }
    }
  }
  cp_async_wait<0>();
  // thread (g, t) holds D[column g and g + 8 of each block][inputs 2t, 2t + 1]
  float* out = a.S == 1 ? a.y : a.partial + (size_t)run * B * a.d_out;
  #pragma unroll
  for (int mb = 0; mb < 2; ++mb) {
    const size_t col = (size_t)tile * kBatchCols + (2 * warp + mb) * 16 + g;
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int b = 2 * t + j;
      if (b < B) {
        out[(size_t)b * a.d_out + col] = d[mb][j];
        out[(size_t)b * a.d_out + col + 8] = d[mb][2 + j];
      }
    }
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

// From 7 sequences the CUDA-core kernel is bound by its B x 8 FMAs per 16
// weight bytes and the tensor-core kernel is faster (gate/up of one layer,
// union of the sequences' halves: 81.3 / 80.4 us against 84.2 / 87.2 us at
// B = 7 / 8; 77.5 against 77.2 at 6; below that the register-streaming
// kernel wins, 38.0 against 50.5 us at 1).
constexpr int kBatchTensorCoreMin = 7;

template <int B>
static cudaError_t launch_b(const cudaLaunchConfig_t& base, const BatchGemvArgs& a) {
  cudaLaunchConfig_t c = base;
  c.gridDim = dim3(a.d_out / kBatchCols, a.S);
  c.blockDim = dim3(kBatchThreads);
  if constexpr (B >= kBatchTensorCoreMin) {
    static bool attr = false;
    const size_t smem = tcb_ring_offset(B) + (size_t)kTcbStages * kTcbStageBytes;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(k_gemv_batch_tc<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    c.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&c, k_gemv_batch_tc<B>, a);
  } else {
    c.dynamicSmemBytes = (size_t)kBatchRunCap * (4 + 4 * B);
    return cudaLaunchKernelEx(&c, k_gemv_batch<B>, a);
  }
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
