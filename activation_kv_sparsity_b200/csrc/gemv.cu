// Column-gathered bf16 GEMV with fp32 accumulation: the projection kernel of
// every decode mode.
//
//   y[j] = sum over listed input channels c of x[c] * W[c][j]
//
// W is input-channel-major ([d_in][d_out]), so each selected channel is one
// contiguous row and the activation-sparse projection (the ByteCross README's
// projection branch, "Timing and quality on a GPU") reads exactly the rows of
// the kept channels; dense mode is the same kernel over every row.
//
// Work split: CTA (tile, split) owns 256 output columns and a contiguous run
// of `chunk` listed rows.  Each of its 8 warps streams every 8th row of the
// run, one 16-byte vector per lane per row (512 contiguous bytes per warp and
// row), with 8 rows in flight per warp.  Warps are reduced in shared memory;
// splits are reduced by the last CTA of each column tile to arrive (an atomic
// ticket, no spinning), which sums the partials in split order -- the result
// is deterministic -- and applies the epilogue:
//   STORE  y = r
//   RESID  y += r (residual stream), optional copy for the layer trace
//   QKV    raw output, rotary embedding of q and k heads, bf16 append of the
//          new k and v at position pos, refresh of the page's key bounds
#include "common.cuh"
#include "kernels.h"

#include <math.h>
#include <algorithm>

namespace bc {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvRowsInFlight = 8;

__device__ __forceinline__ void fma8(float* acc, float xv, const uint4& w) {
  acc[0] = fmaf(xv, bf16_lo(w.x), acc[0]);
  acc[1] = fmaf(xv, bf16_hi(w.x), acc[1]);
  acc[2] = fmaf(xv, bf16_lo(w.y), acc[2]);
  acc[3] = fmaf(xv, bf16_hi(w.y), acc[3]);
  acc[4] = fmaf(xv, bf16_lo(w.z), acc[4]);
  acc[5] = fmaf(xv, bf16_hi(w.z), acc[5]);
  acc[6] = fmaf(xv, bf16_lo(w.w), acc[6]);
  acc[7] = fmaf(xv, bf16_hi(w.w), acc[7]);
}

// Rotary embedding, bf16 append and key-bound refresh for one 256-column tile
// of the q/k/v output.  Heads never straddle a tile (256 is a multiple of hd).
__device__ void qkv_epilogue(const QkvEpilogue& e, int col0, float v, float* s_v) {
  const int tid = threadIdx.x;
  const int col = col0 + tid;
  s_v[tid] = v;
  __syncthreads();
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
    return;
  }
  const int head = is_v ? (col - qcols - kcols) / hd : (col - qcols) / hd;
  const int page = e.pos / kPage, slot = e.pos % kPage;
  __nv_bfloat16* pg = e.kv_layer + ((size_t)head * e.Pmax + page) * (2 * kPage * hd);
  const __nv_bfloat16 b = __float2bfloat16_rn(out);
  if (is_v) {
    pg[kPage * hd + slot * hd + i] = b;
    return;
  }
  pg[slot * hd + i] = b;
  // bounds over the page's valid keys: earlier slots from the pool, this one
  float mn = __bfloat162float(b), mx = mn;
  for (int t = 0; t < slot; ++t) {
    const float kt = __bfloat162float(pg[t * hd + i]);
    mn = fminf(mn, kt);
    mx = fmaxf(mx, kt);
  }
  __nv_bfloat16* mt = e.meta_layer + ((size_t)head * e.Pmax + page) * (2 * hd);
  mt[i] = __float2bfloat16_rn(mn);
  mt[hd + i] = __float2bfloat16_rn(mx);
}

__global__ void __launch_bounds__(kGemvThreads, 2) k_gemv(GemvArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* s_idx = reinterpret_cast<int*>(smem);
  float* s_x = reinterpret_cast<float*>(smem + sizeof(int) * a.chunk);
  __shared__ __align__(16) float s_red[kGemvWarps][kColTile];
  __shared__ int s_last;

  const int tile = blockIdx.x, split = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int col0 = tile * kColTile;
  const int r0 = split * a.chunk;
  const int nr = min(a.k, r0 + a.chunk) - r0;

  pdl_wait();
  for (int r = tid; r < nr; r += kGemvThreads) {
    const int c = a.idx ? a.idx[r0 + r] : r0 + r;
    s_idx[r] = c;
    s_x[r] = a.x[c];
  }
  __syncthreads();
  pdl_trigger();

  float acc[8];
  #pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  const __nv_bfloat16* wcol = a.W + col0 + lane * 8;
  const size_t ld = (size_t)a.d_out;
  for (int r = warp; r < nr; r += kGemvWarps * kGemvRowsInFlight) {
    uint4 w[kGemvRowsInFlight];
    float xv[kGemvRowsInFlight];
    #pragma unroll
    for (int u = 0; u < kGemvRowsInFlight; ++u) {
      const int rr = r + u * kGemvWarps;
      if (rr < nr) {
        w[u] = ld_stream(wcol + (size_t)s_idx[rr] * ld);
        xv[u] = s_x[rr];
      } else {
        w[u] = make_uint4(0, 0, 0, 0);
        xv[u] = 0.f;
      }
    }
    #pragma unroll
    for (int u = 0; u < kGemvRowsInFlight; ++u) fma8(acc, xv[u], w[u]);
  }
  float4* red4 = reinterpret_cast<float4*>(&s_red[warp][lane * 8]);
  red4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  red4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  __syncthreads();
  float r = 0.f;
  #pragma unroll
  for (int w = 0; w < kGemvWarps; ++w) r += s_red[w][tid];

  const int col = col0 + tid;
  if (a.n_chunks > 1) {
    a.partial[(size_t)split * a.d_out + col] = r;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&a.counters[tile], 1u) == (unsigned)(a.n_chunks - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    r = 0.f;
    for (int s = 0; s < a.n_chunks; ++s) r += ld_cg(&a.partial[(size_t)s * a.d_out + col]);
    if (tid == 0) a.counters[tile] = 0u;
  }
  if (a.epi == EPI_STORE) {
    a.y[col] = r;
  } else if (a.epi == EPI_RESID) {
    const float nx = a.y[col] + r;
    a.y[col] = nx;
    if (a.y_copy) a.y_copy[col] = nx;
  } else {
    a.y[col] = r;
    __syncthreads();
    qkv_epilogue(a.qkv, col0, r, &s_red[0][0]);
  }
}

void gemv_plan(int k, int d_out, int sms, int max_chunks, int* chunk, int* n_chunks) {
  const int tiles = d_out / kColTile;
  const int target = 2 * sms;                       // two resident CTAs per SM
  int want = (target + tiles - 1) / tiles;
  const int lo = (k + kGemvMaxChunkRows - 1) / kGemvMaxChunkRows;
  const int hi = std::max(1, (k + 31) / 32);          // at least 32 rows per split
  want = std::max(lo, std::min(want, hi));
  want = std::max(1, std::min(want, max_chunks));
  int c = (k + want - 1) / want;
  *chunk = c;
  *n_chunks = (k + c - 1) / c;
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)a.chunk * (sizeof(int) + sizeof(float));
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_gemv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kGemvMaxChunkRows * (sizeof(int) + sizeof(float))));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.d_out / kColTile, a.n_chunks);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_gemv, a);
}

}  // namespace bc
