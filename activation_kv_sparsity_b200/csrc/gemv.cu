// Column-gathered bf16 GEMV with fp32 accumulation: the projection kernel of
// every decode mode.
//
//   y[j] = s * sum over listed input channels c of v[c] * W[c][j]
//
// W is input-channel-major ([d_in][d_out]), so each selected channel is one
// contiguous row and the activation-sparse projection (the ByteCross README's
// projection branch, "Timing and quality on a GPU") reads exactly the rows of
// the kept channels; dense mode is the same kernel over every row.
//
// The GEMV input v is produced while staging, from the previous step's
// output, so no separate kernel runs for it:
//   NONE        v = x
//   NORM        v = x * g, s = 1 / sqrt(mean(x^2) + eps)   (RMSNorm; the
//               scale factors out of the sum and is applied to the partials)
//   EMBED_NORM  the same with x = the token's bf16 embedding row; CTA 0 also
//               initialises the residual stream with it
//   SWIGLU      v = silu(gate) * up
//
// Work split: a column tile of TW = 256 outputs (128 when there would be
// fewer than 24 wide tiles) is shared by the CTAs of one or more thread-block
// clusters, and the tile's k listed rows are cut into one contiguous run per
// CTA.  A row segment is TW*2 bytes read by TW/8 lanes at 16 bytes each; a
// CTA's 8 warps stream its run with 8 to 16 row segments per lane in flight
// (two halves of 8 in registers, each refilled as soon as it is multiplied);
// warps are reduced in shared memory.  The CTAs of a cluster then sum their partials
// through distributed shared memory after a hardware cluster barrier (rank 0
// reads them in rank order).  A tile split over several clusters adds one
// stage through global scratch: each cluster's rank 0 writes its partial and
// takes an atomic ticket; the last to arrive (no spinning) sums the clusters'
// partials in order.  Both stages sum in a fixed order: deterministic.  The
// CTA that holds the tile's complete sum applies the epilogue:
//   STORE   y = r
//   RESID   y += r (the residual stream), optionally copied
//   QKV     rotary embedding of q and k, bf16 append of k and v to their
//           page, refresh of that page's key bounds
//   SWIGLU  the tile pairs TW/2 gate columns with the up columns of the same
//           channels, and y = silu(gate) * up for those channels
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

#include <cooperative_groups.h>
#include <math.h>
#include <algorithm>

namespace cg = cooperative_groups;

namespace bc {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kRowsInFlight = 16;

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

// x0^2 + x1^2 + x2^2 + x3^2 in one fixed order.
__device__ __forceinline__ float sumsq4(float x0, float x1, float x2, float x3) {
  return fmaf(x3, x3, fmaf(x2, x2, fmaf(x1, x1, x0 * x0)));
}

__device__ __forceinline__ float prep_value(const GemvArgs& a, int c) {
  switch (a.prep) {
    case GP_NORM: return a.x[c] * bf16f(a.gain[c]);
    case GP_EMBED_NORM: return bf16f(a.embed_row[c]) * bf16f(a.gain[c]);
    case GP_SWIGLU: {
      const float g = a.x[c], u = a.x[a.d_in + c];
      return g / (1.0f + expf(-g)) * u;
    }
    default: return a.x[c];
  }
}

// TW: columns per tile (256 or 128).  A row segment is TW*2 bytes read by
// TW/8 lanes at 16 bytes each, so a warp instruction covers 32/(TW/8) rows.
template <int TW>
__global__ void __launch_bounds__(kGemvThreads, 2) k_gemv(GemvArgs a) {
  constexpr int LPR = TW / 8;                      // lanes per row
  constexpr int RPI = 32 / LPR;                    // rows per warp instruction
  constexpr int ROWS_STEP = kGemvWarps * RPI;      // rows between a lane's consecutive rows
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ __align__(16) float s_red[kGemvWarps][TW];
  __shared__ __align__(16) float s_part[TW];
  __shared__ float s_v[kColTile];
  __shared__ float s_sum[kGemvWarps];
  __shared__ int s_last;
  cg::cluster_group cluster = cg::this_cluster();

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lrow = lane / LPR, lcol = lane % LPR;
  const int t = blockIdx.y;                       // column tile
  const int split = blockIdx.x;                   // run of rows: cluster * S + rank
  const int nsplit = a.S * a.C;
  const int r0 = (int)(((long long)a.k * split) / nsplit);
  const int nr = (int)(((long long)a.k * (split + 1)) / nsplit) - r0;
  const int col0 = t * TW;
  int* s_idx = reinterpret_cast<int*>(smem);
  float* s_x = reinterpret_cast<float*>(smem + sizeof(int) * a.max_rows);
  const bool norm = a.prep == GP_NORM || a.prep == GP_EMBED_NORM;
  // SWIGLU epilogue: the tile pairs gate columns t*TW/2 .. +TW/2 (lanes of
  // the first half of a row) with the up columns of the same channels
  const bool paired = a.epi == EPI_SWIGLU;
  const int hcol0 = t * (TW / 2);
  const __nv_bfloat16* wcol =
      a.W + (!paired ? col0 + lcol * 8
                     : (lcol < LPR / 2 ? hcol0 + lcol * 8 : a.d_out / 2 + hcol0 + (lcol - LPR / 2) * 8));
  const size_t ld = (size_t)a.d_out;
  const int my0 = warp * RPI + lrow;              // this lane's first row in the run

  uint4 w0[kRowsInFlight];
  float ss = 0.f;
  // the q/k/v epilogue's rotation and earlier key bounds, kept in shared
  // memory until the tile's sum is known (they depend only on the position)
  __shared__ QkvPre s_pre[TW];
  if (a.epi == EPI_QKV && tid < TW && (a.C > 1 || cluster.block_rank() == 0))
    s_pre[tid] = qkv_prologue(a.qkv, col0 + tid);     // only a CTA that may hold the tile's sum
  // Weights do not depend on the previous kernel: in dense mode issue this
  // lane's first batch of rows before waiting for it, so the stream overlaps
  // the previous kernel's tail.  (Pulling further rows into L2 as well was
  // measured to cost more than it saved.)
  bool first_loaded = false;
  if (!a.idx) {
    #pragma unroll
    for (int u = 0; u < kRowsInFlight; ++u) {
      const int rr = my0 + u * ROWS_STEP;
      w0[u] = rr < nr ? ld_stream(wcol + (size_t)(r0 + rr) * ld) : make_uint4(0, 0, 0, 0);
    }
    first_loaded = true;
  }
  pdl_wait();
  pdl_trigger();
  int cs0[4];                                     // the staging's first round of channels
  if (!first_loaded) {
    // the warp's first 16*RPI listed rows: lane e fetches the index of batch
    // element e = u*RPI + lrow, so the weight loads skip the staging barrier;
    // the staging's first round of the list is loaded in the same round trip
    int c = -1;
    if (lane < kRowsInFlight * RPI) {
      const int rr = warp * RPI + (lane % RPI) + (lane / RPI) * ROWS_STEP;
      if (rr < nr) c = a.idx[r0 + rr];
    }
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = u * kGemvThreads + tid;
      cs0[u] = r < nr ? a.idx[r0 + r] : -1;
    }
    #pragma unroll
    for (int u = 0; u < kRowsInFlight; ++u) {
      const int cu = __shfl_sync(0xffffffffu, c, u * RPI + lrow);
      w0[u] = cu >= 0 ? ld_stream(wcol + (size_t)cu * ld) : make_uint4(0, 0, 0, 0);
    }
  }

  // RMSNorm statistics over the whole input: independent loads, 4 in flight
  if (norm) {
    if (a.prep == GP_NORM) {
      const float4* x4 = reinterpret_cast<const float4*>(a.x);
      #pragma unroll 4
      for (int c = tid; c < a.d_in / 4; c += kGemvThreads) {
        const float4 v = x4[c];
        ss += sumsq4(v.x, v.y, v.z, v.w);
      }
    } else if (a.d_in % 4 == 0) {
      const uint2* e4 = reinterpret_cast<const uint2*>(a.embed_row);
      #pragma unroll 4
      for (int c = tid; c < a.d_in / 4; c += kGemvThreads) {
        const uint2 e = e4[c];
        const float e0 = bf16_lo(e.x), e1 = bf16_hi(e.x), e2 = bf16_lo(e.y), e3 = bf16_hi(e.y);
        ss += sumsq4(e0, e1, e2, e3);
        if (blockIdx.x == 0 && blockIdx.y == 0)
          reinterpret_cast<float4*>(a.x_init)[c] = make_float4(e0, e1, e2, e3);
      }
    } else {
      #pragma unroll 4
      for (int c = tid; c < a.d_in; c += kGemvThreads) {
        const float xv = bf16f(a.embed_row[c]);
        ss = fmaf(xv, xv, ss);
        if (blockIdx.x == 0 && blockIdx.y == 0) a.x_init[c] = xv;
      }
    }
  }

  // staging: 4 rows per thread per round, loads of a round in flight together
  for (int rb = 0; rb < nr; rb += 4 * kGemvThreads) {
    int cs[4];
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = rb + u * kGemvThreads + tid;
      cs[u] = rb == 0 && !first_loaded ? cs0[u] : (r < nr ? (a.idx ? a.idx[r0 + r] : r0 + r) : -1);
    }
    float vs[4];
    #pragma unroll
    for (int u = 0; u < 4; ++u) vs[u] = cs[u] >= 0 ? prep_value(a, cs[u]) : 0.f;
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = rb + u * kGemvThreads + tid;
      if (r < nr) {
        s_idx[r] = cs[u];
        s_x[r] = vs[u];
      }
    }
  }
  if (norm) {
    float v = ss;
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_sum[warp] = v;
  }
  __syncthreads();

  float acc[8];
  #pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  // Rolling pipeline over halves of 8 rows: w0[0..7] and w0[8..15] hold two
  // halves; a half is refilled with the half two ahead as soon as it has been
  // multiplied, so 8 to 16 rows per lane are always in flight.
  constexpr int HALF = kRowsInFlight / 2;
  const int rows_w = nr > warp * RPI ? (nr - warp * RPI + ROWS_STEP - 1) / ROWS_STEP : 0;
  const int nh = (rows_w + HALF - 1) / HALF;
  auto consume = [&](const uint4* w, int h) {
    #pragma unroll
    for (int u = 0; u < HALF; ++u) {
      const int rr = my0 + (h * HALF + u) * ROWS_STEP;
      fma8(acc, rr < nr ? s_x[rr] : 0.f, w[u]);
    }
  };
  auto refill = [&](uint4* w, int h) {
    #pragma unroll
    for (int u = 0; u < HALF; ++u) {
      const int rr = my0 + (h * HALF + u) * ROWS_STEP;
      w[u] = rr < nr ? ld_stream(wcol + (size_t)s_idx[rr] * ld) : make_uint4(0, 0, 0, 0);
    }
  };
  for (int h = 0; h < nh; h += 2) {
    consume(w0, h);
    if (h + 2 < nh) refill(w0, h + 2);
    if (h + 1 < nh) {
      consume(w0 + HALF, h + 1);
      if (h + 3 < nh) refill(w0 + HALF, h + 3);
    }
  }
  // lanes of the same columns (different rows) first, then the warps
  #pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
    #pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
  if (lrow == 0) {
    float4* red4 = reinterpret_cast<float4*>(&s_red[warp][lcol * 8]);
    red4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    red4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  __syncthreads();
  float scale = 1.f;
  if (norm) {
    float tot = 0.f;
    #pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) tot += s_sum[w];
    scale = 1.0f / sqrtf(tot / (float)a.d_in + a.eps);
  }
  float r = 0.f;
  if (tid < TW) {
    #pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) r += s_red[w][tid];
    s_part[tid] = r * scale;
  }

  // cluster stage: rank 0 sums the cluster's partials in rank order
  cluster.sync();
  const unsigned rank = cluster.block_rank();
  bool have_total = false;
  if (rank == 0) {
    r = 0.f;
    if (tid < TW)
      for (int q = 0; q < a.S; ++q) r += cluster.map_shared_rank(s_part, q)[tid];
    have_total = a.C == 1;
  }
  cluster.sync();                                  // peers' shared memory stays alive until read
  if (rank != 0) return;

  // global stage, when the tile is split over several clusters
  if (a.C > 1) {
    const int c = blockIdx.x / a.S;
    if (tid < TW) a.partial[((size_t)t * kGemvMaxContrib + c) * TW + tid] = r;
    __syncthreads();
    if (tid == 0) {
      __threadfence();   // the CTA's partials (ordered by the barrier) before the ticket
      s_last = (atomicAdd(&a.counters[t], 1u) == (unsigned)(a.C - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid < TW) {
      const float* pp = &a.partial[(size_t)t * kGemvMaxContrib * TW + tid];
      float v[kGemvMaxContrib];
      #pragma unroll
      for (int q = 0; q < kGemvMaxContrib; ++q) v[q] = q < a.C ? ld_cg(pp + (size_t)q * TW) : 0.f;
      r = 0.f;
      #pragma unroll
      for (int q = 0; q < kGemvMaxContrib; ++q) r += v[q];
    }
    if (tid == 0) a.counters[t] = 0u;
    have_total = true;
  }
  if (!have_total) return;
  const int col = col0 + tid;
  if (a.epi == EPI_QKV) {
    if (tid < TW) a.y[col] = r;
    qkv_epilogue<TW>(a.qkv, col0, r, s_v, tid < TW ? s_pre[tid] : QkvPre{});
  } else if (a.epi == EPI_SWIGLU) {
    // h = silu(gate) * up for the tile's TW/2 channels
    if (tid < TW) s_v[tid] = r;
    __syncthreads();
    if (tid < TW / 2) {
      const float g = s_v[tid], u = s_v[tid + TW / 2];
      a.y[hcol0 + tid] = g / (1.0f + expf(-g)) * u;
    }
  } else if (tid < TW) {
    if (a.epi == EPI_STORE) {
      a.y[col] = r;
    } else {
      const float nx = a.y[col] + r;
      a.y[col] = nx;
      if (a.y_copy) a.y_copy[col] = nx;
    }
  }
}

static int g_max_cluster = 0;   // largest cluster size the GPU schedules for k_gemv

template <int TW>
static cudaError_t set_attrs() {
  cudaError_t e = cudaFuncSetAttribute(k_gemv<TW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(kGemvMaxPer * (sizeof(int) + sizeof(float))));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_gemv<TW>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

static cudaError_t init_gemv_attrs() {
  if (g_max_cluster) return cudaSuccess;
  cudaError_t e = set_attrs<256>();
  if (e == cudaSuccess) e = set_attrs<128>();
  g_max_cluster = 8;
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 1);
    cfg.blockDim = dim3(kGemvThreads);
    cfg.dynamicSmemBytes = kGemvMaxPer * (sizeof(int) + sizeof(float));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_gemv<256>, &cfg) == cudaSuccess && n > 0) g_max_cluster = 16;
  }
  cudaGetLastError();   // a refused query leaves no sticky state; clear the last-error slot
  return cudaSuccess;
}

void gemv_plan(int k, int d_out, int sms, int* TW, int* S, int* C) {
  init_gemv_attrs();
  // 256-column tiles when there are enough of them, else 128-column tiles
  int tw = 256;
  if (d_out / 256 < 24 && d_out % 128 == 0) tw = 128;
  const int tiles = d_out / tw;
  // row runs per tile: about two CTAs per SM in all, at least 32 rows a run,
  // at most kGemvMaxPer rows a run
  int p = std::max(1, (2 * sms) / tiles);
  p = std::min(p, std::max(1, k / 32));
  p = std::max(p, (k + kGemvMaxPer - 1) / kGemvMaxPer);
  // clusters of at most 8 (portable) unless a bigger one avoids the global stage
  const int cap = std::max(1, g_max_cluster);
  int s = 1;
  while (s * 2 <= std::min(p, 8)) s *= 2;
  if (p >= 16 && cap >= 16 && p < 32) s = 16;
  // whole clusters only, never more row runs than planned (no extra wave);
  // runs stay within the staging limit
  int c = std::max(1, p / s);
  while ((k + s * c - 1) / (s * c) > kGemvMaxPer) ++c;
  c = std::min(c, kGemvMaxContrib);
  *TW = tw;
  *S = s;
  *C = c;
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st, bool pdl) {
  cudaError_t e = init_gemv_attrs();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S * a.C, a.d_out / a.TW);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = (size_t)a.max_rows * (sizeof(int) + sizeof(float));
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  if (a.TW == 128) return cudaLaunchKernelEx(&cfg, k_gemv<128>, a);
  return cudaLaunchKernelEx(&cfg, k_gemv<256>, a);
}

}  // namespace bc
