// Once-after-prefill page scores: the pages' own KV mode (ByteCross README,
// "Timing and quality on a GPU": an attention-scored selection made once
// after prefill, in the manner of SnapKV, listed on the mlsanity page).
//
// A window of observation queries per query head (the last prompt
// positions' queries, post-rotary) votes for the cached tokens with its
// softmax attention over the whole prefix, scale 1/sqrt(hd).  A page's score
// is the attention mass its valid tokens receive from every observation
// query of the kv head's group:
//
//   score_p = sum_q sum_{t in p} exp(s_qt - M_q) / L_q,
//   M_q = max_t s_qt,  L_q = sum_t exp(s_qt - M_q)   (t over all n tokens).
//
// Three kernels per layer: per-chunk (max, sum) of every query, their merge,
// and the page masses (logits recomputed).  The logits are a dense
// contraction (queries x keys x hd), so they run on the tensor cores with the
// attention kernel's operand layout: mma m16n8k16 with 8 observation queries
// per A block (rows 0-7 their bf16 "hi" parts, rows 8-15 the residues, so the
// sum of both keeps about 16 bits of the fp32 query) and 8 keys per B block.
// A CTA takes a chunk of 32 pages of one kv head; each of its 4 warps takes
// every 4th page, with the next page's keys in flight (lane (g, t) loads dims
// u*32 + t*8 .. +8 of key rows g and g+8, and the contraction dims are
// permuted alike in the query fragments).  The query fragments of all blocks
// are staged once per CTA in shared memory, one 16-byte read per lane, block
// and k16 step; each key fragment feeds 4 query blocks in turn, so a warp has
// 8 independent accumulator chains in flight.  Base-2 logits throughout.  It runs once per selection, not
// per decode step.
#include "common.cuh"
#include "kernels.h"
#include "tensor_map.h"

#include <math.h>
#include <string.h>
#include <algorithm>

namespace bc {

constexpr int kSnapWarps = 4;
constexpr int kSnapPages = 32;                // pages per chunk (CTA)
constexpr int kSnapTok = kSnapPages * kPage;  // tokens per chunk
constexpr int kSnapBlocks = kSnapMaxQ / 8;    // query blocks of 8
constexpr int kSnapGrp = 4;                   // blocks per key-fragment pass: 8 independent mma chains

// PASS 0: per-chunk (max, sum) of every query.  PASS 1: page masses.
template <int HD, int PASS>
__global__ void __launch_bounds__(kSnapWarps * 32, 2) k_snap(SnapArgs a) {
  constexpr int KSTEPS = HD / 16;
  constexpr int U4 = HD / 32;                 // 16-byte vectors per lane and key row
  constexpr int PAGE_ELEMS = 2 * kPage * HD;
  extern __shared__ __align__(16) uint4 s_qa[];   // [blocks][KSTEPS][32 lanes]
  __shared__ float s_m[kSnapWarps][kSnapMaxQ], s_l[kSnapWarps][kSnapMaxQ];
  const int chunk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int Q = a.n_obs * a.G;
  const int NB = ((Q + 8 * kSnapGrp - 1) / (8 * kSnapGrp)) * kSnapGrp;   // blocks, zero-padded
  const float qscale = 1.4426950408889634f * rsqrtf((float)HD);
  pdl_wait();
  pdl_trigger();

  // query fragments: block b holds queries 8b .. 8b+7 (query qi = j*G + gg is
  // observation j of head h*G + gg); lane (g, t) of k-step s takes dims
  // (s/2)*32 + 4*(s%2) + t*8 + 0..3 of query 8b + g
  for (int e = tid; e < NB * KSTEPS * 32; e += kSnapWarps * 32) {
    const int ln = e % 32, s = (e / 32) % KSTEPS, blk = e / (32 * KSTEPS);
    const int qi = 8 * blk + (ln >> 2), tt = ln & 3;
    const int d0 = (s / 2) * 32 + 4 * (s % 2) + tt * 8;
    float q[4] = {0.f, 0.f, 0.f, 0.f};
    if (qi < Q) {
      const int j = qi / a.G, gg = qi % a.G;
      const float* qp = a.q_obs + ((size_t)j * a.Hkv * a.G + h * a.G + gg) * HD + d0;
      #pragma unroll
      for (int c = 0; c < 4; ++c) q[c] = qp[c] * qscale;
    }
    uint4 f;
    split2(q[0], q[1], f.x, f.y);
    split2(q[2], q[3], f.z, f.w);
    s_qa[e] = f;
  }
  __syncthreads();

  // per lane: query g of every block, running (max, sum) or its (M, 1/L)
  float m_run[kSnapBlocks], l_run[kSnapBlocks];
  #pragma unroll
  for (int b = 0; b < kSnapBlocks; ++b) {
    m_run[b] = -INFINITY;
    l_run[b] = 0.f;
    if (PASS == 1 && b < NB && 8 * b + g < Q) {
      const float2 st = a.stats[(size_t)h * Q + 8 * b + g];
      m_run[b] = st.x;
      l_run[b] = 1.0f / st.y;
    }
  }
  const __nv_bfloat16* head = a.kv + (size_t)h * a.Pmax * PAGE_ELEMS;
  const int p0 = chunk * kSnapPages;
  const int p_end = min(p0 + kSnapPages, (a.n_tok + kPage - 1) / kPage);
  auto load = [&](int page, uint4* k0, uint4* k1) {
    const __nv_bfloat16* pk = head + (size_t)page * PAGE_ELEMS + t * 8;
    #pragma unroll
    for (int u = 0; u < U4; ++u) {
      k0[u] = ld_stream(pk + g * HD + 32 * u);
      k1[u] = ld_stream(pk + (g + 8) * HD + 32 * u);
    }
  };
  auto process = [&](int page, const uint4* k0, const uint4* k1) {
    const uint32_t* kr0 = reinterpret_cast<const uint32_t*>(k0);
    const uint32_t* kr1 = reinterpret_cast<const uint32_t*>(k1);
    const int valid = min(kPage, a.n_tok - page * kPage);
    const int tok[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
    float mass = 0.f;
    #pragma unroll
    for (int b0 = 0; b0 < kSnapBlocks; b0 += kSnapGrp) {
      if (b0 >= NB) break;
      float c[kSnapGrp][2][4];
      #pragma unroll
      for (int i = 0; i < kSnapGrp; ++i)
        #pragma unroll
        for (int r = 0; r < 4; ++r) c[i][0][r] = c[i][1][r] = 0.f;
      #pragma unroll
      for (int s = 0; s < KSTEPS; ++s)
        #pragma unroll
        for (int i = 0; i < kSnapGrp; ++i) {
          const uint4 f = s_qa[((b0 + i) * KSTEPS + s) * 32 + lane];
          const uint32_t qa[4] = {f.x, f.y, f.z, f.w};
          mma16816(c[i][0], qa, kr0[2 * s], kr0[2 * s + 1]);
          mma16816(c[i][1], qa, kr1[2 * s], kr1[2 * s + 1]);
        }
      #pragma unroll
      for (int i = 0; i < kSnapGrp; ++i) {
        const int b = b0 + i;
        const float sc[4] = {c[i][0][0] + c[i][0][2], c[i][0][1] + c[i][0][3],
                             c[i][1][0] + c[i][1][2], c[i][1][1] + c[i][1][3]};
        if (PASS == 0) {
          float mx = -INFINITY;
          #pragma unroll
          for (int j = 0; j < 4; ++j)
            if (tok[j] < valid) mx = fmaxf(mx, sc[j]);
          const float m_new = fmaxf(m_run[b], mx);
          float add = 0.f;
          #pragma unroll
          for (int j = 0; j < 4; ++j)
            if (tok[j] < valid) add += exp2f(sc[j] - m_new);
          l_run[b] = (m_run[b] == -INFINITY ? 0.f : l_run[b] * exp2f(m_run[b] - m_new)) + add;
          m_run[b] = m_new;
        } else if (8 * b + g < Q) {
          #pragma unroll
          for (int j = 0; j < 4; ++j)
            if (tok[j] < valid) mass += exp2f(sc[j] - m_run[b]) * l_run[b];
        }
      }
    }
    if (PASS == 1) {
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) mass += __shfl_xor_sync(0xffffffffu, mass, o);
      if (lane == 0) a.scores[(size_t)h * a.Pmax + page] = mass;
    }
  };
  uint4 ka0[U4], ka1[U4], kb0[U4], kb1[U4];
  int p = p0 + warp;
  if (p < p_end) load(p, ka0, ka1);
  while (p < p_end) {
    int q = p + kSnapWarps;
    if (q < p_end) load(q, kb0, kb1);
    process(p, ka0, ka1);
    p = q;
    if (p >= p_end) break;
    q = p + kSnapWarps;
    if (q < p_end) load(q, ka0, ka1);
    process(p, kb0, kb1);
    p = q;
  }
  if (PASS == 0) {
    // the quad's lanes hold the same query: merge them, then the warps
    #pragma unroll
    for (int b = 0; b < kSnapBlocks; ++b) {
      if (b >= NB) break;
      float m = m_run[b], l = l_run[b];
      #pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
        const float mm = fmaxf(m, m2);
        l = (m == -INFINITY ? 0.f : l * exp2f(m - mm)) + (m2 == -INFINITY ? 0.f : l2 * exp2f(m2 - mm));
        m = mm;
      }
      if (t == 0) {
        s_m[warp][8 * b + g] = m;
        s_l[warp][8 * b + g] = l;
      }
    }
    __syncthreads();
    for (int qi = tid; qi < Q; qi += kSnapWarps * 32) {
      float M = -INFINITY;
      #pragma unroll
      for (int w = 0; w < kSnapWarps; ++w) M = fmaxf(M, s_m[w][qi]);
      float L = 0.f;
      #pragma unroll
      for (int w = 0; w < kSnapWarps; ++w)
        if (s_m[w][qi] != -INFINITY) L += s_l[w][qi] * exp2f(s_m[w][qi] - M);
      a.part[((size_t)h * gridDim.x + chunk) * Q + qi] = make_float2(M, L);
    }
  }
}

// Merges the chunks' (max, sum) of every query: one thread per (kv head, query).
__global__ void k_snap_merge(SnapArgs a, int chunks) {
  const int Q = a.n_obs * a.G;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (e >= a.Hkv * Q) return;
  const int h = e / Q, qi = e % Q;
  float M = -INFINITY;
  for (int c = 0; c < chunks; ++c) M = fmaxf(M, a.part[((size_t)h * chunks + c) * Q + qi].x);
  float L = 0.f;
  for (int c = 0; c < chunks; ++c) {
    const float2 p = a.part[((size_t)h * chunks + c) * Q + qi];
    if (p.x != -INFINITY) L += p.y * exp2f(p.x - M);
  }
  a.stats[(size_t)h * Q + qi] = make_float2(M, L);
}

int snap_chunks(int n_tok) { return (n_tok + kSnapTok - 1) / kSnapTok; }

// ------------------------------------------------------------------ tcgen05 scorer
// For head_dim 128 and at most 64 observation queries per kv head: one pass
// over the keys, with the logits of a tile of 256 keys (16 pages) computed on
// the fifth-generation tensor cores into tensor memory.  For every page and
// query it keeps the page's own (max m_pq, sum l_pq) of exp2(s - m_pq), and
// per chunk of pages the running (max, sum) of every query; after the merge
// of the chunks (M_q, L_q), a small kernel forms each page's mass
//
//   score_p = sum_q l_pq * exp2(m_pq - M_q) / L_q,
//
// the same sum as above regrouped by page, so the keys are read once (the
// page partials add 512 bytes per page, an eighth of the page's keys).
//
// Operands.  A (shared memory, 128 rows x 128 dims bf16, K-major, 128-byte
// swizzle, written by the CTA): row 2q holds the bf16 "hi" part of
// observation query q scaled by log2(e)/sqrt(hd), row 2q+1 its residue, so
// D[2q] + D[2q+1] is the base-2 logit with about 16 bits of the fp32 query.
// B (shared memory, 256 keys x 128 dims): two tensor copies of 64 dims each
// through a 3-D tensor map over [page][token][dim] whose page stride skips
// the values.  D: 128 lanes x 256 fp32 columns of tensor memory; two such
// accumulators, so one tile's epilogue runs while the next is multiplied.
//
// Roles (18 warps): warp 0 issues the tensor copies into a 2-stage ring of
// 64 KB; warp 1 owns the tensor memory, and one of its threads issues the
// MMAs (8 per tile: two 64-dim halves x four k16 steps, M 128, N 256) and
// commits them to the stage's and the accumulator's mbarriers; warps 2-17
// read the accumulator, each a 32-lane subpartition (its warp index mod 4,
// as tensor memory requires) and a group of 64 columns (4 pages).  A lane
// holds one row, so lanes 2q and 2q+1 hold query q; they swap half their
// columns so that each ends with the 16 logits of one page.  Sixteen reading
// warps keep the exponentials and shuffles of a tile within the time its
// keys take to arrive.  A kv head's tiles are split evenly over its CTAs
// (the chunks), one CTA per SM, and the first two tiles' copies start before
// the dependency wait.  Every wait is bounded; a timeout sets g_snap_status
// (read by the host after the selection) and the CTA still releases its
// tensor memory after its own copies and MMAs.
constexpr int kTcKeys = 256;                          // keys per tile
constexpr int kTcPagesPerTile = kTcKeys / kPage;      // 16
constexpr int kTcHalfBytes = kTcKeys * 128;           // 64 dims of a tile: 32 KB
constexpr int kTcStageBytes = 2 * kTcHalfBytes;       // 64 KB
constexpr int kTcStages = 2;
constexpr int kTcABytes = 2 * 128 * 128;              // two 64-dim halves of 128 rows
constexpr int kTcSmem = 1024 + kTcABytes + kTcStages * kTcStageBytes;
constexpr int kTcEpiWarps = 16;                       // 4 subpartitions x 4 column groups
constexpr int kTcColGroup = kTcKeys / (kTcEpiWarps / 4);   // 64 columns
constexpr int kTcThreads = (2 + kTcEpiWarps) * 32;
constexpr uint32_t kTcCols = 512;                     // two 256-column accumulators
// instruction descriptor: fp32 D, bf16 A and B, both K-major, N 256, M 128
constexpr uint32_t kTcIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcKeys >> 3) << 17) |
                              ((uint32_t)(128 >> 4) << 24);

__device__ unsigned g_snap_status;

struct SnapTcParams {
  CUtensorMap tm;          // keys of the layer: [Hkv*Pmax pages][16 tokens][128 dims], box 64 x 16 x 16
  SnapArgs a;
  int chunks;              // CTAs per kv head; chunk c takes tiles [c*T/chunks, (c+1)*T/chunks)
};

// Shared-memory matrix descriptor: K-major rows of 128 bytes, 128-byte
// swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(kTcIdesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_load_tile(uint32_t dst, const void* tmap, int d0, int page, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(tmap), "r"(d0), "r"(0), "r"(page), "r"(bar)
      : "memory");
}
// 2^x by the hardware approximation (flushes results below 2^-126 to 0: the
// arguments here are logit minus a maximum, whose tiny terms do not matter).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 32 consecutive fp32 columns of this warp's 32 lanes (complete after
// tcgen05.wait::ld).
__device__ __forceinline__ void tc_ld32_nowait(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

__global__ void __launch_bounds__(kTcThreads, 1) k_snap_tc(const __grid_constant__ SnapTcParams prm) {
  const SnapArgs& a = prm.a;
  extern __shared__ __align__(1024) unsigned char tc_smem[];
  __shared__ __align__(8) uint64_t full_b[kTcStages], empty_b[kTcStages], acc_full[2], acc_empty[2];
  __shared__ uint32_t s_taddr;
  __shared__ int s_err;
  __shared__ float2 s_ml[4][128];                     // [column group][row] (max, sum)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, h = blockIdx.y;
  const int Q = a.n_obs * a.G;
  const int P = (a.n_tok + kPage - 1) / kPage;
  const int T = (P + kTcPagesPerTile - 1) / kTcPagesPerTile;
  const int t0 = (int)((long long)chunk * T / prm.chunks);
  const int nt = (int)((long long)(chunk + 1) * T / prm.chunks) - t0;
  const uint32_t s0 = smem_addr(tc_smem);
  const uint32_t sA = (s0 + 1023u) & ~1023u, sB = sA + kTcABytes;
  unsigned char* gA = tc_smem + (sA - s0);

  if (tid == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(smem_addr(&full_b[i]), 1);
      mbar_init(smem_addr(&empty_b[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&acc_full[i]), 1);
      mbar_init(smem_addr(&acc_empty[i]), kTcEpiWarps);
    }
    mbar_init_fence();
    s_err = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_taddr)),
                 "r"(kTcCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // the keys do not depend on the previous kernel: the first tiles' copies
  // start before waiting for it and before A is built (barrier init is
  // ordered by the same thread)
  auto issue = [&](int it) {
    const int st = it & 1;
    const uint32_t fb = smem_addr(&full_b[st]);
    mbar_arrive_expect_tx(fb, kTcStageBytes);
    const int page = h * a.Pmax + (t0 + it) * kTcPagesPerTile;
    tc_load_tile(sB + st * kTcStageBytes, &prm.tm, 0, page, fb);
    tc_load_tile(sB + st * kTcStageBytes + kTcHalfBytes, &prm.tm, 64, page, fb);
  };
  const int pre = min(nt, kTcStages);
  if (tid == 0)
    for (int it = 0; it < pre; ++it) issue(it);
  pdl_wait();
  pdl_trigger();

  // A: row r = 2q + (0 hi | 1 lo), 16-byte chunk c of dims 8c .. 8c+7 (half
  // c / 8), stored at chunk (c % 8) ^ (r % 8) of the row: the 128-byte swizzle
  const float qscale = 1.4426950408889634f * rsqrtf(128.f);
  for (int e = tid; e < 128 * 16; e += kTcThreads) {
    const int row = e >> 4, c = e & 15, q = row >> 1;
    float v[8];
    #pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    if (q < Q) {
      const int j = q / a.G, gg = q % a.G;
      const float4* qp = reinterpret_cast<const float4*>(a.q_obs + ((size_t)j * a.Hkv * a.G + h * a.G + gg) * 128 + c * 8);
      const float4 x0 = qp[0], x1 = qp[1];
      v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
      v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
    }
    uint32_t w[4];
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t hi, lo;
      split2(v[2 * i] * qscale, v[2 * i + 1] * qscale, hi, lo);
      w[i] = (row & 1) ? lo : hi;
    }
    const uint32_t off = (c >> 3) * (128 * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4);
    *reinterpret_cast<uint4*>(gA + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // A is read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_taddr;

  if (warp == 0) {
    if (lane == 0) {
      int issued = pre;
      for (int it = pre; it < nt; ++it) {
        if (!mbar_wait(smem_addr(&empty_b[it & 1]), ((it >> 1) - 1) & 1)) {
          atomicOr(&g_snap_status, 1u);
          break;
        }
        issue(it);
        issued = it + 1;
      }
      // the last copies have landed before the CTA ends (they have, unless a
      // wait above gave up)
      for (int it = max(0, issued - kTcStages); it < issued; ++it)
        mbar_wait(smem_addr(&full_b[it & 1]), (it >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nt; ++it) {
        const int st = it & 1;
        if (!mbar_wait(smem_addr(&full_b[st]), (it >> 1) & 1) ||
            (it >= 2 && !mbar_wait(smem_addr(&acc_empty[st]), ((it >> 1) - 1) & 1))) {
          atomicOr(&g_snap_status, 2u);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + st * kTcKeys;
        #pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          #pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tc_mma(d, tc_desc(sA + hh * (128 * 128) + ks * 32),
                   tc_desc(sB + st * kTcStageBytes + hh * kTcHalfBytes + ks * 32), (hh | ks) != 0);
        tc_commit(smem_addr(&empty_b[st]));
        tc_commit(smem_addr(&acc_full[st]));
        issued = it + 1;
      }
      // every MMA issued has completed before the tensor memory is released
      if (issued > 0) mbar_wait(smem_addr(&acc_full[(issued - 1) & 1]), ((issued - 1) >> 1) & 1);
    }
  } else {
    const int ew = warp - 2, sp = warp & 3;          // tensor-memory subpartition: lanes 32*sp ..
    const int cg = ew >> 2;                          // column group: columns 64*cg .. 64*cg + 63
    const int q = (32 * sp + lane) >> 1;
    const bool odd = lane & 1, qv = q < Q;
    float m_run = -INFINITY, l_run = 0.f;
    for (int it = 0; it < nt; ++it) {
      const int st = it & 1;
      bool ok = *reinterpret_cast<volatile int*>(&s_err) == 0;
      if (ok && !mbar_wait(smem_addr(&acc_full[st]), (it >> 1) & 1)) {
        ok = false;
        s_err = 1;
        atomicOr(&g_snap_status, 4u);
      }
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const int key_t = (t0 + it) * kTcKeys + cg * kTcColGroup;
      if (ok) {
        // this warp's 64 columns: two loads in flight, one wait
        uint32_t v[2][32];
        const uint32_t ta = tmem + ((uint32_t)(32 * sp) << 16) + st * kTcKeys + cg * kTcColGroup;
        tc_ld32_nowait(ta, v[0]);
        tc_ld32_nowait(ta + 32, v[1]);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        #pragma unroll
        for (int c = 0; c < 2; ++c) {
          // lanes 2q (hi) and 2q+1 (lo): the even lane keeps columns 0-15, the odd one 16-31
          float lg[16];
          #pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t send = odd ? v[c][j] : v[c][16 + j];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 1);
            lg[j] = __uint_as_float(odd ? v[c][16 + j] : v[c][j]) + __uint_as_float(recv);
          }
          const int key0 = key_t + c * 32 + (odd ? 16 : 0);
          const int valid = qv ? min(kPage, max(0, a.n_tok - key0)) : 0;
          if (valid > 0) {
            // this page's (max, sum) for query q (pairwise trees), then the running pair
            #pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j >= valid) lg[j] = -INFINITY;
            float t8[8], t4[4];
            #pragma unroll
            for (int j = 0; j < 8; ++j) t8[j] = fmaxf(lg[j], lg[j + 8]);
            #pragma unroll
            for (int j = 0; j < 4; ++j) t4[j] = fmaxf(t8[j], t8[j + 4]);
            const float mp = fmaxf(fmaxf(t4[0], t4[2]), fmaxf(t4[1], t4[3]));
            #pragma unroll
            for (int j = 0; j < 8; ++j) t8[j] = ex2(lg[j] - mp) + ex2(lg[j + 8] - mp);
            #pragma unroll
            for (int j = 0; j < 4; ++j) t4[j] = t8[j] + t8[j + 4];
            const float lp = (t4[0] + t4[2]) + (t4[1] + t4[3]);
            a.pp[((size_t)h * a.Pmax + key0 / kPage) * Q + q] = make_float2(mp, lp);
            // one exponential: the smaller maximum is rescaled to the larger
            if (mp > m_run) {
              l_run = (m_run == -INFINITY ? 0.f : l_run * ex2(m_run - mp)) + lp;
              m_run = mp;
            } else {
              l_run += lp * ex2(mp - m_run);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&acc_empty[st]));
    }
    {
      // the pair's two halves of each page, then the four column groups in order
      const float m2 = __shfl_xor_sync(0xffffffffu, m_run, 1), l2 = __shfl_xor_sync(0xffffffffu, l_run, 1);
      const float mm = fmaxf(m_run, m2);
      const float l = mm == -INFINITY ? 0.f
                                      : (m_run == -INFINITY ? 0.f : l_run * exp2f(m_run - mm)) +
                                            (m2 == -INFINITY ? 0.f : l2 * exp2f(m2 - mm));
      s_ml[cg][32 * sp + lane] = make_float2(mm, l);
      asm volatile("bar.sync 1, %0;" ::"n"(kTcEpiWarps * 32) : "memory");
      if (cg == 0 && !odd && qv) {
        float M2 = -INFINITY;
        #pragma unroll
        for (int g = 0; g < 4; ++g) M2 = fmaxf(M2, s_ml[g][32 * sp + lane].x);
        float L2 = 0.f;
        #pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float2 p = s_ml[g][32 * sp + lane];
          if (p.x != -INFINITY) L2 += p.y * exp2f(p.x - M2);
        }
        a.part[((size_t)h * gridDim.x + chunk) * Q + q] = make_float2(M2, L2);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols) : "memory");
  }
}

// Page masses from the page partials: a warp per page, lane l holding
// queries l and l + 32; the butterfly sum fixes the order.
constexpr int kMassWarps = 8;
constexpr int kMassPagesPerBlock = 64;

__global__ void __launch_bounds__(kMassWarps * 32) k_snap_mass(SnapArgs a) {
  const int h = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int Q = a.n_obs * a.G, P = (a.n_tok + kPage - 1) / kPage;
  pdl_wait();
  pdl_trigger();
  float M[2], invL[2];
  #pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int q = lane + 32 * u;
    M[u] = 0.f;
    invL[u] = 0.f;
    if (q < Q) {
      const float2 st = a.stats[(size_t)h * Q + q];
      M[u] = st.x;
      invL[u] = 1.0f / st.y;
    }
  }
  const int p_end = min(P, (blockIdx.x + 1) * kMassPagesPerBlock);
  for (int page = blockIdx.x * kMassPagesPerBlock + warp; page < p_end; page += kMassWarps) {
    const float2* pp = a.pp + ((size_t)h * a.Pmax + page) * Q;
    float mass = 0.f;
    #pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = lane + 32 * u;
      if (q < Q) {
        const float2 v = pp[q];
        mass += v.y * exp2f(v.x - M[u]) * invL[u];
      }
    }
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) mass += __shfl_xor_sync(0xffffffffu, mass, o);
    if (lane == 0) a.scores[(size_t)h * a.Pmax + page] = mass;
  }
}

static int device_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 1;
  }
  return sms;
}

static cudaError_t launch_tc(const SnapArgs& a, cudaStream_t st, bool pdl) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_snap_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const EncodeTiledFn encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  SnapTcParams prm;
  memset(&prm, 0, sizeof prm);
  prm.a = a;
  // the layer's keys as [Hkv*Pmax pages][16 tokens][128 dims]: the page
  // stride (keys and values of a page) skips the values
  cuuint64_t gdim[3] = {128, (cuuint64_t)kPage, (cuuint64_t)a.Hkv * a.Pmax};
  cuuint64_t gstride[2] = {128 * sizeof(__nv_bfloat16), 2 * kPage * 128 * sizeof(__nv_bfloat16)};
  cuuint32_t box[3] = {64, (cuuint32_t)kPage, (cuuint32_t)kTcPagesPerTile};
  cuuint32_t estride[3] = {1, 1, 1};
  if ((uintptr_t)a.kv & 15) return cudaErrorInvalidValue;
  if (encode(&prm.tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)a.kv, gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // one CTA per SM at most: chunks of whole tiles, no more chunks than the
  // (max, sum) buffer holds
  const int P = (a.n_tok + kPage - 1) / kPage;
  const int T = (P + kTcPagesPerTile - 1) / kTcPagesPerTile;
  int chunks = std::min(T, std::min(std::max(1, device_sms() / a.Hkv), snap_chunks(a.n_tok)));
  prm.chunks = chunks;
  const int Q = a.n_obs * a.G;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(chunks, a.Hkv);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = kTcSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_snap_tc, prm);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c2 = cfg;
  c2.gridDim = dim3((a.Hkv * Q + 127) / 128);
  c2.blockDim = dim3(128);
  c2.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&c2, k_snap_merge, a, chunks);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c3 = c2;
  c3.gridDim = dim3((P + kMassPagesPerBlock - 1) / kMassPagesPerBlock, a.Hkv);
  c3.blockDim = dim3(kMassWarps * 32);
  return cudaLaunchKernelEx(&c3, k_snap_mass, a);
}

cudaError_t snap_status(unsigned* status, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(status, g_snap_status, sizeof(unsigned), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return e;
}

template <int HD>
static cudaError_t launch_hd(const SnapArgs& a, cudaStream_t st, bool pdl) {
  constexpr int KSTEPS = HD / 16;
  const int Q = a.n_obs * a.G;
  const int NB = ((Q + 8 * kSnapGrp - 1) / (8 * kSnapGrp)) * kSnapGrp;
  const size_t smem = (size_t)NB * KSTEPS * 32 * sizeof(uint4);
  static bool attr_done = false;
  if (!attr_done) {
    const int max_smem = kSnapBlocks * KSTEPS * 32 * (int)sizeof(uint4);
    cudaError_t e = cudaFuncSetAttribute(k_snap<HD, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_snap<HD, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int chunks = snap_chunks(a.n_tok);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(chunks, a.Hkv);
  cfg.blockDim = dim3(kSnapWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_snap<HD, 0>, a);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c2 = cfg;
  c2.gridDim = dim3((a.Hkv * Q + 127) / 128);
  c2.blockDim = dim3(128);
  c2.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&c2, k_snap_merge, a, chunks);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k_snap<HD, 1>, a);
}

cudaError_t launch_snap_scores(const SnapArgs& a, cudaStream_t st, bool pdl) {
  if (a.n_tok < 1 || a.n_obs < 1 || a.n_obs * a.G > kSnapMaxQ) return cudaErrorInvalidValue;
  if (a.hd == 128 && a.n_obs * a.G <= 64 && a.pp) return launch_tc(a, st, pdl);
  if (a.hd == 128) return launch_hd<128>(a, st, pdl);
  if (a.hd == 64) return launch_hd<64>(a, st, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace bc
