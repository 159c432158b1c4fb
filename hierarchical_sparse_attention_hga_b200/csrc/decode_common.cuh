// Building blocks of the bf16, D = 128 decode attention (attend_decode.cu and
// the one-launch decode step in decode_step.cu).
//
// A decode query's visible tokens form 16-token units, each a contiguous
// 16 x 256 B segment of the cache.  One warp streams its units through a
// private two-stage shared-memory ring (TMA box loads of 16 rows x 64 columns,
// 128-byte swizzle) and runs S^T = Q K^T and O += P V on mma.sync m16n8k16 with
// the G <= 16 query heads as the M rows; the online softmax stays in registers.
// Partials (o, m, l) are merged by log-sum-exp inside the CTA through shared
// memory, then across the cluster through distributed shared memory.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hga {
namespace decode {

constexpr int kD = 128;
constexpr int kUnit = 16;                       // tokens per unit (= group size)
constexpr int kWarps = 4;
constexpr int kStages = 2;
constexpr int kBoxBytes = kUnit * 64 * 2;       // 16 rows x 64 bf16 = 2 KB
constexpr int kTileBytes = 2 * kBoxBytes;       // one tensor, 128 dims
constexpr int kStageBytes = 2 * kTileBytes;     // K and V
constexpr int kWarpBytes = kStages * kStageBytes;
constexpr int kRingBytes = kWarps * kWarpBytes + 1024;  // + alignment slack
constexpr uint32_t kWaitLimit = 1u << 26;       // bounded mbarrier polls
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Address of the 16-byte chunk `chunk` (0..15 over 128 dims) of row `row` in a
// tile stored as two 128B-swizzled boxes of 64 columns.
__device__ __forceinline__ uint32_t swz(uint32_t tile, int row, int chunk) {
  const int box = chunk >> 3, c = chunk & 7;
  return tile + box * kBoxBytes + row * 128 + ((c ^ (row & 7)) << 4);
}

// One warp's online-softmax state: o for query heads (g, g + 8) x 128 dims as
// mma accumulators, running max m (log2 units) and this lane's partial sums l.
struct WarpState {
  float o[16][4];
  float m0, m1, l0, l1;
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    m0 = m1 = -CUDART_INF_F;
    l0 = l1 = 0.f;
  }
};

// Q of (b, KV head h) as m16n8k16 A fragments: rows = query heads (g, g+8), k = dims.
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16* q, const LayerParams& p, int b,
                                             int h, uint32_t (&qa)[8][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t* q0 = reinterpret_cast<const uint32_t*>(
      q + (static_cast<size_t>(b) * p.Hq + h * p.G + g) * kD);
  const uint32_t* q1 = reinterpret_cast<const uint32_t*>(
      q + (static_cast<size_t>(b) * p.Hq + h * p.G + g + 8) * kD);
  const bool r0 = g < p.G, r1 = g + 8 < p.G;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    qa[kk][0] = r0 ? __ldg(q0 + kk * 8 + t) : 0u;
    qa[kk][1] = r1 ? __ldg(q1 + kk * 8 + t) : 0u;
    qa[kk][2] = r0 ? __ldg(q0 + kk * 8 + 4 + t) : 0u;
    qa[kk][3] = r1 ? __ldg(q1 + kk * 8 + 4 + t) : 0u;
  }
}

// Issues the four TMA boxes (K and V, two column halves each) of the unit at
// cache row y into ring stage `st` (lane 0 of the warp only).
__device__ __forceinline__ void issue_unit(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                           uint8_t* st, uint64_t* bar, int32_t y) {
  ptx::mbar_expect_tx(bar, kStageBytes);
  ptx::tma_load_2d(st, tm_k, bar, 0, y);
  ptx::tma_load_2d(st + kBoxBytes, tm_k, bar, 64, y);
  ptx::tma_load_2d(st + kTileBytes, tm_v, bar, 0, y);
  ptx::tma_load_2d(st + kTileBytes + kBoxBytes, tm_v, bar, 64, y);
}

// Attends one landed unit (K tile at kt, V tile at vt, `valid` leading tokens
// visible) into the warp state.  Warp-collective.
__device__ __forceinline__ void attend_unit(uint32_t kt, uint32_t vt, int valid,
                                            const uint32_t (&qa)[8][4], float sc, WarpState& w) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  const int mi = lane >> 3, ri = lane & 7;  // ldmatrix lane roles
  // S^T[head, token] for tokens 0-7 (s[0]) and 8-15 (s[1])
  float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    uint32_t r[4];
    const int tok = (mi >> 1) * 8 + ri;
    ptx::ldmatrix_x4(swz(kt, tok, kk * 2 + (mi & 1)), r);
    ptx::mma_bf16_16816(s[0], qa[kk], r[0], r[1]);
    ptx::mma_bf16_16816(s[1], qa[kk], r[2], r[3]);
  }
  // scale into log2 units, mask tokens past the query
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = nt * 8 + 2 * t + (e & 1);
      s[nt][e] = tok < valid ? s[nt][e] * sc : -CUDART_INF_F;
    }
  }
  float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
  float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float n0 = fmaxf(w.m0, mx0), n1 = fmaxf(w.m1, mx1);
  const float c0 = exp2f(w.m0 - n0), c1 = exp2f(w.m1 - n1);  // 0 while m is -inf
  w.m0 = n0;
  w.m1 = n1;
  float pr[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    pr[nt][0] = exp2f(s[nt][0] - n0);
    pr[nt][1] = exp2f(s[nt][1] - n0);
    pr[nt][2] = exp2f(s[nt][2] - n1);
    pr[nt][3] = exp2f(s[nt][3] - n1);
  }
  w.l0 = w.l0 * c0 + pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
  w.l1 = w.l1 * c1 + pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    w.o[j][0] *= c0; w.o[j][1] *= c0;
    w.o[j][2] *= c1; w.o[j][3] *= c1;
  }
  uint32_t pa[4];
  pa[0] = ptx::pack_bf16x2(pr[0][0], pr[0][1]);
  pa[1] = ptx::pack_bf16x2(pr[0][2], pr[0][3]);
  pa[2] = ptx::pack_bf16x2(pr[1][0], pr[1][1]);
  pa[3] = ptx::pack_bf16x2(pr[1][2], pr[1][3]);
  // Tokens past the query may hold anything (even NaN) in the cache: their V
  // rows must not reach the product, so zero them in the tile.
  if (valid < kUnit) {
    __syncwarp();
    for (int i = lane; i < (kUnit - valid) * 16; i += 32) {
      const int row = valid + i / 16, chunk = i % 16;
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(swz(vt, row, chunk)), "r"(0u));
    }
    ptx::fence_proxy_async();  // the stage is refilled by TMA later
    __syncwarp();
  }
#pragma unroll
  for (int nn = 0; nn < 8; ++nn) {
    uint32_t r[4];
    const int tok = (mi & 1) * 8 + ri;
    ptx::ldmatrix_x4_trans(swz(vt, tok, nn * 2 + (mi >> 1)), r);
    ptx::mma_bf16_16816(w.o[2 * nn], pa, r[0], r[1]);
    ptx::mma_bf16_16816(w.o[2 * nn + 1], pa, r[2], r[3]);
  }
  __syncwarp();
}

// Shared memory of the merge (besides the rings, which it reuses).
struct MergeSmem {
  float ml[kWarps][16][2];   // per-warp (m, l) of each query head
  float rml[8][16][2];       // rank 0: (m, l) pushed by each CTA of the cluster
};

// Merges the warps' partials (state w; `empty` when the warp attended nothing)
// into the CTA, then the CTAs of the cluster into rank 0, which writes out / lse
// of (b, KV head h).  `ring0` is the CTA's 1024-aligned ring area (every copy
// into it has landed).  Block- and cluster-collective.
template <typename TO>
__device__ void merge_and_store(WarpState& w, bool empty, uint8_t* ring0, MergeSmem& ms,
                                const LayerParams& p, int b, int h, TO* out, float* lse) {
  cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int n_cta = static_cast<int>(cluster.num_blocks());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, 1);
  w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, 2);
  w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, 1);
  w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, 2);
  // ---- merge 1: the CTA's warps, through shared memory (each warp's own ring)
  float* wo = reinterpret_cast<float*>(ring0 + warp * kWarpBytes);  // [16 heads][128]
  if (empty) {
    w.m0 = w.m1 = -CUDART_INF_F;
    w.l0 = w.l1 = 0.f;
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      *reinterpret_cast<float2*>(wo + g * kD + j * 8 + 2 * t) = make_float2(w.o[j][0], w.o[j][1]);
      *reinterpret_cast<float2*>(wo + (g + 8) * kD + j * 8 + 2 * t) =
          make_float2(w.o[j][2], w.o[j][3]);
    }
  }
  if (t == 0) {
    ms.ml[warp][g][0] = w.m0;
    ms.ml[warp][g][1] = w.l0;
    ms.ml[warp][g + 8][0] = w.m1;
    ms.ml[warp][g + 8][1] = w.l1;
  }
  __syncthreads();
  const int d = threadIdx.x;  // one output dim per thread (blockDim == D == 128)
  float cta_m[16], cta_l[16], cta_o[16];
#pragma unroll
  for (int hh = 0; hh < 16; ++hh) {
    cta_m[hh] = -CUDART_INF_F;
    cta_l[hh] = 0.f;
    cta_o[hh] = 0.f;
    if (hh >= p.G) continue;
    float mm = -CUDART_INF_F;
#pragma unroll
    for (int v = 0; v < kWarps; ++v) mm = fmaxf(mm, ms.ml[v][hh][0]);
    if (mm == -CUDART_INF_F) continue;
    float ll = 0.f, oo = 0.f;
#pragma unroll
    for (int v = 0; v < kWarps; ++v) {
      const float mw = ms.ml[v][hh][0];
      if (mw == -CUDART_INF_F) continue;
      const float f = exp2f(mw - mm);
      ll += ms.ml[v][hh][1] * f;
      oo += reinterpret_cast<const float*>(ring0 + v * kWarpBytes)[hh * kD + d] * f;
    }
    cta_m[hh] = mm;
    cta_l[hh] = ll;
    cta_o[hh] = oo;
  }
  // ---- merge 2: the cluster's CTAs.  After the first barrier every CTA has
  // finished reading its own ring, so rank 0's ring is free; every CTA then
  // pushes its partial into rank 0's ring (remote shared-memory stores), and
  // after the second barrier rank 0 merges from its own shared memory.
  cluster.sync();
  float* recv = cluster.map_shared_rank(reinterpret_cast<float*>(ring0), 0);  // [8][16][128]
  float(*recv_ml)[16][2] = cluster.map_shared_rank(ms.rml, 0);
#pragma unroll
  for (int hh = 0; hh < 16; ++hh) {
    if (hh >= p.G) continue;
    recv[(rank * 16 + hh) * kD + d] = cta_o[hh];
    if (d == 0) {
      recv_ml[rank][hh][0] = cta_m[hh];
      recv_ml[rank][hh][1] = cta_l[hh];
    }
  }
  cluster.sync();
  if (rank == 0) {
    const float* mine = reinterpret_cast<const float*>(ring0);
    for (int hh = 0; hh < p.G; ++hh) {
      float mm = -CUDART_INF_F;
      for (int r = 0; r < n_cta; ++r) mm = fmaxf(mm, ms.rml[r][hh][0]);
      float ll = 0.f, oo = 0.f;
      if (mm != -CUDART_INF_F) {
        for (int r = 0; r < n_cta; ++r) {
          const float mr = ms.rml[r][hh][0];
          if (mr == -CUDART_INF_F) continue;
          const float f = exp2f(mr - mm);
          ll += ms.rml[r][hh][1] * f;
          oo += mine[(r * 16 + hh) * kD + d] * f;
        }
      }
      const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + hh;
      store_out(out + row * kD + d, ll > 0.f ? oo / ll : 0.f);
      if (lse && d == 0) lse[row] = ll > 0.f ? (mm + log2f(ll)) * kLn2 : -CUDART_INF_F;
    }
  }
}

}  // namespace decode
}  // namespace hga
