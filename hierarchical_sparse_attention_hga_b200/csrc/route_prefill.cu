// Steps 2 and 3 for prefill: two-level routing of every query block of a
// prompt, eight consecutive blocks of one (sequence, KV head) per CTA.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", item 2: level 1 scores a query
// block against the chunk key summaries of the earlier chunks and keeps the
// top-kc; level 2 scores the group summaries inside those chunks and keeps the
// top-kg.  The sink, local and current chunks are always visible, so they are
// not candidates.
//
// Consecutive blocks see nearly the same candidate chunks (block j's are
// chunks sink .. cur_j - local - 1), so a CTA scores the union once for all
// its blocks: every summary row is read once per eight blocks instead of once
// per block and dotted with the eight routing queries held in shared memory.
// Each warp then owns one block: a warp top-k of its level-1 scores, then
// level 2 over the groups of its chunks.
//
// The routing query of a block is the mean of its G*C post-RoPE query rows,
// summed in a fixed order; the same kernel serves the level-1-only, the
// level-2-only and the fused call, so their results agree bit for bit.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kNB = kWarps;  // query blocks per CTA, one per warp after scoring

enum { kL1 = 1, kL2 = 2 };

// Dynamic shared memory in 4-byte words:
//   qbar [kNB][D] | scores [kNB][n_pad] | survivor keys, ids [kWarps][64] x 2 |
//   selected chunks [kNB][kc] | selected group positions [kNB][kg]
__host__ __device__ inline int prefill_route_pad(const LayerParams& p) {
  const int n = max(p.n_chunks, p.kc * p.Ng);
  return (n + 3) & ~3;
}
__host__ __device__ inline size_t prefill_route_words(const LayerParams& p) {
  return static_cast<size_t>(kNB) * p.D + static_cast<size_t>(kNB) * prefill_route_pad(p) +
         2 * kWarps * kWarpTopkList + static_cast<size_t>(kNB) * (p.kc + p.kg);
}

// 16 bytes of q as floats (a zero word widens to zeros in both types).
__device__ __forceinline__ void widen16(const uint4& v, float (&x)[4]) {
  x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
  x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void widen16(const uint4& v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// dst[0..D) = mean of the G*C query rows of block blk of (b, KV head h).
// Warp-collective.  The block's rows of one head are C*D contiguous elements,
// read 16 bytes per lane (a lane always meets the same VEC dimensions), sixteen
// loads in flight per lane.
template <typename T, int D>
__device__ void block_query_mean(const T* __restrict__ q, const LayerParams& p, int b, int h,
                                 int blk, float* dst) {
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
  constexpr int LPR = D / VEC;         // lanes per row
  constexpr int UNR = 16;
  const int lane = threadIdx.x & 31;
  const int seg = p.C * D / (32 * VEC);  // warp loads per head (C*D is a multiple of 32*VEC)
  float acc[VEC];
#pragma unroll
  for (int u = 0; u < VEC; ++u) acc[u] = 0.f;
  for (int hh = 0; hh < p.G; ++hh) {
    const uint4* src = reinterpret_cast<const uint4*>(
        q + ((static_cast<size_t>(b) * p.Hq + h * p.G + hh) * p.q_len +
             static_cast<size_t>(blk) * p.C) * D) + lane;
    for (int i0 = 0; i0 < seg; i0 += UNR) {
      uint4 x[UNR];
#pragma unroll
      for (int k = 0; k < UNR; ++k)
        x[k] = i0 + k < seg ? __ldg(src + (i0 + k) * 32) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int k = 0; k < UNR; ++k) {
        float f[VEC];
        widen16(x[k], f);
#pragma unroll
        for (int u = 0; u < VEC; ++u) acc[u] += f[u];
      }
    }
  }
  // lanes l, l + LPR, l + 2 LPR, ... hold the same dimensions
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int u = 0; u < VEC; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
  if (lane < LPR) {
    const float inv = 1.f / static_cast<float>(p.G * p.C);
#pragma unroll
    for (int u = 0; u < VEC; ++u) dst[lane * VEC + u] = acc[u] * inv;
  }
}

// a + x . y, in a fixed order.
__device__ __forceinline__ float dot4(const float4& x, const float4& y, float a) {
  a = fmaf(x.x, y.x, a);
  a = fmaf(x.y, y.y, a);
  a = fmaf(x.z, y.z, a);
  return fmaf(x.w, y.w, a);
}

// Sums v[j] over the eight lanes of an aligned lane octet for j = 0..7 and
// returns the sum of v[s8] in lane s8 of the octet (three exchange stages; each
// lane sends the half of its values that its partner keeps).
__device__ __forceinline__ float butterfly8(float (&v)[8], int s8) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = (s8 & 4) != 0;
    const float send = hi ? v[i] : v[i + 4], keep = hi ? v[i + 4] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = (s8 & 2) != 0;
    const float send = hi ? v[i] : v[i + 2], keep = hi ? v[i + 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  const bool hi = (s8 & 1) != 0;
  const float send = hi ? v[0] : v[1], keep = hi ? v[1] : v[0];
  return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kThreads, 2)
route_prefill_kernel(const T* __restrict__ q, const int64_t* __restrict__ pos,
                     const float* __restrict__ chunk_sum, const float* __restrict__ group_sum,
                     LayerParams p, int32_t* __restrict__ chunk_idx, float* __restrict__ chunk_score,
                     int32_t* __restrict__ group_idx, float* __restrict__ group_score,
                     unsigned* err) {
  extern __shared__ __align__(16) float dyn[];
  const int n_pad = prefill_route_pad(p);
  float* qb = dyn;                                                  // [kNB][D]
  float* sc = qb + kNB * D;                                         // [kNB][n_pad]
  unsigned* lkey = reinterpret_cast<unsigned*>(sc + static_cast<size_t>(kNB) * n_pad);
  int* lidx = reinterpret_cast<int*>(lkey + kWarps * kWarpTopkList);
  int* csel = lidx + kWarps * kWarpTopkList;                        // [kNB][kc]
  int* gpos = csel + kNB * p.kc;                                    // [kNB][kg]

  constexpr int kF4 = D / 32;  // float4 columns of a row per lane (eight lanes per row)
  constexpr int kUnr1 = 2;     // level 1: passes of four rows in flight per warp
  constexpr int kUnr2 = 4;     // level 2: the same
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane >> 3, s8 = lane & 7;  // row of the warp's four, lane within the row
  const int groups = (p.nblk + kNB - 1) / kNB;
  const int bh = blockIdx.x / groups, j0 = (blockIdx.x % groups) * kNB;
  const int h = bh % p.Hkv, b = bh / p.Hkv;
  const int nb = min(kNB, p.nblk - j0);
  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, threadIdx.x == 0 && j0 == 0 ? err : nullptr);
  const int chunk0 = ok ? static_cast<int>((pb - p.q_len + 1) / p.C) : 0;  // block 0's chunk

  // routing queries (q is an input, never written by this library)
  if (ok && warp < nb) block_query_mean<T, D>(q, p, b, h, j0 + warp, qb + warp * D);
  else
    for (int d = lane; d < D; d += 32) qb[warp * D + d] = 0.f;
  pdl_wait();  // the summaries may come from the kernel just before
  __syncthreads();

  const int j = warp, blk = j0 + j;
  const int cur = chunk0 + blk;
  const int n_cand = ok && j < nb ? max(0, cur - p.local - p.sink) : 0;
  int* cs = csel + j * p.kc;
  int ns = 0;

  if constexpr ((MODE & kL1) != 0) {
    // ---- level 1: the union of the blocks' candidates, scored once.  Eight
    // lanes share a summary row (lane s8 of the eight holds its float4 columns
    // s8, s8 + 8, ...), so rows are read in coalesced 128-byte pieces, four rows
    // per warp and pass; the eight lanes' partial dot products with the eight
    // routing queries are then summed by a butterfly that leaves block s8's
    // score in lane s8.
    const int n_union = ok ? max(0, chunk0 + j0 + nb - 1 - p.local - p.sink) : 0;
    const float4* rows4 =
        reinterpret_cast<const float4*>(chunk_sum + (static_cast<size_t>(bh) * p.n_chunks + p.sink) * D);
    const float4* qb4 = reinterpret_cast<const float4*>(qb);
    for (int r0 = warp * 4 * kUnr1; r0 < n_union; r0 += kWarps * 4 * kUnr1) {
      float4 x[kUnr1][kF4];
#pragma unroll
      for (int u = 0; u < kUnr1; ++u) {
        const int i = min(r0 + u * 4 + sub, n_union - 1);
#pragma unroll
        for (int k = 0; k < kF4; ++k) x[u][k] = __ldg(rows4 + static_cast<size_t>(i) * (D / 4) + s8 + 8 * k);
      }
      float acc[kUnr1][kNB];
#pragma unroll
      for (int jj = 0; jj < kNB; ++jj) {
#pragma unroll
        for (int u = 0; u < kUnr1; ++u) acc[u][jj] = 0.f;
#pragma unroll
        for (int k = 0; k < kF4; ++k) {
          const float4 qv = qb4[jj * (D / 4) + s8 + 8 * k];
#pragma unroll
          for (int u = 0; u < kUnr1; ++u) acc[u][jj] = dot4(x[u][k], qv, acc[u][jj]);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnr1; ++u) {
        const float v = butterfly8(acc[u], s8);
        const int i = r0 + u * 4 + sub;
        if (i < n_union) sc[static_cast<size_t>(s8) * n_pad + i] = v;
      }
    }
    __syncthreads();
    // ---- level-1 top-k, one warp per block
    float* s = sc + static_cast<size_t>(j) * n_pad;
    ns = warp_topk(s, n_cand, p.kc, cs, lkey + warp * kWarpTopkList, lidx + warp * kWarpTopkList);
    if (j < nb) {
      const size_t item = static_cast<size_t>(bh) * p.nblk + blk;
      for (int i = lane; i < p.kc; i += 32) {
        const bool have = ok && i < ns;
        const int c = have ? cs[i] + p.sink : -1;
        chunk_idx[item * p.kc + i] = c;
        if (chunk_score) chunk_score[item * p.kc + i] = have ? s[cs[i]] : CUDART_NAN_F;
      }
    }
    __syncwarp();
    for (int i = lane; i < ns; i += 32) cs[i] += p.sink;  // chunk ids
    __syncwarp();
  } else {
    // ---- level 2 only: the chunks come from chunk_idx (validated)
    if (ok && j < nb) {
      bool bad = false;
      const int32_t* cidx = chunk_idx + (static_cast<size_t>(bh) * p.nblk + blk) * p.kc;
      ns = warp_keep_ascending(
          cidx, p.kc, [&](int c) { return c >= p.sink && c < cur - p.local; }, cs, &bad);
      if (bad && lane == 0) flag_error(err, kErrChunkIdx);
    }
    __syncwarp();
  }

  if constexpr ((MODE & kL2) != 0) {
    // ---- level 2: the groups of the block's chunks, one warp per block
    if (j < nb) {
      float* gs = sc + static_cast<size_t>(j) * n_pad;  // level-1 scores are consumed
      const int n_g = ok ? ns * p.Ng : 0;
      const float* gbase = group_sum + static_cast<size_t>(bh) * p.n_chunks * p.Ng * D;
      float4 qv[kF4];  // this lane's columns of the block's routing query
#pragma unroll
      for (int k = 0; k < kF4; ++k) qv[k] = reinterpret_cast<const float4*>(qb + j * D)[s8 + 8 * k];
      const float4* g4 = reinterpret_cast<const float4*>(gbase);
      for (int r0 = 0; r0 < n_g; r0 += 4 * kUnr2) {
        float4 x[kUnr2][kF4];
#pragma unroll
        for (int u = 0; u < kUnr2; ++u) {
          const int i = min(r0 + u * 4 + sub, n_g - 1);
          const size_t row = static_cast<size_t>(cs[i / p.Ng]) * p.Ng + i % p.Ng;
#pragma unroll
          for (int k = 0; k < kF4; ++k) x[u][k] = __ldg(g4 + row * (D / 4) + s8 + 8 * k);
        }
#pragma unroll
        for (int u = 0; u < kUnr2; ++u) {
          float a = 0.f;
#pragma unroll
          for (int k = 0; k < kF4; ++k) a = dot4(x[u][k], qv[k], a);
          a += __shfl_xor_sync(0xffffffffu, a, 4);  // the same sum in all eight lanes
          a += __shfl_xor_sync(0xffffffffu, a, 2);
          a += __shfl_xor_sync(0xffffffffu, a, 1);
          const int i = r0 + u * 4 + sub;
          if (s8 == 0 && i < n_g) gs[i] = a;
        }
      }
      __syncwarp();
      int* gout_pos = gpos + j * p.kg;
      const int ng = warp_topk(gs, n_g, p.kg, gout_pos, lkey + warp * kWarpTopkList,
                               lidx + warp * kWarpTopkList);
      const size_t item = static_cast<size_t>(bh) * p.nblk + blk;
      for (int i = lane; i < p.kg; i += 32) {
        const bool have = ok && i < ng;
        const int s = have ? gout_pos[i] : 0;
        group_idx[item * p.kg + i] = have ? cs[s / p.Ng] * p.Ng + s % p.Ng : -1;
        if (group_score) group_score[item * p.kg + i] = have ? gs[s] : CUDART_NAN_F;
      }
    }
  }
  pdl_trigger();
}

template <typename T, int D, int MODE>
cudaError_t launch_t(const LayerParams& p, const void* q, const int64_t* pos,
                     const float* chunk_sum, const float* group_sum, int32_t* chunk_idx,
                     float* chunk_score, int32_t* group_idx, float* group_score, unsigned* err,
                     cudaStream_t s) {
  const size_t smem = prefill_route_words(p) * 4;
  cudaError_t e = ensure_smem<route_prefill_kernel<T, D, MODE>>(smem);
  if (e != cudaSuccess) return e;
  const int groups = (p.nblk + kNB - 1) / kNB;
  return launch_pdl(route_prefill_kernel<T, D, MODE>, dim3(p.B * p.Hkv * groups), dim3(kThreads),
                    smem, s, 1, static_cast<const T*>(q), pos, chunk_sum, group_sum, p, chunk_idx,
                    chunk_score, group_idx, group_score, err);
}

template <int MODE>
cudaError_t launch_mode(const LayerParams& p, int dtype, const void* q, const int64_t* pos,
                        const float* chunk_sum, const float* group_sum, int32_t* chunk_idx,
                        float* chunk_score, int32_t* group_idx, float* group_score, unsigned* err,
                        cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (dtype == 0)
    return p.D == 64 ? launch_t<float, 64, MODE>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s)
                     : launch_t<float, 128, MODE>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s);
  return p.D == 64 ? launch_t<bf, 64, MODE>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s)
                   : launch_t<bf, 128, MODE>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s);
}

}  // namespace

bool prefill_route_path(const LayerParams& p, int dtype) {
  const int elem = dtype == 0 ? 4 : 2;
  return p.q_len > 1 && (p.D == 64 || p.D == 128) && (p.C * p.D * elem) % 512 == 0 &&
         prefill_route_words(p) * 4 <= 200 * 1024;
}

cudaError_t launch_route_prefill(const LayerParams& p, int dtype, bool level1, bool level2,
                                 const void* q, const int64_t* pos, const float* chunk_sum,
                                 const float* group_sum, int32_t* chunk_idx, float* chunk_score,
                                 int32_t* group_idx, float* group_score, unsigned* err,
                                 cudaStream_t s) {
  if (level1 && level2)
    return launch_mode<kL1 | kL2>(p, dtype, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score,
                                  group_idx, group_score, err, s);
  if (level1)
    return launch_mode<kL1>(p, dtype, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score,
                            group_idx, group_score, err, s);
  return launch_mode<kL2>(p, dtype, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score,
                          group_idx, group_score, err, s);
}

}  // namespace hga
