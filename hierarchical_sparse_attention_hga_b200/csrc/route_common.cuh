// Routing building blocks of the 128-thread decode kernels (route_decode.cu and
// the one-launch decode step in decode_step.cu): the routing query, summary-row
// scoring and the top-k, so that both kernels compute identical scores and
// selections.
#pragma once

#include "common.cuh"
#include "topk.cuh"

namespace hga {
namespace route {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;

__host__ __device__ constexpr int round4(int n) { return (n + 3) & ~3; }

// qbar[0..D) = mean of the G query heads' rows of (b, KV head h) of a decode
// query (q [B, Hq, 1, D]), summed in head order.  Block-collective writes; the
// caller synchronises before reading qbar.
template <typename T, int D>
__device__ __forceinline__ void decode_query_mean(const T* __restrict__ q, const LayerParams& p,
                                                  int b, int h, float* qbar) {
  for (int d = threadIdx.x; d < D; d += kThreads) {
    float s = 0.f;
    for (int hh = 0; hh < p.G; ++hh)
      s += to_f32(q[(static_cast<size_t>(b) * p.Hq + h * p.G + hh) * D + d]);
    qbar[d] = s / static_cast<float>(p.G);
  }
}

// Scores n summary rows, row(i) a float4 pointer to D floats, against qv (this
// lane's float4 columns s8, s8 + 8, ... of the query, s8 = lane % 8) into
// sc[0..n).  Eight lanes share a row, four rows per warp and pass, UNR passes
// of loads in flight; each row's dot product is summed in a fixed order.
template <int D, int UNR, typename RowFn>
__device__ __forceinline__ void score_rows8(int n, const float4 (&qv)[D / 32], float* sc, RowFn row) {
  constexpr int F4 = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane >> 3, s8 = lane & 7;
  for (int r0 = warp * 4 * UNR; r0 < n; r0 += kWarps * 4 * UNR) {
    float4 x[UNR][F4];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const float4* src = row(min(r0 + u * 4 + sub, n - 1));
#pragma unroll
      for (int k = 0; k < F4; ++k) x[u][k] = __ldg(src + s8 + 8 * k);
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < F4; ++k) {
        a = fmaf(x[u][k].x, qv[k].x, a);
        a = fmaf(x[u][k].y, qv[k].y, a);
        a = fmaf(x[u][k].z, qv[k].z, a);
        a = fmaf(x[u][k].w, qv[k].w, a);
      }
      a += __shfl_xor_sync(0xffffffffu, a, 4);  // the same sum in all eight lanes
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      const int i = r0 + u * 4 + sub;
      if (s8 == 0 && i < n) sc[i] = a;
    }
  }
}

constexpr int kRankMax = kThreads;  // rank-count top-k up to this many candidates

// Top-k of sc[0..n), n <= kRankMax, by rank counting: thread t owns the
// candidates [t * ipt, (t + 1) * ipt) and takes each one that fewer than k
// candidates beat (j beats i if s_j > s_i, or s_j == s_i and j < i); the taken
// indices are then compacted in index order.  Block-collective; sc is 16-byte
// aligned shared memory; s_cnt holds kWarps ints.
__device__ __forceinline__ int cta_rank_topk(const float* sc, int n, int k, int* out, int* s_cnt) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int ipt = (n + kThreads - 1) / kThreads;  // 1..4
  const int beg = min(n, t * ipt), end = min(n, beg + ipt);
  unsigned take = 0u;
  for (int i = beg; i < end; ++i) {
    const float si = sc[i];
    int beats = 0;
    int j = 0;
#pragma unroll 4
    for (; j + 4 <= n; j += 4) {
      const float4 x = *reinterpret_cast<const float4*>(sc + j);
      beats += (x.x > si || (x.x == si && j < i)) + (x.y > si || (x.y == si && j + 1 < i)) +
               (x.z > si || (x.z == si && j + 2 < i)) + (x.w > si || (x.w == si && j + 3 < i));
    }
    for (; j < n; ++j) beats += sc[j] > si || (sc[j] == si && j < i);
    if (beats < k) take |= 1u << (i - beg);
  }
  // exclusive prefix of the taken counts over threads (warp scan, then warps)
  const int c = __popc(take);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) s_cnt[w] = incl;
  __syncthreads();
  int at = incl - c, total = 0;
#pragma unroll
  for (int x = 0; x < kWarps; ++x) {
    if (x < w) at += s_cnt[x];
    total += s_cnt[x];
  }
  for (int i = beg; i < end; ++i)
    if (take >> (i - beg) & 1u) out[at++] = i;
  __syncthreads();
  return total;
}

// Top-k of sc[0..n) (ties to the lower index) into out[0..), ascending; block-
// collective, out complete on return.  Up to kRankMax candidates (every decode
// set of the usual shapes) by rank counting over the 128 threads; larger sets
// by one warp's threshold top-k.
__device__ __forceinline__ int cta_topk(const float* sc, int n, int k, int* out, unsigned* lkey,
                                        int* lidx, int* s_n) {
  if (n <= kRankMax) return cta_rank_topk(sc, n, k, out, s_n);
  if ((threadIdx.x >> 5) == 0) {
    const int r = warp_topk(sc, n, k, out, lkey, lidx);
    if ((threadIdx.x & 31) == 0) *s_n = r;
  }
  __syncthreads();
  const int r = *s_n;
  __syncthreads();
  return r;
}

}  // namespace route
}  // namespace hga
