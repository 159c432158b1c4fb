// Steps 2 and 3: two-level routing.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", item 2: level 1 scores the
// current block against the compact table of chunk key summaries of earlier
// chunks; level 2 scores the group summaries inside the selected chunks.  The
// sink, local and current chunks are always visible, so they are not
// candidates: content routing covers the intermediate context only.
//
// This file holds the general routing kernels and the entry points' dispatch:
// decode goes to route_decode.cu and prefill to route_prefill.cu whenever their
// shared-memory layouts fit (every shape up to millions of tokens); the kernels
// below serve the rest.
//
// One cluster per (sequence, KV head, query block).  The routing query is the mean
// of the block's post-RoPE query rows over the G heads sharing the KV head,
// summed in a fixed order (deterministic).  Summary rows are streamed with
// 16-byte loads, one row per D/4 lanes, eight rows in flight per lane; scores
// land in shared memory and a block radix select keeps the top-k.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Below this many candidates the one-pass rank count beats the 4-pass radix
// select; above it the rank count's O(n) serial compare chain per thread loses.
constexpr int kRankTopkMax = 128;

// qbar[0..D) = mean of the q rows (G heads x nr rows) of (b, KV head h).
template <typename T, int D>
__device__ void routing_query(const T* __restrict__ q, const LayerParams& p, int b, int h, int r0,
                              int nr, float* qbar, float (*part)[D]) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float acc[DPL];
#pragma unroll
  for (int u = 0; u < DPL; ++u) acc[u] = 0.f;
  const int rows = p.G * nr;
  for (int r = wid; r < rows; r += kWarps) {
    const int hh = r / nr, rr = r % nr;
    const T* src = q + ((static_cast<size_t>(b) * p.Hq + h * p.G + hh) * p.q_len + r0 + rr) * D +
                   lane * DPL;
    float x[DPL];
    if constexpr (DPL == 4) load4(src, x); else load2(src, x);
#pragma unroll
    for (int u = 0; u < DPL; ++u) acc[u] += x[u];
  }
#pragma unroll
  for (int u = 0; u < DPL; ++u) part[wid][lane * DPL + u] = acc[u];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += part[w][threadIdx.x];
    qbar[threadIdx.x] = s / static_cast<float>(rows);
  }
  __syncthreads();
}

// sc[i] = qbar . row(i) for i < n; row(i) returns a pointer to D floats (16 B aligned).
template <int D, typename RowFn>
__device__ void score_rows(int n, const float* qbar, float* sc, RowFn row) {
  constexpr int LPR = D / 4;          // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp step
  constexpr int UNR = 8;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int sub = lane / LPR, l = lane % LPR;
  const float4 qv = reinterpret_cast<const float4*>(qbar)[l];
  const int step = kWarps * RPW;
  // The loop bound is uniform across the warp (all lanes join the shuffles);
  // rows past n are masked per lane.
  for (int wbase = wid * RPW; wbase < n; wbase += step * UNR) {
    const int base = wbase + sub;
    float4 v[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = base + u * step;
      v[u] = i < n ? __ldg(reinterpret_cast<const float4*>(row(i)) + l) : make_float4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      float d = v[u].x * qv.x + v[u].y * qv.y + v[u].z * qv.z + v[u].w * qv.w;
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      const int i = base + u * step;
      if (l == 0 && i < n) sc[i] = d;
    }
  }
}

// Decode (q_len == 1): one block, the query's chunk.  Prefill: block blk holds
// queries blk*C .. blk*C+C-1 and its current chunk is their chunk.
__device__ __forceinline__ void block_rows(const LayerParams& p, int64_t pos, int blk, int* r0,
                                           int* nr, int* cur) {
  const int64_t first = pos - p.q_len + 1;
  *r0 = p.q_len == 1 ? 0 : blk * p.C;
  *nr = p.q_len == 1 ? 1 : p.C;
  *cur = static_cast<int>((first + *r0 + *nr - 1) / p.C);
}

// Dynamic shared memory of route_chunks_kernel, in 4-byte words (every part a
// multiple of 4 words, so each part stays 16-byte aligned):
//   local [per] | lsel [lsel_n] | pushed scores, pushed ids, merged scores,
//   merged ids [4 x 8 x kc4] | sel [kc4]
struct RouteSmem {
  int per, lsel_n, kc4;
  __host__ __device__ size_t words() const { return per + lsel_n + 4 * 8 * kc4 + kc4; }
};
__host__ __device__ inline RouteSmem route_smem(const LayerParams& p, int cl, bool fuse) {
  RouteSmem L;
  L.kc4 = (p.kc + 3) & ~3;
  L.per = ((p.n_chunks + cl - 1) / cl + 3) & ~3;
  if (fuse && L.per < p.kc * p.Ng) L.per = (p.kc * p.Ng + 3) & ~3;  // level-2 scores reuse it
  L.lsel_n = fuse && p.kg > L.kc4 ? ((p.kg + 3) & ~3) : L.kc4;       // level-2 ids reuse it
  return L;
}

// One cluster of `cl` CTAs per (sequence, KV head, block): CTA r scores the
// r-th slice of the candidates and selects that slice's top-kc, then pushes
// those (score, index) pairs into CTA 0's shared memory (distributed shared
// memory stores).  CTA 0 takes the top-kc of the pushed pairs: the global
// top-kc is always among the slices' top-kc, and the slices are pushed in
// candidate order, so ties still go to the lower index.  With FUSE, CTA 0
// continues into level 2 (the work of route_groups_kernel) with the selected
// chunks still in shared memory; results are identical to the two launches.
template <typename T, int D, bool FUSE>
__global__ void __launch_bounds__(kThreads)
route_chunks_kernel(const T* __restrict__ q, const int64_t* __restrict__ pos,
                    const float* __restrict__ chunk_sum, const float* __restrict__ group_sum,
                    LayerParams p, int32_t* __restrict__ chunk_idx,
                    float* __restrict__ chunk_score, int32_t* __restrict__ group_idx,
                    float* __restrict__ group_score, unsigned* err) {
  __shared__ __align__(16) float qbar[D];
  __shared__ float part[kWarps][D];
  __shared__ TopkSmem tsm;
  __shared__ int s_cnt[8];
  extern __shared__ __align__(16) float dyn[];
  cg::cluster_group cluster = cg::this_cluster();
  cluster.barrier_arrive();  // paired with barrier_wait() before the first remote store
  const int cl = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int item = blockIdx.x / cl;
  const int blk = item % p.nblk;
  const int bh = item / p.nblk;
  const int h = bh % p.Hkv, b = bh / p.Hkv;
  int32_t* out = chunk_idx + static_cast<size_t>(item) * p.kc;
  float* out_sc = chunk_score ? chunk_score + static_cast<size_t>(item) * p.kc : nullptr;
  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, threadIdx.x == 0 && rank == 0 ? err : nullptr);
  int r0 = 0, nr = 0, cur = 0;
  if (ok) {
    block_rows(p, pb, blk, &r0, &nr, &cur);
    routing_query<T, D>(q, p, b, h, r0, nr, qbar, part);  // q is never written by this library
  }
  pdl_wait();

  const int n_cand = ok ? max(0, cur - p.local - p.sink) : 0;
  const RouteSmem L = route_smem(p, cl, FUSE);
  const int kc4 = L.kc4;
  float* local = dyn;                                             // [per]
  int* lsel = reinterpret_cast<int*>(local + L.per);              // [lsel_n]
  float* rsc = reinterpret_cast<float*>(lsel + L.lsel_n);         // [8 * kc4] pushed scores
  int* ridx = reinterpret_cast<int*>(rsc + 8 * kc4);              // [8 * kc4] pushed indices
  float* msc = reinterpret_cast<float*>(ridx + 8 * kc4);          // [8 * kc4] merged, compact
  int* midx = reinterpret_cast<int*>(msc + 8 * kc4);              // [8 * kc4]
  int* sel = reinterpret_cast<int*>(midx + 8 * kc4);              // [kc4]
  const int slice = (n_cand + cl - 1) / cl;
  const int lo = min(n_cand, rank * slice), hi = min(n_cand, lo + slice);
  const float* rows = chunk_sum + (static_cast<size_t>(bh) * p.n_chunks + p.sink + lo) * D;
  score_rows<D>(hi - lo, qbar, local, [&](int i) { return rows + static_cast<size_t>(i) * D; });
  __syncthreads();
  const int nl = hi - lo <= kRankTopkMax ? block_topk_rank<kThreads>(local, hi - lo, p.kc, lsel, tsm)
                                         : block_topk<kThreads>(local, hi - lo, p.kc, lsel, tsm);
  cluster.barrier_wait();  // every CTA of the cluster is running
  {
    float* dst_sc = cluster.map_shared_rank(rsc, 0);
    int* dst_idx = cluster.map_shared_rank(ridx, 0);
    for (int j = threadIdx.x; j < nl; j += kThreads) {
      dst_sc[rank * kc4 + j] = local[lsel[j]];
      dst_idx[rank * kc4 + j] = lo + lsel[j];
    }
    if (threadIdx.x == 0) cluster.map_shared_rank(s_cnt, 0)[rank] = nl;
  }
  cluster.sync();  // pushes visible to CTA 0
  if (rank != 0) return;
  int32_t* gout = FUSE ? group_idx + static_cast<size_t>(item) * p.kg : nullptr;
  float* gout_sc = FUSE && group_score ? group_score + static_cast<size_t>(item) * p.kg : nullptr;
  if (!ok) {
    for (int i = threadIdx.x; i < p.kc; i += kThreads) {
      out[i] = -1;
      if (out_sc) out_sc[i] = CUDART_NAN_F;
    }
    if constexpr (FUSE) {
      for (int i = threadIdx.x; i < p.kg; i += kThreads) {
        gout[i] = -1;
        if (gout_sc) gout_sc[i] = CUDART_NAN_F;
      }
    }
    return;
  }
  // compact the pushed lists in rank order (= ascending candidate index)
  int n_m = 0;
  for (int r = 0; r < cl; ++r) {
    const int c = s_cnt[r];
    for (int j = threadIdx.x; j < c; j += kThreads) {
      msc[n_m + j] = rsc[r * kc4 + j];
      midx[n_m + j] = ridx[r * kc4 + j];
    }
    n_m += c;
  }
  __syncthreads();
  const int ns = n_m <= kRankTopkMax ? block_topk_rank<kThreads>(msc, n_m, p.kc, sel, tsm)
                                     : block_topk<kThreads>(msc, n_m, p.kc, sel, tsm);
  for (int i = threadIdx.x; i < p.kc; i += kThreads) {
    out[i] = i < ns ? midx[sel[i]] + p.sink : -1;
    if (out_sc) out_sc[i] = i < ns ? msc[sel[i]] : CUDART_NAN_F;
  }
  pdl_trigger();  // the other CTAs of the cluster have exited
  if constexpr (FUSE) {
    // level 2 over the groups of the ns selected chunks (ascending chunk ids)
    float* gsc = local;                                      // reuse: [kc * Ng] (fits: see launcher)
    int* gsel = lsel;                                        // reuse: [kg]
    const int n_g = ns * p.Ng;
    const float* gbase = group_sum + static_cast<size_t>(bh) * p.n_chunks * p.Ng * D;
    __syncthreads();  // everyone is done with local / lsel
    score_rows<D>(n_g, qbar, gsc, [&](int i) {
      const int c = midx[sel[i / p.Ng]] + p.sink, gi = i % p.Ng;
      return gbase + (static_cast<size_t>(c) * p.Ng + gi) * D;
    });
    __syncthreads();
    const int ng = n_g <= kRankTopkMax ? block_topk_rank<kThreads>(gsc, n_g, p.kg, gsel, tsm)
                                       : block_topk<kThreads>(gsc, n_g, p.kg, gsel, tsm);
    for (int i = threadIdx.x; i < p.kg; i += kThreads) {
      if (i < ng) {
        const int sidx = gsel[i];
        gout[i] = (midx[sel[sidx / p.Ng]] + p.sink) * p.Ng + sidx % p.Ng;
        if (gout_sc) gout_sc[i] = gsc[sidx];
      } else {
        gout[i] = -1;
        if (gout_sc) gout_sc[i] = CUDART_NAN_F;
      }
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
route_groups_kernel(const T* __restrict__ q, const int64_t* __restrict__ pos,
                    const float* __restrict__ group_sum, const int32_t* __restrict__ chunk_idx,
                    LayerParams p, int32_t* __restrict__ group_idx,
                    float* __restrict__ group_score, unsigned* err) {
  __shared__ __align__(16) float qbar[D];
  __shared__ float part[kWarps][D];
  __shared__ TopkSmem tsm;
  __shared__ int n_sel;
  extern __shared__ __align__(16) float dyn[];
  const int item = blockIdx.x;
  const int blk = item % p.nblk;
  const int bh = item / p.nblk;
  const int h = bh % p.Hkv, b = bh / p.Hkv;
  int32_t* out = group_idx + static_cast<size_t>(item) * p.kg;
  float* out_sc = group_score ? group_score + static_cast<size_t>(item) * p.kg : nullptr;
  const int64_t pb = pos[b];
  if (!valid_position(pb, p, threadIdx.x == 0 ? err : nullptr)) {
    pdl_wait();
    for (int i = threadIdx.x; i < p.kg; i += kThreads) {
      out[i] = -1;
      if (out_sc) out_sc[i] = CUDART_NAN_F;
    }
    return;
  }
  int r0, nr, cur;
  block_rows(p, pb, blk, &r0, &nr, &cur);
  routing_query<T, D>(q, p, b, h, r0, nr, qbar, part);  // q is never written by this library
  pdl_wait();

  const int n_cand_max = p.kc * p.Ng;
  float* sc = dyn;                                        // [kc * Ng]
  int* sel = reinterpret_cast<int*>(dyn + n_cand_max);    // [kg]
  int* chunks = sel + p.kg;                               // [kc]
  const int32_t* cidx = chunk_idx + static_cast<size_t>(item) * p.kc;
  if (threadIdx.x < 32) {
    // Keep the ascending complete candidate chunks; flag anything else.
    bool bad = false;
    const int n = warp_keep_ascending(
        cidx, p.kc, [&](int c) { return c >= p.sink && c < cur - p.local; }, chunks, &bad);
    if (threadIdx.x == 0) {
      n_sel = n;
      if (bad) flag_error(err, kErrChunkIdx);
    }
  }
  __syncthreads();

  const int n_cand = n_sel * p.Ng;
  const float* base = group_sum + static_cast<size_t>(bh) * p.n_chunks * p.Ng * D;
  score_rows<D>(n_cand, qbar, sc, [&](int i) {
    const int c = chunks[i / p.Ng], gi = i % p.Ng;
    return base + (static_cast<size_t>(c) * p.Ng + gi) * D;
  });
  __syncthreads();
  const int ns = n_cand <= kRankTopkMax ? block_topk_rank<kThreads>(sc, n_cand, p.kg, sel, tsm)
                                       : block_topk<kThreads>(sc, n_cand, p.kg, sel, tsm);
  for (int i = threadIdx.x; i < p.kg; i += kThreads) {
    if (i < ns) {
      const int s = sel[i];
      out[i] = chunks[s / p.Ng] * p.Ng + s % p.Ng;
      if (out_sc) out_sc[i] = sc[s];
    } else {
      out[i] = -1;
      if (out_sc) out_sc[i] = CUDART_NAN_F;
    }
  }
  pdl_trigger();
}

// CTAs per cluster for the chunk scan: at most 8 (the portable cluster size),
// no more CTAs in total than fit at once (4 per SM), slices of >= 32 rows.
int chunk_cluster_size(const LayerParams& p) {
  const int64_t items = static_cast<int64_t>(p.B) * p.Hkv * p.nblk;
  const int64_t sms = device_sm_count();
  int cl = 1;
  while (cl < 8 && items * cl * 2 <= sms * 4 && p.n_chunks / (cl * 2) >= 32) cl *= 2;
  return cl;
}

template <typename T, int D, bool FUSE>
cudaError_t launch_route_chunks_t(const LayerParams& p, const void* q, const int64_t* pos,
                                  const float* chunk_sum, const float* group_sum,
                                  int32_t* chunk_idx, float* chunk_score, int32_t* group_idx,
                                  float* group_score, unsigned* err, cudaStream_t s) {
  const int cl = chunk_cluster_size(p);
  const size_t smem = route_smem(p, cl, FUSE).words() * 4;
  cudaError_t e = ensure_smem<route_chunks_kernel<T, D, FUSE>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(route_chunks_kernel<T, D, FUSE>, dim3(p.B * p.Hkv * p.nblk * cl),
                    dim3(kThreads), smem, s, cl, static_cast<const T*>(q), pos, chunk_sum,
                    group_sum, p, chunk_idx, chunk_score, group_idx, group_score, err);
}

template <typename T, int D>
cudaError_t launch_route_groups_t(const LayerParams& p, const void* q, const int64_t* pos,
                                  const float* group_sum, const int32_t* chunk_idx,
                                  int32_t* group_idx, float* group_score, unsigned* err,
                                  cudaStream_t s) {
  const size_t smem = static_cast<size_t>(p.kc) * p.Ng * sizeof(float) +
                      static_cast<size_t>(p.kg + p.kc) * sizeof(int);
  cudaError_t e = ensure_smem<route_groups_kernel<T, D>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(route_groups_kernel<T, D>, dim3(p.B * p.Hkv * p.nblk), dim3(kThreads), smem,
                    s, 1, static_cast<const T*>(q), pos, group_sum, chunk_idx, p, group_idx,
                    group_score, err);
}

}  // namespace

cudaError_t launch_route_chunks(const LayerParams& p, int dtype, const void* q, const int64_t* pos,
                                const float* chunk_sum, int32_t* chunk_idx, float* chunk_score,
                                unsigned* err, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (prefill_route_path(p, dtype))
    return launch_route_prefill(p, dtype, true, false, q, pos, chunk_sum, nullptr, chunk_idx,
                                chunk_score, nullptr, nullptr, err, s);
  if (decode_route_path(p))
    return launch_route_decode(p, dtype, true, false, q, pos, chunk_sum, nullptr, chunk_idx,
                               chunk_score, nullptr, nullptr, err, s);
  if (dtype == 0)
    return p.D == 64 ? launch_route_chunks_t<float, 64, false>(p, q, pos, chunk_sum, nullptr, chunk_idx, chunk_score, nullptr, nullptr, err, s)
                     : launch_route_chunks_t<float, 128, false>(p, q, pos, chunk_sum, nullptr, chunk_idx, chunk_score, nullptr, nullptr, err, s);
  return p.D == 64 ? launch_route_chunks_t<bf, 64, false>(p, q, pos, chunk_sum, nullptr, chunk_idx, chunk_score, nullptr, nullptr, err, s)
                   : launch_route_chunks_t<bf, 128, false>(p, q, pos, chunk_sum, nullptr, chunk_idx, chunk_score, nullptr, nullptr, err, s);
}

cudaError_t launch_route(const LayerParams& p, int dtype, const void* q, const int64_t* pos,
                         const float* chunk_sum, const float* group_sum, int32_t* chunk_idx,
                         float* chunk_score, int32_t* group_idx, float* group_score,
                         unsigned* err, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (prefill_route_path(p, dtype))
    return launch_route_prefill(p, dtype, true, true, q, pos, chunk_sum, group_sum, chunk_idx,
                                chunk_score, group_idx, group_score, err, s);
  if (decode_route_path(p))
    return launch_route_decode(p, dtype, true, true, q, pos, chunk_sum, group_sum, chunk_idx,
                               chunk_score, group_idx, group_score, err, s);
  if (dtype == 0)
    return p.D == 64 ? launch_route_chunks_t<float, 64, true>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s)
                     : launch_route_chunks_t<float, 128, true>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s);
  return p.D == 64 ? launch_route_chunks_t<bf, 64, true>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s)
                   : launch_route_chunks_t<bf, 128, true>(p, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx, group_score, err, s);
}

cudaError_t launch_route_groups(const LayerParams& p, int dtype, const void* q, const int64_t* pos,
                                const float* group_sum, const int32_t* chunk_idx,
                                int32_t* group_idx, float* group_score, unsigned* err,
                                cudaStream_t s) {
  if (prefill_route_path(p, dtype))
    return launch_route_prefill(p, dtype, false, true, q, pos, nullptr, group_sum,
                                const_cast<int32_t*>(chunk_idx), nullptr, group_idx, group_score,
                                err, s);
  if (decode_route_path(p))
    return launch_route_decode(p, dtype, false, true, q, pos, nullptr, group_sum,
                               const_cast<int32_t*>(chunk_idx), nullptr, group_idx, group_score,
                               err, s);
  if (dtype == 0)
    return p.D == 64 ? launch_route_groups_t<float, 64>(p, q, pos, group_sum, chunk_idx, group_idx, group_score, err, s)
                     : launch_route_groups_t<float, 128>(p, q, pos, group_sum, chunk_idx, group_idx, group_score, err, s);
  return p.D == 64
             ? launch_route_groups_t<__nv_bfloat16, 64>(p, q, pos, group_sum, chunk_idx, group_idx, group_score, err, s)
             : launch_route_groups_t<__nv_bfloat16, 128>(p, q, pos, group_sum, chunk_idx, group_idx, group_score, err, s);
}

}  // namespace hga
