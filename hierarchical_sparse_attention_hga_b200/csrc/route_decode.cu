// Steps 2 and 3 for decode (one query per sequence): two-level routing with one
// thread-block cluster per (sequence, KV head).
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", item 2: level 1 scores the
// routing query against the chunk key summaries of the earlier chunks and keeps
// the top-kc; level 2 scores the group summaries inside those chunks and keeps
// the top-kg.  The sink, local and current chunks are always visible, so they
// are not candidates.
//
// A decode step has few (sequence, KV head) items, so each item gets a cluster
// of up to eight small CTAs: CTA r scores the r-th slice of the candidate
// chunks (eight lanes per summary row, four rows per warp and pass, eight
// rows in flight per warp) and takes the slice's top-kc with a warp top-k;
// the slices' picks go to CTA 0 through distributed shared memory, in
// candidate order, and CTA 0 takes the top-kc of them (the global top-kc is
// always among the slices' top-kc, and ties still go to the lower index).
// CTA 0 then scores the groups of its chunks and keeps the top-kg.  The same
// kernel serves the level-1-only, level-2-only and fused calls, so their
// results agree bit for bit.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "route_common.cuh"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace hga {
namespace {

using route::kThreads;
using route::kWarps;
using route::round4;
using route::score_rows8;
using route::cta_topk;
constexpr int kMaxCluster = 8;

enum { kL1 = 1, kL2 = 2 };

// Dynamic shared memory, in 4-byte words (each part a multiple of 4 words):
//   qbar [D] | slice scores [per] | warp top-k scratch keys, ids [2 x kWarps x 64] |
//   picks [kc] | pushed scores, ids [2 x cl x kc] | pushed counts [cl] |
//   merged scores, ids [2 x cl x kc] | chunks [kc] | group scores [kc x Ng] | groups [kg]
struct DecodeRouteSmem {
  int D, per, kc, cl, ng, kg;
  __host__ __device__ int o_sc() const { return D; }
  __host__ __device__ int o_lkey() const { return o_sc() + per; }
  __host__ __device__ int o_lidx() const { return o_lkey() + kWarps * kWarpTopkList; }
  __host__ __device__ int o_pick() const { return o_lidx() + kWarps * kWarpTopkList; }
  __host__ __device__ int o_psc() const { return o_pick() + round4(kc); }
  __host__ __device__ int o_pidx() const { return o_psc() + round4(cl * kc); }
  __host__ __device__ int o_pcnt() const { return o_pidx() + round4(cl * kc); }
  __host__ __device__ int o_msc() const { return o_pcnt() + round4(cl); }
  __host__ __device__ int o_midx() const { return o_msc() + round4(cl * kc); }
  __host__ __device__ int o_chunks() const { return o_midx() + round4(cl * kc); }
  __host__ __device__ int o_gsc() const { return o_chunks() + round4(kc); }
  __host__ __device__ int o_gsel() const { return o_gsc() + round4(ng); }
  __host__ __device__ int words() const { return o_gsel() + round4(kg); }
};
__host__ __device__ inline DecodeRouteSmem decode_route_smem(const LayerParams& p, int cl) {
  DecodeRouteSmem L;
  L.D = p.D;
  L.per = round4((p.n_chunks + cl - 1) / cl);
  L.kc = p.kc;
  L.cl = cl;
  L.ng = p.kc * p.Ng;
  L.kg = p.kg;
  return L;
}

constexpr int kCtasPerSm = 7;  // resident CTAs per SM (registers: 72 per thread at most)

// Clusters of `cl` CTAs of Kern (with `smem` bytes each) that fit on the GPU at
// once; cached per device and shape.
template <auto Kern>
int max_active_clusters(int cl, size_t smem) {
  struct Entry {
    int dev, cl;
    size_t smem;
    int n;
  };
  static Entry cache[32];
  static std::atomic<int> used{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int m = std::min(used.load(), 32);
  for (int i = 0; i < m; ++i)
    if (cache[i].dev == dev && cache[i].cl == cl && cache[i].smem == smem) return cache[i].n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cl * 64);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = cl;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, Kern, &cfg) != cudaSuccess) {
    cudaGetLastError();  // clears the error; the caller falls back to smaller clusters
    n = 0;
  }
  const int slot = used.fetch_add(1);
  if (slot < 32) cache[slot] = Entry{dev, cl, smem, n};
  return n;
}

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
route_decode_kernel(const T* __restrict__ q, const int64_t* __restrict__ pos,
                    const float* __restrict__ chunk_sum, const float* __restrict__ group_sum,
                    LayerParams p, int32_t* __restrict__ chunk_idx, float* __restrict__ chunk_score,
                    int32_t* __restrict__ group_idx, float* __restrict__ group_score,
                    unsigned* err) {
  constexpr bool kLevel1 = (MODE & kL1) != 0;
  constexpr bool kLevel2 = (MODE & kL2) != 0;
  constexpr int F4 = D / 32;
  extern __shared__ __align__(16) float dyn[];
  __shared__ int s_n;
  __shared__ int s_cnt[kWarps];
  cg::cluster_group cluster = cg::this_cluster();
  const int cl = kLevel1 ? static_cast<int>(cluster.num_blocks()) : 1;
  const int rank = kLevel1 ? static_cast<int>(cluster.block_rank()) : 0;
  if constexpr (kLevel1) cluster.barrier_arrive();  // paired with barrier_wait() before the pushes
  const DecodeRouteSmem L = decode_route_smem(p, cl);
  float* qbar = dyn;
  float* sc = dyn + L.o_sc();
  unsigned* lkey = reinterpret_cast<unsigned*>(dyn + L.o_lkey());
  int* lidx = reinterpret_cast<int*>(dyn + L.o_lidx());
  int* pick = reinterpret_cast<int*>(dyn + L.o_pick());
  float* psc = dyn + L.o_psc();
  int* pidx = reinterpret_cast<int*>(dyn + L.o_pidx());
  int* pcnt = reinterpret_cast<int*>(dyn + L.o_pcnt());
  float* msc = dyn + L.o_msc();
  int* midx = reinterpret_cast<int*>(dyn + L.o_midx());
  int* chunks = reinterpret_cast<int*>(dyn + L.o_chunks());
  float* gsc = dyn + L.o_gsc();
  int* gsel = reinterpret_cast<int*>(dyn + L.o_gsel());

  const int item = blockIdx.x / cl;  // (sequence, KV head) = b * Hkv + h; one block per item
  const int h = item % p.Hkv, b = item / p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, threadIdx.x == 0 && rank == 0 ? err : nullptr);
  const int cur = ok ? static_cast<int>(pb / p.C) : 0;

  // routing query: mean of the G heads' query rows (q is never written by this library)
  route::decode_query_mean<T, D>(q, p, b, h, qbar);
  pdl_wait();  // the summaries may come from the kernel just before
  __syncthreads();
  float4 qv[F4];
#pragma unroll
  for (int k = 0; k < F4; ++k) qv[k] = reinterpret_cast<const float4*>(qbar)[(lane & 7) + 8 * k];

  const int n_cand = ok ? max(0, cur - p.local - p.sink) : 0;
  int ns = 0;
  if constexpr (kLevel1) {
    // ---- level 1, this CTA's slice of the candidates
    const int slice = (n_cand + cl - 1) / cl;
    const int lo = min(n_cand, rank * slice), hi = min(n_cand, lo + slice);
    const float* rows = chunk_sum + (static_cast<size_t>(item) * p.n_chunks + p.sink + lo) * D;
    score_rows8<D, 8 / (D / 32)>(hi - lo, qv, sc, [&](int i) {
      return reinterpret_cast<const float4*>(rows + static_cast<size_t>(i) * D);
    });
    __syncthreads();
    const int nl = cta_topk(sc, hi - lo, p.kc, pick, lkey, lidx, s_cnt);
    cluster.barrier_wait();  // every CTA of the cluster is running
    {
      float* dsc = cluster.map_shared_rank(psc, 0);
      int* didx = cluster.map_shared_rank(pidx, 0);
      for (int j = threadIdx.x; j < nl; j += kThreads) {
        dsc[rank * p.kc + j] = sc[pick[j]];
        didx[rank * p.kc + j] = lo + pick[j];
      }
      if (threadIdx.x == 0) cluster.map_shared_rank(pcnt, 0)[rank] = nl;
    }
    cluster.sync();  // the pushes are visible to CTA 0
    // The next kernel may launch now: its prologue (which reads no output of
    // this kernel) overlaps the merge and level 2 below; it still waits for
    // this grid to complete before reading group_idx.
    pdl_trigger();
    if (rank != 0) return;
    // ---- merge: the slices' picks in rank order (= ascending candidate index)
    int n_m = 0;
    for (int r = 0; r < cl; ++r) {
      const int c = pcnt[r];
      for (int j = threadIdx.x; j < c; j += kThreads) {
        msc[n_m + j] = psc[r * p.kc + j];
        midx[n_m + j] = pidx[r * p.kc + j];
      }
      n_m += c;
    }
    __syncthreads();
    ns = cta_topk(msc, n_m, p.kc, pick, lkey, lidx, s_cnt);
    for (int i = threadIdx.x; i < p.kc; i += kThreads) {
      const int c = i < ns ? midx[pick[i]] + p.sink : -1;
      if (i < ns) chunks[i] = c;
      chunk_idx[static_cast<size_t>(item) * p.kc + i] = c;
      if (chunk_score)
        chunk_score[static_cast<size_t>(item) * p.kc + i] = i < ns ? msc[pick[i]] : CUDART_NAN_F;
    }
    if (threadIdx.x == 0) s_n = ns;
  } else {
    // ---- level 2 only: the chunks come from chunk_idx (validated)
    if (warp == 0) {
      int n = 0;
      if (ok) {
        bool bad = false;
        n = warp_keep_ascending(
            chunk_idx + static_cast<size_t>(item) * p.kc, p.kc,
            [&](int c) { return c >= p.sink && c < cur - p.local; }, chunks, &bad);
        if (bad && lane == 0) flag_error(err, kErrChunkIdx);
      }
      if (lane == 0) s_n = n;
    }
  }
  if constexpr (kLevel2) {
    __syncthreads();
    ns = s_n;
    // ---- level 2: the groups of the selected chunks (ascending chunk ids)
    const int n_g = ns * p.Ng;
    const float* gbase = group_sum + static_cast<size_t>(item) * p.n_chunks * p.Ng * D;
    score_rows8<D, 8 / (D / 32)>(n_g, qv, gsc, [&](int i) {
      return reinterpret_cast<const float4*>(
          gbase + (static_cast<size_t>(chunks[i / p.Ng]) * p.Ng + i % p.Ng) * D);
    });
    __syncthreads();
    const int ng = cta_topk(gsc, n_g, p.kg, gsel, lkey, lidx, s_cnt);
    for (int i = threadIdx.x; i < p.kg; i += kThreads) {
      const bool have = i < ng;
      const int sg = have ? gsel[i] : 0;
      group_idx[static_cast<size_t>(item) * p.kg + i] = have ? chunks[sg / p.Ng] * p.Ng + sg % p.Ng : -1;
      if (group_score)
        group_score[static_cast<size_t>(item) * p.kg + i] = have ? gsc[sg] : CUDART_NAN_F;
    }
  }
  pdl_trigger();
}

// CTAs per cluster: 8, 4 or 2 while the slices keep at least 64 candidate
// chunks and every (sequence, KV head) item's cluster fits on the GPU at once
// (otherwise some clusters would wait for a second wave); else 1.
template <auto Kern>
int decode_cluster_size(const LayerParams& p) {
  const int items = p.B * p.Hkv;
  for (int cl = kMaxCluster; cl > 1; cl /= 2) {
    if (p.n_chunks / cl < 64) continue;
    const size_t smem = static_cast<size_t>(decode_route_smem(p, cl).words()) * 4;
    if (ensure_smem<Kern>(smem) != cudaSuccess) continue;
    if (max_active_clusters<Kern>(cl, smem) >= items) return cl;
  }
  return 1;
}

template <typename T, int D, int MODE>
cudaError_t launch_t(const LayerParams& p, const void* q, const int64_t* pos,
                     const float* chunk_sum, const float* group_sum, int32_t* chunk_idx,
                     float* chunk_score, int32_t* group_idx, float* group_score, unsigned* err,
                     cudaStream_t s) {
  const int cl = (MODE & kL1) ? decode_cluster_size<route_decode_kernel<T, D, MODE>>(p) : 1;
  const size_t smem = static_cast<size_t>(decode_route_smem(p, cl).words()) * 4;
  cudaError_t e = ensure_smem<route_decode_kernel<T, D, MODE>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(route_decode_kernel<T, D, MODE>, dim3(p.B * p.Hkv * cl), dim3(kThreads), smem,
                    s, cl, static_cast<const T*>(q), pos, chunk_sum, group_sum, p, chunk_idx,
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

bool decode_route_path(const LayerParams& p) {
  return p.q_len == 1 && (p.D == 64 || p.D == 128) &&
         static_cast<size_t>(decode_route_smem(p, 1).words()) * 4 <= 200 * 1024;
}

cudaError_t launch_route_decode(const LayerParams& p, int dtype, bool level1, bool level2,
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
