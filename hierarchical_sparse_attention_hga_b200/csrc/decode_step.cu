// One decode step of one attention layer in one launch: steps 2-5 (two-level
// routing, gather of the original K/V, exact attention) for bf16 K/V, D = 128.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core": item 2 (level 1 over the
// chunk summaries, level 2 over the group summaries of the chosen chunks,
// sink / local / current chunks always visible) and item 4 (the original K/V
// of the chosen tokens, attended exactly with a standard softmax).
//
// One thread-block cluster of cl CTAs (4 warps each) per (sequence, KV head):
//   1. every CTA starts the TMA loads of its first forced units (the sink,
//      local and current chunks do not depend on routing), scores its slice of
//      the chunk summaries, takes the slice's top-kc and pushes the picks to
//      CTA 0 through distributed shared memory;
//   2. CTA 0 takes the top-kc of the picks, scores the groups of those chunks,
//      takes the top-kg and hands the group list to every CTA of the cluster,
//      while the other CTAs attend the forced units (with one CTA, it attends
//      them afterwards);
//   3. every warp of the cluster attends its share of the routed groups, and
//      the partials are merged by log-sum-exp inside the cluster.
// The routing uses the same scoring and top-k code as the routing kernel, so
// chunk_idx / group_idx are bit-identical to hga_route; the output matches
// hga_attend up to the order in which the softmax partials are merged.
#include <cuda.h>

#include <cooperative_groups.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "route_common.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace hga {
namespace {

using namespace decode;
using route::round4;

constexpr int kThreads = kWarps * 32;
constexpr int kMaxCluster = 8;
static_assert(kThreads == route::kThreads, "the routing helpers assume 128 threads");

// Routing words after the rings (4-byte words, each part a multiple of 4):
//   qbar [D] | slice scores [per] | warp top-k scratch keys, ids [2 x kWarps x 64], only
//   when a candidate set can exceed route::kRankMax |
//   picks [kc] | pushed scores, ids [2 x cl x kc] | pushed counts [cl] |
//   merged scores, ids [2 x cl x kc] | chunks [kc] | group scores [kc x Ng] |
//   chosen group positions [kg] | group list [kg]
struct StepSmem {
  int per, kc, cl, ng, kg;
  int lst;  // warp top-k scratch words (only for candidate sets above route::kRankMax)
  __host__ __device__ int o_sc() const { return kD; }
  __host__ __device__ int o_lkey() const { return o_sc() + per; }
  __host__ __device__ int o_lidx() const { return o_lkey() + lst; }
  __host__ __device__ int o_pick() const { return o_lidx() + lst; }
  __host__ __device__ int o_psc() const { return o_pick() + round4(kc); }
  __host__ __device__ int o_pidx() const { return o_psc() + round4(cl * kc); }
  __host__ __device__ int o_pcnt() const { return o_pidx() + round4(cl * kc); }
  __host__ __device__ int o_msc() const { return o_pcnt() + round4(cl); }
  __host__ __device__ int o_midx() const { return o_msc() + round4(cl * kc); }
  __host__ __device__ int o_chunks() const { return o_midx() + round4(cl * kc); }
  __host__ __device__ int o_gsc() const { return o_chunks() + round4(kc); }
  __host__ __device__ int o_gsel() const { return o_gsc() + round4(ng); }
  __host__ __device__ int o_glist() const { return o_gsel() + round4(kg); }
  __host__ __device__ int words() const { return o_glist() + round4(kg); }
};
__host__ __device__ inline StepSmem step_smem(const LayerParams& p, int cl) {
  StepSmem L;
  L.per = round4((p.n_chunks + cl - 1) / cl);
  L.kc = p.kc;
  L.cl = cl;
  L.ng = p.kc * p.Ng;
  L.kg = p.kg;
  const bool big = L.per > route::kRankMax || cl * p.kc > route::kRankMax || L.ng > route::kRankMax;
  L.lst = big ? kWarps * kWarpTopkList : 0;
  return L;
}
__host__ __device__ inline size_t step_smem_bytes(const LayerParams& p, int cl) {
  return kRingBytes + static_cast<size_t>(step_smem(p, cl).words()) * 4;
}

template <typename TO>
struct StepArgs {
  const __nv_bfloat16* q;
  const int64_t* pos;
  const float* chunk_sum;
  const float* group_sum;
  int32_t* chunk_idx;
  float* chunk_score;
  int32_t* group_idx;
  float* group_score;
  TO* out;
  float* lse;
  unsigned* err;
};

template <typename TO>
__global__ void __launch_bounds__(kThreads)
decode_step_kernel(const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, StepArgs<TO> a, LayerParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[kWarps][kStages];
  __shared__ MergeSmem s_merge;
  __shared__ int s_cnt[kWarps];
  __shared__ int s_ng;

  cg::cluster_group cluster = cg::this_cluster();
  const int cl = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  cluster.barrier_arrive();  // (1) paired with the wait before the first remote store
  const int item = blockIdx.x / cl;  // (sequence, KV head) = b * Hkv + h
  const int b = item / p.Hkv, h = item % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = rank * kWarps + warp;  // warp index within the cluster

  uint8_t* ring0 = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  float* rw = reinterpret_cast<float*>(ring0 + kWarps * kWarpBytes);
  const StepSmem L = step_smem(p, cl);
  float* qbar = rw;
  float* sc = rw + L.o_sc();
  unsigned* lkey = reinterpret_cast<unsigned*>(rw + L.o_lkey());
  int* lidx = reinterpret_cast<int*>(rw + L.o_lidx());
  int* pick = reinterpret_cast<int*>(rw + L.o_pick());
  float* psc = rw + L.o_psc();
  int* pidx = reinterpret_cast<int*>(rw + L.o_pidx());
  int* pcnt = reinterpret_cast<int*>(rw + L.o_pcnt());
  float* msc = rw + L.o_msc();
  int* midx = reinterpret_cast<int*>(rw + L.o_midx());
  int* chunks = reinterpret_cast<int*>(rw + L.o_chunks());
  float* gsc = rw + L.o_gsc();
  int* gsel = reinterpret_cast<int*>(rw + L.o_gsel());
  int* glist = reinterpret_cast<int*>(rw + L.o_glist());

  if (threadIdx.x == 0) {
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
    for (int w = 0; w < kWarps; ++w)
      for (int s = 0; s < kStages; ++s) ptx::mbar_init(&bars[w][s], 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();

  const int64_t pb = a.pos[b];  // pos, q, k and v are never written by this library
  const bool ok = valid_position(pb, p, threadIdx.x == 0 && rank == 0 ? a.err : nullptr);
  const int cur = ok ? static_cast<int>(pb / p.C) : 0;
  const int b0 = max(0, cur - p.local);
  // forced units: sink [0, su), then local + current up to the query [su, n_forced)
  const int ng_per_c = p.C / kUnit;
  const int su = ok ? min(p.sink, b0) * ng_per_c : 0;
  const int u_first_local = b0 * ng_per_c;
  const int n_forced = ok ? su + static_cast<int>(pb / kUnit) - u_first_local + 1 : 0;
  auto forced_token = [&](int u) -> int64_t {
    return static_cast<int64_t>(u < su ? u : u_first_local + (u - su)) * kUnit;
  };
  // The forced units go to the warps of CTAs 1..cl-1 (all warps when cl == 1).
  const int fw0 = cl > 1 ? kWarps : 0;
  const int fpw = (n_forced + cl * kWarps - fw0 - 1) / (cl * kWarps - fw0);
  const int f_lo = wg >= fw0 ? min(n_forced, (wg - fw0) * fpw) : 0;
  const int f_hi = wg >= fw0 ? min(n_forced, f_lo + fpw) : 0;

  // this warp's ring: units issued and consumed so far
  uint8_t* wsm = ring0 + warp * kWarpBytes;
  const uint32_t wsm_u32 = ptx::smem_u32(wsm);
  uint64_t* wbar = bars[warp];
  const int64_t row_base = static_cast<int64_t>(item) * p.n_alloc;
  int issued = 0, done = 0;
  auto issue_token = [&](int64_t tok) {
    if (lane == 0)
      issue_unit(&tm_k, &tm_v, wsm + (issued & 1) * kStageBytes, &wbar[issued & 1],
                 static_cast<int32_t>(row_base + tok));
    ++issued;
  };
  int f_next = f_lo;
  while (f_next < f_hi && issued < kStages) issue_token(forced_token(f_next++));

  route::decode_query_mean<__nv_bfloat16, kD>(a.q, p, b, h, qbar);
  pdl_wait();  // the summaries may come from the kernel just before
  __syncthreads();
  float4 qv[kD / 32];
#pragma unroll
  for (int k = 0; k < kD / 32; ++k) qv[k] = reinterpret_cast<const float4*>(qbar)[(lane & 7) + 8 * k];

  // ---- 1. level 1 on this CTA's slice of the candidate chunks
  const int n_cand = ok ? max(0, cur - p.local - p.sink) : 0;
  const int slice = (n_cand + cl - 1) / cl;
  const int lo = min(n_cand, rank * slice), hi = min(n_cand, lo + slice);
  {
    const float* rows = a.chunk_sum + (static_cast<size_t>(item) * p.n_chunks + p.sink + lo) * kD;
    route::score_rows8<kD, 4>(hi - lo, qv, sc, [&](int i) {
      return reinterpret_cast<const float4*>(rows + static_cast<size_t>(i) * kD);
    });
  }
  __syncthreads();
  const int nl = route::cta_topk(sc, hi - lo, p.kc, pick, lkey, lidx, s_cnt);
  cluster.barrier_wait();  // (1) every CTA of the cluster is running
  {
    float* dsc = cluster.map_shared_rank(psc, 0);
    int* didx = cluster.map_shared_rank(pidx, 0);
    for (int j = threadIdx.x; j < nl; j += kThreads) {
      dsc[rank * p.kc + j] = sc[pick[j]];
      didx[rank * p.kc + j] = lo + pick[j];
    }
    if (threadIdx.x == 0) cluster.map_shared_rank(pcnt, 0)[rank] = nl;
  }
  cluster.barrier_arrive();  // (2) this CTA's picks are in CTA 0

  // Q fragments and the softmax state are set up where each CTA first needs
  // them (CTA 0: after level 2), so that they hold no registers during the
  // level-2 scan.
  uint32_t qa[8][4];
  const float scale = kLog2e * rsqrtf(static_cast<float>(kD));
  WarpState w;
  bool timed_out = false;
  auto consume = [&](int valid) -> bool {
    const int st = done & 1;
    if (!ptx::mbar_wait(&wbar[st], (done >> 1) & 1, kWaitLimit)) return false;
    const uint32_t kt = wsm_u32 + st * kStageBytes;
    attend_unit(kt, kt + kTileBytes, valid, qa, scale, w);
    ++done;
    return true;
  };
  auto run_forced = [&]() {
    for (int u = f_lo; u < f_hi && !timed_out; ++u) {
      if (!consume(u == n_forced - 1 ? static_cast<int>(pb % kUnit) + 1 : kUnit)) {
        timed_out = true;
        break;
      }
      if (f_next < f_hi) issue_token(forced_token(f_next++));
    }
  };
  if (rank != 0) {
    load_q_frags(a.q, p, b, h, qa);
    w.init();
    run_forced();
  }
  cluster.barrier_wait();  // (2) every CTA's picks are in CTA 0

  if (rank == 0) {
    // ---- 2. merge the picks (rank order = ascending candidate index), level 2
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
    const int ns = route::cta_topk(msc, n_m, p.kc, pick, lkey, lidx, s_cnt);
    for (int i = threadIdx.x; i < p.kc; i += kThreads) {
      const int c = i < ns ? midx[pick[i]] + p.sink : -1;
      if (i < ns) chunks[i] = c;
      a.chunk_idx[static_cast<size_t>(item) * p.kc + i] = c;
      if (a.chunk_score)
        a.chunk_score[static_cast<size_t>(item) * p.kc + i] = i < ns ? msc[pick[i]] : CUDART_NAN_F;
    }
    __syncthreads();
    const int n_g = ns * p.Ng;
    const float* gbase = a.group_sum + static_cast<size_t>(item) * p.n_chunks * p.Ng * kD;
    route::score_rows8<kD, 4>(n_g, qv, gsc, [&](int i) {
      return reinterpret_cast<const float4*>(
          gbase + (static_cast<size_t>(chunks[i / p.Ng]) * p.Ng + i % p.Ng) * kD);
    });
    __syncthreads();
    const int ng = route::cta_topk(gsc, n_g, p.kg, gsel, lkey, lidx, s_cnt);
    for (int i = threadIdx.x; i < p.kg; i += kThreads) {
      const bool have = i < ng;
      const int sg = have ? gsel[i] : 0;
      const int gid = have ? chunks[sg / p.Ng] * p.Ng + sg % p.Ng : -1;
      a.group_idx[static_cast<size_t>(item) * p.kg + i] = gid;
      if (a.group_score)
        a.group_score[static_cast<size_t>(item) * p.kg + i] = have ? gsc[sg] : CUDART_NAN_F;
      if (have) glist[i] = gid;
    }
    __syncthreads();
    // hand the group list to the other CTAs of the cluster
    for (int r = 1; r < cl; ++r) {
      int* dst = cluster.map_shared_rank(glist, r);
      for (int i = threadIdx.x; i < ng; i += kThreads) dst[i] = glist[i];
      if (threadIdx.x == 0) *cluster.map_shared_rank(&s_ng, r) = ng;
    }
    if (threadIdx.x == 0) s_ng = ng;
    load_q_frags(a.q, p, b, h, qa);
    w.init();
  }
  cluster.barrier_arrive();  // (3) the group list is in every CTA
  if (cl == 1) run_forced();
  cluster.barrier_wait();  // (3)

  // ---- 3. the routed groups, split over the warps of the cluster
  const int n_r = s_ng;
  const int rpw = (n_r + cl * kWarps - 1) / (cl * kWarps);
  const int r_lo = min(n_r, wg * rpw), r_hi = min(n_r, r_lo + rpw);
  int r_next = r_lo;
  if (!timed_out)
    while (r_next < r_hi && issued - done < kStages)
      issue_token(static_cast<int64_t>(glist[r_next++]) * kUnit);
  for (int u = r_lo; u < r_hi && !timed_out; ++u) {
    if (!consume(kUnit)) {
      timed_out = true;
      break;
    }
    if (r_next < r_hi) issue_token(static_cast<int64_t>(glist[r_next++]) * kUnit);
  }
  if (timed_out) {
    // The warp gave up waiting on its copies: its partial is dropped (the
    // output is wrong and flagged), it waits once more, again bounded, for the
    // copies still in flight, and it still joins every barrier.
    if (lane == 0) flag_error(a.err, kErrTimeout);
    for (; done < issued; ++done) ptx::mbar_wait(&wbar[done & 1], (done >> 1) & 1, kWaitLimit);
    w.m0 = w.m1 = -CUDART_INF_F;
    w.l0 = w.l1 = 0.f;
  }
  merge_and_store<TO>(w, done == 0, ring0, s_merge, p, b, h, a.out, a.lse);
  pdl_trigger();
}

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

// CTAs per cluster: the largest cl <= 8 whose clusters all fit on the GPU at
// once (one wave) with slices of at least 32 candidate chunks; else 1.
template <auto Kern>
int step_cluster_size(const LayerParams& p) {
  const int items = p.B * p.Hkv;
  for (int cl = kMaxCluster; cl > 1; --cl) {
    if (p.n_chunks / cl < 32) continue;
    const size_t smem = step_smem_bytes(p, cl);
    if (ensure_smem<Kern>(smem) != cudaSuccess) continue;
    if (max_active_clusters<Kern>(cl, smem) >= items) return cl;
  }
  return 1;
}

template <typename TO>
cudaError_t launch_t(const LayerParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                     const StepArgs<TO>& a, cudaStream_t s) {
  const int cl = step_cluster_size<decode_step_kernel<TO>>(p);
  const size_t smem = step_smem_bytes(p, cl);
  cudaError_t e = ensure_smem<decode_step_kernel<TO>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_step_kernel<TO>, dim3(cl * p.B * p.Hkv), dim3(kThreads), smem, s, cl,
                    tk, tv, a, p);
}

}  // namespace

bool decode_step_path(const LayerParams& p, int dtype) {
  return decode_fast_path(p, dtype) && step_smem_bytes(p, 1) <= 200 * 1024 &&
         static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc < (static_cast<int64_t>(1) << 31);
}

cudaError_t launch_decode_step(const LayerParams& p, int out_dtype, const void* q,
                               const int64_t* pos, const float* chunk_sum, const float* group_sum,
                               const void* k, const void* v, int32_t* chunk_idx,
                               float* chunk_score, int32_t* group_idx, float* group_score,
                               void* out, float* lse, unsigned* err, cudaStream_t s) {
  CUtensorMap tk, tv;
  const int64_t all_rows = static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc;
  cudaError_t e = make_bf16_map(&tk, k, all_rows, kUnit);
  if (e == cudaSuccess) e = make_bf16_map(&tv, v, all_rows, kUnit);
  if (e != cudaSuccess) return e;
  if (out_dtype == 0) {
    StepArgs<float> a{static_cast<const __nv_bfloat16*>(q), pos, chunk_sum, group_sum, chunk_idx,
                      chunk_score, group_idx, group_score, static_cast<float*>(out), lse, err};
    return launch_t<float>(p, tk, tv, a, s);
  }
  StepArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(q), pos, chunk_sum, group_sum,
                            chunk_idx, chunk_score, group_idx, group_score,
                            static_cast<__nv_bfloat16*>(out), lse, err};
  return launch_t<__nv_bfloat16>(p, tk, tv, a, s);
}

}  // namespace hga
