// Host tier: K/V history in pinned host memory, only the routed groups (and the
// newest window rows) brought to the GPU per step.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Architettura della Memoria": hot tier in VRAM (chunk summaries
// and the always-visible windows), cold tier in host RAM (the whole K/V
// history); and "Meccanismo Core", item 4: the router fetches the original
// token K/V of the selected groups from host RAM into VRAM before the exact
// attention.
//
// Per (sequence, KV head) the device keeps a working buffer of rows
//   [sink chunks | ring of local+1 chunks (chunk c at slot c mod (local+1)) |
//    kg routed groups (slot j = entry j of group_idx)].
// The gather kernel reads pinned host memory directly (zero-copy 16-byte loads
// over the host link, several in flight per thread) and writes those rows:
// every call stages the routed groups and the current chunk's rows up to the
// query; with refresh_window it also copies the sink and local chunks (after a
// prefill, or when positions jump).  The decode attention then reads the
// working buffer with the same row map (attend_decode.cu, hot mode).
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kRowVec = 16;   // uint4 per 128-dim bf16 row
constexpr int kSplits = 4;    // CTAs per (sequence, KV head)

// Copies `rows` rows (16 uint4 each) from src to dst with this CTA's threads,
// four 16-byte loads in flight per thread per tensor.
__device__ __forceinline__ void copy_rows(const uint4* __restrict__ ks, const uint4* __restrict__ vs,
                                          uint4* __restrict__ kd, uint4* __restrict__ vd,
                                          int rows) {
  const int n = rows * kRowVec;
  for (int base = threadIdx.x; base < n; base += kThreads * 4) {
    uint4 kx[4], vx[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * kThreads;
      if (e < n) { kx[u] = ks[e]; vx[u] = vs[e]; }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * kThreads;
      if (e < n) { kd[e] = kx[u]; vd[e] = vx[u]; }
    }
  }
}

__global__ void __launch_bounds__(kThreads)
gather_host_kernel(const uint4* __restrict__ k_host, const uint4* __restrict__ v_host,
                   const int64_t* __restrict__ pos, const int32_t* __restrict__ group_idx,
                   LayerParams p, int refresh, uint4* __restrict__ k_work,
                   uint4* __restrict__ v_work, unsigned* err) {
  __shared__ int s_gid[1024], s_slot[1024];
  __shared__ int s_n;
  const int bh = blockIdx.x, b = bh / p.Hkv;
  const int split = blockIdx.y;
  const int64_t R = hot_rows(p);
  const int64_t W = static_cast<int64_t>(p.sink + p.local + 1) * p.C;
  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, threadIdx.x == 0 && split == 0 ? err : nullptr);
  pdl_wait();
  const int cur = ok ? static_cast<int>(pb / p.C) : 0;
  const int b0 = max(0, cur - p.local);
  if (threadIdx.x < 32) {
    int n = 0;
    bool bad = false;
    if (ok) {
      n = warp_keep_ascending(
          group_idx + static_cast<size_t>(bh) * p.kg, p.kg,
          [&](int gid) { return gid / p.Ng >= p.sink && gid / p.Ng < cur - p.local; }, s_gid,
          &bad, s_slot);
    }
    if (threadIdx.x == 0) s_n = n;
  }
  __syncthreads();
  if (!ok) return;
  const uint4* kh = k_host + static_cast<size_t>(bh) * p.n_alloc * kRowVec;
  const uint4* vh = v_host + static_cast<size_t>(bh) * p.n_alloc * kRowVec;
  uint4* kw = k_work + static_cast<size_t>(bh) * R * kRowVec;
  uint4* vw = v_work + static_cast<size_t>(bh) * R * kRowVec;
  // routed groups, split over the CTAs of this (sequence, KV head)
  const int n = s_n;
  for (int i = split; i < n; i += kSplits) {
    const size_t src = static_cast<size_t>(s_gid[i]) * p.g * kRowVec;
    const size_t dst = static_cast<size_t>(W + static_cast<int64_t>(s_slot[i]) * p.g) * kRowVec;
    copy_rows(kh + src, vh + src, kw + dst, vw + dst, p.g);
  }
  // window rows
  auto ring_row = [&](int c) { return static_cast<int64_t>(p.sink + c % (p.local + 1)) * p.C; };
  if (split == 0) {  // the current chunk up to the query
    const int64_t c0 = static_cast<int64_t>(cur) * p.C;
    copy_rows(kh + c0 * kRowVec, vh + c0 * kRowVec, kw + ring_row(cur) * kRowVec,
              vw + ring_row(cur) * kRowVec, static_cast<int>(pb - c0 + 1));
  }
  if (refresh) {
    for (int c = split; c < min(p.sink, b0); c += kSplits)
      copy_rows(kh + static_cast<size_t>(c) * p.C * kRowVec, vh + static_cast<size_t>(c) * p.C * kRowVec,
                kw + static_cast<size_t>(c) * p.C * kRowVec, vw + static_cast<size_t>(c) * p.C * kRowVec,
                p.C);
    for (int c = b0 + split; c < cur; c += kSplits)
      copy_rows(kh + static_cast<size_t>(c) * p.C * kRowVec, vh + static_cast<size_t>(c) * p.C * kRowVec,
                kw + ring_row(c) * kRowVec, vw + ring_row(c) * kRowVec, p.C);
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_gather_host(const LayerParams& p, const void* k_host, const void* v_host,
                               const int64_t* pos, const int32_t* group_idx, void* k_work,
                               void* v_work, int refresh_window, unsigned* err, cudaStream_t s) {
  return launch_pdl(gather_host_kernel, dim3(p.B * p.Hkv, kSplits), dim3(kThreads), 0, s, 1,
                    static_cast<const uint4*>(k_host), static_cast<const uint4*>(v_host), pos,
                    group_idx, p, refresh_window, static_cast<uint4*>(k_work),
                    static_cast<uint4*>(v_work), err);
}

}  // namespace hga
