// Internal launchers of the HGA kernels (host side, C++; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "common.cuh"

namespace hga {

// Launches `kern`, with programmatic stream serialization (see pdl_wait in
// common.cuh) unless kNoPdl is passed as `cluster` flag bit, and, when the
// cluster size is > 1, with that many CTAs per cluster along x.
constexpr int kNoPdl = 1 << 16;
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, int cluster_and_flags, Args&&... args) {
  const int cluster = cluster_and_flags & 0xffff;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (cluster_and_flags & kNoPdl) ? 0 : 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Raises the dynamic shared-memory limit of kernel Kern on the current device
// to at least `bytes`, calling cudaFuncSetAttribute only the first time a
// larger value is needed on that device.
template <auto Kern>
cudaError_t ensure_smem(size_t bytes) {
  static std::atomic<int> done[64];
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int want = static_cast<int>(bytes);
  if (dev >= 0 && dev < 64 && done[dev].load() >= want) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
  if (e == cudaSuccess && dev >= 0 && dev < 64) {
    int cur = done[dev].load();
    while (cur < want && !done[dev].compare_exchange_weak(cur, want)) {
    }
  }
  return e;
}

// SMs of the current device (cached per device; 148 if the query fails).
inline int device_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load();
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev].store(n);
  }
  return n;
}

// dtype: 0 = float32, 1 = bfloat16 (hga_dtype values).
cudaError_t launch_summaries(const LayerParams& p, int dtype, const void* k, int64_t t_begin,
                             int64_t t_end, float* chunk_sum, float* group_sum, cudaStream_t s);

cudaError_t launch_route_chunks(const LayerParams& p, int dtype, const void* q, const int64_t* pos,
                                const float* chunk_sum, int32_t* chunk_idx, float* chunk_score,
                                unsigned* err, cudaStream_t s);

cudaError_t launch_route_groups(const LayerParams& p, int dtype, const void* q, const int64_t* pos,
                                const float* group_sum, const int32_t* chunk_idx,
                                int32_t* group_idx, float* group_score, unsigned* err,
                                cudaStream_t s);

// Both routing levels in one launch (same results as the two launches above).
cudaError_t launch_route(const LayerParams& p, int dtype, const void* q, const int64_t* pos,
                         const float* chunk_sum, const float* group_sum, int32_t* chunk_idx,
                         float* chunk_score, int32_t* group_idx, float* group_score,
                         unsigned* err, cudaStream_t s);

// Prefill routing, several consecutive query blocks per CTA (level 1, level 2
// from chunk_idx, or both in one launch); applies to p when prefill_route_path.
bool prefill_route_path(const LayerParams& p, int dtype);
cudaError_t launch_route_prefill(const LayerParams& p, int dtype, bool level1, bool level2,
                                 const void* q, const int64_t* pos, const float* chunk_sum,
                                 const float* group_sum, int32_t* chunk_idx, float* chunk_score,
                                 int32_t* group_idx, float* group_score, unsigned* err,
                                 cudaStream_t s);

// Decode routing, one cluster of small CTAs per (sequence, KV head); same modes.
bool decode_route_path(const LayerParams& p);
cudaError_t launch_route_decode(const LayerParams& p, int dtype, bool level1, bool level2,
                                const void* q, const int64_t* pos, const float* chunk_sum,
                                const float* group_sum, int32_t* chunk_idx, float* chunk_score,
                                int32_t* group_idx, float* group_score, unsigned* err,
                                cudaStream_t s);

// One decode step (optional summary append + routing + attention): one launch of
// decode_step_kernel when decode_item_path (kc <= 64, kg <= 128 and the shared
// memory fits, with n_pt block-table entries staged per item for a paged pool),
// else the append, routing and attention kernels; applies when
// decode_step_path (bf16, D = 128 decode, device-resident K/V).  With
// kv.block_table, k and v are page pools and only the one launch is taken.
bool decode_item_path(const LayerParams& p, int n_pt = 0);
bool decode_step_path(const LayerParams& p, int dtype);
cudaError_t launch_decode_step(const LayerParams& p, int out_dtype, const void* q,
                               const int64_t* pos, float* chunk_sum, float* group_sum,
                               const void* k, const void* v, int32_t* chunk_idx,
                               float* chunk_score, int32_t* group_idx, float* group_score,
                               void* out, float* lse, int append, unsigned* err, cudaStream_t s,
                               const KvPages& kv = KvPages{nullptr, 0, 0, 0, -1});

// Backward pass of the prefill attention over the routed index sets
// (attend_backward.cu): bf16, D = 128, group 16, whole aligned query chunks.
bool backward_path(const LayerParams& p, int dtype);
size_t backward_workspace_bytes(const LayerParams& p);
cudaError_t launch_attend_backward(const LayerParams& p, const void* q, const void* k,
                                   const void* v, const void* out, int out_f32, const float* lse,
                                   const void* d_out, const int64_t* pos, const int32_t* group_idx,
                                   float* dq, float* dk, float* dv, void* workspace,
                                   unsigned* err, cudaStream_t s);

// Summaries of paged pools: every group and chunk row that ends before
// seq_len[b], per sequence (summaries.cu).
cudaError_t launch_summaries_paged(const LayerParams& p, int dtype, const void* k_pages,
                                   const KvPages& kv, const int64_t* seq_len, float* chunk_sum,
                                   float* group_sum, unsigned* err, cudaStream_t s);

// The summary rows each sequence's token pos[b] closes (one warp per (sequence,
// KV head) item; the rows hga_build_summaries(pos, pos + 1) writes, per sequence).
cudaError_t launch_append_per_sequence(const LayerParams& p, int dtype, const void* k,
                                       const int64_t* pos, float* chunk_sum, float* group_sum,
                                       cudaStream_t s);

// Workspace bytes of launch_attend for p (0 when the launch needs none).
size_t attend_workspace_bytes(const LayerParams& p, int dtype);

// The bf16, D = 128 decode kernel (TMA + mma.sync, in-cluster merge, no
// workspace) applies to p.
bool decode_fast_path(const LayerParams& p, int dtype);
// hot != 0: k / v are the host tier's device working buffers (hot_rows(p,
// slots) rows per (sequence, KV head)) instead of the device cache.  With
// slot_map (warm tier) routed entry j sits at cached slot slot_map[j] of
// `slots`; without, at slot j.
cudaError_t launch_attend_decode_bf16(const LayerParams& p, int out_dtype, const void* q,
                                      const int64_t* pos, const void* k, const void* v,
                                      const int32_t* group_idx, void* out, float* lse,
                                      unsigned* err, int hot, cudaStream_t s,
                                      const int32_t* slot_map = nullptr, int slots = 0);

// Host tier: rows per (sequence, KV head) of the device working buffers:
// sink chunks, a ring of local+1 chunks, and kg routed groups (or, with the
// warm tier, `slots` cached groups).
__host__ __device__ inline int64_t hot_rows(const LayerParams& p, int slots = 0) {
  return static_cast<int64_t>(p.sink + p.local + 1) * p.C +
         static_cast<int64_t>(slots > 0 ? slots : p.kg) * p.g;
}
cudaError_t launch_gather_host(const LayerParams& p, const void* k_host, const void* v_host,
                               const int64_t* pos, const int32_t* group_idx, void* k_work,
                               void* v_work, int refresh_window, unsigned* err, cudaStream_t s);

// Window rows a host-tier step copies for a query at pb, in the order a cold
// store stages them: with refresh mode 1 the sink chunks (c < min(sink, b0)),
// then the local chunks [b0, cur); then the current chunk from its first row
// (modes 0 and 1) or only the row at pb (mode 2), up to pb.
__host__ __device__ inline int64_t window_row_count(const LayerParams& p, int64_t pb, int mode) {
  const int64_t cur = pb / p.C, b0 = cur - p.local > 0 ? cur - p.local : 0;
  const int64_t n_sink = mode == 1 ? (p.sink < b0 ? p.sink : b0) * p.C : 0;
  const int64_t n_local = mode == 1 ? (cur - b0) * p.C : 0;
  return n_sink + n_local + (pb - (mode == 2 ? pb : cur * p.C) + 1);
}
__host__ __device__ inline int64_t window_row_token(const LayerParams& p, int64_t pb, int mode,
                                                    int64_t i) {
  const int64_t cur = pb / p.C, b0 = cur - p.local > 0 ? cur - p.local : 0;
  const int64_t n_sink = mode == 1 ? (p.sink < b0 ? p.sink : b0) * p.C : 0;
  const int64_t n_local = mode == 1 ? (cur - b0) * p.C : 0;
  if (i < n_sink) return i;
  if (i < n_sink + n_local) return b0 * p.C + (i - n_sink);
  return (mode == 2 ? pb : cur * p.C) + (i - n_sink - n_local);
}
// Rows per (sequence, KV head) of a cold store's window staging.
__host__ __device__ inline int64_t window_row_capacity(const LayerParams& p) {
  return static_cast<int64_t>(p.sink + p.local + 1) * p.C;
}

// Warm tier: at most kWarmMax cached groups per (sequence, KV head).
constexpr int kWarmMax = 2048;
// One step of the warm tier (host_tier.cu): LRU lookup and eviction in
// tags / stamps [B*Hkv][slots], slot_map [B*Hkv][kg] written, misses and the
// window rows copied from the host cache.  counters (hits, misses) may be null.
cudaError_t launch_gather_warm(const LayerParams& p, const void* k_host, const void* v_host,
                               const int64_t* pos, const int32_t* group_idx, int slots,
                               int32_t* tags, int32_t* stamps, int32_t* slot_map, void* k_work,
                               void* v_work, int refresh_window, unsigned long long* counters,
                               unsigned* err, cudaStream_t s, int2* plan = nullptr,
                               int32_t* n_plan = nullptr);
// With plan / n_plan the warm step above only decides: the table and slot map
// are written, and each (sequence, KV head)'s misses as (group, slot) pairs
// [B*Hkv][kg] with their count [B*Hkv]; no row is copied.  launch_warm_fill then
// copies the rows a cold store staged (pinned host memory, read in place):
// staging per (sequence, KV head) = [K | V][kg][16 rows][128] of the misses in
// plan order, then [K | V][window_row_capacity][128] of the window rows.
cudaError_t launch_warm_fill(const LayerParams& p, const void* staging, const int2* plan,
                             const int32_t* n_plan, const int64_t* pos, int slots, int mode,
                             void* k_work, void* v_work, unsigned* err, cudaStream_t s);
// Bytes of staging per (sequence, KV head).
__host__ __device__ inline int64_t cold_stage_unit_bytes(const LayerParams& p) {
  return 2 * (static_cast<int64_t>(p.kg) * 16 + window_row_capacity(p)) * p.D * 2;
}

// The bf16, D = 128 prefill kernel (64-query blocks on tcgen05 / TMEM) applies to p.
bool prefill_tc_path(const LayerParams& p, int dtype);
cudaError_t launch_attend_prefill_bf16(const LayerParams& p, int out_dtype, const void* q,
                                       const int64_t* pos, const void* k, const void* v,
                                       const int32_t* group_idx, void* out, float* lse,
                                       unsigned* err, cudaStream_t s);

// Log-sum-exp merge of nsplit decode partials into out / lse.
cudaError_t launch_combine(const LayerParams& p, int out_dtype, int nsplit, const float* ws_o,
                           const float* ws_ml, void* out, float* lse, cudaStream_t s);

cudaError_t launch_attend(const LayerParams& p, int dtype, int out_dtype, const void* q,
                          const int64_t* pos, const void* k, const void* v,
                          const int32_t* group_idx, void* out, float* lse, void* ws,
                          unsigned* err, cudaStream_t s);

}  // namespace hga
