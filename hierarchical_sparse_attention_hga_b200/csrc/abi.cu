// C ABI of the HGA hot path: argument validation, the per-device error word
// and dispatch to the kernels.  Every entry point returns a status and never
// aborts; see include/hga.h for the contract of each call.
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <new>
#include <string>

#include "../../include/hga.h"
#include "cold_tier.h"
#include "kernels.h"

namespace hga {
namespace {

thread_local char g_msg[512] = "";

// Test hooks (kDebug* bits) copied into every launch's parameters.
std::atomic<unsigned> g_debug{0};

// NVTX range around an entry point (a no-op unless a profiler is attached).
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

hga_status fail(hga_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

hga_status cuda_fail(cudaError_t e, const char* where) {
  return fail(HGA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Sticky device error word: one per device that loads the library.
__device__ unsigned g_device_error;

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
unsigned* g_err_ptr[kMaxDevices] = {};

// Device address of g_device_error on the current device (looked up once per device).
hga_status device_error_ptr(unsigned** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(HGA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_device_error);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(device error word)");
    g_err_ptr[dev] = static_cast<unsigned*>(ptr);
  }
  *out = g_err_ptr[dev];
  return HGA_OK;
}

// Host-side checks of cfg and the derived kernel parameters.
hga_status make_params(const hga_config* cfg, int64_t n_alloc, int32_t q_len, LayerParams* p) {
  if (!cfg) return fail(HGA_ERR_INVALID_ARG, "cfg is NULL");
  const hga_config& c = *cfg;
  if (c.batch <= 0 || c.heads_q <= 0 || c.heads_kv <= 0 || c.head_dim <= 0 || c.chunk <= 0 ||
      c.group <= 0 || c.sink_chunks < 0 || c.local_chunks < 0 || c.topk_chunks <= 0 ||
      c.topk_groups <= 0 || c.n_high_pairs < 0)
    return fail(HGA_ERR_INVALID_ARG, "config sizes must be positive (sink/local/n_high >= 0)");
  if (!(c.rope_theta > 1.0)) return fail(HGA_ERR_INVALID_ARG, "rope_theta must be > 1");
  if (c.dtype != HGA_F32 && c.dtype != HGA_BF16) return fail(HGA_ERR_INVALID_ARG, "dtype %d", c.dtype);
  if (c.out_dtype != HGA_F32 && c.out_dtype != HGA_BF16)
    return fail(HGA_ERR_INVALID_ARG, "out_dtype %d", c.out_dtype);
  if (c.kv_loc != HGA_KV_DEVICE && c.kv_loc != HGA_KV_HOST_PINNED)
    return fail(HGA_ERR_INVALID_ARG, "kv_loc %d", c.kv_loc);
  if (c.heads_q % c.heads_kv) return fail(HGA_ERR_SHAPE, "heads_q %% heads_kv != 0");
  if (c.heads_q / c.heads_kv > 16) return fail(HGA_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
  if (c.head_dim != 64 && c.head_dim != 128) return fail(HGA_ERR_UNSUPPORTED, "head_dim %d", c.head_dim);
  if (c.chunk != 64 && c.chunk != 128) return fail(HGA_ERR_UNSUPPORTED, "chunk %d", c.chunk);
  if (c.group != 16) return fail(HGA_ERR_UNSUPPORTED, "group %d (16 is built)", c.group);
  if (c.n_high_pairs > c.head_dim / 2) return fail(HGA_ERR_SHAPE, "n_high_pairs > head_dim/2");
  if (c.topk_chunks > 256) return fail(HGA_ERR_UNSUPPORTED, "topk_chunks > 256");
  if (c.topk_groups > 1024) return fail(HGA_ERR_UNSUPPORTED, "topk_groups > 1024");
  if (n_alloc <= 0 || n_alloc % c.chunk) return fail(HGA_ERR_SHAPE, "n_alloc must be a positive multiple of chunk");
  if (n_alloc / c.chunk > 32768) return fail(HGA_ERR_UNSUPPORTED, "n_alloc / chunk > 32768");
  if (q_len <= 0) return fail(HGA_ERR_INVALID_ARG, "q_len must be positive");
  if (q_len > 1 && q_len % c.chunk) return fail(HGA_ERR_UNSUPPORTED, "prefill q_len must be a multiple of chunk");
  if (q_len > n_alloc) return fail(HGA_ERR_SHAPE, "q_len > n_alloc");
  const int64_t rows = static_cast<int64_t>(c.batch) * c.heads_kv * q_len;
  if (rows > 0x7fffffffLL) return fail(HGA_ERR_UNSUPPORTED, "batch * heads_kv * q_len too large");
  if (static_cast<int64_t>(c.topk_chunks) * (c.chunk / c.group) > 8192)
    return fail(HGA_ERR_UNSUPPORTED, "topk_chunks * chunk/group > 8192");
  p->B = c.batch; p->Hq = c.heads_q; p->Hkv = c.heads_kv; p->G = c.heads_q / c.heads_kv;
  p->D = c.head_dim; p->C = c.chunk; p->g = c.group; p->Ng = c.chunk / c.group;
  p->sink = c.sink_chunks; p->local = c.local_chunks;
  p->kc = c.topk_chunks; p->kg = c.topk_groups; p->n_high = c.n_high_pairs;
  p->q_len = q_len; p->nblk = q_len == 1 ? 1 : q_len / c.chunk;
  p->n_alloc = n_alloc; p->n_chunks = static_cast<int>(n_alloc / c.chunk);
  p->theta = c.rope_theta;
  p->debug = g_debug.load();
  return HGA_OK;
}

}  // namespace

// Sets the message hga_last_error() returns on this thread (for entry points
// defined in other files of the library).
void set_last_error(const char* msg) { snprintf(g_msg, sizeof(g_msg), "%s", msg); }

}  // namespace hga

using namespace hga;

extern "C" {

int32_t hga_abi_version(void) { return HGA_ABI_VERSION; }

const char* hga_status_string(hga_status s) {
  switch (s) {
    case HGA_OK: return "HGA_OK";
    case HGA_ERR_INVALID_ARG: return "HGA_ERR_INVALID_ARG";
    case HGA_ERR_SHAPE: return "HGA_ERR_SHAPE";
    case HGA_ERR_UNSUPPORTED: return "HGA_ERR_UNSUPPORTED";
    case HGA_ERR_CUDA: return "HGA_ERR_CUDA";
    case HGA_ERR_TIMEOUT: return "HGA_ERR_TIMEOUT";
    case HGA_ERR_DEVICE_CHECK: return "HGA_ERR_DEVICE_CHECK";
    case HGA_ERR_WORKSPACE: return "HGA_ERR_WORKSPACE";
  }
  return "HGA_ERR_UNKNOWN";
}

const char* hga_last_error(void) { return g_msg; }

hga_status hga_device_status(void* stream) {
  unsigned* err = nullptr;
  hga_status st = device_error_ptr(&err);
  if (st != HGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, err, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(err, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "hga_device_status");
  if (host & kErrTimeout)
    return fail(HGA_ERR_TIMEOUT, "a bounded device wait gave up, bits 0x%x", host);
  if (host) return fail(HGA_ERR_DEVICE_CHECK, "device check failed, bits 0x%x", host);
  return HGA_OK;
}

int32_t hga_debug_inject(int32_t flags) {
  return static_cast<int32_t>(g_debug.exchange(static_cast<unsigned>(flags)));
}

hga_status hga_workspace_size(const hga_config* cfg, int64_t n_alloc, int32_t q_len, size_t* bytes) {
  if (!bytes) return fail(HGA_ERR_INVALID_ARG, "bytes is NULL");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, q_len, &p);
  if (st != HGA_OK) return st;
  *bytes = attend_workspace_bytes(p, cfg->dtype);
  return HGA_OK;
}

hga_status hga_build_summaries(const hga_config* cfg, const void* k, int64_t n_alloc,
                               int64_t t_begin, int64_t t_end, float* chunk_sum,
                               float* group_sum, void* stream) {
  Range nvtx_range("hga_build_summaries");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if (!k || !chunk_sum || !group_sum) return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (t_begin < 0 || t_end < t_begin || t_end > n_alloc)
    return fail(HGA_ERR_INVALID_ARG, "need 0 <= t_begin <= t_end <= n_alloc");
  cudaError_t e = launch_summaries(p, cfg->dtype, k, t_begin, t_end, chunk_sum, group_sum,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_build_summaries");
}

hga_status hga_route_chunks(const hga_config* cfg, const void* q, int32_t q_len,
                            const int64_t* pos, const float* chunk_sum, int64_t n_alloc,
                            int32_t* chunk_idx, float* chunk_score, void* stream) {
  Range nvtx_range("hga_route_chunks");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, q_len, &p);
  if (st != HGA_OK) return st;
  if (!q || !pos || !chunk_sum || !chunk_idx) return fail(HGA_ERR_INVALID_ARG, "null pointer");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_route_chunks(p, cfg->dtype, q, pos, chunk_sum, chunk_idx, chunk_score,
                                      err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_route_chunks");
}

hga_status hga_route_groups(const hga_config* cfg, const void* q, int32_t q_len,
                            const int64_t* pos, const float* group_sum, int64_t n_alloc,
                            const int32_t* chunk_idx, int32_t* group_idx, float* group_score,
                            void* stream) {
  Range nvtx_range("hga_route_groups");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, q_len, &p);
  if (st != HGA_OK) return st;
  if (!q || !pos || !group_sum || !chunk_idx || !group_idx)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_route_groups(p, cfg->dtype, q, pos, group_sum, chunk_idx, group_idx,
                                      group_score, err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_route_groups");
}

hga_status hga_route(const hga_config* cfg, const void* q, int32_t q_len, const int64_t* pos,
                     const float* chunk_sum, const float* group_sum, int64_t n_alloc,
                     int32_t* chunk_idx, float* chunk_score, int32_t* group_idx,
                     float* group_score, void* stream) {
  Range nvtx_range("hga_route");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, q_len, &p);
  if (st != HGA_OK) return st;
  if (!q || !pos || !chunk_sum || !group_sum || !chunk_idx || !group_idx)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_route(p, cfg->dtype, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score,
                               group_idx, group_score, err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_route");
}

// The host tier runs bf16, D = 128 decode through the working buffers.
static hga_status check_host_tier(const hga_config* cfg, const LayerParams& p) {
  if (cfg->dtype != HGA_BF16 || p.D != 128 || p.g != 16 || p.kg > 1024 || p.q_len != 1)
    return fail(HGA_ERR_UNSUPPORTED, "the host tier is built for bf16, head_dim 128 decode");
  return HGA_OK;
}

hga_status hga_hot_rows(const hga_config* cfg, int64_t* rows) {
  if (!rows) return fail(HGA_ERR_INVALID_ARG, "rows is NULL");
  LayerParams p;
  hga_status st = make_params(cfg, cfg ? cfg->chunk : 0, 1, &p);
  if (st != HGA_OK) return st;
  *rows = hot_rows(p);
  return HGA_OK;
}

hga_status hga_gather_host(const hga_config* cfg, const void* k_host, const void* v_host,
                           int64_t n_alloc, const int64_t* pos, const int32_t* group_idx,
                           void* k_work, void* v_work, int32_t refresh_window, void* stream) {
  Range nvtx_range("hga_gather_host");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  if (!k_host || !v_host || !pos || !group_idx || !k_work || !v_work)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (refresh_window < 0 || refresh_window > 2)
    return fail(HGA_ERR_INVALID_ARG, "refresh_window %d is not 0, 1 or 2", refresh_window);
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_gather_host(p, k_host, v_host, pos, group_idx, k_work, v_work,
                                     refresh_window, err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_gather_host");
}

static hga_status check_warm(const LayerParams& p, int32_t warm_groups) {
  if (warm_groups < p.kg || warm_groups > kWarmMax)
    return fail(HGA_ERR_INVALID_ARG, "warm_groups %d outside [topk_groups %d, %d]", warm_groups,
                p.kg, kWarmMax);
  return HGA_OK;
}

hga_status hga_warm_rows(const hga_config* cfg, int32_t warm_groups, int64_t* rows) {
  if (!rows) return fail(HGA_ERR_INVALID_ARG, "rows is NULL");
  LayerParams p;
  hga_status st = make_params(cfg, cfg ? cfg->chunk : 0, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_warm(p, warm_groups)) != HGA_OK) return st;
  *rows = hot_rows(p, warm_groups);
  return HGA_OK;
}

hga_status hga_warm_reset(const hga_config* cfg, int32_t warm_groups, int32_t* tags,
                          int32_t* stamps, int32_t seq, void* stream) {
  Range nvtx_range("hga_warm_reset");
  LayerParams p;
  hga_status st = make_params(cfg, cfg ? cfg->chunk : 0, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_warm(p, warm_groups)) != HGA_OK) return st;
  if (!tags || !stamps) return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (seq < -1 || seq >= p.B) return fail(HGA_ERR_INVALID_ARG, "seq %d outside [-1, %d)", seq, p.B);
  const size_t per_seq = static_cast<size_t>(p.Hkv) * warm_groups;
  const size_t off = seq < 0 ? 0 : static_cast<size_t>(seq) * per_seq;
  const size_t count = seq < 0 ? per_seq * p.B : per_seq;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(tags + off, 0xff, count * sizeof(int32_t), s);  // -1: empty
  if (e == cudaSuccess) e = cudaMemsetAsync(stamps + off, 0, count * sizeof(int32_t), s);
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_warm_reset");
}

hga_status hga_gather_warm(const hga_config* cfg, const void* k_host, const void* v_host,
                           int64_t n_alloc, const int64_t* pos, const int32_t* group_idx,
                           int32_t warm_groups, int32_t* tags, int32_t* stamps, int32_t* slot_map,
                           void* k_work, void* v_work, int32_t refresh_window, uint64_t* counters,
                           void* stream) {
  Range nvtx_range("hga_gather_warm");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  if ((st = check_warm(p, warm_groups)) != HGA_OK) return st;
  if (!k_host || !v_host || !pos || !group_idx || !tags || !stamps || !slot_map || !k_work ||
      !v_work)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (refresh_window < 0 || refresh_window > 2)
    return fail(HGA_ERR_INVALID_ARG, "refresh_window %d is not 0, 1 or 2", refresh_window);
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_gather_warm(p, k_host, v_host, pos, group_idx, warm_groups, tags, stamps,
                                     slot_map, k_work, v_work, refresh_window,
                                     reinterpret_cast<unsigned long long*>(counters), err,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_gather_warm");
}

hga_status hga_attend_warm(const hga_config* cfg, const void* q, const int64_t* pos,
                           const void* k_work, const void* v_work, int64_t n_alloc,
                           const int32_t* group_idx, const int32_t* slot_map, int32_t warm_groups,
                           void* out, float* lse, void* stream) {
  Range nvtx_range("hga_attend_warm");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  if ((st = check_warm(p, warm_groups)) != HGA_OK) return st;
  if (!q || !pos || !k_work || !v_work || !group_idx || !slot_map || !out)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_attend_decode_bf16(p, cfg->out_dtype, q, pos, k_work, v_work, group_idx,
                                            out, lse, err, 1, static_cast<cudaStream_t>(stream),
                                            slot_map, warm_groups);
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_attend_warm");
}

hga_status hga_attend(const hga_config* cfg, const void* q, int32_t q_len, const int64_t* pos,
                      const void* k, const void* v, int64_t n_alloc, const int32_t* group_idx,
                      void* out, float* lse, void* workspace, size_t workspace_bytes,
                      void* stream) {
  Range nvtx_range("hga_attend");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, q_len, &p);
  if (st != HGA_OK) return st;
  if (!q || !pos || !k || !v || !group_idx || !out) return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (cfg->kv_loc == HGA_KV_HOST_PINNED) {
    if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
    unsigned* err = nullptr;
    if ((st = device_error_ptr(&err)) != HGA_OK) return st;
    cudaError_t e = launch_attend_decode_bf16(p, cfg->out_dtype, q, pos, k, v, group_idx, out, lse,
                                              err, 1, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_attend (host tier)");
  }
  const size_t need = attend_workspace_bytes(p, cfg->dtype);
  if (need && (!workspace || workspace_bytes < need))
    return fail(HGA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_attend(p, cfg->dtype, cfg->out_dtype, q, pos, k, v, group_idx, out, lse,
                                workspace, err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_attend");
}

hga_status hga_decode_step(const hga_config* cfg, const void* q, const int64_t* pos,
                           float* chunk_sum, float* group_sum, int64_t n_alloc, const void* k,
                           const void* v, int32_t* chunk_idx, float* chunk_score,
                           int32_t* group_idx, float* group_score, void* out, float* lse,
                           int32_t append, void* stream) {
  Range nvtx_range("hga_decode_step");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if (!q || !pos || !chunk_sum || !group_sum || !k || !v || !chunk_idx || !group_idx || !out)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (cfg->kv_loc != HGA_KV_DEVICE || !decode_step_path(p, cfg->dtype))
    return fail(HGA_ERR_UNSUPPORTED,
                "hga_decode_step is built for bf16, head_dim 128, group 16 decode with K/V in "
                "device memory; use hga_route + hga_attend");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_decode_step(p, cfg->out_dtype, q, pos, chunk_sum, group_sum, k, v,
                                     chunk_idx, chunk_score, group_idx, group_score, out, lse,
                                     append != 0, err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_decode_step");
}

hga_status hga_decode_step_launches(const hga_config* cfg, int64_t n_alloc, int32_t* launches) {
  if (!launches) return fail(HGA_ERR_INVALID_ARG, "launches is NULL");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if (cfg->kv_loc != HGA_KV_DEVICE || !decode_step_path(p, cfg->dtype))
    return fail(HGA_ERR_UNSUPPORTED, "hga_decode_step does not take this shape");
  *launches = decode_item_path(p) ? 1 : 2;
  return HGA_OK;
}

// Checks a paged pool and derives p for n_alloc = max_pages * page_size.
static hga_status paged_params(const hga_config* cfg, const hga_kv_pages* kv, LayerParams* p,
                               KvPages* out) {
  if (!kv || !kv->block_table) return fail(HGA_ERR_INVALID_ARG, "null block table");
  if (kv->page_size <= 0 || kv->page_size % 16 != 0)
    return fail(HGA_ERR_INVALID_ARG, "page_size %d is not a positive multiple of 16", kv->page_size);
  if (kv->max_pages <= 0 || kv->n_pages <= 0)
    return fail(HGA_ERR_INVALID_ARG, "max_pages and n_pages must be positive");
  const int64_t n_alloc = static_cast<int64_t>(kv->max_pages) * kv->page_size;
  hga_status st = make_params(cfg, n_alloc, 1, p);
  if (st != HGA_OK) return st;
  if (kv->n_pages * p->Hkv * kv->page_size >= (static_cast<int64_t>(1) << 31) ||
      n_alloc >= (static_cast<int64_t>(1) << 31))
    return fail(HGA_ERR_UNSUPPORTED, "the pool, or a sequence's capacity, has 2^31 rows or more");
  int shift = -1;
  for (int s = 0; s < 31; ++s)
    if ((1 << s) == kv->page_size) shift = s;
  *out = KvPages{kv->block_table, kv->page_size, kv->max_pages, kv->n_pages, shift};
  return HGA_OK;
}

hga_status hga_build_summaries_paged(const hga_config* cfg, const void* k_pages,
                                     const hga_kv_pages* kv, const int64_t* seq_len,
                                     float* chunk_sum, float* group_sum, void* stream) {
  Range nvtx_range("hga_build_summaries_paged");
  LayerParams p;
  KvPages pages;
  hga_status st = paged_params(cfg, kv, &p, &pages);
  if (st != HGA_OK) return st;
  if (!k_pages || !seq_len || !chunk_sum || !group_sum)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_summaries_paged(p, cfg->dtype, k_pages, pages, seq_len, chunk_sum,
                                         group_sum, err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_build_summaries_paged");
}

hga_status hga_decode_step_paged(const hga_config* cfg, const void* q, const int64_t* pos,
                                 float* chunk_sum, float* group_sum, const void* k_pages,
                                 const void* v_pages, const hga_kv_pages* kv, int32_t* chunk_idx,
                                 float* chunk_score, int32_t* group_idx, float* group_score,
                                 void* out, float* lse, int32_t append, void* stream) {
  Range nvtx_range("hga_decode_step_paged");
  LayerParams p;
  KvPages pages;
  hga_status st = paged_params(cfg, kv, &p, &pages);
  if (st != HGA_OK) return st;
  if (!q || !pos || !chunk_sum || !group_sum || !k_pages || !v_pages || !chunk_idx ||
      !group_idx || !out)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (cfg->kv_loc != HGA_KV_DEVICE || !decode_fast_path(p, cfg->dtype) ||
      !decode_item_path(p, pages.max_pages))
    return fail(HGA_ERR_UNSUPPORTED,
                "hga_decode_step_paged is one launch of the decode-step kernel: bf16, head_dim "
                "128, group 16, top-k within its limits and a block-table row that fits in "
                "shared memory");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_decode_step(p, cfg->out_dtype, q, pos, chunk_sum, group_sum, k_pages,
                                     v_pages, chunk_idx, chunk_score, group_idx, group_score,
                                     out, lse, append != 0, err,
                                     static_cast<cudaStream_t>(stream), pages);
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_decode_step_paged");
}

hga_status hga_attend_backward_workspace_size(const hga_config* cfg, int64_t n_alloc,
                                              int32_t q_len, size_t* bytes) {
  if (!bytes) return fail(HGA_ERR_INVALID_ARG, "bytes is NULL");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, q_len, &p);
  if (st != HGA_OK) return st;
  if (!backward_path(p, cfg->dtype))
    return fail(HGA_ERR_UNSUPPORTED,
                "the backward pass is built for bf16, head_dim 128, group 16 prefill of whole "
                "chunks, G <= 16, topk_groups <= 128");
  *bytes = backward_workspace_bytes(p);
  return HGA_OK;
}

hga_status hga_attend_backward(const hga_config* cfg, const void* q, int32_t q_len,
                               const int64_t* pos, const void* k, const void* v, int64_t n_alloc,
                               const int32_t* group_idx, const void* out, const float* lse,
                               const void* d_out, float* dq, float* dk, float* dv,
                               void* workspace, size_t workspace_bytes, void* stream) {
  Range nvtx_range("hga_attend_backward");
  size_t need = 0;
  hga_status st = hga_attend_backward_workspace_size(cfg, n_alloc, q_len, &need);
  if (st != HGA_OK) return st;
  if (!q || !pos || !k || !v || !group_idx || !out || !lse || !d_out || !dq || !dk || !dv)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (!workspace || workspace_bytes < need)
    return fail(HGA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                workspace_bytes);
  LayerParams p;
  make_params(cfg, n_alloc, q_len, &p);
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_attend_backward(p, q, k, v, out, cfg->out_dtype == HGA_F32 ? 1 : 0, lse,
                                         d_out, pos, group_idx, dq, dk, dv, workspace, err,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_attend_backward");
}

hga_status hga_warm_plan(const hga_config* cfg, int64_t n_alloc, const int64_t* pos,
                         const int32_t* group_idx, int32_t warm_groups, int32_t* tags,
                         int32_t* stamps, int32_t* slot_map, int32_t* plan, int32_t* n_plan,
                         uint64_t* counters, void* stream) {
  Range nvtx_range("hga_warm_plan");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  if ((st = check_warm(p, warm_groups)) != HGA_OK) return st;
  if (!pos || !group_idx || !tags || !stamps || !slot_map || !plan || !n_plan)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_gather_warm(p, nullptr, nullptr, pos, group_idx, warm_groups, tags, stamps,
                                     slot_map, nullptr, nullptr, 0,
                                     reinterpret_cast<unsigned long long*>(counters), err,
                                     static_cast<cudaStream_t>(stream),
                                     reinterpret_cast<int2*>(plan), n_plan);
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_warm_plan");
}

hga_status hga_warm_fill(const hga_config* cfg, int64_t n_alloc, const int64_t* pos,
                         const void* staging, const int32_t* plan, const int32_t* n_plan,
                         int32_t warm_groups, int32_t window_mode, void* k_work, void* v_work,
                         void* stream) {
  Range nvtx_range("hga_warm_fill");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  if ((st = check_warm(p, warm_groups)) != HGA_OK) return st;
  if (!pos || !staging || !plan || !n_plan || !k_work || !v_work)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (window_mode < 0 || window_mode > 2)
    return fail(HGA_ERR_INVALID_ARG, "window_mode %d is not 0, 1 or 2", window_mode);
  unsigned* err = nullptr;
  if ((st = device_error_ptr(&err)) != HGA_OK) return st;
  cudaError_t e = launch_warm_fill(p, staging, reinterpret_cast<const int2*>(plan), n_plan, pos,
                                   warm_groups, window_mode, k_work, v_work, err,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "hga_warm_fill");
}

}  // extern "C"

struct hga_cold_store {
  hga::ColdStore s;
  int32_t B, Hkv;
};

extern "C" {

hga_status hga_cold_stage_bytes(const hga_config* cfg, size_t* bytes) {
  if (!bytes) return fail(HGA_ERR_INVALID_ARG, "bytes is NULL");
  LayerParams p;
  hga_status st = make_params(cfg, cfg ? cfg->chunk : 0, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  *bytes = static_cast<size_t>(p.B) * p.Hkv * cold_stage_unit_bytes(p);
  return HGA_OK;
}

hga_status hga_cold_open(const char* path, const hga_config* cfg, int64_t n_alloc,
                         int32_t create, hga_cold_store** store) {
  if (!path || !store) return fail(HGA_ERR_INVALID_ARG, "null pointer");
  LayerParams p;
  hga_status st = make_params(cfg, n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  hga_cold_store* h = new (std::nothrow) hga_cold_store;
  if (!h) return fail(HGA_ERR_INVALID_ARG, "out of host memory");
  const std::string e = cold_open(path, static_cast<int64_t>(p.B) * p.Hkv, n_alloc, p.D * 2,
                                  create != 0, &h->s);
  if (!e.empty()) {
    delete h;
    return fail(HGA_ERR_INVALID_ARG, "hga_cold_open: %s", e.c_str());
  }
  h->B = p.B;
  h->Hkv = p.Hkv;
  *store = h;
  return HGA_OK;
}

hga_status hga_cold_close(hga_cold_store* store) {
  if (!store) return fail(HGA_ERR_INVALID_ARG, "store is NULL");
  cold_close(&store->s);
  delete store;
  return HGA_OK;
}

hga_status hga_cold_write(hga_cold_store* store, const void* k, const void* v, int64_t t0,
                          int64_t t1, int32_t threads) {
  Range nvtx_range("hga_cold_write");
  if (!store || !k || !v) return fail(HGA_ERR_INVALID_ARG, "null pointer");
  if (t0 < 0 || t1 < t0 || t1 > store->s.n_alloc)
    return fail(HGA_ERR_INVALID_ARG, "need 0 <= t0 <= t1 <= n_alloc");
  const std::string e = cold_write(store->s, k, v, t0, t1, threads);
  return e.empty() ? HGA_OK : fail(HGA_ERR_INVALID_ARG, "hga_cold_write: %s", e.c_str());
}

hga_status hga_cold_stage(hga_cold_store* store, const hga_config* cfg, const int64_t* pos,
                          const int32_t* plan, const int32_t* n_plan, int32_t window_mode,
                          void* staging, int32_t threads) {
  Range nvtx_range("hga_cold_stage");
  if (!store || !pos || !plan || !n_plan || !staging)
    return fail(HGA_ERR_INVALID_ARG, "null pointer");
  LayerParams p;
  hga_status st = make_params(cfg, store->s.n_alloc, 1, &p);
  if (st != HGA_OK) return st;
  if ((st = check_host_tier(cfg, p)) != HGA_OK) return st;
  if (p.B != store->B || p.Hkv != store->Hkv)
    return fail(HGA_ERR_SHAPE, "the store was opened for another batch or head count");
  if (window_mode < 0 || window_mode > 2)
    return fail(HGA_ERR_INVALID_ARG, "window_mode %d is not 0, 1 or 2", window_mode);
  const std::string e = cold_stage(store->s, p, pos, reinterpret_cast<const int2*>(plan), n_plan,
                                   window_mode, staging, threads);
  return e.empty() ? HGA_OK : fail(HGA_ERR_INVALID_ARG, "hga_cold_stage: %s", e.c_str());
}

}  // extern "C"
