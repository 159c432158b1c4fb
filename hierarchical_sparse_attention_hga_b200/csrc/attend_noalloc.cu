// hga_attend_noalloc: hga_attend for callers that cannot allocate device memory.
//
// Some callers cannot hand this library a workspace: frameworks that own all
// device memory through their own pool and give an attention plugin only its
// input and output buffers, and latency-critical loops in which a cudaMalloc
// or cudaFree (which may synchronise the whole device) is not allowed.  This
// entry point runs the same attention as hga_attend, with the split-K scratch
// held in one fixed array inside the library instead of a caller buffer.
//
// The array has a fixed size (kNoAllocScratchBytes below) and lives on every
// GPU that loads the library until the process exits.  All calls on a device
// share it and it keeps the previous call's contents; nothing in it needs to
// start at zero, because each call writes every byte it later reads.  Calls
// whose kernels overlap on the GPU (several streams, several host threads)
// race on the array and give wrong results: serialise them.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/hga.h"

namespace hga {
void set_last_error(const char* msg);
}

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per GPU

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with that device current (cudaGetSymbolAddress) and cached.
hga_status scratch_ptr(void** out) {
  int dev = 0;
  char msg[256];
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "hga_attend_noalloc: cudaGetDevice failed: %s",
             cudaGetErrorString(e));
    hga::set_last_error(msg);
    return HGA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof(msg), "hga_attend_noalloc: device ordinal %d (at most %d devices)", dev,
             kMaxDevices);
    hga::set_last_error(msg);
    return HGA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      snprintf(msg, sizeof(msg), "hga_attend_noalloc: cudaGetSymbolAddress failed: %s",
               cudaGetErrorString(e));
      hga::set_last_error(msg);
      return HGA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HGA_OK;
}

}  // namespace

extern "C" hga_status hga_attend_noalloc(const hga_config* cfg, const void* q, int32_t q_len,
                                         const int64_t* pos, const void* k, const void* v,
                                         int64_t n_alloc, const int32_t* group_idx, void* out,
                                         float* lse, void* stream) {
  size_t need = 0;
  hga_status st = hga_workspace_size(cfg, n_alloc, q_len, &need);
  if (st != HGA_OK) return st;
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "hga_attend_noalloc: this shape needs %zu bytes of scratch, more than the %zu-byte "
             "built-in array; use hga_attend with a caller workspace",
             need, kNoAllocScratchBytes);
    hga::set_last_error(msg);
    return HGA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0 && (st = scratch_ptr(&scratch)) != HGA_OK) return st;
  return hga_attend(cfg, q, q_len, pos, k, v, n_alloc, group_idx, out, lse, scratch,
                    kNoAllocScratchBytes, stream);
}
