// Shared device helpers of the HGA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

namespace hga {

// Bits of the sticky device error word.
enum DeviceErr : unsigned {
  kErrPos = 1u << 0,          // pos[b] out of range for n_alloc / q_len
  kErrPrefillAlign = 1u << 1, // prefill queries not on whole aligned chunks
  kErrChunkIdx = 1u << 2,     // chunk_idx entry not a complete candidate chunk / not ascending
  kErrGroupIdx = 1u << 3,     // group_idx entry not a group of a candidate chunk
  kErrTimeout = 1u << 4,      // a bounded wait gave up
  kErrPage = 1u << 5,         // a block-table entry a step needs is not a page of the pool
};

// Layer parameters as the kernels see them (derived from hga_config).
struct LayerParams {
  int B, Hq, Hkv, G, D;
  int C, g, Ng;               // chunk, group, groups per chunk
  int sink, local, kc, kg;
  int n_high;                 // high-frequency RoPE pairs
  int q_len, nblk;            // queries per sequence, routing blocks per sequence
  int64_t n_alloc;            // cache rows per (b, h)
  int n_chunks;               // n_alloc / C
  double theta;
  unsigned debug;             // test hooks (kDebug* bits); 0 in normal use
};

// Paged K/V: k and v are pools [n_pages][Hkv][page_size][D]; token t of
// sequence b lives in page block_table[b * max_pages + t / page_size], row
// t % page_size.  page_size is a multiple of 16, so a group (and every 16-row
// tile the kernels move) never straddles two pages.  block_table == nullptr:
// the dense layout [B][Hkv][n_alloc][D].
struct KvPages {
  const int32_t* block_table;
  int page_size;
  int max_pages;   // entries per sequence; n_alloc = max_pages * page_size < 2^31
  int64_t n_pages;
  int page_shift;  // log2(page_size) when it is a power of two, else -1
};

// Block-table index of token t (t < 2^31).
__host__ __device__ __forceinline__ uint32_t page_index(const KvPages& kv, uint32_t t) {
  return kv.page_shift >= 0 ? t >> kv.page_shift : t / static_cast<uint32_t>(kv.page_size);
}

// Row of token t of (b, h) in the [rows][D] view of a paged pool, given its
// page (validated by the caller).
__host__ __device__ __forceinline__ int64_t paged_row(const KvPages& kv, int Hkv, int h,
                                                     int32_t page, int64_t t) {
  const uint32_t tt = static_cast<uint32_t>(t);
  return (static_cast<int64_t>(page) * Hkv + h) * kv.page_size +
         (tt - page_index(kv, tt) * static_cast<uint32_t>(kv.page_size));
}

// Test hook of the one-launch decode step: warp 0 skips its first group-summary
// copy of the first item of each CTA but still waits for it, so that bounded wait
// runs out (nothing is in flight into that stage) and the kernel reports
// HGA_ERR_TIMEOUT through the device error word.
constexpr unsigned kDebugSkipRouteArrive = 1u;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void store_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Load 4 consecutive elements starting at p (16 B aligned for float, 8 B for bf16).
__device__ __forceinline__ void load4(const float* p, float (&o)[4]) {
  float4 v = __ldg(reinterpret_cast<const float4*>(p));
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&o)[4]) {
  uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
  o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xffff0000u);
  o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xffff0000u);
}
__device__ __forceinline__ void load2(const float* p, float (&o)[2]) {
  float2 v = __ldg(reinterpret_cast<const float2*>(p));
  o[0] = v.x; o[1] = v.y;
}
__device__ __forceinline__ void load2(const __nv_bfloat16* p, float (&o)[2]) {
  unsigned v = __ldg(reinterpret_cast<const unsigned*>(p));
  o[0] = __uint_as_float(v << 16); o[1] = __uint_as_float(v & 0xffff0000u);
}

// Programmatic dependent launch.  Every kernel of the library launches with the
// programmatic-serialization attribute, waits for its stream predecessor before
// reading anything a predecessor may have written, and lets its own dependents
// launch only after that wait, near the end of its work (so that waiting
// dependent CTAs do not take SM slots the kernel still needs).  The code a
// kernel runs before pdl_wait() overlaps the tail of its predecessor and may
// read only data no kernel of this library writes (q, pos, k, v).  Without
// the attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void flag_error(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Position check shared by every kernel: 0 <= pos < n_alloc, pos >= q_len-1,
// and for prefill (q_len > 1) whole aligned chunks.
__device__ __forceinline__ bool valid_position(int64_t pos, const LayerParams& p, unsigned* err) {
  if (pos < 0 || pos >= p.n_alloc || pos < p.q_len - 1) {
    flag_error(err, kErrPos);
    return false;
  }
  if (p.q_len > 1 && ((pos + 1) % p.C != 0 || p.q_len % p.C != 0)) {
    flag_error(err, kErrPrefillAlign);
    return false;
  }
  return true;
}

}  // namespace hga
