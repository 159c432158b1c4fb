// Internal launchers of the HGA kernels (host side, C++; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace hga {

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

// Workspace bytes of launch_attend for p (0 when the launch needs none).
size_t attend_workspace_bytes(const LayerParams& p);

cudaError_t launch_attend(const LayerParams& p, int dtype, int out_dtype, const void* q,
                          const int64_t* pos, const void* k, const void* v,
                          const int32_t* group_idx, void* out, float* lse, void* ws,
                          unsigned* err, cudaStream_t s);

}  // namespace hga
