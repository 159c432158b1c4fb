// Cold tier: the K/V history in a file (an NVMe drive behind host RAM), read
// with positioned reads by a pool of host threads into pinned staging.
#pragma once

#include <cstdint>
#include <string>

#include "kernels.h"

namespace hga {

struct ColdStore {
  int fd = -1;
  int64_t units = 0;      // B * Hkv
  int64_t n_alloc = 0;    // rows per (sequence, KV head)
  int64_t row_bytes = 0;  // D * 2 (bf16)
};

// Each returns an empty string on success, else what failed.
std::string cold_open(const char* path, int64_t units, int64_t n_alloc, int64_t row_bytes,
                      bool create, ColdStore* out);
void cold_close(ColdStore* s);
// Rows [t0, t1) of every (sequence, KV head) from host k, v [units][n_alloc][D].
std::string cold_write(const ColdStore& s, const void* k, const void* v, int64_t t0, int64_t t1,
                       int threads);
// Stages one warm step: per (sequence, KV head) u, the n_plan[u] missed groups
// plan[u * kg + r].x and the window rows of pos[u / Hkv] under `mode`, in the
// layout launch_warm_fill reads.
std::string cold_stage(const ColdStore& s, const LayerParams& p, const int64_t* pos,
                       const int2* plan, const int32_t* n_plan, int mode, void* staging,
                       int threads);

}  // namespace hga
