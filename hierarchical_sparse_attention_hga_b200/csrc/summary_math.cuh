// Arithmetic of the RoPE-aware key summaries (step 1), shared by the batch
// builder (summaries.cu) and the summary append fused into the decode step
// (decode_step.cu), so that both write the same bits for the same row.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", item 3: high-frequency RoPE
// pairs are averaged as stored (already rotated per token); low-frequency pairs
// are averaged as raw keys and rotated to the span's representative position,
// its centre t0 + (L-1)/2.  With post-RoPE keys that is one rotation of token
// t by (r - t) * omega_i before the mean.
//
// Every product and sum is written with an explicit rounding (__fmul_rn,
// __fadd_rn, fmaf), so no compiler contraction choice can make two kernels
// disagree.
#pragma once

#include "common.cuh"

namespace hga {
namespace summ {

constexpr int kGroup = 16;

// Entries of the rotation table (float2 = (cos, sin)) of p: [g][n_lo] for the
// rotation by (g-1)/2 - o of a group's token o, then [Ng][n_lo] for the
// rotation by (C-g)/2 - w*g that takes group w's centre to the chunk's.
__host__ __device__ inline int table_entries(const LayerParams& p, int D) {
  return (kGroup + p.Ng) * (D / 2 - p.n_high);
}

// Entry idx of the table.  The angle is formed in double from
// omega_i = theta^(-2i/D) and the exact half-integer offset, then rounded once
// to float for sincosf.
__device__ inline float2 table_entry(const LayerParams& p, int D, int idx) {
  const int n_lo = D / 2 - p.n_high;
  const bool is_g = idx < kGroup * n_lo;
  const int j = is_g ? idx : idx - kGroup * n_lo;
  const int o = j / n_lo;
  const double omega = pow(p.theta, -2.0 * (p.n_high + j % n_lo) / D);
  const double off = is_g ? 0.5 * (kGroup - 1) - o : 0.5 * (p.C - kGroup) - o * kGroup;
  float s, c;
  sincosf(static_cast<float>(off * omega), &s, &c);
  return make_float2(c, s);
}

// Adds the (x, y) pair of dims (i, i + D/2) rotated by r = (cos, sin) to (sx, sy).
__device__ __forceinline__ void add_rotated(float& sx, float& sy, float x, float y, float2 r) {
  sx = __fadd_rn(sx, fmaf(x, r.x, __fmul_rn(-y, r.y)));
  sy = __fadd_rn(sy, fmaf(x, r.y, __fmul_rn(y, r.x)));
}

// Raw (unnormalised) sum of one group of kGroup keys for the PPL pairs
// i = lane*PPL + u this lane owns: x[o][u] = key o, dim i; y[o][u] = dim i + D/2.
// tab_g is the [g][n_lo] part of the table.
template <int PPL>
__device__ __forceinline__ void group_raw_sum(const float (&x)[kGroup][PPL],
                                              const float (&y)[kGroup][PPL], const float2* tab_g,
                                              int n_high, int n_lo, int lane, float (&gx)[PPL],
                                              float (&gy)[PPL]) {
#pragma unroll
  for (int u = 0; u < PPL; ++u) gx[u] = gy[u] = 0.f;
#pragma unroll
  for (int o = 0; o < kGroup; ++o) {
#pragma unroll
    for (int u = 0; u < PPL; ++u) {
      const int i = lane * PPL + u;
      if (i < n_high) {
        gx[u] = __fadd_rn(gx[u], x[o][u]);
        gy[u] = __fadd_rn(gy[u], y[o][u]);
      } else {
        add_rotated(gx[u], gy[u], x[o][u], y[o][u], tab_g[o * n_lo + i - n_high]);
      }
    }
  }
}

// Pair i of a chunk row from the raw group sums gsum[w][0..D) of its Ng groups
// (x part at [i], y part at [D/2 + i]); tab_s is the [Ng][n_lo] part of the
// table.  Returns the unnormalised (sx, sy).
template <int D>
__device__ __forceinline__ float2 chunk_pair(const float (*gsum)[D], const float2* tab_s, int ng,
                                             int n_high, int n_lo, int i) {
  constexpr int P = D / 2;
  float sx = 0.f, sy = 0.f;
  for (int w = 0; w < ng; ++w) {
    const float gx = gsum[w][i], gy = gsum[w][P + i];
    if (i < n_high) {
      sx = __fadd_rn(sx, gx);
      sy = __fadd_rn(sy, gy);
    } else {
      add_rotated(sx, sy, gx, gy, tab_s[w * n_lo + i - n_high]);
    }
  }
  return make_float2(sx, sy);
}

// PPL = D / 64 pairs per lane: loads of the (x, y) halves of one key row.
template <typename T, int PPL> struct PairLoad;
template <> struct PairLoad<float, 2> {
  static __device__ __forceinline__ void run(const float* p, float (&o)[2]) { load2(p, o); }
};
template <> struct PairLoad<__nv_bfloat16, 2> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, float (&o)[2]) { load2(p, o); }
};
template <> struct PairLoad<float, 1> {
  static __device__ __forceinline__ void run(const float* p, float (&o)[1]) { o[0] = __ldg(p); }
};
template <> struct PairLoad<__nv_bfloat16, 1> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, float (&o)[1]) {
    o[0] = __bfloat162float(p[0]);
  }
};

// The summary rows of one (sequence, KV head) item whose last token is pb: the
// group that pb ends, and the chunk when pb ends it too (a chunk row needs the
// raw sums of all its groups, recomputed here from the cache).  One warp;
// group_rows(t0) gives the item's key row t0 of a group start t0 (the group's
// rows follow it contiguously), or null when that group is not available;
// chunk_sum / group_sum are the item's tables, tab the full rotation table,
// gsum [Ng][D] scratch.  Nothing is written unless pb ends a group; false
// (and nothing written) when a group the rows need is not available.
template <typename T, int D, typename GroupRows>
__device__ bool append_closed_rows(GroupRows group_rows, float* chunk_sum, float* group_sum,
                                   const LayerParams& p, int64_t pb, const float2* tab,
                                   float (*gsum)[D]) {
  constexpr int P = D / 2, PPL = P / 32;
  if ((pb + 1) % kGroup != 0) return true;
  const int lane = threadIdx.x & 31;
  const int n_lo = P - p.n_high;
  const int c = static_cast<int>(pb / p.C);
  const bool closes_chunk = (pb + 1) % p.C == 0;
  const int w_close = static_cast<int>(pb % p.C) / kGroup;
  for (int w = closes_chunk ? 0 : w_close; w <= w_close; ++w) {
    const int64_t g0 = static_cast<int64_t>(c) * p.C + static_cast<int64_t>(w) * kGroup;
    const T* grp = group_rows(g0);
    if (grp == nullptr) return false;
    float x[kGroup][PPL], y[kGroup][PPL];
#pragma unroll
    for (int o = 0; o < kGroup; ++o) {
      const T* row = grp + o * D + lane * PPL;
      PairLoad<T, PPL>::run(row, x[o]);
      PairLoad<T, PPL>::run(row + P, y[o]);
    }
    float gx[PPL], gy[PPL];
    group_raw_sum<PPL>(x, y, tab, p.n_high, n_lo, lane, gx, gy);
    if (w == w_close) {
      float* dst = group_sum + (static_cast<size_t>(c) * p.Ng + w) * D;
#pragma unroll
      for (int u = 0; u < PPL; ++u) {
        dst[lane * PPL + u] = __fmul_rn(gx[u], 1.0f / kGroup);
        dst[P + lane * PPL + u] = __fmul_rn(gy[u], 1.0f / kGroup);
      }
    }
#pragma unroll
    for (int u = 0; u < PPL; ++u) {
      gsum[w][lane * PPL + u] = gx[u];
      gsum[w][P + lane * PPL + u] = gy[u];
    }
  }
  if (closes_chunk) {
    __syncwarp();
    const float inv_c = 1.0f / p.C;
    float* dst = chunk_sum + static_cast<size_t>(c) * D;
    for (int i = lane; i < P; i += 32) {
      const float2 sc = chunk_pair<D>(gsum, tab + kGroup * n_lo, p.Ng, p.n_high, n_lo, i);
      dst[i] = __fmul_rn(sc.x, inv_c);
      dst[P + i] = __fmul_rn(sc.y, inv_c);
    }
  }
  __syncwarp();
  return true;
}

}  // namespace summ
}  // namespace hga
