// Step 1: RoPE-aware chunk and group key summaries.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", items 1 and 3: the sequence is
// cut into chunks of C tokens and each chunk into groups; a summary averages the
// high-frequency RoPE pairs of the rotated keys, and averages the low-frequency
// pairs in raw-key space before rotating them to the span's representative
// position (its centre, t0 + (L-1)/2).
//
// Because k is stored post-RoPE, un-rotating token t and re-rotating at r is
// one rotation by (r - t) * omega, and r - t = (L-1)/2 - o depends only on the
// token's offset o inside the span.  The kernel therefore keeps one table of
// cos/sin per (offset, low pair) in shared memory and sums R((L-1)/2 - o) k[t]
// over the span: a fixed linear map per span, one HBM read of k.
//
// Work split: a warp owns whole chunks of one (b, h); lane l owns the RoPE pairs
// l*PPL .. l*PPL+PPL-1 (both halves of each pair, dims i and i + D/2), so a
// warp reads a key row as two contiguous 4*D/2-byte halves.  Every chunk or
// group row whose last token lies in [t_begin, t_end) is computed in token
// order from the cache alone: a decode append and a batch build produce the
// same bits.
#include "common.cuh"
#include "kernels.h"

namespace hga {
namespace {

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

constexpr int kWarps = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
summaries_kernel(const T* __restrict__ k, LayerParams p, int64_t t_begin, int64_t t_end,
                 int c_first, int c_count, int chunks_per_warp, int with_chunk_table,
                 float* __restrict__ chunk_sum, float* __restrict__ group_sum) {
  constexpr int P = D / 2;
  constexpr int PPL = P / 32;
  extern __shared__ float2 smem_tab[];
  const int n_lo = P - p.n_high;
  const int rows_c = with_chunk_table ? p.C : 0;
  float2* tab_c = smem_tab;                   // [C][n_lo]: rotation by (C-1)/2 - o
  float2* tab_g = smem_tab + rows_c * n_lo;   // [g][n_lo]: rotation by (g-1)/2 - o
  // Angles are formed in double from omega_i = theta^(-2i/D) and the exact
  // half-integer offset, then rounded once to float for sincosf.
  for (int idx = threadIdx.x; idx < (rows_c + p.g) * n_lo; idx += blockDim.x) {
    const bool is_c = idx < rows_c * n_lo;
    const int j = is_c ? idx : idx - rows_c * n_lo;
    const int o = j / n_lo;
    const int i = p.n_high + j % n_lo;
    const double omega = pow(p.theta, -2.0 * i / D);
    const double half = is_c ? 0.5 * (p.C - 1) : 0.5 * (p.g - 1);
    float s, c;
    sincosf(static_cast<float>((half - o) * omega), &s, &c);
    smem_tab[idx] = make_float2(c, s);
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const T* kb = k + static_cast<size_t>(bh) * p.n_alloc * D;
  const float inv_c = 1.0f / p.C, inv_g = 1.0f / p.g;

  for (int j = 0; j < chunks_per_warp; ++j) {
    const int ci = (blockIdx.x * kWarps + warp) * chunks_per_warp + j;
    if (ci >= c_count) break;
    const int c = c_first + ci;
    const int64_t c0 = static_cast<int64_t>(c) * p.C;
    const bool fin_c = c0 + p.C - 1 >= t_begin && c0 + p.C - 1 < t_end;
    float cx[PPL], cy[PPL];
#pragma unroll
    for (int u = 0; u < PPL; ++u) cx[u] = cy[u] = 0.f;

    for (int gi = 0; gi < p.Ng; ++gi) {
      const int64_t g0 = c0 + static_cast<int64_t>(gi) * p.g;
      const bool fin_g = g0 + p.g - 1 >= t_begin && g0 + p.g - 1 < t_end;
      if (!fin_c && !fin_g) continue;
      float gx[PPL], gy[PPL];
#pragma unroll
      for (int u = 0; u < PPL; ++u) gx[u] = gy[u] = 0.f;
#pragma unroll 4
      for (int o = 0; o < p.g; ++o) {
        const T* row = kb + (g0 + o) * D + lane * PPL;
        float x[PPL], y[PPL];
        PairLoad<T, PPL>::run(row, x);
        PairLoad<T, PPL>::run(row + P, y);
        const int oc = gi * p.g + o;
#pragma unroll
        for (int u = 0; u < PPL; ++u) {
          const int i = lane * PPL + u;
          if (i < p.n_high) {
            cx[u] += x[u]; cy[u] += y[u];
            gx[u] += x[u]; gy[u] += y[u];
          } else {
            const int il = i - p.n_high;
            if (fin_c) {
              const float2 r = tab_c[oc * n_lo + il];
              cx[u] += x[u] * r.x - y[u] * r.y;
              cy[u] += x[u] * r.y + y[u] * r.x;
            }
            const float2 r = tab_g[o * n_lo + il];
            gx[u] += x[u] * r.x - y[u] * r.y;
            gy[u] += x[u] * r.y + y[u] * r.x;
          }
        }
      }
      if (fin_g) {
        float* dst = group_sum + ((static_cast<size_t>(bh) * p.n_chunks + c) * p.Ng + gi) * D;
#pragma unroll
        for (int u = 0; u < PPL; ++u) {
          dst[lane * PPL + u] = gx[u] * inv_g;
          dst[P + lane * PPL + u] = gy[u] * inv_g;
        }
      }
    }
    if (fin_c) {
      float* dst = chunk_sum + (static_cast<size_t>(bh) * p.n_chunks + c) * D;
#pragma unroll
      for (int u = 0; u < PPL; ++u) {
        dst[lane * PPL + u] = cx[u] * inv_c;
        dst[P + lane * PPL + u] = cy[u] * inv_c;
      }
    }
  }
}

template <typename T, int D>
cudaError_t launch_summaries_t(const LayerParams& p, const void* k, int64_t t_begin, int64_t t_end,
                               float* chunk_sum, float* group_sum, cudaStream_t stream) {
  // First group end and first chunk end at or after t_begin.
  const int64_t first_g_end = (t_begin / p.g) * p.g + p.g - 1;
  if (t_end <= t_begin || first_g_end >= t_end) return cudaSuccess;  // no row closes
  const int64_t first_c_end = (t_begin / p.C) * p.C + p.C - 1;
  const int with_chunk_table = first_c_end < t_end ? 1 : 0;
  const int c_first = static_cast<int>(t_begin / p.C);
  const int c_last = static_cast<int>((t_end - 1) / p.C);
  const int c_count = c_last - c_first + 1;
  const int cpw = c_count >= 64 ? 4 : 1;
  const int per_cta = kWarps * cpw;
  dim3 grid((c_count + per_cta - 1) / per_cta, p.B * p.Hkv);
  const int n_lo = D / 2 - p.n_high;
  const size_t smem = static_cast<size_t>((with_chunk_table ? p.C : 0) + p.g) * n_lo * sizeof(float2);
  auto kern = summaries_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kWarps * 32, smem, stream>>>(static_cast<const T*>(k), p, t_begin, t_end, c_first,
                                            c_count, cpw, with_chunk_table, chunk_sum, group_sum);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_summaries(const LayerParams& p, int dtype, const void* k, int64_t t_begin,
                             int64_t t_end, float* chunk_sum, float* group_sum, cudaStream_t s) {
  if (dtype == 0) {
    return p.D == 64 ? launch_summaries_t<float, 64>(p, k, t_begin, t_end, chunk_sum, group_sum, s)
                     : launch_summaries_t<float, 128>(p, k, t_begin, t_end, chunk_sum, group_sum, s);
  }
  return p.D == 64
             ? launch_summaries_t<__nv_bfloat16, 64>(p, k, t_begin, t_end, chunk_sum, group_sum, s)
             : launch_summaries_t<__nv_bfloat16, 128>(p, k, t_begin, t_end, chunk_sum, group_sum, s);
}

}  // namespace hga
