// Step 1: RoPE-aware chunk and group key summaries.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", items 1 and 3: the sequence is
// cut into chunks of C tokens and each chunk into groups; a summary averages the
// high-frequency RoPE pairs of the rotated keys, and averages the low-frequency
// pairs in raw-key space before rotating them to the span's representative
// position (its centre, t0 + (L-1)/2).
//
// k is stored post-RoPE, so un-rotating token t and re-rotating at the centre r
// is one rotation by (r - t) * omega_i.  For a group, r_g - t = (g-1)/2 - o
// depends only on the token's offset o in the group: one shared-memory table of
// g x (low pairs) cos/sin serves every group.  A chunk's sum is composed from
// its groups' sums: R(r_c - t) = R(r_c - r_w) R(r_w - t), so the chunk sum is
// sum_w R(delta_w) S_w with delta_w = (C-g)/2 - w*g, one more small table.
//
// One CTA per chunk (looping over chunks when a whole cache is built), one warp
// per group; lane l owns the pairs l*PPL .. l*PPL+PPL-1 (dims i and i + D/2).
// Every row whose last token lies in [t_begin, t_end) is computed from the
// cache alone in a fixed order, so a decode append and a batch build produce
// the same bits.
#include "common.cuh"
#include "kernels.h"
#include "summary_math.cuh"

namespace hga {
namespace {

using summ::PairLoad;
using summ::kGroup;

// Paged pools (PAGED): sequence b's rows past seq_len[b] are never read (their
// pages need not exist), and a group whose block-table entry is not a page of
// the pool is skipped and flagged, with the chunk row it belongs to.
template <typename T, int D, bool PRELOAD, bool PAGED>
__global__ void __launch_bounds__(256)
summaries_kernel(const T* __restrict__ k, LayerParams p, int64_t t_begin, int64_t t_end,
                 int c_first, int c_count, float* __restrict__ chunk_sum,
                 float* __restrict__ group_sum, KvPages kv, const int64_t* __restrict__ seq_len,
                 unsigned* err) {
  constexpr int P = D / 2;
  constexpr int PPL = P / 32;
  extern __shared__ float2 smem_tab[];
  __shared__ float s_gsum[8][D];             // raw group sums of one chunk
  __shared__ int s_missing[2];               // a group of the chunk had no page (by iteration parity)
  const int n_lo = P - p.n_high;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  if (PAGED) {  // this sequence's rows end at seq_len[b]
    const int64_t len = seq_len[b];
    t_end = min(t_end, max(static_cast<int64_t>(0), len));
  }
  // key row g0 of a group (its rows follow contiguously), or null
  auto group_rows = [&](int64_t g0) -> const T* {
    if (!PAGED) return k + (static_cast<size_t>(bh) * p.n_alloc + g0) * D;
    const int32_t pg = __ldg(kv.block_table + static_cast<size_t>(b) * kv.max_pages + page_index(kv, static_cast<uint32_t>(g0)));
    if (pg < 0 || pg >= kv.n_pages) {
      if (lane == 0) flag_error(err, kErrPage);
      return nullptr;
    }
    return k + static_cast<size_t>(paged_row(kv, p.Hkv, h, pg, g0)) * D;
  };
  // With PRELOAD (each CTA finishes one chunk: a decode append), the chunk's key
  // rows are loaded before the tables are built (k is never written by this
  // library), so their latency overlaps the table setup.
  float x0[kGroup][PPL], y0[kGroup][PPL];
  bool pre = PRELOAD && static_cast<int>(blockIdx.x) < c_count && warp < p.Ng;
  if (pre) {  // only rows the chunk or this warp's group finishes are read
    const int64_t c0 = static_cast<int64_t>(c_first + blockIdx.x) * p.C;
    const int64_t g0 = c0 + static_cast<int64_t>(warp) * kGroup;
    pre = (c0 + p.C - 1 >= t_begin && c0 + p.C - 1 < t_end) ||
          (g0 + kGroup - 1 >= t_begin && g0 + kGroup - 1 < t_end);
  }
  if (pre) {
    const int64_t g0 = static_cast<int64_t>(c_first + blockIdx.x) * p.C + static_cast<int64_t>(warp) * kGroup;
    const T* grp = group_rows(g0);
    pre = grp != nullptr;
    if (pre) {
#pragma unroll
      for (int o = 0; o < kGroup; ++o) {
        const T* row = grp + o * D + lane * PPL;
        PairLoad<T, PPL>::run(row, x0[o]);
        PairLoad<T, PPL>::run(row + P, y0[o]);
      }
    }
  }
  float2* tab_g = smem_tab;                  // [g][n_lo]: rotation by (g-1)/2 - o
  float2* tab_s = smem_tab + kGroup * n_lo;  // [Ng][n_lo]: rotation by (C-g)/2 - w*g
  for (int idx = threadIdx.x; idx < summ::table_entries(p, D); idx += blockDim.x)
    smem_tab[idx] = summ::table_entry(p, D, idx);
  if (threadIdx.x == 0) s_missing[0] = s_missing[1] = 0;
  __syncthreads();
  pdl_wait();

  for (int ci = blockIdx.x, it = 0; ci < c_count; ci += gridDim.x, ++it) {
    const int c = c_first + ci;
    // the other flag was last read before the previous iteration's final barrier
    // and is next written after this iteration's
    if (threadIdx.x == 0) s_missing[(it + 1) & 1] = 0;
    const int64_t c0 = static_cast<int64_t>(c) * p.C;
    const bool fin_c = c0 + p.C - 1 >= t_begin && c0 + p.C - 1 < t_end;
    // warp w: group w of the chunk
    if (warp < p.Ng) {
      const int64_t g0 = c0 + static_cast<int64_t>(warp) * kGroup;
      const bool fin_g = g0 + kGroup - 1 >= t_begin && g0 + kGroup - 1 < t_end;
      if (fin_c || fin_g) {
        float gx[PPL], gy[PPL];
        float x[kGroup][PPL], y[kGroup][PPL];
        bool have = true;
        if (PRELOAD && pre && ci == static_cast<int>(blockIdx.x)) {
#pragma unroll
          for (int o = 0; o < kGroup; ++o)
#pragma unroll
            for (int u = 0; u < PPL; ++u) {
              x[o][u] = x0[o][u];
              y[o][u] = y0[o][u];
            }
        } else {
          const T* grp = group_rows(g0);
          have = grp != nullptr;
          if (have) {
#pragma unroll
            for (int o = 0; o < kGroup; ++o) {
              const T* row = grp + o * D + lane * PPL;
              PairLoad<T, PPL>::run(row, x[o]);
              PairLoad<T, PPL>::run(row + P, y[o]);
            }
          } else if (lane == 0) {
            s_missing[it & 1] = 1;
          }
        }
        if (have) {
        summ::group_raw_sum<PPL>(x, y, tab_g, p.n_high, n_lo, lane, gx, gy);
        if (fin_g) {
          float* dst = group_sum + ((static_cast<size_t>(bh) * p.n_chunks + c) * p.Ng + warp) * D;
#pragma unroll
          for (int u = 0; u < PPL; ++u) {
            dst[lane * PPL + u] = __fmul_rn(gx[u], 1.0f / kGroup);
            dst[P + lane * PPL + u] = __fmul_rn(gy[u], 1.0f / kGroup);
          }
        }
#pragma unroll
        for (int u = 0; u < PPL; ++u) {
          s_gsum[warp][lane * PPL + u] = gx[u];
          s_gsum[warp][P + lane * PPL + u] = gy[u];
        }
        }
      }
    }
    if (fin_c) {  // uniform over the CTA
      __syncthreads();
      const float inv_c = 1.0f / p.C;
      float* dst = chunk_sum + (static_cast<size_t>(bh) * p.n_chunks + c) * D;
      if (!s_missing[it & 1]) {
        for (int i = threadIdx.x; i < P; i += blockDim.x) {
          const float2 sc = summ::chunk_pair<D>(s_gsum, tab_s, p.Ng, p.n_high, n_lo, i);
          dst[i] = __fmul_rn(sc.x, inv_c);
          dst[P + i] = __fmul_rn(sc.y, inv_c);
        }
      }
    }
    __syncthreads();
  }
  pdl_trigger();
}

template <typename T, int D, bool PAGED>
cudaError_t launch_summaries_t(const LayerParams& p, const void* k, int64_t t_begin, int64_t t_end,
                               float* chunk_sum, float* group_sum, const KvPages& kv,
                               const int64_t* seq_len, unsigned* err, cudaStream_t stream) {
  // First group end at or after t_begin: nothing to do if it is past t_end.
  const int64_t first_g_end = (t_begin / p.g) * p.g + p.g - 1;
  if (t_end <= t_begin || first_g_end >= t_end) return cudaSuccess;
  const int c_first = static_cast<int>(t_begin / p.C);
  const int c_last = static_cast<int>((t_end - 1) / p.C);
  const int c_count = c_last - c_first + 1;
  const int bh = p.B * p.Hkv;
  // enough CTAs for ~8 per SM, each looping over several chunks of one (b, h)
  int gx = static_cast<int>((device_sm_count() * 8 + bh - 1) / bh);
  gx = gx < 1 ? 1 : (gx > c_count ? c_count : gx);
  dim3 grid(gx, bh);
  const int n_lo = D / 2 - p.n_high;
  const size_t smem = static_cast<size_t>(kGroup + p.Ng) * n_lo * sizeof(float2);
  if (c_count <= gx)  // one chunk per CTA
    return launch_pdl(summaries_kernel<T, D, true, PAGED>, grid, dim3(32 * p.Ng), smem, stream, 1,
                      static_cast<const T*>(k), p, t_begin, t_end, c_first, c_count, chunk_sum,
                      group_sum, kv, seq_len, err);
  return launch_pdl(summaries_kernel<T, D, false, PAGED>, grid, dim3(32 * p.Ng), smem, stream, 1,
                    static_cast<const T*>(k), p, t_begin, t_end, c_first, c_count, chunk_sum,
                    group_sum, kv, seq_len, err);
}

// Summary append of a decode step with per-sequence positions: one warp per
// (sequence, KV head) item writes the rows its token pos[b] closes, with the
// batch builder's arithmetic.
template <typename T, int D>
__global__ void __launch_bounds__(32)
append_kernel(const T* __restrict__ k, const int64_t* __restrict__ pos, LayerParams p,
              float* __restrict__ chunk_sum, float* __restrict__ group_sum) {
  extern __shared__ float2 smem_tab[];
  __shared__ float s_gsum[8][D];
  for (int i = threadIdx.x; i < summ::table_entries(p, D); i += 32) smem_tab[i] = summ::table_entry(p, D, i);
  __syncwarp();
  pdl_wait();
  const int item = blockIdx.x;
  const int64_t pb = pos[item / p.Hkv];
  const T* kb = k + static_cast<size_t>(item) * p.n_alloc * D;
  if (pb >= 0 && pb < p.n_alloc)
    summ::append_closed_rows<T, D>([&](int64_t g0) { return kb + g0 * D; },
                                   chunk_sum + static_cast<size_t>(item) * p.n_chunks * D,
                                   group_sum + static_cast<size_t>(item) * p.n_chunks * p.Ng * D,
                                   p, pb, smem_tab, s_gsum);
  pdl_trigger();
}

template <typename T, int D>
cudaError_t launch_append_t(const LayerParams& p, const void* k, const int64_t* pos,
                            float* chunk_sum, float* group_sum, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(summ::table_entries(p, D)) * sizeof(float2);
  return launch_pdl(append_kernel<T, D>, dim3(p.B * p.Hkv), dim3(32), smem, s, 1,
                    static_cast<const T*>(k), pos, p, chunk_sum, group_sum);
}

}  // namespace

cudaError_t launch_append_per_sequence(const LayerParams& p, int dtype, const void* k,
                                       const int64_t* pos, float* chunk_sum, float* group_sum,
                                       cudaStream_t s) {
  if (dtype == 0)
    return p.D == 64 ? launch_append_t<float, 64>(p, k, pos, chunk_sum, group_sum, s)
                     : launch_append_t<float, 128>(p, k, pos, chunk_sum, group_sum, s);
  return p.D == 64 ? launch_append_t<__nv_bfloat16, 64>(p, k, pos, chunk_sum, group_sum, s)
                   : launch_append_t<__nv_bfloat16, 128>(p, k, pos, chunk_sum, group_sum, s);
}

cudaError_t launch_summaries(const LayerParams& p, int dtype, const void* k, int64_t t_begin,
                             int64_t t_end, float* chunk_sum, float* group_sum, cudaStream_t s) {
  const KvPages dense{nullptr, 0, 0, 0, -1};
  if (dtype == 0) {
    return p.D == 64 ? launch_summaries_t<float, 64, false>(p, k, t_begin, t_end, chunk_sum,
                                                           group_sum, dense, nullptr, nullptr, s)
                     : launch_summaries_t<float, 128, false>(p, k, t_begin, t_end, chunk_sum,
                                                            group_sum, dense, nullptr, nullptr, s);
  }
  return p.D == 64 ? launch_summaries_t<__nv_bfloat16, 64, false>(p, k, t_begin, t_end, chunk_sum,
                                                                 group_sum, dense, nullptr,
                                                                 nullptr, s)
                   : launch_summaries_t<__nv_bfloat16, 128, false>(p, k, t_begin, t_end, chunk_sum,
                                                                  group_sum, dense, nullptr,
                                                                  nullptr, s);
}

cudaError_t launch_summaries_paged(const LayerParams& p, int dtype, const void* k_pages,
                                   const KvPages& kv, const int64_t* seq_len, float* chunk_sum,
                                   float* group_sum, unsigned* err, cudaStream_t s) {
  if (dtype == 0) {
    return p.D == 64 ? launch_summaries_t<float, 64, true>(p, k_pages, 0, p.n_alloc, chunk_sum,
                                                          group_sum, kv, seq_len, err, s)
                     : launch_summaries_t<float, 128, true>(p, k_pages, 0, p.n_alloc, chunk_sum,
                                                           group_sum, kv, seq_len, err, s);
  }
  return p.D == 64 ? launch_summaries_t<__nv_bfloat16, 64, true>(p, k_pages, 0, p.n_alloc,
                                                                chunk_sum, group_sum, kv, seq_len,
                                                                err, s)
                   : launch_summaries_t<__nv_bfloat16, 128, true>(p, k_pages, 0, p.n_alloc,
                                                                 chunk_sum, group_sum, kv, seq_len,
                                                                 err, s);
}

}  // namespace hga
