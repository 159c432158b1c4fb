// One decode step (steps 2-5) in one launch, for batches with about one
// (sequence, KV head) item per SM: one CTA of eight warps per item, no cluster.
// bf16 K/V, D = 128.  Other batches take the routing and attention kernels.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core": item 2 (level 1 over the
// chunk summaries, level 2 over the group summaries of the chosen chunks,
// sink / local / current chunks always visible) and item 4 (the original K/V
// of the chosen tokens, attended exactly with a standard softmax).
//
// Per item, in one CTA:
//   1. the warps start the TMA loads of their first forced units, and one
//      thread streams the item's candidate chunk summaries (contiguous fp32
//      rows) through a two-stage shared-memory ring with bulk copies, so the
//      scan runs at the SM's share of the HBM bandwidth; the warps score each
//      64-row tile from shared memory with the routing kernel's arithmetic;
//   2. top-kc of the scores; the chosen chunks' group summaries are
//      bulk-loaded while the warps attend the forced units;
//   3. level 2 (top-kg), then the routed groups; the eight warps' partials are
//      merged by log-sum-exp in shared memory.
// Routing is bit-identical to hga_route; the output matches hga_attend up to
// the bf16 rounding of P.
#include <cuda.h>

#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "route_common.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace hga {
namespace {

using namespace decode;
using route::round4;

constexpr int kIW = 8;                            // warps
constexpr int kIT = kIW * 32;                     // threads
constexpr int kTileRows = 64;                     // summary rows per scan tile
constexpr int kRowBytes = kD * 4;                 // one fp32 summary row
constexpr int kScanTileBytes = kTileRows * kRowBytes;  // 32 KB
constexpr int kScanStages = 2;
constexpr int kRingsBytes = kIW * kWarpBytes;     // 128 KB of per-warp K/V rings

// Words after the rings and the scan ring:
//   qbar [D] | scores [per] | picks [kc] | chunks [kc] | group scores [kc x Ng] |
//   chosen group positions [kg] | group list [kg]
struct ItemSmem {
  int per, kc, ng, kg;
  __host__ __device__ int o_sc() const { return kD; }
  __host__ __device__ int o_pick() const { return o_sc() + per; }
  __host__ __device__ int o_chunks() const { return o_pick() + round4(kc); }
  __host__ __device__ int o_gsc() const { return o_chunks() + round4(kc); }
  __host__ __device__ int o_gsel() const { return o_gsc() + round4(ng); }
  __host__ __device__ int o_glist() const { return o_gsel() + round4(kg); }
  __host__ __device__ int words() const { return o_glist() + round4(kg); }
};
__host__ __device__ inline ItemSmem item_smem(const LayerParams& p) {
  ItemSmem L;
  L.per = round4(p.n_chunks);
  L.kc = p.kc;
  L.ng = p.kc * p.Ng;
  L.kg = p.kg;
  return L;
}
__host__ __device__ inline size_t item_smem_bytes(const LayerParams& p) {
  return 1024 + kRingsBytes + kScanStages * kScanTileBytes +
         static_cast<size_t>(item_smem(p).words()) * 4;
}

template <typename TO>
struct ItemArgs {
  const __nv_bfloat16* q;
  const int64_t* pos;
  const float* chunk_sum;
  const float* group_sum;
  int32_t* chunk_idx;
  float* chunk_score;
  int32_t* group_idx;
  float* group_score;
  TO* out;
  float* lse;
  unsigned* err;
};

// Scores rows [0, n) held in shared memory at `rows` (kD floats each) against
// qv into sc[0..n): eight lanes per row, the routing kernel's arithmetic.
__device__ __forceinline__ void score_smem_rows(const float* rows, int n, const float4 (&qv)[kD / 32],
                                                float* sc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane >> 3, s8 = lane & 7;
  for (int r0 = warp * 8; r0 < n; r0 += kIW * 8) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = r0 + u * 4 + sub;
      const float4* src = reinterpret_cast<const float4*>(rows + static_cast<size_t>(min(i, n - 1)) * kD);
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < kD / 32; ++k) {
        const float4 x = src[s8 + 8 * k];
        a = fmaf(x.x, qv[k].x, a);
        a = fmaf(x.y, qv[k].y, a);
        a = fmaf(x.z, qv[k].z, a);
        a = fmaf(x.w, qv[k].w, a);
      }
      a += __shfl_xor_sync(0xffffffffu, a, 4);  // the same sum in all eight lanes
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      if (s8 == 0 && i < n) sc[i] = a;
    }
  }
}

// Top-k of sc[0..n) into out[0..), ascending (block-collective, kIT threads).
__device__ __forceinline__ int item_topk(const float* sc, int n, int k, int* out, int* s_cnt,
                                         TopkSmem& tsm) {
  if (n <= kIT) return block_rank_topk<kIT>(sc, n, k, out, s_cnt);
  return block_topk<kIT>(sc, n, k, out, tsm);
}

template <typename TO>
__global__ void __launch_bounds__(kIT, 1)
decode_step_kernel(const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, ItemArgs<TO> a, LayerParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[kIW][kStages];
  __shared__ uint64_t bar_scan[kScanStages], bar_l2;
  __shared__ float s_ml[kIW][16][2];
  __shared__ int s_cnt[kIW];
  __shared__ TopkSmem tsm;

  const int item = blockIdx.x;  // (sequence, KV head) = b * Hkv + h
  const int b = item / p.Hkv, h = item % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* ring0 = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* scan = ring0 + kRingsBytes;
  float* rw = reinterpret_cast<float*>(scan + kScanStages * kScanTileBytes);
  const ItemSmem L = item_smem(p);
  float* qbar = rw;
  float* sc = rw + L.o_sc();
  int* pick = reinterpret_cast<int*>(rw + L.o_pick());
  int* chunks = reinterpret_cast<int*>(rw + L.o_chunks());
  float* gsc = rw + L.o_gsc();
  int* gsel = reinterpret_cast<int*>(rw + L.o_gsel());
  int* glist = reinterpret_cast<int*>(rw + L.o_glist());

  if (threadIdx.x == 0) {
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
    for (int w = 0; w < kIW; ++w)
      for (int s = 0; s < kStages; ++s) ptx::mbar_init(&bars[w][s], 1);
    for (int s = 0; s < kScanStages; ++s) ptx::mbar_init(&bar_scan[s], 1);
    ptx::mbar_init(&bar_l2, 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();

  const int64_t pb = a.pos[b];  // pos, q, k and v are never written by this library
  const bool ok = valid_position(pb, p, threadIdx.x == 0 ? a.err : nullptr);
  const int cur = ok ? static_cast<int>(pb / p.C) : 0;
  const int b0 = max(0, cur - p.local);
  // forced units: sink [0, su), then local + current up to the query [su, n_forced)
  const int ng_per_c = p.C / kUnit;
  const int su = ok ? min(p.sink, b0) * ng_per_c : 0;
  const int u_first_local = b0 * ng_per_c;
  const int n_forced = ok ? su + static_cast<int>(pb / kUnit) - u_first_local + 1 : 0;
  auto forced_token = [&](int u) -> int64_t {
    return static_cast<int64_t>(u < su ? u : u_first_local + (u - su)) * kUnit;
  };
  const int fpw = (n_forced + kIW - 1) / kIW;
  const int f_lo = min(n_forced, warp * fpw), f_hi = min(n_forced, f_lo + fpw);

  uint8_t* wsm = ring0 + warp * kWarpBytes;
  const uint32_t wsm_u32 = ptx::smem_u32(wsm);
  uint64_t* wbar = bars[warp];
  const int64_t row_base = static_cast<int64_t>(item) * p.n_alloc;
  int issued = 0, done = 0;
  auto issue_token = [&](int64_t tok) {
    if (lane == 0)
      issue_unit(&tm_k, &tm_v, wsm + (issued & 1) * kStageBytes, &wbar[issued & 1],
                 static_cast<int32_t>(row_base + tok));
    ++issued;
  };
  int f_next = f_lo;
  while (f_next < f_hi && issued < kStages) issue_token(forced_token(f_next++));

  route::decode_query_mean<__nv_bfloat16, kD>(a.q, p, b, h, qbar);  // threads < D
  pdl_wait();  // the summaries may come from the kernel just before

  // ---- 1. level 1: stream the candidate chunk summaries through the scan ring
  const int n_cand = ok ? max(0, cur - p.local - p.sink) : 0;
  const int n_tiles = (n_cand + kTileRows - 1) / kTileRows;
  const float* cbase = a.chunk_sum + (static_cast<size_t>(item) * p.n_chunks + p.sink) * kD;
  auto issue_tile = [&](int t) {  // one thread
    const int nr = min(kTileRows, n_cand - t * kTileRows);
    uint64_t* bar = &bar_scan[t % kScanStages];
    ptx::mbar_expect_tx(bar, static_cast<uint32_t>(nr) * kRowBytes);
    ptx::bulk_load(scan + (t % kScanStages) * kScanTileBytes,
                   cbase + static_cast<size_t>(t) * kTileRows * kD,
                   static_cast<uint32_t>(nr) * kRowBytes, bar);
  };
  if (threadIdx.x == 0)
    for (int t = 0; t < min(n_tiles, kScanStages); ++t) issue_tile(t);
  __syncthreads();  // qbar
  float4 qv[kD / 32];
#pragma unroll
  for (int k = 0; k < kD / 32; ++k) qv[k] = reinterpret_cast<const float4*>(qbar)[(lane & 7) + 8 * k];

  bool timed_out = false;
  for (int t = 0; t < n_tiles; ++t) {
    const bool landed = ptx::mbar_wait(&bar_scan[t % kScanStages], (t / kScanStages) & 1, kWaitLimit);
    if (!landed) timed_out = true;
    const int nr = min(kTileRows, n_cand - t * kTileRows);
    if (landed)
      score_smem_rows(reinterpret_cast<const float*>(scan + (t % kScanStages) * kScanTileBytes), nr,
                      qv, sc + t * kTileRows);
    __syncthreads();  // the stage is free again
    if (threadIdx.x == 0 && t + kScanStages < n_tiles) issue_tile(t + kScanStages);
  }
  const bool scan_ok = !__syncthreads_or(timed_out);
  if (!scan_ok && threadIdx.x == 0)  // every tile was issued: wait (bounded) for the last ones
    for (int t = max(0, n_tiles - kScanStages); t < n_tiles; ++t)
      ptx::mbar_wait(&bar_scan[t % kScanStages], (t / kScanStages) & 1, kWaitLimit);
  const int ns = scan_ok ? item_topk(sc, n_cand, p.kc, pick, s_cnt, tsm) : 0;
  for (int i = threadIdx.x; i < p.kc; i += kIT) {
    const int c = i < ns ? pick[i] + p.sink : -1;
    if (i < ns) chunks[i] = c;
    a.chunk_idx[static_cast<size_t>(item) * p.kc + i] = c;
    if (a.chunk_score)
      a.chunk_score[static_cast<size_t>(item) * p.kc + i] = i < ns ? sc[pick[i]] : CUDART_NAN_F;
  }
  __syncthreads();
  // the chosen chunks' group summaries (Ng contiguous rows each) into the scan ring
  const int n_g = ns * p.Ng;
  const float* gbase = a.group_sum + static_cast<size_t>(item) * p.n_chunks * p.Ng * kD;
  if (threadIdx.x == 0 && n_g > 0) {
    ptx::mbar_expect_tx(&bar_l2, static_cast<uint32_t>(n_g) * kRowBytes);
    for (int i = 0; i < ns; ++i)
      ptx::bulk_load(scan + static_cast<size_t>(i) * p.Ng * kRowBytes,
                     gbase + static_cast<size_t>(chunks[i]) * p.Ng * kD,
                     static_cast<uint32_t>(p.Ng) * kRowBytes, &bar_l2);
  }

  // ---- 2. the forced units, while the group summaries load
  uint32_t qa[8][4];
  load_q_frags(a.q, p, b, h, qa);
  const float scale = kLog2e * rsqrtf(static_cast<float>(kD));
  WarpState w;
  w.init();
  auto consume = [&](int valid) -> bool {
    const int st = done & 1;
    if (!ptx::mbar_wait(&wbar[st], (done >> 1) & 1, kWaitLimit)) return false;
    const uint32_t kt = wsm_u32 + st * kStageBytes;
    attend_unit(kt, kt + kTileBytes, valid, qa, scale, w);
    ++done;
    return true;
  };
  for (int u = f_lo; u < f_hi && !timed_out; ++u) {
    if (!consume(u == n_forced - 1 ? static_cast<int>(pb % kUnit) + 1 : kUnit)) {
      timed_out = true;
      break;
    }
    if (f_next < f_hi) issue_token(forced_token(f_next++));
  }

  // ---- 3. level 2, then the routed groups
  bool l2_ok = true;
  if (n_g > 0) {
    l2_ok = ptx::mbar_wait(&bar_l2, 0, kWaitLimit);
    if (l2_ok) score_smem_rows(reinterpret_cast<const float*>(scan), n_g, qv, gsc);
  }
  l2_ok = !__syncthreads_or(!l2_ok);
  if (!l2_ok) timed_out = true;
  const int ng = l2_ok ? item_topk(gsc, n_g, p.kg, gsel, s_cnt, tsm) : 0;
  for (int i = threadIdx.x; i < p.kg; i += kIT) {
    const bool have = i < ng;
    const int sg = have ? gsel[i] : 0;
    const int gid = have ? chunks[sg / p.Ng] * p.Ng + sg % p.Ng : -1;
    a.group_idx[static_cast<size_t>(item) * p.kg + i] = gid;
    if (a.group_score)
      a.group_score[static_cast<size_t>(item) * p.kg + i] = have ? gsc[sg] : CUDART_NAN_F;
    if (have) glist[i] = gid;
  }
  __syncthreads();
  const int rpw = (ng + kIW - 1) / kIW;
  const int r_lo = min(ng, warp * rpw), r_hi = min(ng, r_lo + rpw);
  int r_next = r_lo;
  if (!timed_out)
    while (r_next < r_hi && issued - done < kStages)
      issue_token(static_cast<int64_t>(glist[r_next++]) * kUnit);
  for (int u = r_lo; u < r_hi && !timed_out; ++u) {
    if (!consume(kUnit)) {
      timed_out = true;
      break;
    }
    if (r_next < r_hi) issue_token(static_cast<int64_t>(glist[r_next++]) * kUnit);
  }
  if (timed_out) {
    // A wait gave up: the partial is dropped (the output is wrong and flagged),
    // the copies still in flight are waited for once more (bounded), and every
    // barrier below is still reached.
    if (lane == 0) flag_error(a.err, kErrTimeout);
    for (; done < issued; ++done) ptx::mbar_wait(&wbar[done & 1], (done >> 1) & 1, kWaitLimit);
    w.m0 = w.m1 = -CUDART_INF_F;
    w.l0 = w.l1 = 0.f;
  }

  // ---- merge the warps' partials (each in its own ring, whose copies all landed)
  const int g = lane >> 2, t4 = lane & 3;
  w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, 1);
  w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, 2);
  w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, 1);
  w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, 2);
  float* wo = reinterpret_cast<float*>(wsm);  // [16 heads][128]
  if (done == 0) {
    w.m0 = w.m1 = -CUDART_INF_F;
    w.l0 = w.l1 = 0.f;
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      *reinterpret_cast<float2*>(wo + g * kD + j * 8 + 2 * t4) = make_float2(w.o[j][0], w.o[j][1]);
      *reinterpret_cast<float2*>(wo + (g + 8) * kD + j * 8 + 2 * t4) =
          make_float2(w.o[j][2], w.o[j][3]);
    }
  }
  if (t4 == 0) {
    s_ml[warp][g][0] = w.m0;
    s_ml[warp][g][1] = w.l0;
    s_ml[warp][g + 8][0] = w.m1;
    s_ml[warp][g + 8][1] = w.l1;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < p.G * kD; idx += kIT) {
    const int hh = idx / kD, d = idx % kD;
    float mm = -CUDART_INF_F;
#pragma unroll
    for (int v = 0; v < kIW; ++v) mm = fmaxf(mm, s_ml[v][hh][0]);
    float ll = 0.f, oo = 0.f;
    if (mm != -CUDART_INF_F) {
#pragma unroll
      for (int v = 0; v < kIW; ++v) {
        const float mv = s_ml[v][hh][0];
        if (mv == -CUDART_INF_F) continue;
        const float f = exp2f(mv - mm);
        ll += s_ml[v][hh][1] * f;
        oo += reinterpret_cast<const float*>(ring0 + v * kWarpBytes)[hh * kD + d] * f;
      }
    }
    const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + hh;
    store_out(a.out + row * kD + d, ll > 0.f ? oo / ll : 0.f);
    if (a.lse && d == 0) a.lse[row] = ll > 0.f ? (mm + log2f(ll)) * kLn2 : -CUDART_INF_F;
  }
  pdl_trigger();
}

template <typename TO>
cudaError_t launch_t(const LayerParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                     const ItemArgs<TO>& a, cudaStream_t s) {
  const size_t smem = item_smem_bytes(p);
  cudaError_t e = ensure_smem<decode_step_kernel<TO>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_step_kernel<TO>, dim3(p.B * p.Hkv), dim3(kIT), smem, s, 1, tk, tv, a, p);
}

}  // namespace

bool decode_item_path(const LayerParams& p) {
  const int64_t items = static_cast<int64_t>(p.B) * p.Hkv;
  const int sms = device_sm_count();
  return items * 2 >= sms && items <= sms && item_smem_bytes(p) <= 220 * 1024 &&
         p.kc * p.Ng <= kScanStages * kTileRows;
}

bool decode_step_path(const LayerParams& p, int dtype) {
  return decode_fast_path(p, dtype) &&
         static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc < (static_cast<int64_t>(1) << 31);
}

cudaError_t launch_decode_step(const LayerParams& p, int out_dtype, const void* q,
                               const int64_t* pos, const float* chunk_sum, const float* group_sum,
                               const void* k, const void* v, int32_t* chunk_idx,
                               float* chunk_score, int32_t* group_idx, float* group_score,
                               void* out, float* lse, unsigned* err, cudaStream_t s) {
  if (!decode_item_path(p)) {  // the routing kernel, then the attention kernel
    cudaError_t e = launch_route(p, 1, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score,
                                 group_idx, group_score, err, s);
    if (e != cudaSuccess) return e;
    return launch_attend_decode_bf16(p, out_dtype, q, pos, k, v, group_idx, out, lse, err, 0, s);
  }
  CUtensorMap tk, tv;
  const int64_t all_rows = static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc;
  cudaError_t e = make_bf16_map(&tk, k, all_rows, kUnit);
  if (e == cudaSuccess) e = make_bf16_map(&tv, v, all_rows, kUnit);
  if (e != cudaSuccess) return e;
  if (out_dtype == 0) {
    ItemArgs<float> a{static_cast<const __nv_bfloat16*>(q), pos, chunk_sum, group_sum, chunk_idx,
                      chunk_score, group_idx, group_score, static_cast<float*>(out), lse, err};
    return launch_t<float>(p, tk, tv, a, s);
  }
  ItemArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(q), pos, chunk_sum, group_sum,
                            chunk_idx, chunk_score, group_idx, group_score,
                            static_cast<__nv_bfloat16*>(out), lse, err};
  return launch_t<__nv_bfloat16>(p, tk, tv, a, s);
}

}  // namespace hga
