// Steps 4-5 for decode, bf16 K/V with D = 128: fused gather + split-K flash
// decoding on sm_100a.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", item 4: the original K/V of
// the selected tokens are fetched and attended exactly with a standard softmax.
//
// Every part of a decode query's token list starts on a group boundary, so the
// list is a sequence of 16-token units, each a contiguous 16 x 256 B segment of
// the cache: the sink chunks, the local chunks, the current chunk up to the
// query (last unit partial) and the routed groups.  One warp owns a split of
// consecutive units (a warp-split) and streams them through a private
// double-buffered shared-memory ring:
//   - lane 0 issues two 2-D TMA box loads per unit and tensor (16 rows x 64
//     columns each, 128-byte swizzle), completing on the stage's mbarrier;
//   - S^T = Q K^T runs on the tensor cores (mma.sync m16n8k16, bf16 -> fp32),
//     with the G <= 16 query heads as the M rows and K fragments read with
//     ldmatrix from the swizzled tile;
//   - online softmax in registers (log2 domain); P stays in registers and is
//     reused as the A operand of O += P V (V fragments via ldmatrix.trans).
// The CTAs of one (sequence, KV head) form a thread-block cluster.  Each warp's
// partial (o, m, l) is merged by log-sum-exp first inside its CTA (shared
// memory), then across the cluster by CTA rank 0 reading the other CTAs'
// partials through distributed shared memory: no workspace, no second kernel.
// No cluster multicast is used anywhere.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace hga {

namespace {

constexpr int kD = 128;
constexpr int kUnit = 16;                       // tokens per unit (= group size)
constexpr int kWarps = 4;
constexpr int kStages = 2;
constexpr int kBoxBytes = kUnit * 64 * 2;       // 16 rows x 64 bf16 = 2 KB
constexpr int kTileBytes = 2 * kBoxBytes;       // one tensor, 128 dims
constexpr int kStageBytes = 2 * kTileBytes;     // K and V
constexpr int kWarpBytes = kStages * kStageBytes;
constexpr int kSmemBytes = kWarps * kWarpBytes + 1024;  // + alignment slack
constexpr uint32_t kWaitLimit = 1u << 26;       // bounded mbarrier polls
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename TO>
struct DecodeArgs {
  const __nv_bfloat16* q;
  const int64_t* pos;
  const int32_t* group_idx;
  TO* out;
  float* lse;
  unsigned* err;
  int units_per_split;
  int nsplit;   // warp-splits per (sequence, KV head) = kWarps * cluster size
  int hot;      // K/V are the host tier's device working buffers (see host_tier.cu)
  int64_t rows; // rows per (sequence, KV head) of k / v: n_alloc, or the working-buffer rows
};

// Address of the 16-byte chunk `chunk` (0..15 over 128 dims) of row `row` in a
// tile stored as two 128B-swizzled boxes of 64 columns.
__device__ __forceinline__ uint32_t swz(uint32_t tile, int row, int chunk) {
  const int box = chunk >> 3, c = chunk & 7;
  return tile + box * kBoxBytes + row * 128 + ((c ^ (row & 7)) << 4);
}

template <typename TO>
__global__ void __launch_bounds__(kWarps * 32)
attend_decode_bf16_kernel(const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, DecodeArgs<TO> a,
                          LayerParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[kWarps][kStages];
  __shared__ int s_gl[1024];
  __shared__ int s_slot[1024];  // input position of each kept routed group
  __shared__ int s_ng;
  __shared__ float s_ml[kWarps][16][2];   // per-warp (m, l) of each query head
  __shared__ float s_rml[8][16][2];       // rank 0: (m, l) pushed by each CTA of the cluster

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());  // grid.x == cluster size
  const int n_cta = static_cast<int>(cluster.num_blocks());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const int split = rank * kWarps + warp;

  if (threadIdx.x == 0) {
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
    for (int w = 0; w < kWarps; ++w)
      for (int s = 0; s < kStages; ++s) ptx::mbar_init(&bars[w][s], 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();

  // Everything up to pdl_wait() reads only pos, k and v (never written by this
  // library), so it overlaps the routing kernel still running ahead of us.
  const int64_t pb = a.pos[b];
  const bool ok = valid_position(pb, p, threadIdx.x == 0 && rank == 0 ? a.err : nullptr);
  const int cur = ok ? static_cast<int>(pb / p.C) : 0;
  const int b0 = max(0, cur - p.local);
  // Unit list: sink units [0, su), local+current units [su, su+lu), routed groups.
  const int ng_per_c = p.C / kUnit;
  const int su = ok ? min(p.sink, b0) * ng_per_c : 0;
  const int u_first_local = b0 * ng_per_c;
  const int lu = ok ? static_cast<int>(pb / kUnit) - u_first_local + 1 : 0;
  const int n_forced = su + lu;
  const int u_lo = split * a.units_per_split;
  const int u_cap = u_lo + a.units_per_split;
  const int64_t row_base = static_cast<int64_t>(bh) * a.rows;
  // Row of unit u in k / v.  The device cache holds token t at row t.  The host
  // tier's working buffer holds [sink chunks | ring of local+1 chunks (chunk c
  // at slot c mod (local+1)) | routed groups in group_idx order].
  auto unit_token = [&](int u) -> int64_t {
    if (u < su) return static_cast<int64_t>(u) * kUnit;
    u -= su;
    if (u < lu) {
      const int unit = u_first_local + u;
      if (!a.hot) return static_cast<int64_t>(unit) * kUnit;
      const int c = unit / ng_per_c, gi = unit % ng_per_c;
      return static_cast<int64_t>(p.sink + c % (p.local + 1)) * p.C + gi * kUnit;
    }
    u -= lu;
    if (!a.hot) return static_cast<int64_t>(s_gl[u]) * kUnit;
    return static_cast<int64_t>(p.sink + p.local + 1) * p.C + static_cast<int64_t>(s_slot[u]) * kUnit;
  };
  // Valid tokens in unit u (only the unit holding the query can be partial).
  auto unit_valid = [&](int u) -> int {
    if (u == n_forced - 1) return static_cast<int>(pb % kUnit) + 1;
    return kUnit;
  };
  uint8_t* wsm = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023) + warp * kWarpBytes;
  const uint32_t wsm_u32 = ptx::smem_u32(wsm);
  uint64_t* wbar = bars[warp];
  auto issue = [&](int u, int stage) {
    if (lane == 0) {
      const int32_t y = static_cast<int32_t>(row_base + unit_token(u));
      uint8_t* st = wsm + stage * kStageBytes;
      ptx::mbar_expect_tx(&wbar[stage], kStageBytes);
      ptx::tma_load_2d(st, &tm_k, &wbar[stage], 0, y);
      ptx::tma_load_2d(st + kBoxBytes, &tm_k, &wbar[stage], 64, y);
      ptx::tma_load_2d(st + kTileBytes, &tm_v, &wbar[stage], 0, y);
      ptx::tma_load_2d(st + kTileBytes + kBoxBytes, &tm_v, &wbar[stage], 64, y);
    }
  };
  // Forced units (sink, local, current) do not depend on routing: start them now.
  const int pre0 = u_lo < n_forced ? 1 : 0;
  const int pre1 = u_lo + 1 < n_forced && u_lo + 1 < u_cap ? 1 : 0;
  if (pre0) issue(u_lo, 0);
  if (pre1) issue(u_lo + 1, 1);

  // Q as m16n8k16 A fragments: rows = query heads (g, g+8), k = dims.
  const int g = lane >> 2, t = lane & 3;
  uint32_t qa[8][4];
  {
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(
        a.q + (static_cast<size_t>(b) * p.Hq + h * p.G + g) * kD);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(
        a.q + (static_cast<size_t>(b) * p.Hq + h * p.G + g + 8) * kD);
    const bool r0 = g < p.G, r1 = g + 8 < p.G;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qa[kk][0] = r0 ? __ldg(q0 + kk * 8 + t) : 0u;
      qa[kk][1] = r1 ? __ldg(q1 + kk * 8 + t) : 0u;
      qa[kk][2] = r0 ? __ldg(q0 + kk * 8 + 4 + t) : 0u;
      qa[kk][3] = r1 ? __ldg(q1 + kk * 8 + 4 + t) : 0u;
    }
  }
  const float sc = kLog2e * rsqrtf(static_cast<float>(kD));

  pdl_wait();

  // Routed groups kept, in order: warp 0 validates and compacts them (a group
  // of a candidate chunk, strictly ascending; anything else is dropped and
  // flagged).  The host tier's gather applies the same rule.
  if (warp == 0) {
    int n = 0;
    bool bad = false;
    if (ok) {
      const int32_t* gl = a.group_idx + static_cast<size_t>(bh) * p.kg;
      n = warp_keep_ascending(
          gl, p.kg, [&](int gid) { return gid / p.Ng >= p.sink && gid / p.Ng < cur - p.local; },
          s_gl, &bad, s_slot);
    }
    if (lane == 0) {
      s_ng = n;
      if (bad && rank == 0) flag_error(a.err, kErrGroupIdx);
    }
  }
  __syncthreads();

  const int n_units = n_forced + s_ng;
  const int u_hi = min(n_units, u_cap);
  if (u_lo < u_hi) {
    if (!pre0) issue(u_lo, 0);
    if (!pre1 && u_lo + 1 < u_hi) issue(u_lo + 1, 1);
  }

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F;  // rows g and g+8
  float l0 = 0.f, l1 = 0.f;                      // this lane's partial sums

  // ldmatrix lane roles
  const int mi = lane >> 3, ri = lane & 7;
  bool timed_out = false;
  int stuck_it = 0;

  for (int u = u_lo; u < u_hi; ++u) {
    const int it = u - u_lo;
    const int stage = it & 1;
    if (!ptx::mbar_wait(&wbar[stage], (it >> 1) & 1, kWaitLimit)) {
      timed_out = true;
      stuck_it = it;
      break;
    }
    const uint32_t kt = wsm_u32 + stage * kStageBytes;
    const uint32_t vt = kt + kTileBytes;
    const int valid = unit_valid(u);

    // S^T[head, token] for tokens 0-7 (s[0]) and 8-15 (s[1])
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t r[4];
      const int tok = (mi >> 1) * 8 + ri;
      ptx::ldmatrix_x4(swz(kt, tok, kk * 2 + (mi & 1)), r);
      ptx::mma_bf16_16816(s[0], qa[kk], r[0], r[1]);
      ptx::mma_bf16_16816(s[1], qa[kk], r[2], r[3]);
    }
    // scale into log2 units, mask tokens past the query
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = nt * 8 + 2 * t + (e & 1);
        s[nt][e] = tok < valid ? s[nt][e] * sc : -CUDART_INF_F;
      }
    }
    float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    const float c0 = exp2f(m0 - n0), c1 = exp2f(m1 - n1);  // 0 while m is -inf
    m0 = n0;
    m1 = n1;
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pr[nt][0] = exp2f(s[nt][0] - n0);
      pr[nt][1] = exp2f(s[nt][1] - n0);
      pr[nt][2] = exp2f(s[nt][2] - n1);
      pr[nt][3] = exp2f(s[nt][3] - n1);
    }
    l0 = l0 * c0 + pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
    l1 = l1 * c1 + pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j][0] *= c0; o[j][1] *= c0;
      o[j][2] *= c1; o[j][3] *= c1;
    }
    uint32_t pa[4];
    pa[0] = ptx::pack_bf16x2(pr[0][0], pr[0][1]);
    pa[1] = ptx::pack_bf16x2(pr[0][2], pr[0][3]);
    pa[2] = ptx::pack_bf16x2(pr[1][0], pr[1][1]);
    pa[3] = ptx::pack_bf16x2(pr[1][2], pr[1][3]);
    // Tokens past the query may hold anything (even NaN) in the cache: their
    // V rows must not reach the product, so zero them in the tile.
    if (valid < kUnit) {
      __syncwarp();
      for (int i = lane; i < (kUnit - valid) * 16; i += 32) {
        const int row = valid + i / 16, chunk = i % 16;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(swz(vt, row, chunk)), "r"(0u));
      }
      ptx::fence_proxy_async();  // the stage is refilled by TMA later
      __syncwarp();
    }
#pragma unroll
    for (int nn = 0; nn < 8; ++nn) {
      uint32_t r[4];
      const int tok = (mi & 1) * 8 + ri;
      ptx::ldmatrix_x4_trans(swz(vt, tok, nn * 2 + (mi >> 1)), r);
      ptx::mma_bf16_16816(o[2 * nn], pa, r[0], r[1]);
      ptx::mma_bf16_16816(o[2 * nn + 1], pa, r[2], r[3]);
    }
    __syncwarp();
    if (u + 2 < u_hi) issue(u + 2, stage);
  }

  if (timed_out) {
    // The warp gave up waiting on its copies: its partial is dropped (the
    // output is wrong and flagged), it waits once more, again bounded, for the
    // copies it still has in flight, and it still joins the merge barriers.
    if (lane == 0) flag_error(a.err, kErrTimeout);
    for (int it = stuck_it; it < stuck_it + 2 && u_lo + it < u_hi; ++it)
      ptx::mbar_wait(&wbar[it & 1], (it >> 1) & 1, kWaitLimit);
    m0 = m1 = -CUDART_INF_F;
    l0 = l1 = 0.f;
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  // ---- merge 1: the CTA's warps, through shared memory.  Every issued TMA
  // copy has been waited for, so a warp's own ring now holds its partial o.
  float* wo = reinterpret_cast<float*>(wsm);  // [16 heads][128] floats
  if (u_lo >= u_hi) {
    m0 = m1 = -CUDART_INF_F;
    l0 = l1 = 0.f;
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      *reinterpret_cast<float2*>(wo + g * kD + j * 8 + 2 * t) = make_float2(o[j][0], o[j][1]);
      *reinterpret_cast<float2*>(wo + (g + 8) * kD + j * 8 + 2 * t) = make_float2(o[j][2], o[j][3]);
    }
  }
  if (t == 0) {
    s_ml[warp][g][0] = m0;
    s_ml[warp][g][1] = l0;
    s_ml[warp][g + 8][0] = m1;
    s_ml[warp][g + 8][1] = l1;
  }
  __syncthreads();
  const int d = threadIdx.x;  // one output dim per thread (blockDim == D == 128)
  uint8_t* ring0 = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  float cta_m[16], cta_l[16], cta_o[16];
#pragma unroll
  for (int hh = 0; hh < 16; ++hh) {
    cta_m[hh] = -CUDART_INF_F;
    cta_l[hh] = 0.f;
    cta_o[hh] = 0.f;
    if (hh >= p.G) continue;
    float mm = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, s_ml[w][hh][0]);
    if (mm == -CUDART_INF_F) continue;
    float ll = 0.f, oo = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = s_ml[w][hh][0];
      if (mw == -CUDART_INF_F) continue;
      const float f = exp2f(mw - mm);
      ll += s_ml[w][hh][1] * f;
      oo += reinterpret_cast<const float*>(ring0 + w * kWarpBytes)[hh * kD + d] * f;
    }
    cta_m[hh] = mm;
    cta_l[hh] = ll;
    cta_o[hh] = oo;
  }
  // ---- merge 2: the cluster's CTAs.  After the first barrier every CTA has
  // finished reading its own ring, so rank 0's ring is free; every CTA then
  // pushes its partial into rank 0's ring (remote shared-memory stores), and
  // after the second barrier rank 0 merges from its own shared memory.
  cluster.sync();
  float* recv = cluster.map_shared_rank(reinterpret_cast<float*>(ring0), 0);  // [8][16][128]
  float (*recv_ml)[16][2] = cluster.map_shared_rank(s_rml, 0);
#pragma unroll
  for (int hh = 0; hh < 16; ++hh) {
    if (hh >= p.G) continue;
    recv[(rank * 16 + hh) * kD + d] = cta_o[hh];
    if (d == 0) {
      recv_ml[rank][hh][0] = cta_m[hh];
      recv_ml[rank][hh][1] = cta_l[hh];
    }
  }
  cluster.sync();
  if (rank == 0) {
    const float* mine = reinterpret_cast<const float*>(ring0);
    for (int hh = 0; hh < p.G; ++hh) {
      float mm = -CUDART_INF_F;
      for (int r = 0; r < n_cta; ++r) mm = fmaxf(mm, s_rml[r][hh][0]);
      float ll = 0.f, oo = 0.f;
      if (mm != -CUDART_INF_F) {
        for (int r = 0; r < n_cta; ++r) {
          const float mr = s_rml[r][hh][0];
          if (mr == -CUDART_INF_F) continue;
          const float f = exp2f(mr - mm);
          ll += s_rml[r][hh][1] * f;
          oo += mine[(r * 16 + hh) * kD + d] * f;
        }
      }
      const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + hh;
      store_out(a.out + row * kD + d, ll > 0.f ? oo / ll : 0.f);
      if (a.lse && d == 0) a.lse[row] = ll > 0.f ? (mm + log2f(ll)) * kLn2 : -CUDART_INF_F;
    }
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ host side

int max_units(const LayerParams& p) {
  return (p.sink + p.local + 1) * (p.C / kUnit) + p.kg;
}

// CTAs per (sequence, KV head), at most 8 (the portable cluster size): enough
// warps for ~12 per SM over the whole batch, but never more CTAs than fit at
// once (3 per SM, bounded by registers and shared memory), so the grid runs
// in a single wave.
int cluster_size(const LayerParams& p) {
  const int64_t bh = static_cast<int64_t>(p.B) * p.Hkv;
  const int64_t want = (148 * 12 + bh * kWarps - 1) / (bh * kWarps);
  const int64_t fit = (148 * 3) / bh;
  const int64_t useful = (max_units(p) + kWarps - 1) / kWarps;
  int64_t cl = want < fit ? want : fit;
  cl = cl < useful ? cl : useful;
  return static_cast<int>(cl < 1 ? 1 : (cl > 8 ? 8 : cl));
}

template <typename TO>
cudaError_t launch_t(const LayerParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                     const void* q, const int64_t* pos, const int32_t* group_idx, void* out,
                     float* lse, unsigned* err, int hot, int64_t rows, cudaStream_t s) {
  const int cl = cluster_size(p);
  DecodeArgs<TO> a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.pos = pos;
  a.group_idx = group_idx;
  a.out = static_cast<TO*>(out);
  a.lse = lse;
  a.err = err;
  a.nsplit = cl * kWarps;
  a.units_per_split = (max_units(p) + a.nsplit - 1) / a.nsplit;
  a.hot = hot;
  a.rows = rows;
  cudaError_t e = ensure_smem<attend_decode_bf16_kernel<TO>>(kSmemBytes);
  if (e != cudaSuccess) return e;
  // A plain (non-programmatic) launch: measured faster here, because CTAs of
  // this kernel launched early would hold SM slots while the routing kernel
  // before it finishes.  pdl_wait() inside is then a no-op.
  return launch_pdl(attend_decode_bf16_kernel<TO>, dim3(cl, p.B * p.Hkv), dim3(kWarps * 32),
                    kSmemBytes, s, cl | kNoPdl, tk, tv, a, p);
}

}  // namespace

bool decode_fast_path(const LayerParams& p, int dtype) {
  return dtype == 1 && p.D == kD && p.q_len == 1 && p.g == kUnit && p.kg <= 1024 && p.G <= 16 &&
         p.B * p.Hkv <= 65535;
}

cudaError_t launch_attend_decode_bf16(const LayerParams& p, int out_dtype, const void* q,
                                      const int64_t* pos, const void* k, const void* v,
                                      const int32_t* group_idx, void* out, float* lse,
                                      unsigned* err, int hot, cudaStream_t s) {
  CUtensorMap tk, tv;
  const int64_t rows = hot ? hot_rows(p) : p.n_alloc;
  const int64_t all_rows = static_cast<int64_t>(p.B) * p.Hkv * rows;
  cudaError_t e = make_bf16_map(&tk, k, all_rows, kUnit);
  if (e == cudaSuccess) e = make_bf16_map(&tv, v, all_rows, kUnit);
  if (e != cudaSuccess) return e;
  return out_dtype == 0
             ? launch_t<float>(p, tk, tv, q, pos, group_idx, out, lse, err, hot, rows, s)
             : launch_t<__nv_bfloat16>(p, tk, tv, q, pos, group_idx, out, lse, err, hot, rows, s);
}

}  // namespace hga
