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
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace hga {

namespace {

using namespace decode;

constexpr int kSmemBytes = kRingBytes;

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
  const int32_t* slot_map;  // warm tier: cached slot of every group_idx entry, or null
  int slots;                // warm tier: cached group slots per (sequence, KV head)
};

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
  __shared__ MergeSmem s_merge;

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());  // grid.x == cluster size
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

  // Everything up to pdl_wait() reads only pos, q and the device K/V cache (never
  // written by this library), so it overlaps the routing kernel still running
  // ahead of us.
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
    if (lane == 0)
      issue_unit(&tm_k, &tm_v, wsm + stage * kStageBytes, &wbar[stage],
                 static_cast<int32_t>(row_base + unit_token(u)));
  };
  // Forced units (sink, local, current) do not depend on routing: start them now
  // from the device cache.  The host tier's working buffers are written by the
  // gather kernel just before, so there they wait for it.
  const int pre0 = !a.hot && u_lo < n_forced ? 1 : 0;
  const int pre1 = !a.hot && u_lo + 1 < n_forced && u_lo + 1 < u_cap ? 1 : 0;
  if (pre0) issue(u_lo, 0);
  if (pre1) issue(u_lo + 1, 1);

  uint32_t qa[8][4];
  load_q_frags(a.q, p, b, h, qa);
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
      if (a.slot_map) {  // warm tier: the kept entries' cached slots
        __syncwarp();
        const int32_t* sm = a.slot_map + static_cast<size_t>(bh) * p.kg;
        bool bad_slot = false;
        for (int i = lane; i < n; i += 32) {
          int s = sm[s_slot[i]];
          if (s < 0 || s >= a.slots) {
            bad_slot = true;
            s = 0;
          }
          s_slot[i] = s;
        }
        bad |= __any_sync(0xffffffffu, bad_slot);
      }
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

  WarpState w;
  w.init();
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
    attend_unit(kt, kt + kTileBytes, unit_valid(u), qa, sc, w);
    if (u + 2 < u_hi) issue(u + 2, stage);
  }

  if (timed_out) {
    // The warp gave up waiting on its copies: its partial is dropped (the
    // output is wrong and flagged), it waits once more, again bounded, for the
    // copies it still has in flight, and it still joins the merge barriers.
    if (lane == 0) flag_error(a.err, kErrTimeout);
    for (int it = stuck_it; it < stuck_it + 2 && u_lo + it < u_hi; ++it)
      ptx::mbar_wait(&wbar[it & 1], (it >> 1) & 1, kWaitLimit);
    w.m0 = w.m1 = -CUDART_INF_F;
    w.l0 = w.l1 = 0.f;
  }
  // Every issued TMA copy has been waited for, so the rings can hold partials.
  uint8_t* ring0 = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  merge_and_store<TO>(w, u_lo >= u_hi, ring0, s_merge, p, b, h, a.out, a.lse);
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
  const int64_t sms = device_sm_count();
  const int64_t want = (sms * 12 + bh * kWarps - 1) / (bh * kWarps);
  const int64_t fit = (sms * 3) / bh;
  const int64_t useful = (max_units(p) + kWarps - 1) / kWarps;
  int64_t cl = want < fit ? want : fit;
  cl = cl < useful ? cl : useful;
  return static_cast<int>(cl < 1 ? 1 : (cl > 8 ? 8 : cl));
}

template <typename TO>
cudaError_t launch_t(const LayerParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                     const void* q, const int64_t* pos, const int32_t* group_idx, void* out,
                     float* lse, unsigned* err, int hot, int64_t rows, const int32_t* slot_map,
                     int slots, cudaStream_t s) {
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
  a.slot_map = slot_map;
  a.slots = slots;
  cudaError_t e = ensure_smem<attend_decode_bf16_kernel<TO>>(kSmemBytes);
  if (e != cudaSuccess) return e;
  // Programmatic launch (the prologue and the forced units' loads overlap the
  // routing kernel's tail) while the grid is small; a grid of more than two
  // CTAs per SM launched early holds slots that the kernels before it (and the
  // summary append beside it) still need, and measured slower.
  const bool early = static_cast<int64_t>(cl) * p.B * p.Hkv <= 2 * device_sm_count();
  return launch_pdl(attend_decode_bf16_kernel<TO>, dim3(cl, p.B * p.Hkv), dim3(kWarps * 32),
                    kSmemBytes, s, cl | (early ? 0 : kNoPdl), tk, tv, a, p);
}

}  // namespace

bool decode_fast_path(const LayerParams& p, int dtype) {
  return dtype == 1 && p.D == kD && p.q_len == 1 && p.g == kUnit && p.kg <= 1024 && p.G <= 16 &&
         p.B * p.Hkv <= 65535;
}

cudaError_t launch_attend_decode_bf16(const LayerParams& p, int out_dtype, const void* q,
                                      const int64_t* pos, const void* k, const void* v,
                                      const int32_t* group_idx, void* out, float* lse,
                                      unsigned* err, int hot, cudaStream_t s,
                                      const int32_t* slot_map, int slots) {
  CUtensorMap tk, tv;
  const int64_t rows = hot ? hot_rows(p, slot_map ? slots : 0) : p.n_alloc;
  const int64_t all_rows = static_cast<int64_t>(p.B) * p.Hkv * rows;
  cudaError_t e = make_bf16_map(&tk, k, all_rows, kUnit);
  if (e == cudaSuccess) e = make_bf16_map(&tv, v, all_rows, kUnit);
  if (e != cudaSuccess) return e;
  return out_dtype == 0
             ? launch_t<float>(p, tk, tv, q, pos, group_idx, out, lse, err, hot, rows,
                                             slot_map, slots, s)
             : launch_t<__nv_bfloat16>(p, tk, tv, q, pos, group_idx, out, lse, err, hot,
                                                     rows, slot_map, slots, s);
}

}  // namespace hga
