// Steps 4-5 for prefill, bf16 K/V with D = 128: gathered-tile attention of a
// 64-query block on the 5th-generation tensor cores (tcgen05, TMEM).
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", item 4: every query attends
// exactly, with a standard softmax, to the original K/V of the bounded token
// set its block routed to (sink, local and current chunks plus the routed
// groups), causal inside the current chunk.
//
// Persistent: one CTA per SM walks a static list of work items, one item per
// (sequence, KV head, query block), latest blocks first.  The block's G*C
// query rows (G heads x C queries) form one or two M = 128 tiles.  Its token
// list is cut into 16-token units ordered [sink | local | routed groups |
// current chunk], and the units into KV tiles of 128 keys, so only the last
// tile(s) carry the causal mask.  Warp roles (320 threads):
//   warps 0-3, 4-7  softmax warpgroups of M-tile 0 and 1 (ping-pong): read
//                   S = Q K^T from TMEM, masked online softmax in the log2
//                   domain with lazy rescaling, write P (bf16) back over S;
//                   then the item's epilogue O / l;
//   warp 8          producer: builds each item's unit list (double-buffered),
//                   then TMA-loads Q and the K and V tiles (two 16 x 64 boxes
//                   per unit and tensor, 128B swizzle) into 2-stage rings;
//   warp 9          tcgen05.mma issuer and TMEM owner (512 columns: per M-tile
//                   128 for S/P and 128 for O).
// S_mt(t) = Q_mt K(t)^T and O_mt += P_mt(t) V(t) run on M = 128, N = 128,
// K = 16 instructions; P is the A operand straight from TMEM, V the B operand
// in MN-major layout.  O accumulates in TMEM; a row's O is rescaled only when
// its running maximum grows by more than 2^8, so rescaling is rare.  Items run
// back to back: the next item's list, Q (once the last S of the current item
// has read Q) and first K/V tiles load while the current item finishes, and
// its first S = Q K^T is issued right after the current item's last PV.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace hga {
namespace {

constexpr int kD = 128;
constexpr int kUnit = 16;
constexpr int kUnitsPerTile = 8;                // 128 keys
constexpr int kMaxUnits = 512;
constexpr int kChunkBytes = 128 * 128;          // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kChunkBytes;     // 128 rows x 128 bf16
constexpr int kStages = 2;
constexpr int kThreads = 320;
constexpr int kSmemBytes = (2 + 2 * kStages) * kTileBytes + 1024;
constexpr uint32_t kWaitLimit = 1u << 26;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.f;

// Routed groups of one block, kept if they name a group of a candidate chunk
// and come in strictly ascending order; writes their first tokens to dst
// (warp-collective; returns the count).
__device__ __forceinline__ int warp_keep_ascending_groups(const int32_t* gl, int kg,
                                                          const LayerParams& p, int cur, int* dst,
                                                          bool* bad) {
  const int m = warp_keep_ascending(
      gl, kg,
      [&](int gid) {
        const int c = gid / p.Ng;
        return c >= p.sink && c < cur - p.local;
      },
      dst, bad);
  __syncwarp();
  for (int i = threadIdx.x & 31; i < m; i += 32) dst[i] *= kUnit;
  __syncwarp();
  return m;
}

template <typename TO>
struct PrefillArgs {
  const int64_t* pos;
  const int32_t* group_idx;
  TO* out;
  float* lse;
  unsigned* err;
};

__device__ __forceinline__ void store_row(float* dst, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 32; j += 4)
    *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
}
__device__ __forceinline__ void store_row(__nv_bfloat16* dst, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 32; j += 8) {
    uint4 w;
    w.x = ptx::pack_bf16x2(v[j], v[j + 1]);
    w.y = ptx::pack_bf16x2(v[j + 2], v[j + 3]);
    w.z = ptx::pack_bf16x2(v[j + 4], v[j + 5]);
    w.w = ptx::pack_bf16x2(v[j + 6], v[j + 7]);
    *reinterpret_cast<uint4*>(dst + j) = w;
  }
}

// Work item k of the persistent schedule: the costliest blocks (latest in the
// prompt, most visible tokens) first, every (sequence, KV head) of one block
// together.
struct Item {
  int b, h, bh, blk;
};
__device__ __forceinline__ Item item_at(int k, const LayerParams& p) {
  const int bhs = p.B * p.Hkv;
  Item it;
  it.blk = p.nblk - 1 - k / bhs;
  it.bh = k % bhs;
  it.h = it.bh % p.Hkv;
  it.b = it.bh / p.Hkv;
  return it;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// First query row (head 0 of the KV head's group, query 0 of the block) in Q.
__device__ __forceinline__ int64_t q_row_of(const Item& it, const LayerParams& p) {
  return (static_cast<int64_t>(it.b) * p.Hq + it.h * p.G) * p.q_len +
         static_cast<int64_t>(it.blk) * p.C;
}

template <typename TO>
__global__ void __launch_bounds__(kThreads, 1)
attend_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, PrefillArgs<TO> a,
                      LayerParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_info_full[2], bar_info_empty[2];
  __shared__ uint64_t bar_q_full, bar_q_empty;
  __shared__ uint64_t bar_k_full[kStages], bar_k_empty[kStages];
  __shared__ uint64_t bar_v_full[kStages], bar_v_empty[kStages];
  __shared__ uint64_t bar_s[2], bar_p[2], bar_o[2], bar_fin;
  __shared__ uint32_t s_tmem;
  __shared__ int s_unit[2][kMaxUnits];  // first token of each unit, per item slot
  __shared__ int s_info[2];             // unit count, per item slot

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mt = p.G * p.C / 128;  // M-tiles (1 or 2)
  const int heads_per_tile = 128 / p.C;
  const int total = p.B * p.Hkv * p.nblk;
  const int stride = static_cast<int>(gridDim.x);

  uint8_t* base = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sq = base;                                 // [2][32 KB] Q tiles
  uint8_t* sk = base + 2 * kTileBytes;                // [kStages][32 KB] K ring
  uint8_t* sv = sk + kStages * kTileBytes;            // [kStages][32 KB] V ring

  auto issue_q = [&](const Item& it) {
    const int64_t q_row0 = q_row_of(it, p);
    ptx::mbar_expect_tx(&bar_q_full, n_mt * kTileBytes);
    for (int mt = 0; mt < n_mt; ++mt)
      for (int hs = 0; hs < heads_per_tile; ++hs)
        for (int rb = 0; rb < p.C / 64; ++rb)
          for (int kc = 0; kc < 2; ++kc) {
            const int hh = mt * heads_per_tile + hs;
            const int64_t row = q_row0 + static_cast<int64_t>(hh) * p.q_len + rb * 64;
            ptx::tma_load_2d(sq + mt * kTileBytes + kc * kChunkBytes + (hs * p.C + rb * 64) * 128,
                             &tm_q, &bar_q_full, kc * 64, static_cast<int32_t>(row));
          }
  };

  if (threadIdx.x == 0) {
    ptx::prefetch_tensormap(&tm_q);
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bar_info_full[s], 1);
      ptx::mbar_init(&bar_info_empty[s], 4 * n_mt + 1);
    }
    ptx::mbar_init(&bar_q_full, 1);
    ptx::mbar_init(&bar_q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&bar_k_full[s], 1);
      ptx::mbar_init(&bar_k_empty[s], 1);
      ptx::mbar_init(&bar_v_full[s], 1);
      ptx::mbar_init(&bar_v_empty[s], 1);
    }
    for (int m = 0; m < 2; ++m) {
      ptx::mbar_init(&bar_s[m], 1);
      ptx::mbar_init(&bar_p[m], 128);
      ptx::mbar_init(&bar_o[m], 1);
    }
    ptx::mbar_init(&bar_fin, 1);
    ptx::fence_barrier_init();
  }
  if (warp == 9) ptx::tmem_alloc(&s_tmem, 512);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;

  // The first item's Q does not depend on routing: the producer starts it
  // before waiting for the kernel that wrote group_idx.
  bool q_pre = false;
  if (warp == 8 && lane == 0 && static_cast<int>(blockIdx.x) < total) {
    const Item it = item_at(blockIdx.x, p);
    if (valid_position(a.pos[it.b], p, nullptr)) {
      issue_q(it);
      q_pre = true;
    }
  }
  pdl_wait();
  bool timed_out = false;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    // Per item: the unit list [sink | local | routed | current] into the item's
    // slot, its count published on bar_info_full, then Q and the K and V tiles.
    uint32_t k_fill = 0, v_fill = 0, q_fill = q_pre ? 1u : 0u;
    int jl = 0;
    for (int k = blockIdx.x; k < total; k += stride, ++jl) {
      const Item it = item_at(k, p);
      const int slot = jl & 1;
      const int64_t pb = a.pos[it.b];  // never written by this library
      const bool ok = valid_position(pb, p, lane == 0 ? a.err : nullptr);
      const int cur = ok ? static_cast<int>((pb - p.q_len + 1) / p.C) + it.blk : 0;
      if (jl >= 2) {  // every consumer has read the slot's previous count
        bool w = true;
        if (lane == 0) w = ptx::mbar_wait(&bar_info_empty[slot], ((jl - 2) >> 1) & 1, kWaitLimit);
        if (!__shfl_sync(~0u, w, 0)) { timed_out = true; break; }
      }
      int* su = s_unit[slot];
      int n = 0;
      if (ok) {
        const int b0 = max(0, cur - p.local);
        const int a_end = min(p.sink, b0);
        const int nf = (a_end + (cur - b0)) * p.Ng;  // sink and local units
        for (int i = lane; i < nf; i += 32) {
          const int ci = i / p.Ng, gi = i % p.Ng;
          const int c = ci < a_end ? ci : b0 + (ci - a_end);
          su[i] = (c * p.Ng + gi) * kUnit;
        }
        n = nf;
        bool bad = false;
        const int32_t* gl = a.group_idx + (static_cast<size_t>(it.bh) * p.nblk + it.blk) * p.kg;
        n += warp_keep_ascending_groups(gl, p.kg, p, cur, su + n, &bad);
        for (int i = lane; i < p.Ng; i += 32) su[n + i] = (cur * p.Ng + i) * kUnit;
        n += p.Ng;
        if (bad && lane == 0) flag_error(a.err, kErrGroupIdx);
      }
      __syncwarp();
      if (lane == 0) {
        s_info[slot] = n;
        ptx::mbar_arrive(&bar_info_full[slot]);  // release: the count and the list
        const int n_tiles = (n + kUnitsPerTile - 1) / kUnitsPerTile;
        if (n > 0 && !(jl == 0 && q_pre)) {
          // Q's buffer is free once the previous item's last S = Q K^T is done
          if (q_fill > 0 && !ptx::mbar_wait(&bar_q_empty, (q_fill - 1) & 1, kWaitLimit))
            timed_out = true;
          else {
            issue_q(it);
            ++q_fill;
          }
        }
        const int64_t kv_row0 = static_cast<int64_t>(it.bh) * p.n_alloc;
        for (int t = 0; t < n_tiles && !timed_out; ++t) {
          // slots past the list reload unit 0 (finite data; masked to zero weight)
          const int st = k_fill % kStages;
          if (k_fill >= kStages &&
              !ptx::mbar_wait(&bar_k_empty[st], ((k_fill - kStages) / kStages) & 1, kWaitLimit)) {
            timed_out = true;
            break;
          }
          ptx::mbar_expect_tx(&bar_k_full[st], kTileBytes);
          for (int us = 0; us < kUnitsPerTile; ++us) {
            const int u = t * kUnitsPerTile + us;
            const int32_t y = static_cast<int32_t>(kv_row0 + su[u < n ? u : 0]);
            for (int kc = 0; kc < 2; ++kc)
              ptx::tma_load_2d(sk + st * kTileBytes + kc * kChunkBytes + us * kUnit * 128, &tm_k,
                               &bar_k_full[st], kc * 64, y);
          }
          ++k_fill;
          if (v_fill >= kStages &&
              !ptx::mbar_wait(&bar_v_empty[st], ((v_fill - kStages) / kStages) & 1, kWaitLimit)) {
            timed_out = true;
            break;
          }
          ptx::mbar_expect_tx(&bar_v_full[st], kTileBytes);
          for (int us = 0; us < kUnitsPerTile; ++us) {
            const int u = t * kUnitsPerTile + us;
            const int32_t y = static_cast<int32_t>(kv_row0 + su[u < n ? u : 0]);
            for (int kc = 0; kc < 2; ++kc)
              ptx::tma_load_2d(sv + st * kTileBytes + kc * kChunkBytes + us * kUnit * 128, &tm_v,
                               &bar_v_full[st], kc * 64, y);
          }
          ++v_fill;
        }
      }
      if (__shfl_sync(~0u, timed_out, 0)) { timed_out = true; break; }
    }
    // Every copy this CTA issued lands before it exits (all have on the normal
    // path; after a timeout the waits are bounded).
    __syncwarp();
    if (lane == 0) {
      if (q_fill > 0) ptx::mbar_wait(&bar_q_full, (q_fill - 1) & 1, kWaitLimit);
      for (int s = 0; s < kStages; ++s) {
        if (k_fill > static_cast<uint32_t>(s))
          ptx::mbar_wait(&bar_k_full[s], ((k_fill - 1 - s) / kStages) & 1, kWaitLimit);
        if (v_fill > static_cast<uint32_t>(s))
          ptx::mbar_wait(&bar_v_full[s], ((v_fill - 1 - s) / kStages) & 1, kWaitLimit);
      }
    }
  } else if (warp == 9) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = ptx::umma_idesc_bf16(128, 128, false, false);
      const uint32_t idesc_o = ptx::umma_idesc_bf16(128, 128, false, true);
      const uint32_t sq_a = ptx::smem_u32(sq), sk_a = ptx::smem_u32(sk), sv_a = ptx::smem_u32(sv);
      auto issue_s = [&](int mt, int stage) {
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          const uint64_t ad = ptx::umma_desc_sw128(sq_a + mt * kTileBytes + koff, 16, 1024);
          const uint64_t bd = ptx::umma_desc_sw128(sk_a + stage * kTileBytes + koff, 16, 1024);
          ptx::umma_ss(tmem + mt * 256, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int mt, int stage, bool first_tile) {
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd =
              ptx::umma_desc_sw128(sv_a + stage * kTileBytes + kk * kUnit * 128, kChunkBytes, 1024);
          ptx::umma_ts(tmem + mt * 256 + 128, tmem + mt * 256 + kk * 8, bd, idesc_o,
                       (!first_tile || kk > 0) ? 1u : 0u);
        }
      };
      int jl = 0, k = blockIdx.x;
      // Next item that has tiles (reads and releases each item's count).
      auto next_item = [&](int& n_tiles) -> bool {
        while (k < total) {
          const int slot = jl & 1;
          if (!ptx::mbar_wait(&bar_info_full[slot], (jl >> 1) & 1, kWaitLimit)) {
            timed_out = true;
            return false;
          }
          const int n = s_info[slot];
          ptx::mbar_arrive(&bar_info_empty[slot]);
          ++jl;
          k += stride;
          if (n > 0) {
            n_tiles = (n + kUnitsPerTile - 1) / kUnitsPerTile;
            return true;
          }
        }
        return false;
      };
      uint32_t kt = 0, vt = 0, qc = 0, pc[2] = {0, 0};
      // Issues S_mt = Q K(kt)^T once K tile kt (and, for an item's first tile, Q) landed.
      auto wait_k = [&](bool new_item) -> bool {
        if (new_item && !ptx::mbar_wait(&bar_q_full, qc++ & 1, kWaitLimit)) return false;
        if (!ptx::mbar_wait(&bar_k_full[kt % kStages], (kt / kStages) & 1, kWaitLimit)) return false;
        ptx::tc_fence_after();
        return true;
      };
      int n_tiles = 0;
      if (next_item(n_tiles)) {
        if (!wait_k(true)) {
          timed_out = true;
        } else {
          for (int mt = 0; mt < n_mt; ++mt) {
            issue_s(mt, kt % kStages);
            ptx::umma_commit(&bar_s[mt]);
          }
          ptx::umma_commit(&bar_k_empty[kt % kStages]);
          if (n_tiles == 1) ptx::umma_commit(&bar_q_empty);
          ++kt;
        }
        int t = 0;
        bool more = !timed_out;
        while (more) {
          // the tile after this one: the same item's next, or the next item's first
          int nt_next = n_tiles;
          const bool next_new = t + 1 == n_tiles;
          const bool has_next = next_new ? next_item(nt_next) : true;
          if (timed_out) break;
          const int t_next = next_new ? 0 : t + 1;
          const int vs = vt % kStages;
          if (!ptx::mbar_wait(&bar_v_full[vs], (vt / kStages) & 1, kWaitLimit)) {
            timed_out = true;
            break;
          }
          for (int mt = 0; mt < n_mt; ++mt) {
            if (!ptx::mbar_wait(&bar_p[mt], pc[mt]++ & 1, kWaitLimit)) { timed_out = true; break; }
            ptx::tc_fence_after();
            issue_pv(mt, vs, t == 0);
            if (mt == n_mt - 1) ptx::umma_commit(&bar_v_empty[vs]);
            if (t + 1 == n_tiles) ptx::umma_commit(&bar_o[mt]);
            if (has_next) {
              if (mt == 0 && !wait_k(next_new)) { timed_out = true; break; }
              issue_s(mt, kt % kStages);
              ptx::umma_commit(&bar_s[mt]);
              if (mt == n_mt - 1) {
                ptx::umma_commit(&bar_k_empty[kt % kStages]);
                if (t_next == nt_next - 1) ptx::umma_commit(&bar_q_empty);
              }
            }
          }
          if (timed_out) break;
          ++vt;
          if (has_next) ++kt;
          t = t_next;
          n_tiles = nt_next;
          more = has_next;
        }
      }
    }
    __syncwarp();
  } else if (warp < 4 * n_mt) {
    // ----------------------------------------------------------- softmax (M-tile)
    const int mt = warp >> 2;
    const int r = (warp & 3) * 32 + lane;                 // row of the M-tile = TMEM lane
    const int hh = mt * heads_per_tile + r / p.C;         // query head within the group
    const int qi = r % p.C;                               // query within the block
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + mt * 256;
    const float sc = kLog2e * rsqrtf(static_cast<float>(kD));
    uint32_t sc_ctr = 0, o_ctr = 0;
    int jl = 0;
    for (int k = blockIdx.x; k < total && !timed_out; k += stride, ++jl) {
      const int slot = jl & 1;
      if (!ptx::mbar_wait(&bar_info_full[slot], (jl >> 1) & 1, kWaitLimit)) {
        timed_out = true;
        break;
      }
      const int n_units = s_info[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bar_info_empty[slot]);
      const Item it = item_at(k, p);
      const int n_tiles = (n_units + kUnitsPerTile - 1) / kUnitsPerTile;
      float m_used = -CUDART_INF_F, l = 0.f;
      // Units [0, u_cur0) are visible to every row; units [u_cur0, n_units) are
      // the current chunk (causal: column offset <= qi); slots >= n_units are
      // padding.  Only tiles reaching u_cur0 need a mask.
      const int u_cur0 = n_units - p.Ng;
      for (int t = 0; t < n_tiles; ++t) {
        if (!ptx::mbar_wait(&bar_s[mt], sc_ctr++ & 1, kWaitLimit)) { timed_out = true; break; }
        ptx::tc_fence_after();
        // Two passes over the row's 128 scores in halves of 64 columns (within a
        // softmax thread's register budget): the running max, then
        // p = 2^(s*sc - m), whose bf16 pairs go back over the S columns read.
        const bool masked = (t + 1) * kUnitsPerTile > u_cur0;
        auto load_half = [&](int hf, uint32_t (&v)[2][32]) {
          ptx::tmem_ld32(trow + hf * 64, v[0]);
          ptx::tmem_ld32(trow + hf * 64 + 32, v[1]);
          ptx::tmem_wait_ld();
          if (masked) {
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              const int c = hf * 64 + j;
              const int u = t * kUnitsPerTile + (c >> 4);
              const bool ok_j = u < u_cur0 || (u < n_units && (u - u_cur0) * kUnit + (c & 15) <= qi);
              if (!ok_j) v[j >> 5][j & 31] = __float_as_uint(-CUDART_INF_F);
            }
          }
        };
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t v[2][32];
          load_half(hf, v);
#pragma unroll
          for (int j = 0; j < 64; ++j)
            mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(v[j >> 5][j & 31]));
        }
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * sc;
        // O is rescaled only when the running max grows by more than 2^8
        if (mx > m_used + kRescaleLog2) {
          if (m_used != -CUDART_INF_F) {  // O holds earlier tiles
            const float f = ex2(m_used - mx);
            l *= f;
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t o[32];
              ptx::tmem_ld32(trow + 128 + ch * 32, o);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
              ptx::tmem_st32(trow + 128 + ch * 32, o);
            }
          }
          m_used = mx;
        }
        // masked scores are -inf and give exactly 0
        const float nm = m_used == -CUDART_INF_F ? 0.f : -m_used;
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t v[2][32];
          load_half(hf, v);
          // pair j of this half lands in v[0][j/2], already consumed
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const float p0 = ex2(fmaf(__uint_as_float(v[j >> 5][j & 31]), sc, nm));
            const float p1 = ex2(fmaf(__uint_as_float(v[j >> 5][(j & 31) + 1]), sc, nm));
            l8[(j >> 1) & 7] += p0 + p1;
            v[0][j >> 1] = ptx::pack_bf16x2(p0, p1);
          }
          ptx::tmem_st32(trow + hf * 32, v[0]);  // P columns 32*hf .. 32*hf+31
        }
        l += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bar_p[mt]);
      }
      // epilogue: O / l (O must be read before the next item's first PV, which
      // waits for this thread's next arrival on bar_p)
      const size_t orow = (static_cast<size_t>(it.b) * p.Hq + it.h * p.G + hh) * p.q_len +
                          static_cast<size_t>(it.blk) * p.C + qi;
      TO* dst = a.out + orow * kD;
      const bool have = n_tiles > 0 && !timed_out && ptx::mbar_wait(&bar_o[mt], o_ctr & 1, kWaitLimit);
      if (n_tiles > 0) {
        ++o_ctr;
        if (!have) timed_out = true;
      }
      if (have) ptx::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        float o[32];
        if (have) {
          ptx::tmem_ld32(trow + 128 + ch * 32, v);
          ptx::tmem_wait_ld();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = have ? __uint_as_float(v[j]) * inv : 0.f;
        store_row(dst + ch * 32, o);
      }
      if (a.lse) a.lse[orow] = have && l > 0.f ? (m_used + log2f(l)) * kLn2 : -CUDART_INF_F;
      ptx::tc_fence_before();
    }
  }
  if (timed_out) flag_error(a.err, kErrTimeout);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    // every MMA this CTA issued has completed before its TMEM is released
    if (lane == 0) {
      ptx::umma_commit(&bar_fin);
      ptx::mbar_wait(&bar_fin, 0, kWaitLimit);
    }
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
  pdl_trigger();
}

template <typename TO>
cudaError_t launch_t(const LayerParams& p, const void* q, const int64_t* pos, const void* k,
                     const void* v, const int32_t* group_idx, void* out, float* lse,
                     unsigned* err, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const int64_t kv_rows = static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc;
  const int64_t q_rows = static_cast<int64_t>(p.B) * p.Hq * p.q_len;
  cudaError_t e = make_bf16_map(&tq, q, q_rows, 64);
  if (e == cudaSuccess) e = make_bf16_map(&tk, k, kv_rows, kUnit);
  if (e == cudaSuccess) e = make_bf16_map(&tv, v, kv_rows, kUnit);
  if (e != cudaSuccess) return e;
  PrefillArgs<TO> a{pos, group_idx, static_cast<TO*>(out), lse, err};
  e = ensure_smem<attend_prefill_kernel<TO>>(kSmemBytes);
  if (e != cudaSuccess) return e;
  static int sms[64];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sms[dev] = n;
  }
  // persistent: one CTA per SM (its shared memory and TMEM admit one)
  const int items = p.B * p.Hkv * p.nblk;
  return launch_pdl(attend_prefill_kernel<TO>, dim3(std::min(items, sms[dev])), dim3(kThreads),
                    kSmemBytes, s, 1, tq, tk, tv, a, p);
}

}  // namespace

bool prefill_tc_path(const LayerParams& p, int dtype) {
  const int64_t units = static_cast<int64_t>(p.sink + p.local + 1) * p.Ng + p.kg;
  return dtype == 1 && p.D == kD && p.q_len > 1 && p.g == kUnit && p.C % 64 == 0 &&
         (p.G * p.C == 128 || p.G * p.C == 256) && units <= kMaxUnits &&
         static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc < (static_cast<int64_t>(1) << 31) &&
         static_cast<int64_t>(p.B) * p.Hq * p.q_len < (static_cast<int64_t>(1) << 31);
}

cudaError_t launch_attend_prefill_bf16(const LayerParams& p, int out_dtype, const void* q,
                                       const int64_t* pos, const void* k, const void* v,
                                       const int32_t* group_idx, void* out, float* lse,
                                       unsigned* err, cudaStream_t s) {
  return out_dtype == 0 ? launch_t<float>(p, q, pos, k, v, group_idx, out, lse, err, s)
                        : launch_t<__nv_bfloat16>(p, q, pos, k, v, group_idx, out, lse, err, s);
}

}  // namespace hga
