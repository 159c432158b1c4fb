// Backward pass of the HGA attention over the routed index sets (prefill).
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709): the layer's output is an exact softmax attention over the tokens
// the routing selects ("Metodologia -> Meccanismo Core", item 4), and the
// method is trained and fine-tuned end to end ("Risultati Sperimentali").  The
// routing is a selection, so gradients flow only through the attention over
// each query block's fixed token set: forced chunks (sink, local, the block's
// own chunk causally) and its kept routed groups.  With P = exp(S - lse),
// S = Q K^T / sqrt(D), Delta = rowsum(dO * O):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),
//   dQ = dS K / sqrt(D),  dK = dS^T Q / sqrt(D).
//
// Kernels, all bf16 operands on mma.sync m16n8k16 with fp32 accumulation:
//   prep_kernel   Delta per query row and lse in log2 units;
//   index_kernel  per (sequence, KV head): the transpose of the routing (for
//                 every key group, the query blocks that routed it, ascending),
//                 and work items: each key group's query blocks (its chunk's
//                 forced blocks, then the routing ones) cut into runs of at
//                 most kSeg blocks;
//   dq_kernel     per query block and 128 of its rows: the block's 16-key units
//                 through a shared double buffer, dQ in registers;
//   dkdv_kernel   one warp per work item: its 16 keys fixed, the query tiles
//                 of its blocks through a private double buffer, dK and dV in
//                 registers, written to dk / dv (a group of one item) or to a
//                 scratch slot;
//   reduce_kernel the scratch slots of each multi-item group summed in item
//                 order; keys no query sees get zeros.
// No atomics on the data: the result does not depend on scheduling.
#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hga {
namespace {

using decode::kD;
using decode::kLog2e;
using decode::kUnit;
using decode::swz;

constexpr int kSeg = 16;          // query blocks per dK/dV work item
constexpr int kTile = 4096;       // bytes of one 16 x 128 bf16 tile (two swizzled boxes)
constexpr int kDqWarps = 8;       // 128 query rows per dQ CTA
constexpr int kKvWarps = 4;       // work items per dK/dV CTA
constexpr int kIdxThreads = 512;

struct BwdArgs {
  const __nv_bfloat16* q;     // [B, Hq, L, D]
  const __nv_bfloat16* k;     // [B, Hkv, n_alloc, D]
  const __nv_bfloat16* v;
  const void* out;            // [B, Hq, L, D] of out_f32 ? float : bf16
  int out_f32;
  const float* lse;           // [B, Hq, L], natural log
  const __nv_bfloat16* dout;  // [B, Hq, L, D]
  const int64_t* pos;
  const int32_t* group_idx;   // [B, Hkv, nblk, kg]
  float* dq;                  // [B, Hq, L, D]
  float* dk;                  // [B, Hkv, n_alloc, D]
  float* dv;
  // workspace
  float* lse2;                // [B, Hq, L]
  float* delta;
  int32_t* off_r;             // [B*Hkv][ng + 1]: routing-transpose offsets
  int32_t* ent_r;             // [B*Hkv][nblk * kg]: query blocks, by key group
  int32_t* off_it;            // [B*Hkv][ng + 1]: first work item of each group
  int2* items;                // [B*Hkv][max_items]: (group, run)
  float* scratch;             // [B*Hkv][max_items][2][16][128]
  int ng;                     // key groups per (sequence, KV head): n_alloc / 16
  int nblk;                   // query blocks per sequence
  int max_items;
  unsigned* err;
};

// Query positions of sequence b: the blocks [blk0, blk1] of C rows.
struct Span {
  bool ok;
  int blk0, blk1;
  int64_t first;
};
__device__ __forceinline__ Span span_of(const BwdArgs& a, const LayerParams& p, int b,
                                        unsigned* err) {
  Span s;
  const int64_t pb = a.pos[b];
  s.ok = valid_position(pb, p, err);
  s.first = pb - p.q_len + 1;
  s.blk0 = s.ok ? static_cast<int>(s.first / p.C) : 0;
  s.blk1 = s.ok ? static_cast<int>(pb / p.C) : -1;
  return s;
}

// Keep rule of the attention for one 32-entry pass of a group_idx row (valid,
// a group of a candidate chunk of block j, above every entry kept before).
__device__ __forceinline__ bool keep_pass(int id, int j, const LayerParams& p, int& run_max) {
  const int lane = threadIdx.x & 31;
  const bool ok = id >= 0 && id / p.Ng >= p.sink && id / p.Ng < j - p.local;
  int incl = ok ? id : -1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl = max(incl, x);
  }
  int excl = __shfl_up_sync(0xffffffffu, incl, 1);
  excl = max(lane == 0 ? -1 : excl, run_max);
  run_max = max(run_max, __shfl_sync(0xffffffffu, incl, 31));
  return ok && id > excl;
}

// Forced query blocks of key chunk c: [jf0, jf1] (empty when jf0 > jf1).  Block j
// sees chunk c as forced when c is its own chunk, a local chunk (j - local <= c),
// or a sink chunk (c < sink), always with c <= j.
__device__ __forceinline__ int2 forced_blocks(int c, const Span& s, const LayerParams& p) {
  const int j0 = max(s.blk0, c);
  const int j1 = c < p.sink ? s.blk1 : min(s.blk1, c + p.local);
  return make_int2(j0, j1);
}

// 16 rows x 128 bf16 from global (row stride 128 elements) into a swizzled tile,
// by one warp (8 x 16-byte asynchronous copies per lane).
__device__ __forceinline__ void warp_tile_load(uint8_t* tile, const __nv_bfloat16* src) {
  const int lane = threadIdx.x & 31;
  const uint32_t t = ptx::smem_u32(tile);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int i = lane + 32 * k, row = i >> 4, c = i & 15;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(swz(t, row, c)),
                 "l"(src + row * kD + c * 8)
                 : "memory");
  }
}

// A fragments (m16n8k16) of rows (g, g + 8) of a row-major bf16 [*, 128] matrix.
__device__ __forceinline__ void load_a_rows(const __nv_bfloat16* r0, const __nv_bfloat16* r1,
                                            uint32_t (&a)[8][4]) {
  const int t = threadIdx.x & 3;
  const uint32_t* x0 = reinterpret_cast<const uint32_t*>(r0);
  const uint32_t* x1 = reinterpret_cast<const uint32_t*>(r1);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    a[kk][0] = __ldg(x0 + kk * 8 + t);
    a[kk][1] = __ldg(x1 + kk * 8 + t);
    a[kk][2] = __ldg(x0 + kk * 8 + 4 + t);
    a[kk][3] = __ldg(x1 + kk * 8 + 4 + t);
  }
}

// s[2][4] += A x K^T and dp[2][4] += A2 x V^T with A, A2 in registers (rows g,
// g + 8) and K, V the 16 rows of tiles kt, vt (rows are the n index), the four
// accumulator chains interleaved.
__device__ __forceinline__ void mma_rows_t2(float (&s)[2][4], float (&dp)[2][4],
                                            const uint32_t (&a)[8][4], const uint32_t (&a2)[8][4],
                                            uint32_t kt, uint32_t vt) {
  const int lane = threadIdx.x & 31, mi = lane >> 3, ri = lane & 7;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    uint32_t rk[4], rv[4];
    ptx::ldmatrix_x4(swz(kt, (mi >> 1) * 8 + ri, kk * 2 + (mi & 1)), rk);
    ptx::ldmatrix_x4(swz(vt, (mi >> 1) * 8 + ri, kk * 2 + (mi & 1)), rv);
    ptx::mma_bf16_16816_pure(s[0], a[kk], rk[0], rk[1]);
    ptx::mma_bf16_16816_pure(s[1], a[kk], rk[2], rk[3]);
    ptx::mma_bf16_16816_pure(dp[0], a2[kk], rv[0], rv[1]);
    ptx::mma_bf16_16816_pure(dp[1], a2[kk], rv[2], rv[3]);
  }
}

// st[2][4] += K Q^T and dpt[2][4] += V dO^T, with K, V (rows the m index) and Q,
// dO (rows the n index) 16-row tiles; the four chains interleaved.
__device__ __forceinline__ void mma_tiles_t2(float (&st)[2][4], float (&dpt)[2][4], uint32_t kt,
                                             uint32_t qt, uint32_t vt, uint32_t dt) {
  const int lane = threadIdx.x & 31, mi = lane >> 3, ri = lane & 7;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    uint32_t ka[4], qb[4], va[4], db[4];
    ptx::ldmatrix_x4(swz(kt, (mi & 1) * 8 + ri, kk * 2 + (mi >> 1)), ka);
    ptx::ldmatrix_x4(swz(qt, (mi >> 1) * 8 + ri, kk * 2 + (mi & 1)), qb);
    ptx::ldmatrix_x4(swz(vt, (mi & 1) * 8 + ri, kk * 2 + (mi >> 1)), va);
    ptx::ldmatrix_x4(swz(dt, (mi >> 1) * 8 + ri, kk * 2 + (mi & 1)), db);
    ptx::mma_bf16_16816_pure(st[0], ka, qb[0], qb[1]);
    ptx::mma_bf16_16816_pure(st[1], ka, qb[2], qb[3]);
    ptx::mma_bf16_16816_pure(dpt[0], va, db[0], db[1]);
    ptx::mma_bf16_16816_pure(dpt[1], va, db[2], db[3]);
  }
}

// acc[16][4] += A (16 x 16, registers) x T, T = tile `bt` (16 rows x 128): the
// A columns index T's rows.
__device__ __forceinline__ void mma_into_rows(float (&acc)[16][4], const uint32_t (&a)[4],
                                              uint32_t bt) {
  const int lane = threadIdx.x & 31, mi = lane >> 3, ri = lane & 7;
#pragma unroll
  for (int nn = 0; nn < 8; ++nn) {
    uint32_t r[4];
    ptx::ldmatrix_x4_trans(swz(bt, (mi & 1) * 8 + ri, nn * 2 + (mi >> 1)), r);
    ptx::mma_bf16_16816_pure(acc[2 * nn], a, r[0], r[1]);
    ptx::mma_bf16_16816_pure(acc[2 * nn + 1], a, r[2], r[3]);
  }
}

// C fragments of a 16 x 16 product as the A operand of the next product.
__device__ __forceinline__ void c_to_a(const float (&c)[2][4], uint32_t (&a)[4]) {
  a[0] = ptx::pack_bf16x2(c[0][0], c[0][1]);
  a[1] = ptx::pack_bf16x2(c[0][2], c[0][3]);
  a[2] = ptx::pack_bf16x2(c[1][0], c[1][1]);
  a[3] = ptx::pack_bf16x2(c[1][2], c[1][3]);
}

// ------------------------------------------------------------------ prep

__global__ void __launch_bounds__(256) prep_kernel(BwdArgs a, int64_t rows) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();
  if (r >= rows) return;
  float o[4], d[4];
  load4(a.dout + r * kD + lane * 4, d);
  if (a.out_f32)
    load4(static_cast<const float*>(a.out) + r * kD + lane * 4, o);
  else
    load4(static_cast<const __nv_bfloat16*>(a.out) + r * kD + lane * 4, o);
  const float s = warp_sum(o[0] * d[0] + o[1] * d[1] + o[2] * d[2] + o[3] * d[3]);
  if (lane == 0) {
    a.delta[r] = s;
    a.lse2[r] = a.lse[r] * kLog2e;
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ index

__global__ void __launch_bounds__(kIdxThreads) index_kernel(BwdArgs a, LayerParams p) {
  extern __shared__ int ism[];
  int* cnt = ism;              // [ng]: routing count, then the routing cursor
  int* segs = ism + a.ng;      // [ng]: work items, then their first item
  int* part = ism + 2 * a.ng;  // [kIdxThreads + 1]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / p.Hkv;
  const Span sp = span_of(a, p, b, tid == 0 ? a.err : nullptr);
  int32_t* off_r = a.off_r + static_cast<size_t>(bh) * (a.ng + 1);
  int32_t* ent_r = a.ent_r + static_cast<size_t>(bh) * a.nblk * p.kg;
  int32_t* off_it = a.off_it + static_cast<size_t>(bh) * (a.ng + 1);
  int2* items = a.items + static_cast<size_t>(bh) * a.max_items;
  const int32_t* gi = a.group_idx + static_cast<size_t>(bh) * a.nblk * p.kg;
  for (int u = tid; u < a.ng; u += kIdxThreads) cnt[u] = 0;
  pdl_wait();
  __syncthreads();
  const int nb = sp.ok ? sp.blk1 - sp.blk0 + 1 : 0;
  // 1. routing counts per key group (order-free)
  for (int jb = warp; jb < nb; jb += kIdxThreads / 32) {
    int run_max = -1;
    for (int base = 0; base < p.kg; base += 32) {
      const int id = base + lane < p.kg ? gi[static_cast<size_t>(jb) * p.kg + base + lane] : -1;
      if (keep_pass(id, sp.blk0 + jb, p, run_max)) atomicAdd(&cnt[id], 1);
    }
  }
  __syncthreads();
  // 2. work items per group: its forced blocks and its routing blocks, in runs
  for (int u = tid; u < a.ng; u += kIdxThreads) {
    const int2 f = forced_blocks(u / p.Ng, sp, p);
    const int len = (sp.ok ? max(0, f.y - f.x + 1) : 0) + cnt[u];
    segs[u] = (len + kSeg - 1) / kSeg;
  }
  __syncthreads();
  // 3. exclusive scans of cnt and segs (each thread a contiguous slice)
  const int per = (a.ng + kIdxThreads - 1) / kIdxThreads;
  const int u0 = min(a.ng, tid * per), u1 = min(a.ng, u0 + per);
  for (int pass = 0; pass < 2; ++pass) {
    int* arr = pass == 0 ? cnt : segs;
    int32_t* dst = pass == 0 ? off_r : off_it;
    int sum = 0;
    for (int u = u0; u < u1; ++u) sum += arr[u];
    part[tid] = sum;
    __syncthreads();
    if (warp == 0) {  // scan of the kIdxThreads partial sums by one warp
      int carry = 0;
      for (int base = 0; base < kIdxThreads; base += 32) {
        int x = part[base + lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        part[base + lane] = carry + x - part[base + lane];  // exclusive
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) part[kIdxThreads] = carry;
    }
    __syncthreads();
    int run = part[tid];
    for (int u = u0; u < u1; ++u) {
      const int x = arr[u];
      arr[u] = run;
      dst[u] = run;
      run += x;
    }
    if (tid == 0) dst[a.ng] = part[kIdxThreads];
    __syncthreads();
  }
  if (tid == 0 && part[kIdxThreads] > a.max_items) flag_error(a.err, kErrGroupIdx);
  // 4a. warp 0: the routing transpose, blocks in ascending order (cnt is the cursor)
  if (warp == 0) {
    constexpr int kAhead = 4;  // rows of group_idx in flight
    int pre[kAhead][4];
    auto fetch = [&](int jb, int (&r)[4]) {
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        const int i = pp * 32 + lane;
        r[pp] = jb < nb && i < p.kg ? gi[static_cast<size_t>(jb) * p.kg + i] : -1;
      }
    };
#pragma unroll
    for (int s = 0; s < kAhead; ++s) fetch(s, pre[s]);
    for (int jb = 0; jb < nb; jb += kAhead) {
#pragma unroll
      for (int s = 0; s < kAhead; ++s) {
        const int jj = jb + s;
        if (jj < nb) {
          int run_max = -1;
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) {
            if (pp * 32 < p.kg) {
              const int id = pre[s][pp];
              if (keep_pass(id, sp.blk0 + jj, p, run_max)) ent_r[cnt[id]++] = sp.blk0 + jj;
            }
          }
        }
        fetch(jj + kAhead, pre[s]);
        __syncwarp();
      }
    }
  } else {
    // 4b. the other warps: the work items (group, run) in group order
    const int nw = kIdxThreads / 32 - 1;
    for (int u = warp - 1; u < a.ng; u += nw) {
      const int first = segs[u];
      const int n = (u + 1 < a.ng ? segs[u + 1] : part[kIdxThreads]) - first;
      for (int s = lane; s < n; s += 32)
        if (first + s < a.max_items) items[first + s] = make_int2(u, s);
    }
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ dQ

__global__ void __launch_bounds__(kDqWarps * 32) dq_kernel(BwdArgs a, LayerParams p) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ int s_units[1024 + 256];
  __shared__ int s_nr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.z, b = bh / p.Hkv, h = bh % p.Hkv;
  const int jb = blockIdx.y;
  const Span sp = span_of(a, p, b, nullptr);
  const int j = sp.blk0 + jb;
  const int b0 = max(0, j - p.local);
  const int su = min(p.sink, b0) * (p.C / kUnit);
  const int nf = su + (j - b0 + 1) * (p.C / kUnit);  // forced units
  // this warp's 16 query rows: head hh, rows r0 .. r0 + 15 of the block
  const int tile = blockIdx.x * kDqWarps + warp;
  const bool active = sp.ok && tile < p.G * (p.C / 16);
  const int hh = tile / (p.C / 16), r0 = (tile % (p.C / 16)) * 16;
  const size_t qrow0 = (static_cast<size_t>(b) * p.Hq + h * p.G + hh) * p.q_len +
                       static_cast<size_t>(jb) * p.C + r0;
  uint32_t qa[8][4], da[8][4];
  float lse_g = 0.f, lse_g8 = 0.f, dl_g = 0.f, dl_g8 = 0.f;
  if (active) {
    load_a_rows(a.q + (qrow0 + g) * kD, a.q + (qrow0 + g + 8) * kD, qa);
    load_a_rows(a.dout + (qrow0 + g) * kD, a.dout + (qrow0 + g + 8) * kD, da);
  }
  pdl_wait();
  if (active) {
    lse_g = a.lse2[qrow0 + g];
    lse_g8 = a.lse2[qrow0 + g + 8];
    dl_g = a.delta[qrow0 + g];
    dl_g8 = a.delta[qrow0 + g + 8];
  }
  if (warp == 0) {  // the block's kept routing groups
    int n = 0, run_max = -1;
    if (sp.ok) {
      const int32_t* row = a.group_idx + (static_cast<size_t>(bh) * a.nblk + jb) * p.kg;
      for (int base = 0; base < p.kg; base += 32) {
        const int id = base + lane < p.kg ? row[base + lane] : -1;
        const bool keep = keep_pass(id, j, p, run_max);
        const unsigned km = __ballot_sync(0xffffffffu, keep);
        if (keep) s_units[n + __popc(km & ((1u << lane) - 1u))] = id;
        n += __popc(km);
      }
    }
    if (lane == 0) s_nr = n;
  }
  __syncthreads();
  const int n_units = sp.ok ? nf + s_nr : 0;
  auto unit_token = [&](int u) -> int64_t {
    if (u < su) return static_cast<int64_t>(u) * kUnit;
    if (u < nf) return static_cast<int64_t>(b0 * (p.C / kUnit) + (u - su)) * kUnit;
    return static_cast<int64_t>(s_units[u - nf]) * kUnit;
  };
  const __nv_bfloat16* kb = a.k + static_cast<size_t>(bh) * p.n_alloc * kD;
  const __nv_bfloat16* vb = a.v + static_cast<size_t>(bh) * p.n_alloc * kD;
  // stage s: K tile at dsm + s * 2 * kTile, V tile after it; 256 threads copy 512 chunks
  auto load_unit = [&](int u, int s) {
    const int64_t t0 = unit_token(u);
    uint8_t* st = dsm + s * 2 * kTile;
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
      const int i = threadIdx.x + k2 * kDqWarps * 32;  // 0 .. 511
      const int which = i >> 8, row = (i >> 4) & 15, c = i & 15;
      const __nv_bfloat16* src = (which ? vb : kb) + (t0 + row) * kD + c * 8;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                       swz(ptx::smem_u32(st + which * kTile), row, c)),
                   "l"(src)
                   : "memory");
    }
    ptx::cp_async_commit();
  };
  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const float sl2 = kLog2e * rsqrtf(static_cast<float>(kD));
  const int64_t tq0 = sp.first + static_cast<int64_t>(jb) * p.C + r0;  // position of row 0
  if (n_units > 0) load_unit(0, 0);
  for (int u = 0; u < n_units; ++u) {
    if (u + 1 < n_units) {
      load_unit(u + 1, (u + 1) & 1);
      ptx::cp_async_wait_group<1>();
    } else {
      ptx::cp_async_wait_group<0>();
    }
    __syncthreads();
    const int64_t tk0 = unit_token(u);
    if (active && tk0 <= tq0 + 15) {
      const uint32_t kt = ptx::smem_u32(dsm + (u & 1) * 2 * kTile);
      const uint32_t vt = kt + kTile;
      float s[2][4] = {}, dp[2][4] = {};
      mma_rows_t2(s, dp, qa, da, kt, vt);
      const bool causal = tk0 + 15 > tq0;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = e < 2 ? g : g + 8;
          const int64_t tk = tk0 + nt * 8 + 2 * t + (e & 1);
          float pr = exp2f(s[nt][e] * sl2 - (e < 2 ? lse_g : lse_g8));
          if (causal && tk > tq0 + row) pr = 0.f;
          s[nt][e] = pr * (dp[nt][e] - (e < 2 ? dl_g : dl_g8));  // dS
        }
      uint32_t dsa[4];
      c_to_a(s, dsa);
      mma_into_rows(acc, dsa, kt);
    }
    __syncthreads();  // the stage is refilled two units later
  }
  if (active) {
    const float sc = rsqrtf(static_cast<float>(kD));
    float* d0 = a.dq + (qrow0 + g) * kD;
    float* d1 = a.dq + (qrow0 + g + 8) * kD;
#pragma unroll
    for (int nn = 0; nn < 16; ++nn) {
      *reinterpret_cast<float2*>(d0 + nn * 8 + 2 * t) = make_float2(acc[nn][0] * sc, acc[nn][1] * sc);
      *reinterpret_cast<float2*>(d1 + nn * 8 + 2 * t) = make_float2(acc[nn][2] * sc, acc[nn][3] * sc);
    }
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ dK, dV

// Per warp: K and V tiles of its group, then two stages of (Q tile, dO tile),
// then two stages of (lse2, delta) x 16.
constexpr int kKvWarpBytes = 2 * kTile + 2 * 2 * kTile + 2 * 2 * 16 * 4;

__global__ void __launch_bounds__(kKvWarps * 32) dkdv_kernel(BwdArgs a, LayerParams p) {
  extern __shared__ __align__(128) uint8_t ksm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.y, b = bh / p.Hkv, h = bh % p.Hkv;
  const int item = blockIdx.x * kKvWarps + warp;
  pdl_wait();
  const int32_t* off_it = a.off_it + static_cast<size_t>(bh) * (a.ng + 1);
  const int n_items = min(off_it[a.ng], a.max_items);
  if (item >= n_items) return;  // warp-uniform; the kernel has no block-wide barrier
  const int2 it = a.items[static_cast<size_t>(bh) * a.max_items + item];
  const int u = it.x, run = it.y;
  const Span sp = span_of(a, p, b, nullptr);
  const int c = u / p.Ng;
  const int2 f = forced_blocks(c, sp, p);
  const int nf = max(0, f.y - f.x + 1);
  const int32_t* off_r = a.off_r + static_cast<size_t>(bh) * (a.ng + 1);
  const int32_t* ent = a.ent_r + static_cast<size_t>(bh) * a.nblk * p.kg + off_r[u];
  const int len = nf + (off_r[u + 1] - off_r[u]);
  const int e0 = run * kSeg, e1 = min(len, e0 + kSeg);
  const int n_runs = off_it[u + 1] - off_it[u];

  uint8_t* wsm = ksm + warp * kKvWarpBytes;
  const uint32_t kt = ptx::smem_u32(wsm), vt = kt + kTile;
  const int64_t tk0 = static_cast<int64_t>(u) * kUnit;  // first key of the group
  const __nv_bfloat16* kb = a.k + (static_cast<size_t>(bh) * p.n_alloc + tk0) * kD;
  const __nv_bfloat16* vb = a.v + (static_cast<size_t>(bh) * p.n_alloc + tk0) * kD;
  warp_tile_load(wsm, kb);
  warp_tile_load(wsm + kTile, vb);
  ptx::cp_async_commit();

  // the tiles of this item: for every query block e in [e0, e1), its G heads x
  // C/16 row tiles (those of the key chunk's own block entirely above the keys
  // are skipped: causally invisible)
  const int tpb = p.G * (p.C / 16);  // tiles per block
  const int n_tiles = (e1 - e0) * tpb;
  auto block_of = [&](int e) { return e < nf ? f.x + e : ent[e - nf]; };
  auto tile_rows = [&](int i, int& jq, int& hh, int& r0) {
    jq = block_of(e0 + i / tpb);
    hh = (i % tpb) / (p.C / 16);
    r0 = (i % (p.C / 16)) * 16;
  };
  auto visible = [&](int jq, int r0) {
    return !(jq == c && static_cast<int64_t>(jq) * p.C + r0 + 15 < tk0);
  };
  auto load_tile = [&](int i, int s) {
    int jq, hh, r0;
    tile_rows(i, jq, hh, r0);
    const size_t row0 = (static_cast<size_t>(b) * p.Hq + h * p.G + hh) * p.q_len +
                        static_cast<size_t>(jq - sp.blk0) * p.C + r0;
    uint8_t* st = wsm + 2 * kTile + s * 2 * kTile;
    warp_tile_load(st, a.q + row0 * kD);
    warp_tile_load(st + kTile, a.dout + row0 * kD);
    float* ld = reinterpret_cast<float*>(wsm + 6 * kTile) + s * 32;
    if (lane < 4)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_u32(ld + lane * 4)),
                   "l"(a.lse2 + row0 + lane * 4)
                   : "memory");
    else if (lane < 8)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(
                       ptx::smem_u32(ld + 16 + (lane - 4) * 4)),
                   "l"(a.delta + row0 + (lane - 4) * 4)
                   : "memory");
    ptx::cp_async_commit();
  };
  // next visible tile at or after i
  auto next_visible = [&](int i) {
    for (; i < n_tiles; ++i) {
      int jq, hh, r0;
      tile_rows(i, jq, hh, r0);
      if (visible(jq, r0)) break;
    }
    return i;
  };

  float dk[16][4], dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
  const float sl2 = kLog2e * rsqrtf(static_cast<float>(kD));
  int cur_i = next_visible(0), stage = 0;
  if (cur_i < n_tiles) load_tile(cur_i, 0);
  while (cur_i < n_tiles) {
    const int nxt = next_visible(cur_i + 1);
    if (nxt < n_tiles) {
      load_tile(nxt, stage ^ 1);
      ptx::cp_async_wait_group<1>();
    } else {
      ptx::cp_async_wait_group<0>();
    }
    __syncwarp();
    int jq, hh, r0;
    tile_rows(cur_i, jq, hh, r0);
    const uint32_t qt = kt + 2 * kTile + stage * 2 * kTile, dt = qt + kTile;
    const float* ld = reinterpret_cast<const float*>(wsm + 6 * kTile) + stage * 32;
    float st[2][4] = {}, dpt[2][4] = {};
    mma_tiles_t2(st, dpt, kt, qt, vt, dt);  // S^T (keys x queries) and dP^T
    const int64_t tq0 = static_cast<int64_t>(jq) * p.C + r0;
    const bool causal = jq == c && tq0 < tk0 + 15;
    float pt[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nt * 8 + 2 * t + (e & 1);
        const int krow = e < 2 ? g : g + 8;
        float pr = exp2f(st[nt][e] * sl2 - ld[col]);
        if (causal && tk0 + krow > tq0 + col) pr = 0.f;
        pt[nt][e] = pr;
        st[nt][e] = pr * (dpt[nt][e] - ld[16 + col]);  // dS^T
      }
    uint32_t pa[4], dsa[4];
    c_to_a(pt, pa);
    c_to_a(st, dsa);
    mma_into_rows(dv, pa, dt);   // dV += P^T dO
    mma_into_rows(dk, dsa, qt);  // dK += dS^T Q
    __syncwarp();  // the stage is refilled by the load two tiles later
    cur_i = nxt;
    stage ^= 1;
  }
  ptx::cp_async_wait_group<0>();
  const float sc = rsqrtf(static_cast<float>(kD));
  float* ok;
  float* ov;
  size_t stride;
  if (n_runs == 1) {  // the group's only item: the result itself
    ok = a.dk + (static_cast<size_t>(bh) * p.n_alloc + tk0) * kD;
    ov = a.dv + (static_cast<size_t>(bh) * p.n_alloc + tk0) * kD;
  } else {
    ok = a.scratch + (static_cast<size_t>(bh) * a.max_items + item) * 2 * kUnit * kD;
    ov = ok + kUnit * kD;
  }
  stride = kD;
#pragma unroll
  for (int nn = 0; nn < 16; ++nn) {
    const int col = nn * 8 + 2 * t;
    *reinterpret_cast<float2*>(ok + g * stride + col) = make_float2(dk[nn][0] * sc, dk[nn][1] * sc);
    *reinterpret_cast<float2*>(ok + (g + 8) * stride + col) = make_float2(dk[nn][2] * sc, dk[nn][3] * sc);
    *reinterpret_cast<float2*>(ov + g * stride + col) = make_float2(dv[nn][0], dv[nn][1]);
    *reinterpret_cast<float2*>(ov + (g + 8) * stride + col) = make_float2(dv[nn][2], dv[nn][3]);
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ reduce

__global__ void __launch_bounds__(256) reduce_kernel(BwdArgs a, LayerParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int u = blockIdx.x * 8 + warp;
  pdl_wait();
  if (u >= a.ng) return;
  const int32_t* off_it = a.off_it + static_cast<size_t>(bh) * (a.ng + 1);
  const int first = off_it[u], n = off_it[u + 1] - first;
  if (n == 1) return;  // written by its item
  float* dk = a.dk + (static_cast<size_t>(bh) * p.n_alloc + static_cast<size_t>(u) * kUnit) * kD;
  float* dv = a.dv + (static_cast<size_t>(bh) * p.n_alloc + static_cast<size_t>(u) * kUnit) * kD;
  for (int i = lane * 4; i < kUnit * kD; i += 128) {
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
    for (int r = 0; r < n && first + r < a.max_items; ++r) {  // item order
      const float* s = a.scratch + (static_cast<size_t>(bh) * a.max_items + first + r) * 2 * kUnit * kD;
      const float4 x = *reinterpret_cast<const float4*>(s + i);
      const float4 y = *reinterpret_cast<const float4*>(s + kUnit * kD + i);
      sk.x += x.x; sk.y += x.y; sk.z += x.z; sk.w += x.w;
      sv.x += y.x; sv.y += y.y; sv.z += y.z; sv.w += y.w;
    }
    *reinterpret_cast<float4*>(dk + i) = sk;
    *reinterpret_cast<float4*>(dv + i) = sv;
  }
  pdl_trigger();
}

}  // namespace

// ------------------------------------------------------------------ host side

namespace {
struct BwdLayout {
  size_t lse2, delta, off_r, ent_r, off_it, items, scratch, total;
  int ng, nblk, max_items;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

BwdLayout bwd_layout(const LayerParams& p) {
  BwdLayout L;
  L.ng = static_cast<int>(p.n_alloc / kUnit);
  L.nblk = p.q_len / p.C;
  const int64_t n_chunks = p.n_alloc / p.C;
  const int64_t pairs = static_cast<int64_t>(p.Ng) * (static_cast<int64_t>(p.sink) * L.nblk +
                                                      n_chunks * (p.local + 1)) +
                        static_cast<int64_t>(L.nblk) * p.kg;
  L.max_items = static_cast<int>(L.ng + (pairs + kSeg - 1) / kSeg);
  const int64_t bh = static_cast<int64_t>(p.B) * p.Hkv;
  const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.q_len;
  size_t o = 0;
  L.lse2 = o;    o += up256(rows * 4);
  L.delta = o;   o += up256(rows * 4);
  L.off_r = o;   o += up256(bh * (L.ng + 1) * 4);
  L.ent_r = o;   o += up256(bh * static_cast<int64_t>(L.nblk) * p.kg * 4);
  L.off_it = o;  o += up256(bh * (L.ng + 1) * 4);
  L.items = o;   o += up256(bh * static_cast<int64_t>(L.max_items) * 8);
  L.scratch = o; o += up256(bh * static_cast<int64_t>(L.max_items) * 2 * kUnit * kD * 4);
  L.total = o;
  return L;
}
}  // namespace

bool backward_path(const LayerParams& p, int dtype) {
  // the index kernel keeps two ints per key group in shared memory (<= 200 KB)
  return dtype == 1 && p.D == kD && p.g == kUnit && p.q_len > 1 && p.q_len % p.C == 0 &&
         p.C % 16 == 0 && p.G <= 16 && p.kg <= 128 &&
         (2 * (p.n_alloc / kUnit) + kIdxThreads + 1) * 4 <= 200 * 1024;
}

size_t backward_workspace_bytes(const LayerParams& p) { return bwd_layout(p).total; }

cudaError_t launch_attend_backward(const LayerParams& p, const void* q, const void* k,
                                   const void* v, const void* out, int out_f32, const float* lse,
                                   const void* d_out, const int64_t* pos, const int32_t* group_idx,
                                   float* dq, float* dk, float* dv, void* workspace,
                                   unsigned* err, cudaStream_t s) {
  const BwdLayout L = bwd_layout(p);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.out = out;
  a.out_f32 = out_f32;
  a.lse = lse;
  a.dout = static_cast<const __nv_bfloat16*>(d_out);
  a.pos = pos;
  a.group_idx = group_idx;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.lse2 = reinterpret_cast<float*>(ws + L.lse2);
  a.delta = reinterpret_cast<float*>(ws + L.delta);
  a.off_r = reinterpret_cast<int32_t*>(ws + L.off_r);
  a.ent_r = reinterpret_cast<int32_t*>(ws + L.ent_r);
  a.off_it = reinterpret_cast<int32_t*>(ws + L.off_it);
  a.items = reinterpret_cast<int2*>(ws + L.items);
  a.scratch = reinterpret_cast<float*>(ws + L.scratch);
  a.ng = L.ng;
  a.nblk = L.nblk;
  a.max_items = L.max_items;
  a.err = err;
  const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.q_len;
  const int bh = p.B * p.Hkv;
  cudaError_t e = launch_pdl(prep_kernel, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256),
                             0, s, 1, a, rows);
  if (e != cudaSuccess) return e;
  const size_t ismem = (2 * static_cast<size_t>(L.ng) + kIdxThreads + 1) * sizeof(int);
  if ((e = ensure_smem<index_kernel>(ismem)) != cudaSuccess) return e;
  if ((e = launch_pdl(index_kernel, dim3(bh), dim3(kIdxThreads), ismem, s, 1, a, p)) != cudaSuccess)
    return e;
  const int dq_ctas = (p.G * (p.C / 16) + kDqWarps - 1) / kDqWarps;
  if ((e = launch_pdl(dq_kernel, dim3(dq_ctas, L.nblk, bh), dim3(kDqWarps * 32), 2 * 2 * kTile, s,
                      1, a, p)) != cudaSuccess)
    return e;
  const size_t kvsmem = static_cast<size_t>(kKvWarps) * kKvWarpBytes;
  if ((e = ensure_smem<dkdv_kernel>(kvsmem)) != cudaSuccess) return e;
  if ((e = launch_pdl(dkdv_kernel, dim3((L.max_items + kKvWarps - 1) / kKvWarps, bh),
                      dim3(kKvWarps * 32), kvsmem, s, 1, a, p)) != cudaSuccess)
    return e;
  return launch_pdl(reduce_kernel, dim3((L.ng + 7) / 8, bh), dim3(256), 0, s, 1, a, p);
}

}  // namespace hga
