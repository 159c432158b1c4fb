// Block-wide deterministic top-k over float scores held in shared memory.
//
// Selects the k largest of n scores, equal scores going to the lower index, and
// writes the chosen indices in ascending order.  A 4-pass 8-bit radix select
// finds the k-th largest order key T and how many keys equal to T are still
// needed; one ordered block scan then takes those in index order.  No sort, no
// atomics outside the shared-memory histogram, no inter-block communication.
#pragma once

#include "common.cuh"

namespace hga {

struct TopkSmem {
  unsigned hist[256];
  int warp_tot[32];
  unsigned pick[2];
};

// Order-preserving map of a float to uint32 (larger float -> larger key);
// -0.0 is folded onto +0.0 so that the two compare equal, as they do as floats.
__device__ __forceinline__ unsigned order_key(float f) {
  unsigned u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of one int per thread, in thread order.  Every thread of
// the block must call it.  NT = blockDim.x, a multiple of 32.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, TopkSmem& sm, int* total = nullptr) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sm.warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int w = lane < NW ? sm.warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < NW) sm.warp_tot[lane] = wi - w;  // exclusive warp offsets
    if (lane == NW - 1 && total) sm.pick[1] = static_cast<unsigned>(wi);
  }
  __syncthreads();
  const int res = sm.warp_tot[wid] + incl - v;
  if (total) *total = static_cast<int>(sm.pick[1]);
  __syncthreads();
  return res;
}

// Warp-cooperative compaction of an id list: keeps, in order, every id with
// in_range(id) true that exceeds every id kept before it (so the output is
// strictly ascending and free of duplicates).  Called by all 32 lanes of one
// warp; writes out[0..count) (and, if given, each kept id's input position to
// out_slot) and returns count in every lane; *bad is set when a non-negative id
// was dropped.
template <typename InRange>
__device__ int warp_keep_ascending(const int32_t* ids, int n, InRange in_range, int* out,
                                   bool* bad, int* out_slot = nullptr) {
  const int lane = threadIdx.x & 31;
  int count = 0, run_max = -1;
  bool dropped = false;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const int id = i < n ? ids[i] : -1;
    const bool ok = id >= 0 && in_range(id);
    int incl = ok ? id : -1;  // inclusive prefix max over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl = max(incl, x);
    }
    int excl = __shfl_up_sync(0xffffffffu, incl, 1);
    excl = max(lane == 0 ? -1 : excl, run_max);
    const bool keep = ok && id > excl;
    dropped |= __any_sync(0xffffffffu, id >= 0 && !keep);
    const unsigned km = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int at = count + __popc(km & ((1u << lane) - 1u));
      out[at] = id;
      if (out_slot) out_slot[at] = i;  // position of the kept id in the input list
    }
    count += __popc(km);
    run_max = max(run_max, __shfl_sync(0xffffffffu, incl, 31));
  }
  *bad = dropped;
  return count;
}

// Top-k by rank counting, for small n (each thread compares its candidates
// against all n): candidate i is taken when fewer than k candidates beat it,
// where j beats i if s_j > s_i, or s_j == s_i and j < i.  Same result and
// contract as block_topk.
template <int NT>
__device__ int block_topk_rank(const float* sc, int n, int k, int* sel, TopkSmem& sm) {
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int i = tid; i < n; i += NT) sel[i] = i;
    __syncthreads();
    return n;
  }
  const int ipt = (n + NT - 1) / NT;
  const int beg = min(n, tid * ipt), end = min(n, beg + ipt);
  unsigned take_bits = 0u;  // ipt <= 32 (n <= 32 * NT)
  int n_take = 0;
  for (int i = beg; i < end; ++i) {
    const float si = sc[i];
    int beats = 0;
    int j = 0;
    for (; j + 4 <= n; j += 4) {  // sc is 16-byte aligned shared memory
      const float4 v = *reinterpret_cast<const float4*>(sc + j);
      beats += (v.x > si) || (v.x == si && j < i);
      beats += (v.y > si) || (v.y == si && j + 1 < i);
      beats += (v.z > si) || (v.z == si && j + 2 < i);
      beats += (v.w > si) || (v.w == si && j + 3 < i);
    }
    for (; j < n; ++j) {
      const float sj = sc[j];
      beats += (sj > si) || (sj == si && j < i);
    }
    if (beats < k) {
      take_bits |= 1u << (i - beg);
      ++n_take;
    }
  }
  int w = block_exclusive_scan<NT>(n_take, sm);
  for (int i = beg; i < end; ++i)
    if (take_bits >> (i - beg) & 1u) sel[w++] = i;
  __syncthreads();
  return k;
}

// Indices of the top k of sc[0..n) (ties to the lower index), ascending, into
// sel[0..min(n,k)).  Returns min(n, k).  Every thread of the block must call it;
// sc and sel are shared memory; sel is complete on return.
template <int NT>
__device__ int block_topk(const float* sc, int n, int k, int* sel, TopkSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (n <= k) {
    for (int i = tid; i < n; i += NT) sel[i] = i;
    __syncthreads();
    return n;
  }
  unsigned prefix = 0u, pmask = 0u;
  unsigned krem = static_cast<unsigned>(k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) sm.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
      // lanes hitting the same bin add once, with the lane count (similar
      // scores share their top bits, so this avoids serialised atomics)
      const unsigned key = order_key(sc[i]);
      const bool hit = (key & pmask) == prefix;
      const unsigned bin = hit ? (key >> shift) & 255u : 0xffffffffu;
      const unsigned peers = __match_any_sync(__activemask(), bin);
      if (hit && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], __popc(peers));
    }
    __syncthreads();
    if (wid == 0) {
      // lane l owns digits 255-8l .. 248-8l, visited from the largest down
      unsigned c[8], tot = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = sm.hist[255 - 8 * lane - j]; tot += c[j]; }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      unsigned run = incl - tot;  // keys with a larger digit
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (run < krem && krem <= run + c[j]) {
          sm.pick[0] = 255u - 8u * lane - j;
          sm.pick[1] = run;
        }
        run += c[j];
      }
    }
    __syncthreads();
    const unsigned d = sm.pick[0];
    krem -= sm.pick[1];
    prefix |= d << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const unsigned thr = prefix;  // k-th largest key; krem of the keys equal to it are taken
  const int ipt = (n + NT - 1) / NT;
  const int beg = min(n, tid * ipt), end = min(n, beg + ipt);
  int n_eq = 0;
  for (int i = beg; i < end; ++i) n_eq += order_key(sc[i]) == thr;
  const int eq_before = block_exclusive_scan<NT>(n_eq, sm);
  int n_sel = 0;
  {
    int eq = eq_before;
    for (int i = beg; i < end; ++i) {
      const unsigned key = order_key(sc[i]);
      const bool take = key > thr || (key == thr && static_cast<unsigned>(eq) < krem);
      eq += key == thr;
      n_sel += take;
    }
  }
  int w = block_exclusive_scan<NT>(n_sel, sm);
  {
    int eq = eq_before;
    for (int i = beg; i < end; ++i) {
      const unsigned key = order_key(sc[i]);
      const bool take = key > thr || (key == thr && static_cast<unsigned>(eq) < krem);
      eq += key == thr;
      if (take) sel[w++] = i;
    }
  }
  __syncthreads();
  return k;
}

}  // namespace hga

namespace hga {

// Top-k of sc[0..n), n <= NT, by rank counting with one candidate per thread
// (j beats i if s_j > s_i, or s_j == s_i and j < i; i is taken when fewer than k
// beat it), compacted in index order.  Block-collective (blockDim == NT); sc is
// 16-byte aligned shared memory; s_cnt holds NT / 32 ints.  Writes out[0..),
// returns min(n, k).
template <int NT>
__device__ int block_rank_topk(const float* sc, int n, int k, int* out, int* s_cnt) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  bool take = false;
  if (t < n) {
    const float si = sc[t];
    int beats = 0;
    int j = 0;
#pragma unroll 4
    for (; j + 4 <= n; j += 4) {
      const float4 x = *reinterpret_cast<const float4*>(sc + j);
      beats += (x.x > si || (x.x == si && j < t)) + (x.y > si || (x.y == si && j + 1 < t)) +
               (x.z > si || (x.z == si && j + 2 < t)) + (x.w > si || (x.w == si && j + 3 < t));
    }
    for (; j < n; ++j) beats += sc[j] > si || (sc[j] == si && j < t);
    take = beats < k;
  }
  const unsigned bal = __ballot_sync(0xffffffffu, take);
  if (lane == 0) s_cnt[w] = __popc(bal);
  __syncthreads();
  int at = __popc(bal & ((1u << lane) - 1u)), total = 0;
#pragma unroll
  for (int x = 0; x < NT / 32; ++x) {
    if (x < w) at += s_cnt[x];
    total += s_cnt[x];
  }
  if (take) out[at] = t;
  __syncthreads();
  return total;
}

// Per-warp scratch of warp_topk: up to kWarpTopkList (key, index) survivors.
constexpr int kWarpTopkList = 64;

// Warp-collective top-k of sc[0..n) (larger score first, equal scores to the
// lower index); writes the chosen indices in ascending order to out[0..) and
// returns their count, min(n, k), in every lane.  lst_key / lst_idx are this
// warp's kWarpTopkList-entry scratch.
//
// For k <= 32 the k-th largest of the 32 lanes' maxima is a lower bound on the
// k-th largest score (those k maxima come from k different scores), so only
// scores at or above it can be chosen; they are usually few and get exact
// ranks by pairwise comparison.  Otherwise (or if too many survive) a
// most-significant-bit-first bisection finds the k-th largest key exactly.
__device__ __forceinline__ int warp_topk(const float* sc, int n, int k, int* out,
                                         unsigned* lst_key, int* lst_idx) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  if (k <= 0) return 0;
  if (n <= k) {
    for (int i = lane; i < n; i += 32) out[i] = i;
    __syncwarp();
    return max(n, 0);
  }
  unsigned thr = 0;
  if (k <= 32) {
    unsigned m = 0;
    for (int i = lane; i < n; i += 32) m = max(m, order_key(sc[i]));
    // bitonic sort of the lane maxima, descending across lanes
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const unsigned o = __shfl_xor_sync(0xffffffffu, m, stride);
        const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
        m = keep_max ? max(m, o) : min(m, o);
      }
    }
    thr = __shfl_sync(0xffffffffu, m, k - 1);
  }
  // survivors (key >= thr), compacted in index order
  int cnt = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const unsigned key = i < n ? order_key(sc[i]) : 0u;
    const bool s = i < n && key >= thr;
    const unsigned bal = __ballot_sync(0xffffffffu, s);
    const int at = cnt + __popc(bal & lt);
    if (s && at < kWarpTopkList) {
      lst_key[at] = key;
      lst_idx[at] = i;
    }
    cnt += __popc(bal);
  }
  __syncwarp();
  if (cnt <= kWarpTopkList) {
    const bool h0 = lane < cnt, h1 = lane + 32 < cnt;
    const unsigned k0 = h0 ? lst_key[lane] : 0u, k1 = h1 ? lst_key[lane + 32] : 0u;
    const int i0 = h0 ? lst_idx[lane] : 0, i1 = h1 ? lst_idx[lane + 32] : 0;
    int r0 = 0, r1 = 0;  // how many survivors come before this one
    for (int j = 0; j < cnt; ++j) {
      const unsigned kj = lst_key[j];
      const int ij = lst_idx[j];
      r0 += (kj > k0 || (kj == k0 && ij < i0)) ? 1 : 0;
      r1 += (kj > k1 || (kj == k1 && ij < i1)) ? 1 : 0;
    }
    const bool s0 = h0 && r0 < k, s1 = h1 && r1 < k;
    const unsigned b0 = __ballot_sync(0xffffffffu, s0), b1 = __ballot_sync(0xffffffffu, s1);
    if (s0) out[__popc(b0 & lt)] = i0;
    if (s1) out[__popc(b0) + __popc(b1 & lt)] = i1;
    __syncwarp();
    return __popc(b0) + __popc(b1);
  }
  // exact k-th largest key t: the largest t with #(key >= t) >= k
  unsigned t = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const unsigned cand = t | (1u << bit);
    unsigned c = 0;
    for (int i = lane; i < n; i += 32) c += order_key(sc[i]) >= cand ? 1u : 0u;
    if (__reduce_add_sync(0xffffffffu, c) >= static_cast<unsigned>(k)) t = cand;
  }
  unsigned gt = 0;
  for (int i = lane; i < n; i += 32) gt += order_key(sc[i]) > t ? 1u : 0u;
  const int ties = k - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
  int w = 0, seen = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const unsigned key = i < n ? order_key(sc[i]) : 0u;
    const bool eq = i < n && key == t;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const bool s = (i < n && key > t) || (eq && seen + __popc(beq & lt) < ties);
    const unsigned bs = __ballot_sync(0xffffffffu, s);
    if (s) out[w + __popc(bs & lt)] = i;
    w += __popc(bs);
    seen += __popc(beq);
  }
  __syncwarp();
  return k;
}

}  // namespace hga
