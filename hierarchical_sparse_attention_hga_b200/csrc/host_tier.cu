// Host tier: K/V history in pinned host memory, only the routed groups (and the
// newest window rows) brought to the GPU per step.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Architettura della Memoria": hot tier in VRAM (chunk summaries
// and the always-visible windows), cold tier in host RAM (the whole K/V
// history); and "Meccanismo Core", item 4: the router fetches the original
// token K/V of the selected groups from host RAM into VRAM before the exact
// attention.
//
// Per (sequence, KV head) the device keeps a working buffer of rows
//   [sink chunks | ring of local+1 chunks (chunk c at slot c mod (local+1)) |
//    kg routed groups (slot j = entry j of group_idx)].
// The gather kernel reads pinned host memory directly (zero-copy 16-byte loads
// over the host link, several in flight per thread) and writes those rows:
// every call stages the routed groups and the current chunk's rows up to the
// query; with refresh_window it also copies the sink and local chunks (after a
// prefill, or when positions jump).  The decode attention then reads the
// working buffer with the same row map (attend_decode.cu, hot mode).
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kRowVec = 16;   // uint4 per 128-dim bf16 row
constexpr int kSplits = 4;    // CTAs per (sequence, KV head)

// Copies `rows` rows (16 uint4 each) from src to dst with the NT threads of this
// CTA, four 16-byte loads in flight per thread per tensor.
template <int NT>
__device__ __forceinline__ void copy_rows(const uint4* __restrict__ ks, const uint4* __restrict__ vs,
                                          uint4* __restrict__ kd, uint4* __restrict__ vd,
                                          int rows) {
  const int n = rows * kRowVec;
  for (int base = threadIdx.x; base < n; base += NT * 4) {
    uint4 kx[4], vx[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * NT;
      if (e < n) { kx[u] = ks[e]; vx[u] = vs[e]; }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * NT;
      if (e < n) { kd[e] = kx[u]; vd[e] = vx[u]; }
    }
  }
}

// The window rows of one (sequence, KV head) whose query sits at pb (chunk
// cur, local chunks from b0): part `part` of `parts` CTAs copies its share.
// refresh 0: the current chunk up to the query; 1: that and the sink and
// local chunks; 2: the query's own row only (the caller's previous step was
// at pb - 1, so every earlier window row is in place: across a chunk boundary
// the finished chunk stays in its ring slot and the new chunk's slot is read
// only up to the query).
template <int NT>
__device__ void copy_window(const uint4* kh, const uint4* vh, uint4* kw, uint4* vw,
                            const LayerParams& p, int64_t pb, int cur, int b0, int refresh,
                            int part, int parts) {
  auto ring_row = [&](int c) { return static_cast<int64_t>(p.sink + c % (p.local + 1)) * p.C; };
  auto chunk_row = [&](int c) { return static_cast<size_t>(c) * p.C * kRowVec; };
  if (part == 0) {
    const int64_t c0 = static_cast<int64_t>(cur) * p.C;
    const int64_t r0 = refresh == 2 ? pb : c0;  // first row copied
    copy_rows<NT>(kh + r0 * kRowVec, vh + r0 * kRowVec, kw + (ring_row(cur) + r0 - c0) * kRowVec,
                  vw + (ring_row(cur) + r0 - c0) * kRowVec, static_cast<int>(pb - r0 + 1));
  }
  if (refresh == 1) {
    for (int c = part; c < min(p.sink, b0); c += parts)
      copy_rows<NT>(kh + chunk_row(c), vh + chunk_row(c), kw + chunk_row(c), vw + chunk_row(c), p.C);
    for (int c = b0 + part; c < cur; c += parts)
      copy_rows<NT>(kh + chunk_row(c), vh + chunk_row(c), kw + ring_row(c) * kRowVec,
                    vw + ring_row(c) * kRowVec, p.C);
  }
}

__global__ void __launch_bounds__(kThreads)
gather_host_kernel(const uint4* __restrict__ k_host, const uint4* __restrict__ v_host,
                   const int64_t* __restrict__ pos, const int32_t* __restrict__ group_idx,
                   LayerParams p, int refresh, uint4* __restrict__ k_work,
                   uint4* __restrict__ v_work, unsigned* err) {
  __shared__ int s_gid[1024], s_slot[1024];
  __shared__ int s_n;
  const int bh = blockIdx.x, b = bh / p.Hkv;
  const int split = blockIdx.y;
  const int64_t R = hot_rows(p);
  const int64_t W = static_cast<int64_t>(p.sink + p.local + 1) * p.C;
  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, threadIdx.x == 0 && split == 0 ? err : nullptr);
  pdl_wait();
  const int cur = ok ? static_cast<int>(pb / p.C) : 0;
  const int b0 = max(0, cur - p.local);
  if (threadIdx.x < 32) {
    int n = 0;
    bool bad = false;
    if (ok) {
      n = warp_keep_ascending(
          group_idx + static_cast<size_t>(bh) * p.kg, p.kg,
          [&](int gid) { return gid / p.Ng >= p.sink && gid / p.Ng < cur - p.local; }, s_gid,
          &bad, s_slot);
    }
    if (threadIdx.x == 0) s_n = n;
  }
  __syncthreads();
  if (!ok) return;
  const uint4* kh = k_host + static_cast<size_t>(bh) * p.n_alloc * kRowVec;
  const uint4* vh = v_host + static_cast<size_t>(bh) * p.n_alloc * kRowVec;
  uint4* kw = k_work + static_cast<size_t>(bh) * R * kRowVec;
  uint4* vw = v_work + static_cast<size_t>(bh) * R * kRowVec;
  // routed groups, split over the CTAs of this (sequence, KV head)
  const int n = s_n;
  for (int i = split; i < n; i += kSplits) {
    const size_t src = static_cast<size_t>(s_gid[i]) * p.g * kRowVec;
    const size_t dst = static_cast<size_t>(W + static_cast<int64_t>(s_slot[i]) * p.g) * kRowVec;
    copy_rows<kThreads>(kh + src, vh + src, kw + dst, vw + dst, p.g);
  }
  copy_window<kThreads>(kh, vh, kw, vw, p, pb, cur, b0, refresh, split, kSplits);
  pdl_trigger();
}

// ------------------------------------------------------------------ warm tier
//
// HGA technical summary, "Architettura della Memoria": a warm tier, a bounded
// LRU in VRAM of recently routed spans, sits between the hot tier and the host
// RAM history.  Here its unit is a routed group: per (sequence, KV head) the
// working buffer's routed region holds M group slots instead of kg, with a
// table tag[M] (group id, -1 empty) and stamp[M] (the step of last use, 0
// empty) in device memory.  One step per (sequence, KV head), one CTA:
//   1. keep the routed groups the attention keeps (valid, candidate chunk,
//      strictly ascending); look every cached tag up among them (binary
//      search): a hit gets the step clock, one more than the largest stamp;
//   2. order the other slots by (empty first, by slot) then (stamp, group id)
//      with a bitonic sort of 64-bit keys; the step's misses, ascending, take
//      the first slots of that order (least recently used first);
//   3. write the table and slot_map (the slot of every group_idx entry, -1
//      where the entry is not kept), then copy the missed groups' rows from
//      pinned host memory into their slots and the window rows as the cold
//      gather does.
// A hit costs no host-link traffic; the attention reads routed group j at
// slot slot_map[j].

constexpr int kWarmThreads = 512;

// Ascending bitonic sort of n (a power of two, <= kWarmMax) keys with a 16-bit
// payload, by all NT threads; returns after a barrier.
template <int NT>
__device__ void block_sort_pairs(unsigned long long* key, short* val, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n / 2; i += NT) {
        const int lo = ((i & ~(j - 1)) << 1) | (i & (j - 1));
        const int hi = lo + j;
        const bool up = (lo & k) == 0;
        const unsigned long long a = key[lo], c = key[hi];
        if ((a > c) == up) {
          key[lo] = c;
          key[hi] = a;
          const short t = val[lo];
          val[lo] = val[hi];
          val[hi] = t;
        }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(kWarmThreads)
gather_warm_kernel(const uint4* __restrict__ k_host, const uint4* __restrict__ v_host,
                   const int64_t* __restrict__ pos, const int32_t* __restrict__ group_idx,
                   LayerParams p, int M, int Mp, int32_t* __restrict__ tags,
                   int32_t* __restrict__ stamps, int32_t* __restrict__ slot_map, int refresh,
                   uint4* __restrict__ k_work, uint4* __restrict__ v_work,
                   unsigned long long* __restrict__ counters, unsigned* err,
                   int2* __restrict__ plan, int32_t* __restrict__ n_plan) {
  __shared__ unsigned long long s_key[kWarmMax];  // eviction order, then the miss list
  __shared__ short s_val[kWarmMax];               // slot of each key
  __shared__ int s_gid[1024], s_in[1024];         // kept groups, their group_idx positions
  __shared__ int s_slot[1024];                    // slot of each kept group (-1: miss)
  __shared__ int s_map[1024];                     // slot of each group_idx entry
  __shared__ int s_n, s_m, s_clock;
  const int tid = threadIdx.x, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / p.Hkv;
  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, tid == 0 ? err : nullptr);
  pdl_wait();
  const int cur = ok ? static_cast<int>(pb / p.C) : 0;
  const int b0 = max(0, cur - p.local);
  if (tid < 32) {
    int n = 0;
    bool bad = false;
    if (ok) {
      n = warp_keep_ascending(
          group_idx + static_cast<size_t>(bh) * p.kg, p.kg,
          [&](int gid) { return gid / p.Ng >= p.sink && gid / p.Ng < cur - p.local; }, s_gid,
          &bad, s_in);
    }
    if (tid == 0) {
      s_n = n;
      s_clock = 0;
    }
  }
  for (int j = tid; j < p.kg; j += kWarmThreads) s_slot[j] = s_map[j] = -1;
  __syncthreads();
  int32_t* sm_row = slot_map + static_cast<size_t>(bh) * p.kg;
  if (!ok) {
    for (int j = tid; j < p.kg; j += kWarmThreads) sm_row[j] = -1;
    if (plan && tid == 0) n_plan[bh] = 0;
    return;
  }
  const int n = s_n;
  int32_t* tg = tags + static_cast<size_t>(bh) * M;
  int32_t* st = stamps + static_cast<size_t>(bh) * M;

  // 1. lookup and eviction keys
  int mx = 0;
  for (int s = tid; s < Mp; s += kWarmThreads) {
    unsigned long long key = ~0ull;
    if (s < M) {
      const int t = tg[s], sv = st[s];
      mx = max(mx, sv);
      int lo = 0, hi = n;  // first kept id >= t
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_gid[mid] < t) lo = mid + 1; else hi = mid;
      }
      if (t >= 0 && lo < n && s_gid[lo] == t) {
        s_slot[lo] = s;  // a hit: tags are distinct, so one writer per entry
      } else {
        key = t < 0 ? static_cast<unsigned long long>(s)
                    : (static_cast<unsigned long long>(static_cast<unsigned>(sv) + 1u) << 32) |
                          static_cast<unsigned>(t);
      }
    }
    s_key[s] = key;
    s_val[s] = static_cast<short>(s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) atomicMax(&s_clock, mx);
  __syncthreads();

  // 2. victims in eviction order for the misses, ascending
  block_sort_pairs<kWarmThreads>(s_key, s_val, Mp);
  const int clock = s_clock + 1;
  if (tid < 32) {
    int m = 0;
    for (int base = 0; base < n; base += 32) {
      const int i = base + lane;
      const bool miss = i < n && s_slot[i] < 0;
      const unsigned mm = __ballot_sync(0xffffffffu, miss);
      if (miss) {
        const int r = m + __popc(mm & ((1u << lane) - 1u));
        const int v = s_val[r];
        s_slot[i] = v;
        s_key[r] = (static_cast<unsigned long long>(static_cast<unsigned>(s_gid[i])) << 32) |
                   static_cast<unsigned>(v);
      }
      m += __popc(mm);
    }
    if (lane == 0) {
      s_m = m;
      if (counters) {
        atomicAdd(&counters[0], static_cast<unsigned long long>(n - m));
        atomicAdd(&counters[1], static_cast<unsigned long long>(m));
      }
    }
  }
  __syncthreads();

  // 3. table, slot map, then the rows
  for (int i = tid; i < n; i += kWarmThreads) {
    const int s = s_slot[i];
    tg[s] = s_gid[i];
    st[s] = clock;
    s_map[s_in[i]] = s;
  }
  __syncthreads();
  for (int j = tid; j < p.kg; j += kWarmThreads) sm_row[j] = s_map[j];
  if (plan) {  // decide only: the misses, for a cold store to stage
    for (int r = tid; r < s_m; r += kWarmThreads) {
      const unsigned long long mk = s_key[r];
      plan[static_cast<size_t>(bh) * p.kg + r] =
          make_int2(static_cast<int>(mk >> 32), static_cast<int>(mk & 0xffffffffu));
    }
    if (tid == 0) n_plan[bh] = s_m;
    pdl_trigger();
    return;
  }

  const uint4* kh = k_host + static_cast<size_t>(bh) * p.n_alloc * kRowVec;
  const uint4* vh = v_host + static_cast<size_t>(bh) * p.n_alloc * kRowVec;
  const int64_t R = hot_rows(p, M);
  const int64_t W = static_cast<int64_t>(p.sink + p.local + 1) * p.C;
  uint4* kw = k_work + static_cast<size_t>(bh) * R * kRowVec;
  uint4* vw = v_work + static_cast<size_t>(bh) * R * kRowVec;
  const int per = p.g * kRowVec;
  const int total = s_m * per;
  for (int base = tid; base < total; base += kWarmThreads * 4) {
    uint4 kx[4], vx[4];
    size_t dst[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * kWarmThreads;
      if (e < total) {
        const int r = e / per, w = e - r * per;
        const unsigned long long mk = s_key[r];
        const size_t src = static_cast<size_t>(mk >> 32) * per + w;
        dst[u] = static_cast<size_t>(W + static_cast<int64_t>(mk & 0xffffffffu) * p.g) * kRowVec + w;
        kx[u] = kh[src];
        vx[u] = vh[src];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * kWarmThreads;
      if (e < total) {
        kw[dst[u]] = kx[u];
        vw[dst[u]] = vx[u];
      }
    }
  }
  copy_window<kWarmThreads>(kh, vh, kw, vw, p, pb, cur, b0, refresh, 0, 1);
  pdl_trigger();
}

// Copies the rows a cold store staged for one warm step (see launch_warm_fill):
// the missed groups into their slots, the window rows into the window.  One CTA
// per (sequence, KV head), zero-copy 16-byte loads of the pinned staging.
__global__ void __launch_bounds__(kWarmThreads)
warm_fill_kernel(const uint4* __restrict__ staging, const int2* __restrict__ plan,
                 const int32_t* __restrict__ n_plan, const int64_t* __restrict__ pos,
                 LayerParams p, int M, int mode, uint4* __restrict__ k_work,
                 uint4* __restrict__ v_work, unsigned* err) {
  const int tid = threadIdx.x, bh = blockIdx.x, b = bh / p.Hkv;
  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, tid == 0 ? err : nullptr);
  pdl_wait();
  if (!ok) return;
  const int64_t WR = window_row_capacity(p);
  const int64_t unit_vec = cold_stage_unit_bytes(p) / 16;
  const uint4* sg = staging + static_cast<size_t>(bh) * unit_vec;   // [K|V][kg][16][16 vec]
  const uint4* sw = sg + static_cast<size_t>(2) * p.kg * p.g * kRowVec;  // [K|V][WR][16 vec]
  const int64_t R = hot_rows(p, M);
  const int64_t W = static_cast<int64_t>(p.sink + p.local + 1) * p.C;
  uint4* kw = k_work + static_cast<size_t>(bh) * R * kRowVec;
  uint4* vw = v_work + static_cast<size_t>(bh) * R * kRowVec;
  const int m = min(n_plan[bh], p.kg);
  const int per = p.g * kRowVec;
  const int64_t cur = pb / p.C, b0 = max(static_cast<int64_t>(0), cur - p.local);
  const int64_t nw = window_row_count(p, pb, mode);
  const int64_t total = static_cast<int64_t>(m) * per + nw * kRowVec;
  for (int64_t e = tid; e < total; e += kWarmThreads) {
    size_t src, dst;
    if (e < static_cast<int64_t>(m) * per) {
      const int r = static_cast<int>(e / per), w = static_cast<int>(e - static_cast<int64_t>(r) * per);
      const int slot = plan[static_cast<size_t>(bh) * p.kg + r].y;
      if (slot < 0 || slot >= M) continue;
      src = static_cast<size_t>(r) * per + w;
      dst = static_cast<size_t>(W + static_cast<int64_t>(slot) * p.g) * kRowVec + w;
      kw[dst] = sg[src];
      vw[dst] = sg[static_cast<size_t>(p.kg) * per + src];
    } else {
      const int64_t f = e - static_cast<int64_t>(m) * per;
      const int64_t i = f / kRowVec, w = f - i * kRowVec;
      const int64_t t = window_row_token(p, pb, mode, i);
      const int64_t c = t / p.C;
      const int64_t row = c < p.sink && c < b0 ? t : (p.sink + c % (p.local + 1)) * p.C + t % p.C;
      dst = static_cast<size_t>(row * kRowVec + w);
      kw[dst] = sw[i * kRowVec + w];
      vw[dst] = sw[(WR + i) * kRowVec + w];
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_gather_host(const LayerParams& p, const void* k_host, const void* v_host,
                               const int64_t* pos, const int32_t* group_idx, void* k_work,
                               void* v_work, int refresh_window, unsigned* err, cudaStream_t s) {
  return launch_pdl(gather_host_kernel, dim3(p.B * p.Hkv, kSplits), dim3(kThreads), 0, s, 1,
                    static_cast<const uint4*>(k_host), static_cast<const uint4*>(v_host), pos,
                    group_idx, p, refresh_window, static_cast<uint4*>(k_work),
                    static_cast<uint4*>(v_work), err);
}

}  // namespace hga

namespace hga {

cudaError_t launch_gather_warm(const LayerParams& p, const void* k_host, const void* v_host,
                               const int64_t* pos, const int32_t* group_idx, int slots,
                               int32_t* tags, int32_t* stamps, int32_t* slot_map, void* k_work,
                               void* v_work, int refresh_window, unsigned long long* counters,
                               unsigned* err, cudaStream_t s, int2* plan, int32_t* n_plan) {
  int mp = 2;
  while (mp < slots) mp <<= 1;
  return launch_pdl(gather_warm_kernel, dim3(p.B * p.Hkv), dim3(kWarmThreads), 0, s, 1,
                    static_cast<const uint4*>(k_host), static_cast<const uint4*>(v_host), pos,
                    group_idx, p, slots, mp, tags, stamps, slot_map, refresh_window,
                    static_cast<uint4*>(k_work), static_cast<uint4*>(v_work), counters, err,
                    plan, n_plan);
}

cudaError_t launch_warm_fill(const LayerParams& p, const void* staging, const int2* plan,
                             const int32_t* n_plan, const int64_t* pos, int slots, int mode,
                             void* k_work, void* v_work, unsigned* err, cudaStream_t s) {
  return launch_pdl(warm_fill_kernel, dim3(p.B * p.Hkv), dim3(kWarmThreads), 0, s, 1,
                    static_cast<const uint4*>(staging), plan, n_plan, pos, p, slots, mode,
                    static_cast<uint4*>(k_work), static_cast<uint4*>(v_work), err);
}

}  // namespace hga
