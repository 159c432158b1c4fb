// One decode step of the HGA hot path in one launch: the summary append
// (step 1), chunk routing (2), group routing (3), and the gather and exact
// attention of the chosen tokens (4, 5), for every (sequence, KV head) item of
// the batch.  bf16 K/V, D = 128, at most 64 chosen chunks and 128 routed groups
// (the routing and attention kernels serve wider routing).
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core": item 3 (RoPE-aware summaries
// of each complete group and chunk), item 2 (level 1 over the chunk summaries,
// level 2 over the group summaries of the chosen chunks, sink / local /
// current chunks always visible) and item 4 (the original K/V of the chosen
// tokens, attended exactly with a standard softmax).
//
// One CTA works on one item at a time (persistent over the items), with W
// streaming warps and one append warp (W = 7, one CTA per SM; or W = 3, two
// CTAs per SM when the batch has more items than SMs: eight warps per SM
// either way, two per SM sub-partition, so each thread may hold 255 registers).  Every streaming warp owns a ring of
// three 8 KB stages and walks its own list of 8 KB units, each one bulk or TMA
// copy group: 16 candidate chunk-summary rows (fp32), or 16 tokens of K and V
// (bf16, 128B-swizzled boxes).  So the whole item is a stream of equal units
// spread over the warps, with up to 3 W units in flight.
//
//   scan:    candidate summary units, round-robin over all warps (the first
//            ones issued before the position is known); each warp scores its
//            rows with the routing kernel's arithmetic and keeps a running
//            top-kc list in registers (insertion by ballot and shuffle, or a
//            bitonic merge for a unit with many winners: score order, then the
//            lower chunk index), then publishes it;
//   level 1: after a barrier, every thread ranks its share of the W lists'
//            keys against all of them; the kc best are the chosen chunks;
//   level 2: each warp streams its chosen chunks' group summaries, scores them,
//            and, after a barrier, the kc * Ng keys are ranked the same way into
//            the routed group list;
//   forced:  each warp's share of the sink, local and current chunks' K/V units,
//            queued right behind its group-summary copies (so their loads land
//            while the level-2 selection runs);
//   routed:  the routed groups' K/V units, round-robin over all warps; every K/V
//            unit is attended as it lands (mma.sync, P in registers);
//   merge:   the warps' (o, m, l) partials, by log-sum-exp in shared memory.
//
// The append warp meanwhile finalises the summary rows that the item's new
// token closes (a group, and the chunk when the token ends it), with the batch
// builder's arithmetic (summary_math.cuh), so the rows are bit-identical to
// hga_build_summaries.  Those rows belong to the current chunk, which this
// step never routes.
//
// Routing is bit-identical to hga_route (same scores, same tie rule); the
// output matches hga_attend up to the bf16 rounding of P.
#include <cuda.h>

#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "route_common.cuh"
#include "summary_math.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace hga {
namespace {

using namespace decode;

constexpr int kS = 3;                        // ring stages per streaming warp
constexpr int kRows = 16;                    // summary rows per unit
constexpr int kRowBytes = kD * 4;            // one fp32 summary row
static_assert(kRows * kRowBytes == kStageBytes, "a summary unit fills one stage");
constexpr int kKcMax = 64;                   // top-kc held as 32 * R1 keys per warp
constexpr int kKgMax = 128;                  // routed groups per item
constexpr unsigned kBarStream = 1;           // named barrier of the streaming warps

// Barrier `id` over `n` threads, in a form that lets different warps reach it at
// different instructions (the append warp and the streaming warps end apart).
__device__ __forceinline__ void named_sync(unsigned id, unsigned n) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void cta_sync() { asm volatile("barrier.sync 0;" ::: "memory"); }

// ---------------------------------------------------------------- 64-bit keys
// Larger key = better: the score's order key, then the lower index.

__device__ __forceinline__ uint64_t make_key(float s, int id) {
  return (static_cast<uint64_t>(order_key(s)) << 32) | static_cast<uint32_t>(~id);
}
__device__ __forceinline__ int key_id(uint64_t k) { return static_cast<int>(~static_cast<uint32_t>(k)); }
__device__ __forceinline__ float key_score(uint64_t k) {
  const uint32_t u = static_cast<uint32_t>(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// One compare-exchange layer of a bitonic network over the warp's 32 R
// elements, element e = r * 32 + lane held in a[r].  Blocks of `size` are
// ordered descending when (e & size) == 0 == DESC. 
template <int R, bool DESC>
__device__ __forceinline__ void bitonic_layer(uint64_t (&a)[R], int size, int j) {
  const int lane = threadIdx.x & 31;
  uint64_t b[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (j >= 32) {  // partner in register r ^ (j / 32) of the same lane
      uint64_t t = a[0];
#pragma unroll
      for (int q = 1; q < R; ++q)
        if (q == (r ^ (j >> 5))) t = a[q];
      b[r] = t;
    } else {
      b[r] = __shfl_xor_sync(0xffffffffu, a[r], j);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = r * 32 + lane;
    const bool desc = ((e & size) == 0) == DESC;
    const bool keep_max = ((e & j) == 0) == desc;
    a[r] = keep_max ? (a[r] > b[r] ? a[r] : b[r]) : (a[r] < b[r] ? a[r] : b[r]);
  }
}

template <int R, bool DESC>
__device__ __forceinline__ void bitonic_sort(uint64_t (&a)[R]) {
#pragma unroll
  for (int size = 2; size <= 32 * R; size <<= 1)
#pragma unroll
    for (int j = size >> 1; j > 0; j >>= 1) bitonic_layer<R, DESC>(a, size, j);
}

// L and N sorted descending; L becomes the 32 R largest of both, descending.
template <int R>
__device__ __forceinline__ void merge_desc(uint64_t (&L)[R], const uint64_t (&N)[R]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const uint64_t n = __shfl_sync(0xffffffffu, N[R - 1 - r], 31 - lane);  // N reversed
    L[r] = L[r] > n ? L[r] : n;
  }
#pragma unroll
  for (int j = 16 * R; j > 0; j >>= 1) bitonic_layer<R, true>(L, 32 * R, j);
}

// Element e of a warp-distributed array.
template <int R>
__device__ __forceinline__ uint64_t element(const uint64_t (&a)[R], int e) {
  uint64_t v = 0;
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (r == (e >> 5)) v = a[r];
  return __shfl_sync(0xffffffffu, v, e & 31);
}

// Inserts key x (the same in every lane) into the sorted list L (descending,
// 32 R entries, element e = r * 32 + lane): entries below x move down one place
// and the last one drops out.
template <int R>
__device__ __forceinline__ void insert_key(uint64_t (&L)[R], uint64_t x) {
  const int lane = threadIdx.x & 31;
  int pos = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) pos += __popc(__ballot_sync(0xffffffffu, L[r] > x));
  uint64_t prev[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const uint64_t up = __shfl_up_sync(0xffffffffu, L[r], 1);
    const uint64_t last = r > 0 ? __shfl_sync(0xffffffffu, L[r > 0 ? r - 1 : 0], 31) : 0ull;
    prev[r] = lane == 0 ? last : up;  // element e - 1
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = r * 32 + lane;
    L[r] = e < pos ? L[r] : (e == pos ? x : prev[r]);
  }
}

// Adds the 16 new keys of lanes 0..15 (0 = none) to the running list L
// (descending; the first k entries are the k best so far).  The keys that beat
// the k-th entry are inserted one at a time (usually a few); a batch with many
// winners (the first units) is sorted and merged instead.
template <int R>
__device__ __forceinline__ void offer16(uint64_t (&L)[R], uint64_t nk, int k) {
  unsigned m = __ballot_sync(0xffffffffu, nk > element<R>(L, k - 1));
  if (__popc(m) > 6) {
    uint64_t n[R];
#pragma unroll
    for (int r = 0; r < R; ++r) n[r] = r == 0 ? nk : 0ull;
    bitonic_sort<R, true>(n);
    merge_desc<R>(L, n);
    return;
  }
  while (m) {
    const int src = __ffs(m) - 1;
    m &= m - 1;
    insert_key<R>(L, __shfl_sync(0xffffffffu, nk, src));
  }
}

// Scores of 16 fp32 summary rows in shared memory against the routing query
// (qv: this lane's float4 columns s8, s8 + 8, ... with s8 = lane % 8), with the
// routing kernel's arithmetic (eight lanes per row, the same sum order).  Lane
// L < 16 returns the score of row L.
__device__ __forceinline__ float score16(const float* rows, const float4 (&qv)[kD / 32]) {
  const int lane = threadIdx.x & 31, sub = lane >> 3, s8 = lane & 7;
  float mine = 0.f;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const float4* src = reinterpret_cast<const float4*>(rows + (it * 4 + sub) * kD);
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
    const float v = __shfl_sync(0xffffffffu, a, (lane & 3) * 8);
    if ((lane >> 2) == it) mine = v;
  }
  return mine;
}

// ------------------------------------------------------------ shared memory

constexpr int kL2Max = kKcMax * 8;  // level-2 candidates: chosen chunks x groups per chunk

struct StepSmem {  // byte offsets into the dynamic shared memory (after alignment)
  int W, n_tab, n_pt;  // n_pt: block-table entries staged per item (paged pools), else 0
  int peer_floats;     // clusters: the CTAs' partials gathered in rank 0, else 0
  __host__ __device__ size_t rings() const { return static_cast<size_t>(W) * kS * kStageBytes; }
  __host__ __device__ size_t o_union() const { return rings(); }                    // u64 [W][kKcMax]
  __host__ __device__ size_t o_ckey() const { return o_union() + static_cast<size_t>(W) * kKcMax * 8; }
  __host__ __device__ size_t o_gkey() const { return o_ckey() + kKcMax * 8; }       // u64 [kL2Max]
  __host__ __device__ size_t o_gsc() const { return o_gkey() + kL2Max * 8; }        // float [kKgMax]
  __host__ __device__ size_t o_qbar() const { return o_gsc() + kKgMax * 4; }        // float [kD]
  __host__ __device__ size_t o_chunks() const { return o_qbar() + kD * 4; }         // int [kKcMax]
  __host__ __device__ size_t o_glist() const { return o_chunks() + kKcMax * 4; }    // int [kKgMax]
  __host__ __device__ size_t o_gsum() const { return o_glist() + kKgMax * 4; }      // float [8][kD]
  __host__ __device__ size_t o_tab() const { return o_gsum() + 8 * kD * 4; }        // float2 [n_tab]
  __host__ __device__ size_t o_pages() const {  // int [n_pt], 16-byte aligned
    return (o_tab() + static_cast<size_t>(n_tab) * 8 + 15) & ~static_cast<size_t>(15);
  }
  __host__ __device__ size_t o_peer() const {  // float [peer_floats], 16-byte aligned
    return (o_pages() + static_cast<size_t>(n_pt) * 4 + 15) & ~static_cast<size_t>(15);
  }
  __host__ __device__ size_t bytes() const {
    return 1024 + o_peer() + static_cast<size_t>(peer_floats) * 4;
  }
};

template <typename TO>
struct StepArgs {
  const __nv_bfloat16* q;
  const int64_t* pos;
  const __nv_bfloat16* k;   // the cache (the append warp's reads; address warming)
  const __nv_bfloat16* v;
  float* chunk_sum;
  float* group_sum;
  int32_t* chunk_idx;
  float* chunk_score;
  int32_t* group_idx;
  float* group_score;
  TO* out;
  float* lse;
  unsigned* err;
  int append;
  int n_items;
  KvPages kv;               // paged pools (the PAGED kernels); block_table null otherwise
};

// 2 MB pages of each of the item's group-summary, K and V regions whose address
// translation is warmed at the start of an item (covers 16 MB, a 64K context).
constexpr int kTlbPages = 8;

// Place of `key` among the n keys at `keys` (shared memory): the number above it.
__device__ __forceinline__ int rank_among(const uint64_t* keys, int n, uint64_t key) {
  int r0 = 0, r1 = 0, i = 0;
#pragma unroll 4
  for (; i + 2 <= n; i += 2) {
    r0 += keys[i] > key;
    r1 += keys[i + 1] > key;
  }
  if (i < n) r0 += keys[i] > key;
  return r0 + r1;
}

// ------------------------------------------------------------------ kernel
//
// Per item, every streaming warp walks one stream of units through its ring:
//
//   [scan units] | B1 top-kc by rank B2 | [group-summary units of its chosen
//   chunks] [window units] | B3 top-kg by rank B4 | [routed units]
//
// where B1..B4 are barriers of the streaming warps.  The group-summary fetch is
// the critical path after the scan, so each warp queues its window (sink, local,
// current) loads right behind its own group-summary copies; they land while the
// level-2 selection runs.

// PAGED: k and v are page pools (KvPages); each item stages its sequence's
// block-table row in shared memory (asynchronous copies issued at the item's
// start, validated before the first barrier), and every K/V tile's row comes
// from it.  An entry that is not a page of the pool is flagged and read as
// zeros (its tiles start at a negative row, which the tensor copy fills).
//
// NC > 1 (small batches, NC items' worth of SMs each): each item on a cluster of
// NC CTAs, one per SM.  Every CTA scans a slice of the candidate summaries
// (units round-robin over the cluster's NC x W warps), takes its slice's
// top-kc and writes it into rank 0's shared memory (distributed shared memory,
// then a remote mbarrier arrival); rank 0 selects the chunks among the NC lists,
// runs level 2 and broadcasts the routed list the same way; every CTA attends
// its share of the window units at once and of the routed units on arrival,
// and sends its partial (o, m, l) to rank 0, which merges them and writes the
// outputs.  Every wait on another CTA is bounded.
template <int W, int R1, typename TO, bool PAGED, int NC>
__global__ void __launch_bounds__((W + 1) * 32, W == 7 ? 1 : 2)
decode_step_kernel(const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, StepArgs<TO> a, LayerParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[W][kS];
  __shared__ float s_ml[W][16][2];
  __shared__ int s_abort;
  __shared__ uint64_t s_l1all[NC > 1 ? NC : 1][kKcMax];  // rank 0: every CTA's slice top-kc
  __shared__ uint64_t s_l1bar;   // rank 0: the NC slice lists arrived
  __shared__ uint64_t s_hand;    // ranks > 0: the routed list arrived
  __shared__ uint64_t s_peerbar; // rank 0: the NC - 1 partials arrived
  __shared__ int s_ng_in;        // ranks > 0: routed groups in the list received
  __shared__ int s_bad[2];       // rank 0: a wait of this item gave up (by item parity)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;  // streaming threads: 0 .. W * 32 - 1
  uint8_t* base = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  StepSmem L{W, summ::table_entries(p, kD), PAGED ? a.kv.max_pages : 0,
             NC > 1 ? NC * p.G * (kD + 2) : 0};
  // clusters: this CTA's rank, and its warps' place among the cluster's NW warps
  const int crank = NC > 1 ? static_cast<int>(ptx::cluster_ctarank()) : 0;
  constexpr int NW = NC * W;
  float* peer = reinterpret_cast<float*>(base + L.o_peer());  // rank 0: [NC][G][kD] o, [NC][G] (m, l)
  uint64_t* s_union = reinterpret_cast<uint64_t*>(base + L.o_union());
  uint64_t* ckey = reinterpret_cast<uint64_t*>(base + L.o_ckey());  // chosen chunks' keys, rank order
  uint64_t* gkey = reinterpret_cast<uint64_t*>(base + L.o_gkey());
  float* gsc = reinterpret_cast<float*>(base + L.o_gsc());
  float* qbar = reinterpret_cast<float*>(base + L.o_qbar());
  int* chunks = reinterpret_cast<int*>(base + L.o_chunks());  // chosen chunks, rank order
  int* glist = reinterpret_cast<int*>(base + L.o_glist());    // routed groups, rank order
  float(*gsum)[kD] = reinterpret_cast<float(*)[kD]>(base + L.o_gsum());
  float2* tab = reinterpret_cast<float2*>(base + L.o_tab());
  int* s_pages = reinterpret_cast<int*>(base + L.o_pages());  // PAGED: the item's block-table row

  if (threadIdx.x == 0) {
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
    for (int w = 0; w < W; ++w)
      for (int s = 0; s < kS; ++s) ptx::mbar_init(&bars[w][s], 1);
    ptx::mbar_init(&s_l1bar, NC);
    ptx::mbar_init(&s_hand, 1);
    ptx::mbar_init(&s_peerbar, NC > 1 ? NC - 1 : 1);
    s_abort = 0;
    s_bad[0] = s_bad[1] = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (NC > 1) ptx::cluster_barrier();  // every CTA's barriers exist before any remote arrival
  const int item0 = NC > 1 ? static_cast<int>(blockIdx.x) / NC : static_cast<int>(blockIdx.x);
  const int istride = NC > 1 ? static_cast<int>(gridDim.x) / NC : static_cast<int>(gridDim.x);

  // ------------------------------------------------------------ append warp
  if (warp == W) {
    if (a.append) {
      for (int i = lane; i < L.n_tab; i += 32) tab[i] = summ::table_entry(p, kD, i);
      __syncwarp();
      pdl_wait();  // the rows read and written may belong to the kernel just before
      for (int item = item0; item < a.n_items && crank == 0; item += istride) {
        const int b = item / p.Hkv, h = item % p.Hkv;
        const int64_t pb = a.pos[b];
        if (pb < 0 || pb >= p.n_alloc) continue;
        auto group_rows = [&](int64_t g0) -> const __nv_bfloat16* {
          if (!PAGED) return a.k + (static_cast<size_t>(item) * p.n_alloc + g0) * kD;
          const int32_t pg = __ldg(a.kv.block_table + static_cast<size_t>(b) * a.kv.max_pages +
                                   page_index(a.kv, static_cast<uint32_t>(g0)));
          if (pg < 0 || pg >= a.kv.n_pages) return nullptr;
          return a.k + static_cast<size_t>(paged_row(a.kv, p.Hkv, h, pg, g0)) * kD;
        };
        const bool rows_ok = summ::append_closed_rows<__nv_bfloat16, kD>(
            group_rows, a.chunk_sum + static_cast<size_t>(item) * p.n_chunks * kD,
            a.group_sum + static_cast<size_t>(item) * p.n_chunks * p.Ng * kD, p, pb, tab, gsum);
        if (!rows_ok && lane == 0) flag_error(a.err, kErrPage);
      }
    }
    cta_sync();
    if (NC > 1) ptx::cluster_barrier();
    pdl_trigger();
    return;
  }

  // ------------------------------------------------------- streaming warps
  const float scale = kLog2e * rsqrtf(static_cast<float>(kD));
  uint8_t* ring = base + static_cast<size_t>(warp) * kS * kStageBytes;
  uint64_t* wbar = bars[warp];
  int issued = 0, done = 0;  // this warp's ring counters, continued over items
  int item_no = 0;           // items this CTA has started
  auto stage = [&](int i) { return ring + (i % kS) * kStageBytes; };
  // a debug run that withholds a copy gives up after 2 ms instead of 50 ms
  const uint64_t limit_ns = (p.debug & kDebugSkipRouteArrive) ? 2000000ull : 50000000ull;
  auto wait_stage = [&](int i) { return ptx::mbar_wait_ns(&wbar[i % kS], (i / kS) & 1, kWaitLimit, limit_ns); };
  // candidate summary rows that exist past the sink chunks (whatever the position)
  const int rows_max = max(0, p.n_chunks - p.sink);
  const int n_su_max = (rows_max + kRows - 1) / kRows;
  const int cpu = kRows / p.Ng;  // chosen chunks per group-summary unit

  pdl_wait();  // summaries may come from the kernel just before
  for (int item = item0; item < a.n_items; item += istride, ++item_no) {
    const int b = item / p.Hkv, h = item % p.Hkv;
    if (NC == 1 && s_abort) {  // an earlier item of this CTA timed out: write the empty result, no waits
      if (warp == 0) {
        for (int i = lane; i < p.kc; i += 32) a.chunk_idx[static_cast<size_t>(item) * p.kc + i] = -1;
        for (int i = lane; i < p.kg; i += 32) a.group_idx[static_cast<size_t>(item) * p.kg + i] = -1;
      }
      for (int idx = tid; idx < p.G * kD; idx += W * 32) {
        const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + idx / kD;
        store_out(a.out + row * kD + idx % kD, 0.f);
        if (a.lse && idx % kD == 0) a.lse[row] = -CUDART_INF_F;
      }
      continue;
    }
    const float* cbase = a.chunk_sum + (static_cast<size_t>(item) * p.n_chunks + p.sink) * kD;
    const float* gbase = a.group_sum + static_cast<size_t>(item) * p.n_chunks * p.Ng * kD;
    const int64_t row_base = static_cast<int64_t>(item) * p.n_alloc;
    if (PAGED) {  // the sequence's block-table row, landing while the scan runs
      const int32_t* bt = a.kv.block_table + static_cast<size_t>(b) * a.kv.max_pages;
      if (a.kv.max_pages % 4 == 0 && (reinterpret_cast<uintptr_t>(a.kv.block_table) & 15) == 0) {
        for (int i = 4 * tid; i < a.kv.max_pages; i += 4 * W * 32) ptx::cp_async16(s_pages + i, bt + i);
      } else {
        for (int i = tid; i < a.kv.max_pages; i += W * 32) ptx::cp_async4(s_pages + i, bt + i);
      }
    }
    // row of token t of this item in the [rows][D] view of k / v
    auto kv_row = [&](int64_t t) -> int32_t {
      if (!PAGED) return static_cast<int32_t>(row_base + t);
      const uint32_t tt = static_cast<uint32_t>(t);
      const uint32_t j = page_index(a.kv, tt);
      return (s_pages[j] * p.Hkv + h) * a.kv.page_size + static_cast<int32_t>(tt - j * a.kv.page_size);
    };

    // 1. position, routing query and Q fragments: independent loads, issued first so
    //    that they do not queue behind the bulk copies below
    const int64_t pb = a.pos[b];
    constexpr int kQD = (kD + W * 32 - 1) / (W * 32);  // routing-query dims per thread
    unsigned short v[kQD][16];  // bf16 bits; converted after the bulk copies are issued
    const unsigned short* qraw = reinterpret_cast<const unsigned short*>(a.q);
#pragma unroll
    for (int j = 0; j < kQD; ++j) {
      const int d = min(kD - 1, tid + j * W * 32);
#pragma unroll
      for (int hh = 0; hh < 16; ++hh)
        v[j][hh] = hh < p.G ? __ldg(qraw + (static_cast<size_t>(b) * p.Hq + h * p.G + hh) * kD + d) : 0;
    }
    uint32_t qa[8][4];
    load_q_frags(a.q, p, b, h, qa);
    // warm the address translation of the item's group-summary and K/V regions
    // (read later at scattered places) while the scan runs
    if (warp == 0 && lane < (PAGED ? 1 : 3) * kTlbPages) {
      const int which = lane / kTlbPages, page = lane % kTlbPages;
      const size_t span = which == 0 ? static_cast<size_t>(p.n_chunks) * p.Ng * kD * 4
                                     : static_cast<size_t>(p.n_alloc) * kD * 2;
      const uint8_t* region = which == 0 ? reinterpret_cast<const uint8_t*>(gbase)
                              : which == 1 ? reinterpret_cast<const uint8_t*>(a.k + row_base * kD)
                                           : reinterpret_cast<const uint8_t*>(a.v + row_base * kD);
      const size_t off = static_cast<size_t>(page) << 21;
      if (off < span) asm volatile("prefetch.global.L2 [%0];" ::"l"(region + off));
    }

    // 2. the warp's first scan units before the position is known: the rows that
    //    exist past the sink (the units beyond this item's candidates are dropped)
    const int gw = crank * W + warp;  // this warp among the cluster's NW warps
    const int n_spec = min(kS, n_su_max > gw ? (n_su_max - gw + NW - 1) / NW : 0);
    for (int i = 0; i < n_spec; ++i) {
      const int su = gw + i * NW;
      if (lane == 0) {
        const int nr = min(kRows, rows_max - su * kRows);
        ptx::mbar_expect_tx(&wbar[issued % kS], static_cast<uint32_t>(nr) * kRowBytes);
        ptx::bulk_load(stage(issued), cbase + static_cast<size_t>(su) * kRows * kD,
                       static_cast<uint32_t>(nr) * kRowBytes, &wbar[issued % kS]);
      }
      ++issued;
    }
#pragma unroll
    for (int j = 0; j < kQD; ++j) {
      const int d = tid + j * W * 32;
      float s = 0.f;
#pragma unroll
      for (int hh = 0; hh < 16; ++hh)
        if (hh < p.G) s += __uint_as_float(static_cast<unsigned>(v[j][hh]) << 16);
      if (d < kD) qbar[d] = s / static_cast<float>(p.G);
    }

    // 3. this item's stream: [scan | group summaries | window | routed]
    const bool ok = valid_position(pb, p, (warp == 0 && lane == 0) ? a.err : nullptr);
    const int cur = ok ? static_cast<int>(pb / p.C) : 0;
    const int b0 = max(0, cur - p.local);
    const int n_cand = ok ? max(0, cur - p.local - p.sink) : 0;
    const int n_su = (n_cand + kRows - 1) / kRows;
    const int upc = p.C / kUnit;  // K/V units per chunk
    const int su_sink = ok ? min(p.sink, b0) * upc : 0;
    const int u_first_local = b0 * upc;
    const int n_forced = ok ? su_sink + static_cast<int>(pb / kUnit) - u_first_local + 1 : 0;
    const int ns = min(p.kc, n_cand);       // chosen chunks
    const int n_l2 = ns * p.Ng;             // level-2 candidates
    const int ng = min(p.kg, n_l2);         // routed groups
    auto count = [&](int n) { return n > gw ? (n - gw + NW - 1) / NW : 0; };  // i = gw + k NW < n
    auto count_cta = [&](int n) { return n > warp ? (n - warp + W - 1) / W : 0; };
    const int n_head = max(count(n_su), n_spec);  // scan units (those past n_su are dropped)
    const int n_mine = crank == 0 ? count_cta(ns) : 0;  // chosen chunks warp, warp + W, ... (rank 0)
    const int n_fw = count(n_forced);             // window units warp, warp + W, ...
    const int n_l2u = (n_mine + cpu - 1) / cpu;
    const int n_rw = count(ng);
    // stream index -> unit: [0, e_l2) scan; [e_l2, e_fw) group summaries; [e_fw, e_rt)
    // window; [e_rt, e_all) routed
    const int e_l2 = n_head, e_fw = e_l2 + n_l2u, e_rt = e_fw + n_fw;
    int e_all = e_rt + n_rw;
    auto forced_token = [&](int f) -> int64_t {
      return static_cast<int64_t>(f < su_sink ? f : u_first_local + (f - su_sink)) * kUnit;
    };
    int next = n_spec;  // next stream unit to issue
    bool timed_out = false;
    auto issue_upto = [&](int limit) {
      while (next < limit && issued - done < kS) {
        const int i = next++;
        uint8_t* st = stage(issued);
        uint64_t* bar = &wbar[issued % kS];
        if (lane == 0) {
          if (i < e_l2) {
            const int su = gw + i * NW;
            const int nr = min(kRows, n_cand - su * kRows);
            ptx::mbar_expect_tx(bar, static_cast<uint32_t>(nr) * kRowBytes);
            ptx::bulk_load(st, cbase + static_cast<size_t>(su) * kRows * kD,
                           static_cast<uint32_t>(nr) * kRowBytes, bar);
          } else if (i < e_fw) {
            // a debug run withholds warp 0's first group-summary copy: its bounded wait
            // on that stage then runs out with nothing in flight
            const bool skip = (p.debug & kDebugSkipRouteArrive) && warp == 0 && item_no == 0 && i == e_l2;
            const int k0 = (i - e_l2) * cpu, k1 = min(n_mine, k0 + cpu);
            if (!skip) {
              ptx::mbar_expect_tx(bar, static_cast<uint32_t>((k1 - k0) * p.Ng) * kRowBytes);
              for (int kk = k0; kk < k1; ++kk)
                ptx::bulk_load(st + static_cast<size_t>(kk - k0) * p.Ng * kRowBytes,
                               gbase + static_cast<size_t>(chunks[warp + kk * W]) * p.Ng * kD,
                               static_cast<uint32_t>(p.Ng) * kRowBytes, bar);
            }
          } else if (i < e_rt) {
            issue_unit(&tm_k, &tm_v, st, bar, kv_row(forced_token(gw + (i - e_fw) * NW)));
          } else {
            issue_unit(&tm_k, &tm_v, st, bar,
                       kv_row(static_cast<int64_t>(glist[gw + (i - e_rt) * NW]) * kUnit));
          }
        }
        ++issued;
      }
    };
    // consumes stream units [from, to) with `fn`, topping the ring up to `limit`
    auto consume = [&](int from, int to, int limit, auto&& fn) {
      for (int i = from; i < to && !timed_out; ++i) {
        if (!wait_stage(done)) {
          timed_out = true;
          break;
        }
        fn(i, stage(done));
        ++done;
        __syncwarp();
        issue_upto(limit);
      }
    };
    issue_upto(e_l2);

    named_sync(kBarStream, W * 32);  // qbar
    float4 qv[kD / 32];
#pragma unroll
    for (int k = 0; k < kD / 32; ++k) qv[k] = reinterpret_cast<const float4*>(qbar)[(lane & 7) + 8 * k];

    // ---- scan: score the warp's candidate units into a running top-kc list
    uint64_t l1[R1];
#pragma unroll
    for (int r = 0; r < R1; ++r) l1[r] = 0ull;
    consume(0, e_l2, e_l2, [&](int i, uint8_t* st) {
      if (i * NW + gw < n_su) {
        const int su = gw + i * NW;
        const float sc = score16(reinterpret_cast<const float*>(st), qv);
        const int r = su * kRows + lane;
        offer16<R1>(l1, lane < kRows && r < n_cand ? make_key(sc, p.sink + r) : 0ull, p.kc);
      }
    });
#pragma unroll
    for (int r = 0; r < R1; ++r)
      if (r * 32 + lane < p.kc) s_union[warp * p.kc + r * 32 + lane] = l1[r];
    if (PAGED) {  // this thread's block-table copies: landed; the entries the item reads, checked
      ptx::cp_async_wait_all();
      const int last = ok ? static_cast<int>(pb / a.kv.page_size) : -1;
      const bool wide = a.kv.max_pages % 4 == 0 && (reinterpret_cast<uintptr_t>(a.kv.block_table) & 15) == 0;
      const int step = wide ? 4 : 1;  // entries per copy of this thread
      for (int i0 = step * tid; i0 <= last; i0 += step * W * 32)
        for (int i = i0; i < i0 + step && i <= last; ++i) {
          const int pg = s_pages[i];
          if (pg < 0 || pg >= a.kv.n_pages) {
            flag_error(a.err, kErrPage);
            s_pages[i] = -1;
          }
        }
    }
    if (NC > 1)
      for (int c = tid; c < p.kc; c += W * 32) ckey[c] = 0ull;  // this CTA's slice top-kc
    named_sync(kBarStream, W * 32);  // B1

    // ---- level 1: the kc best of the W lists, by rank, into chunks (rank order);
    // in a cluster, each CTA's slice top-kc first, then rank 0 over the NC lists
    for (int c = tid; c < W * p.kc; c += W * 32) {
      const uint64_t key = s_union[c];
      if (key == 0ull) continue;
      const int rank = rank_among(s_union, W * p.kc, key);
      if (NC > 1) {
        if (rank < p.kc) ckey[rank] = key;
      } else if (rank < ns) {
        chunks[rank] = key_id(key);
        ckey[rank] = key;
      }
    }
    if (NC > 1) {
      named_sync(kBarStream, W * 32);
      const uint32_t dst = ptx::map_to_rank(ptx::smem_u32(&s_l1all[crank][0]), 0);
      for (int c = tid; c < p.kc; c += W * 32) ptx::st_cluster_u64(dst + 8u * c, ckey[c]);
      ptx::fence_cluster();
      named_sync(kBarStream, W * 32);
      if (tid == 0) ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(&s_l1bar), 0));
      if (crank == 0) {
        if (!ptx::mbar_wait_cluster(&s_l1bar, item_no & 1, kWaitLimit, limit_ns)) timed_out = true;
        for (int c = tid; c < NC * p.kc; c += W * 32) {
          const uint64_t key = s_l1all[c / p.kc][c % p.kc];
          if (key == 0ull) continue;
          int rank = 0;
          for (int r = 0; r < NC; ++r) rank += rank_among(s_l1all[r], p.kc, key);
          if (rank < ns) {
            chunks[rank] = key_id(key);
            ckey[rank] = key;
          }
        }
      }
    }
    named_sync(kBarStream, W * 32);  // B2

    WarpState ws;
    int attended = 0;
    // attends one landed K/V unit of stream position i (window units may end at the query)
    auto attend_fn = [&](int i, uint8_t* st) {
      const uint32_t kt = ptx::smem_u32(st);
      int valid = kUnit;
      if (i < e_rt && gw + (i - e_fw) * NW == n_forced - 1) valid = static_cast<int>(pb % kUnit) + 1;
      attend_unit(kt, kt + kTileBytes, valid, qa, scale, ws);
      ++attended;
    };
    if (NC == 1 || crank == 0) {
      // ---- level 2: this warp's chosen chunks' group rows (then its window units
      // queue behind them and land while the selection runs)
      issue_upto(e_rt);
      consume(e_l2, e_fw, e_rt, [&](int i, uint8_t* st) {
        const float sc = score16(reinterpret_cast<const float*>(st), qv);
        const int k0 = (i - e_l2) * cpu;
        const int rows = (min(n_mine, k0 + cpu) - k0) * p.Ng;
        if (lane < rows) {
          const int e = warp + (k0 + lane / p.Ng) * W;  // chosen chunk (rank order)
          const int g = lane % p.Ng;
          gkey[e * p.Ng + g] = make_key(sc, chunks[e] * p.Ng + g);
        }
      });
      named_sync(kBarStream, W * 32);  // B3
      // the kg best group keys, by rank, into glist (rank order)
      for (int j = tid; j < n_l2; j += W * 32) {
        const uint64_t key = gkey[j];
        const int rank = rank_among(gkey, n_l2, key);
        if (rank < ng) {
          glist[rank] = key_id(key);
          gsc[rank] = key_score(key);
        }
      }
      if (NC > 1 && timed_out) s_bad[item_no & 1] = 1;  // read after B4 by warp 0
      named_sync(kBarStream, W * 32);  // B4

      if (NC > 1 && warp == 0) {  // the routed list to the other CTAs of the cluster
        const bool bad = s_bad[item_no & 1] != 0;
        for (int r = 1; r < NC; ++r) {
          const uint32_t dst = ptx::map_to_rank(ptx::smem_u32(glist), r);
          for (int i = lane; i < ng; i += 32) ptx::st_cluster(dst + 4u * i, static_cast<uint32_t>(glist[i]));
          if (lane == 0)
            ptx::st_cluster(ptx::map_to_rank(ptx::smem_u32(&s_ng_in), r), static_cast<uint32_t>(bad ? 0 : ng));
        }
        ptx::fence_cluster();
        __syncwarp();
        if (lane == 0)
          for (int r = 1; r < NC; ++r) ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(&s_hand), r));
      }
      // ---- window and routed units
      ws.init();
      issue_upto(e_all);
      if (warp == 0) {  // outputs, ascending ids, while the units load
        int32_t* cidx = a.chunk_idx + static_cast<size_t>(item) * p.kc;
        float* cscore = a.chunk_score ? a.chunk_score + static_cast<size_t>(item) * p.kc : nullptr;
        for (int e = lane; e < p.kc; e += 32) {
          if (e < ns) {
            const int id = chunks[e];
            int at = 0;
            for (int f = 0; f < ns; ++f) at += chunks[f] < id;
            cidx[at] = id;
            if (cscore) cscore[at] = key_score(ckey[e]);
          } else {
            cidx[e] = -1;
            if (cscore) cscore[e] = CUDART_NAN_F;
          }
        }
        int32_t* gidx = a.group_idx + static_cast<size_t>(item) * p.kg;
        float* gscore = a.group_score ? a.group_score + static_cast<size_t>(item) * p.kg : nullptr;
        for (int e = lane; e < p.kg; e += 32) {
          if (e < ng) {
            const int id = glist[e];
            int at = 0;
            for (int f = 0; f < ng; ++f) at += glist[f] < id;
            gidx[at] = id;
            if (gscore) gscore[at] = gsc[e];
          } else {
            gidx[e] = -1;
            if (gscore) gscore[e] = CUDART_NAN_F;
          }
        }
      }
      consume(e_fw, e_all, e_all, attend_fn);
    } else {
      // ---- the cluster's other CTAs: their window units now, their routed units on arrival
      ws.init();
      issue_upto(e_rt);
      consume(e_fw, e_rt, e_rt, attend_fn);
      int ng_in = 0;
      if (ptx::mbar_wait_cluster(&s_hand, item_no & 1, kWaitLimit, limit_ns)) {
        ng_in = min(s_ng_in, p.kg);
      } else {
        timed_out = true;
      }
      e_all = e_rt + count(ng_in);
      issue_upto(e_all);
      consume(e_rt, e_all, e_all, attend_fn);
    }
    bool drained = true;
    if (timed_out) {
      // A wait gave up: the partial is dropped (the output is wrong and flagged),
      // the copies still in flight are waited for once more (bounded), and every
      // barrier below is still reached.  Later items of this CTA are skipped.
      if (lane == 0) {
        flag_error(a.err, kErrTimeout);
        if (NC == 1) s_abort = 1;
      }
      for (; done < issued; ++done) drained &= wait_stage(done);
      ws.m0 = ws.m1 = -CUDART_INF_F;
      ws.l0 = ws.l1 = 0.f;
    }

    // ---- merge the warps' partials through shared memory (each warp's stage 0)
    const int g = lane >> 2, t4 = lane & 3;
    ws.l0 += __shfl_xor_sync(0xffffffffu, ws.l0, 1);
    ws.l0 += __shfl_xor_sync(0xffffffffu, ws.l0, 2);
    ws.l1 += __shfl_xor_sync(0xffffffffu, ws.l1, 1);
    ws.l1 += __shfl_xor_sync(0xffffffffu, ws.l1, 2);
    float* wo = reinterpret_cast<float*>(ring);  // [16 heads][128]
    const bool write_o = drained && attended > 0;
    if (!write_o) {
      ws.m0 = ws.m1 = -CUDART_INF_F;
      ws.l0 = ws.l1 = 0.f;
    } else {
      // row hh, column c at hh * 128 + (c ^ ((hh & 7) << 3)): the eight rows a
      // store touches land in different banks
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int c = (j * 8 + 2 * t4) ^ (g << 3);
        *reinterpret_cast<float2*>(wo + g * kD + c) = make_float2(ws.o[j][0], ws.o[j][1]);
        *reinterpret_cast<float2*>(wo + (g + 8) * kD + c) = make_float2(ws.o[j][2], ws.o[j][3]);
      }
    }
    if (t4 == 0) {
      s_ml[warp][g][0] = ws.m0;
      s_ml[warp][g][1] = ws.l0;
      s_ml[warp][g + 8][0] = ws.m1;
      s_ml[warp][g + 8][1] = ws.l1;
    }
    named_sync(kBarStream, W * 32);
    if (NC > 1 && crank == 0 &&
        !ptx::mbar_wait_cluster(&s_peerbar, item_no & 1, kWaitLimit, limit_ns) && lane == 0)
      flag_error(a.err, kErrTimeout);  // a partial did not come: flagged
    // peer layout: o [NC][G][kD], then (m, l) [NC][G]
    const uint32_t peer0 = NC > 1 && crank > 0 ? ptx::map_to_rank(ptx::smem_u32(peer), 0) : 0u;
    for (int idx = tid; idx < p.G * kD; idx += W * 32) {
      const int hh = idx / kD, d = idx % kD;
      float mm = -CUDART_INF_F;
#pragma unroll
      for (int v = 0; v < W; ++v) mm = fmaxf(mm, s_ml[v][hh][0]);
      float ll = 0.f, oo = 0.f;
      if (mm != -CUDART_INF_F) {
#pragma unroll
        for (int v = 0; v < W; ++v) {
          const float mv = s_ml[v][hh][0];
          if (mv == -CUDART_INF_F) continue;
          const float f = exp2f(mv - mm);
          ll += s_ml[v][hh][1] * f;
          oo += reinterpret_cast<const float*>(base + static_cast<size_t>(v) * kS * kStageBytes)
                    [hh * kD + (d ^ ((hh & 7) << 3))] * f;
        }
      }
      if (NC > 1 && crank > 0) {  // this CTA's partial, to rank 0
        ptx::st_cluster(peer0 + 4u * ((crank * p.G + hh) * kD + d), __float_as_uint(oo));
        if (d == 0) {
          const uint32_t ml = peer0 + 4u * (NC * p.G * kD + 2 * (crank * p.G + hh));
          ptx::st_cluster(ml, __float_as_uint(mm));
          ptx::st_cluster(ml + 4u, __float_as_uint(ll));
        }
        continue;
      }
      for (int r = 1; r < NC; ++r) {  // rank 0: the other CTAs' partials, by log-sum-exp
        const float pm = peer[NC * p.G * kD + 2 * (r * p.G + hh)];
        const float pl = peer[NC * p.G * kD + 2 * (r * p.G + hh) + 1];
        const float po = peer[(r * p.G + hh) * kD + d];
        const float mx = fmaxf(mm, pm);
        if (mx != -CUDART_INF_F) {
          const float f0 = mm == -CUDART_INF_F ? 0.f : exp2f(mm - mx);
          const float f1 = pm == -CUDART_INF_F ? 0.f : exp2f(pm - mx);
          ll = ll * f0 + pl * f1;
          oo = oo * f0 + po * f1;
          mm = mx;
        }
      }
      const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + hh;
      store_out(a.out + row * kD + d, ll > 0.f ? oo / ll : 0.f);
      if (a.lse && d == 0) a.lse[row] = ll > 0.f ? (mm + log2f(ll)) * kLn2 : -CUDART_INF_F;
    }
    if (NC > 1 && crank > 0) {  // the partial is in rank 0's shared memory: say so
      ptx::fence_cluster();
      named_sync(kBarStream, W * 32);
      if (tid == 0) ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(&s_peerbar), 0));
    }
    if (NC > 1 && tid == 0) s_bad[(item_no + 1) & 1] = 0;  // the next item's flag, before its writes
    // the rings and the lists are reused by the next item (its copies are
    // ordered after this item's shared-memory writes)
    ptx::fence_proxy_async();
    named_sync(kBarStream, W * 32);
  }
  cta_sync();
  if (NC > 1) ptx::cluster_barrier();  // no CTA leaves while another may still write to it
  pdl_trigger();
}

// ------------------------------------------------------------------ launch

struct StepShape {
  int W;           // streaming warps per CTA (7: one CTA per SM; 3: two per SM), plus one append warp
  int R1;          // key registers per lane of the level-1 lists (top-kc <= 32 R1)
  int grid;
  int nc;          // CTAs per item (a cluster): small batches spread each item over nc SMs
};

size_t step_smem_bytes(const LayerParams& p, int W, int n_pt, int nc) {
  return StepSmem{W, summ::table_entries(p, kD), n_pt, nc > 1 ? nc * p.G * (kD + 2) : 0}.bytes();
}

// Dynamic shared memory a CTA may take: 225 KB with one CTA per SM, 112 KB with
// two, less the static slice lists that a cluster of nc CTAs adds (the CTA's
// whole shared memory stays within the 227 KB a block may have).
size_t step_smem_limit(int W, int nc) {
  return (W == 7 ? 225 * 1024 : 112 * 1024) - static_cast<size_t>(nc - 1) * kKcMax * 8;
}

// More items than SMs: three-warp CTAs, two per SM.  Up to one item per SM: one
// seven-warp CTA per SM, and when at most half the SMs would be busy, each item
// on a cluster of nc CTAs (the largest of 8, 4, 2 that keeps one CTA per SM and
// fits the shared memory of n_pt staged block-table entries).
StepShape step_shape(const LayerParams& p, int n_pt) {
  const int64_t items = static_cast<int64_t>(p.B) * p.Hkv;
  const int sms = device_sm_count();
  StepShape s;
  s.W = items <= sms ? 7 : 3;
  s.R1 = p.kc <= 32 ? 1 : 2;
  s.nc = 1;
  if (s.W == 7)
    for (int nc = 8; nc >= 2; nc /= 2)
      if (items * nc <= sms && step_smem_bytes(p, 7, n_pt, nc) <= step_smem_limit(7, nc)) {
        s.nc = nc;
        break;
      }
  const int64_t slots = static_cast<int64_t>(sms) * (s.W == 7 ? 1 : 2);
  s.grid = s.nc > 1 ? static_cast<int>(items * s.nc)
                    : static_cast<int>(items < slots ? items : slots);
  return s;
}

template <int W, int R1, typename TO, bool PAGED, int NC>
cudaError_t launch_t(const LayerParams& p, int grid, const CUtensorMap& tk, const CUtensorMap& tv,
                     const StepArgs<TO>& a, cudaStream_t s) {
  const size_t smem = step_smem_bytes(p, W, PAGED ? a.kv.max_pages : 0, NC);
  cudaError_t e = ensure_smem<decode_step_kernel<W, R1, TO, PAGED, NC>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_step_kernel<W, R1, TO, PAGED, NC>, dim3(grid), dim3((W + 1) * 32), smem,
                    s, NC, tk, tv, a, p);
}

template <int W, int R1, typename TO, bool PAGED>
cudaError_t launch_nc(const LayerParams& p, const StepShape& sh, const CUtensorMap& tk,
                      const CUtensorMap& tv, const StepArgs<TO>& a, cudaStream_t s) {
  switch (sh.nc) {
    case 8: return launch_t<W, R1, TO, PAGED, 8>(p, sh.grid, tk, tv, a, s);
    case 4: return launch_t<W, R1, TO, PAGED, 4>(p, sh.grid, tk, tv, a, s);
    case 2: return launch_t<W, R1, TO, PAGED, 2>(p, sh.grid, tk, tv, a, s);
    default: return launch_t<W, R1, TO, PAGED, 1>(p, sh.grid, tk, tv, a, s);
  }
}

template <typename TO, bool PAGED>
cudaError_t dispatch(const LayerParams& p, const StepShape& sh, const CUtensorMap& tk,
                     const CUtensorMap& tv, const StepArgs<TO>& a, cudaStream_t s) {
  if (sh.W == 7)
    return sh.R1 == 1 ? launch_nc<7, 1, TO, PAGED>(p, sh, tk, tv, a, s)
                      : launch_nc<7, 2, TO, PAGED>(p, sh, tk, tv, a, s);
  return sh.R1 == 1 ? launch_t<3, 1, TO, PAGED, 1>(p, sh.grid, tk, tv, a, s)
                    : launch_t<3, 2, TO, PAGED, 1>(p, sh.grid, tk, tv, a, s);
}

template <typename TO>
cudaError_t dispatch_kv(const LayerParams& p, const StepShape& sh, const CUtensorMap& tk,
                        const CUtensorMap& tv, const StepArgs<TO>& a, cudaStream_t s) {
  return a.kv.block_table ? dispatch<TO, true>(p, sh, tk, tv, a, s)
                          : dispatch<TO, false>(p, sh, tk, tv, a, s);
}

}  // namespace

bool decode_item_path(const LayerParams& p, int n_pt) {
  const StepShape sh = step_shape(p, n_pt);
  return p.kc <= kKcMax && p.kg <= kKgMax && p.Ng <= 8 && kRows % p.Ng == 0 &&
         step_smem_bytes(p, sh.W, n_pt, sh.nc) <= step_smem_limit(sh.W, sh.nc);
}

bool decode_step_path(const LayerParams& p, int dtype) {
  return decode_fast_path(p, dtype) &&
         static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc < (static_cast<int64_t>(1) << 31);
}

cudaError_t launch_decode_step(const LayerParams& p, int out_dtype, const void* q,
                               const int64_t* pos, float* chunk_sum, float* group_sum,
                               const void* k, const void* v, int32_t* chunk_idx,
                               float* chunk_score, int32_t* group_idx, float* group_score,
                               void* out, float* lse, int append, unsigned* err, cudaStream_t s,
                               const KvPages& kv) {
  const bool paged = kv.block_table != nullptr;
  if (!decode_item_path(p, paged ? kv.max_pages : 0)) {
    // the summary append, the routing kernel, then the attention kernel (dense
    // caches only: the caller checks that a paged step fits the one launch)
    if (paged) return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (append) e = launch_append_per_sequence(p, 1, k, pos, chunk_sum, group_sum, s);
    if (e == cudaSuccess)
      e = launch_route(p, 1, q, pos, chunk_sum, group_sum, chunk_idx, chunk_score, group_idx,
                       group_score, err, s);
    if (e != cudaSuccess) return e;
    return launch_attend_decode_bf16(p, out_dtype, q, pos, k, v, group_idx, out, lse, err, 0, s);
  }
  CUtensorMap tk, tv;
  const int64_t all_rows = paged ? kv.n_pages * p.Hkv * kv.page_size
                                 : static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc;
  cudaError_t e = make_bf16_map(&tk, k, all_rows, kUnit);
  if (e == cudaSuccess) e = make_bf16_map(&tv, v, all_rows, kUnit);
  if (e != cudaSuccess) return e;
  const StepShape sh = step_shape(p, paged ? kv.max_pages : 0);
  const int n_items = p.B * p.Hkv;
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
  if (out_dtype == 0) {
    StepArgs<float> a{qb, pos, kb, static_cast<const __nv_bfloat16*>(v), chunk_sum, group_sum, chunk_idx, chunk_score, group_idx,
                      group_score, static_cast<float*>(out), lse, err, append, n_items, kv};
    return dispatch_kv<float>(p, sh, tk, tv, a, s);
  }
  StepArgs<__nv_bfloat16> a{qb, pos, kb, static_cast<const __nv_bfloat16*>(v), chunk_sum, group_sum, chunk_idx, chunk_score, group_idx,
                            group_score, static_cast<__nv_bfloat16*>(out), lse, err, append,
                            n_items, kv};
  return dispatch_kv<__nv_bfloat16>(p, sh, tk, tv, a, s);
}

}  // namespace hga
