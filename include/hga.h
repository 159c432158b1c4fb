/*
 * hga.h - C ABI of the Hierarchical Global Attention (HGA) hot path on B200.
 *
 * HGA replaces dense causal attention over a long K/V cache without touching
 * the model's weights (technical summary of "Hierarchical Global Attention
 * (HGA)", gist.science paper 2606.30709, section "Metodologia", and "Contributi
 * Chiave" item 1: drop-in compatibility).  One layer's decode or prefill step
 * is four calls, in this order:
 *
 *   hga_build_summaries  RoPE-aware chunk and group key summaries
 *   hga_route_chunks     level-1 routing against the chunk-summary table
 *   hga_route_groups     level-2 routing inside the selected chunks
 *   hga_attend           exact softmax over the routed tokens' original K/V
 *
 * Conventions shared by every call
 *  - Plain pointers and sizes only.  Device pointers are CUDA device memory of
 *    the current device; the caller owns and frees every buffer.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  They validate what they can on the
 *    host and return a status; they never abort the process.
 *  - Conditions only the device can see (a position out of range, an index
 *    set that breaks its contract) set a sticky device error word, read and
 *    cleared by hga_device_status().  The offending work item writes -1
 *    indices / zero outputs instead of faulting.
 *  - Layouts are row-major and contiguous:
 *      q      [B, Hq, q_len, D]   post-RoPE queries (dtype)
 *      k, v   [B, Hkv, n_alloc, D] post-RoPE key cache and value cache (dtype);
 *             token t sits at row t and at RoPE position t
 *      chunk_sum [B, Hkv, n_alloc/C, D]          float32
 *      group_sum [B, Hkv, n_alloc/C, C/g, D]     float32
 *      chunk_idx [B, Hkv, nblk, kc] int32, group_idx [B, Hkv, nblk, kg] int32
 *      out    [B, Hq, q_len, D] (out_dtype), lse [B, Hq, q_len] float32
 *    Query head hq reads KV head hq / (Hq/Hkv).
 *  - Query blocks.  The queries of sequence b sit at positions
 *    pos[b]-q_len+1 .. pos[b].  Decode is q_len == 1 (one block).  Prefill
 *    takes q_len a multiple of C with pos[b]+1 a multiple of C; every chunk of
 *    C queries is one routing block (nblk = q_len / C).
 *  - pos is a DEVICE array int64[B] so that a decode loop can advance it on
 *    the GPU; 0 <= pos[b] < n_alloc and pos[b] >= q_len-1 is checked on the
 *    device.
 *  - All sequences share n_alloc (the cache capacity in tokens, a multiple of
 *    C).
 */
#ifndef HGA_H_
#define HGA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HGA_ABI_VERSION 6

typedef enum hga_status {
  HGA_OK = 0,
  HGA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum */
  HGA_ERR_SHAPE = 2,         /* inconsistent sizes (Hq % Hkv, n_alloc % C, ...) */
  HGA_ERR_UNSUPPORTED = 3,   /* valid but not built: head_dim, chunk, group, k limits */
  HGA_ERR_CUDA = 4,          /* a CUDA runtime call failed; see hga_last_error() */
  HGA_ERR_TIMEOUT = 5,       /* a bounded wait ran out */
  HGA_ERR_DEVICE_CHECK = 6,  /* a device-side argument check failed */
  HGA_ERR_WORKSPACE = 7      /* workspace missing or smaller than hga_workspace_size() */
} hga_status;

typedef enum hga_dtype { HGA_F32 = 0, HGA_BF16 = 1 } hga_dtype;

typedef enum hga_kv_loc { HGA_KV_DEVICE = 0, HGA_KV_HOST_PINNED = 1 } hga_kv_loc;

/* Layer shape and method parameters.  Field names follow the pages' notation. */
typedef struct hga_config {
  int32_t batch;          /* B */
  int32_t heads_q;        /* Hq */
  int32_t heads_kv;       /* Hkv; G = Hq / Hkv query heads share one KV head (1..16) */
  int32_t head_dim;       /* D: 64 or 128 */
  int32_t chunk;          /* C: fixed chunk size, 64 or 128 */
  int32_t group;          /* g: tokens per group inside a chunk; 16 */
  int32_t sink_chunks;    /* initial chunks that are always visible (>= 0) */
  int32_t local_chunks;   /* recent chunks before the current one that are always visible (>= 0) */
  int32_t topk_chunks;    /* kc: level-1 top-k, 1..256 */
  int32_t topk_groups;    /* kg: level-2 top-k, 1..1024 */
  int32_t n_high_pairs;   /* RoPE pairs i < n_high_pairs are "high frequency" (0..D/2) */
  int32_t dtype;          /* hga_dtype of q, k, v */
  int32_t out_dtype;      /* hga_dtype of out */
  int32_t kv_loc;         /* hga_kv_loc of k and v (HGA_KV_DEVICE for the calls below) */
  double rope_theta;      /* RoPE base: omega_i = rope_theta^(-2i/D) */
} hga_config;

/*
 * A paged K/V pool (hga_build_summaries_paged, hga_decode_step_paged), the
 * block-table layout of serving engines: k and v are pools
 * [n_pages, Hkv, page_size, D] (page-major, then KV head: one (page, head) is
 * page_size contiguous rows), and token t of sequence b lives at row
 * t % page_size of page block_table[b * max_pages + t / page_size].  Entries
 * past a sequence's last token are never read (they may be -1).  Summary
 * tables stay dense per sequence, with max_pages * page_size rows of capacity.
 */
typedef struct hga_kv_pages {
  const int32_t* block_table; /* device int32 [B, max_pages] */
  int64_t n_pages;            /* pages in each of the k and v pools */
  int32_t page_size;          /* tokens per page: a positive multiple of 16 */
  int32_t max_pages;          /* block-table entries per sequence */
} hga_kv_pages;

/* Version of this ABI (HGA_ABI_VERSION of the built library). */
int32_t hga_abi_version(void);

/* Human-readable name of a status. Never NULL. */
const char* hga_status_string(hga_status status);

/* Detail message of the last failing call on this host thread ("" if none). */
const char* hga_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device: HGA_ERR_TIMEOUT if a kernel of this library gave up a bounded
 * wait since the last call, else HGA_ERR_DEVICE_CHECK if a device-side argument
 * check failed, HGA_OK otherwise (HGA_ERR_CUDA if the sync failed).  Every wait
 * inside the kernels is bounded (a poll count and 50 ms), so a kernel always
 * returns; the work item that gave up writes an empty result.
 */
hga_status hga_device_status(void* stream);

/*
 * Test hook, not for production use: sets the debug flags that every later
 * launch of this process copies (returns the previous flags; 0 = none).  Flag 1
 * makes the one-launch kernel of hga_decode_step skip one warp's group-summary
 * copy for the first item of each CTA while the warp still waits for it, so that
 * bounded wait (nothing is in flight into that stage; limited to 2 ms under this
 * flag) runs out; the kernel still reaches every barrier and returns, and
 * hga_device_status() then reports HGA_ERR_TIMEOUT.
 */
int32_t hga_debug_inject(int32_t flags);

/*
 * Bytes of device workspace hga_attend needs for (cfg, n_alloc, q_len).  Zero
 * is a valid answer (bf16 decode with D = 128 merges its split-K partials inside
 * a thread-block cluster and needs none).  Otherwise the workspace holds the
 * per-split partial results of the split-K decode; its contents need no
 * initialisation and are scratch.
 */
hga_status hga_workspace_size(const hga_config* cfg, int64_t n_alloc, int32_t q_len,
                              size_t* bytes);

/*
 * Step 1 - RoPE-aware key summaries (HGA technical summary, "Metodologia ->
 * Meccanismo Core", item 1 partitioning and item 3 RoPE-aware summaries).
 *
 * For every chunk (C tokens) and every group (g tokens) whose LAST token lies
 * in [t_begin, t_end), computes its summary row from the keys in k and stores
 * it; rows whose last token is outside that range are left untouched, so a
 * whole cache is summarised with (0, n) and a decode step appending token p
 * calls (p, p+1) (a no-op unless p closes a group).  Each row is computed from
 * the cache alone, the same way whatever the call pattern, so appending token
 * by token gives bit-identical rows to one batch call.
 *
 * Summary of the span t0..t0+L-1 with centre r = t0 + (L-1)/2:
 *   high-frequency pairs (i < n_high_pairs): mean of the stored (rotated) keys;
 *   low-frequency pairs: mean of the raw keys R(-t) k[t], rotated to r;
 *   equivalently mean over t of R(r - t) k[t] on those pairs.
 *
 *   k          device, [B, Hkv, n_alloc, D] of cfg->dtype, post-RoPE keys
 *   n_alloc    cache capacity in tokens (multiple of C)
 *   t_begin, t_end   0 <= t_begin <= t_end <= n_alloc (same for every sequence)
 *   chunk_sum  device float32 [B, Hkv, n_alloc/C, D] (written rows only)
 *   group_sum  device float32 [B, Hkv, n_alloc/C, C/g, D] (written rows only)
 * Errors: INVALID_ARG / SHAPE / UNSUPPORTED for bad arguments, CUDA on launch
 * failure.  No workspace.
 */
hga_status hga_build_summaries(const hga_config* cfg, const void* k, int64_t n_alloc,
                               int64_t t_begin, int64_t t_end, float* chunk_sum,
                               float* group_sum, void* stream);

/*
 * Step 2 - level-1 chunk routing with deterministic visibility (HGA technical
 * summary, "Metodologia -> Meccanismo Core", item 2: "Livello 1 (Chunk
 * Routing)" and "Visibilita Deterministica"; "Contributi Chiave" item 3).
 *
 * For each (sequence b, KV head h, query block): the routing query is the mean
 * of the block's post-RoPE query vectors over the G query heads of h.  With
 * cur = the chunk of the block's last query, the candidates are the chunks j
 * with sink_chunks <= j < cur - local_chunks (the always-visible sink, local
 * and current chunks are not candidates: they are attended in full).  Each
 * candidate is scored by the dot product of the routing query with its chunk
 * summary; the kc best are kept (equal scores: lower chunk index first) and
 * written in ascending order, padded with -1.
 *
 *   q          device [B, Hq, q_len, D] (cfg->dtype)
 *   pos        device int64 [B], position of each sequence's last query
 *   chunk_sum  device float32 [B, Hkv, n_alloc/C, D]; candidate rows complete
 *   chunk_idx  device int32 [B, Hkv, nblk, kc] (output)
 *   chunk_score optional device float32 [B, Hkv, nblk, kc]: the selected
 *              chunks' scores (NaN on padding); may be NULL
 * Limits: n_alloc / C <= 32768.  No workspace.
 */
hga_status hga_route_chunks(const hga_config* cfg, const void* q, int32_t q_len,
                            const int64_t* pos, const float* chunk_sum, int64_t n_alloc,
                            int32_t* chunk_idx, float* chunk_score, void* stream);

/*
 * Step 3 - level-2 group routing inside the selected chunks (HGA technical
 * summary, "Metodologia -> Meccanismo Core", item 2: "Livello 2 (Group
 * Routing)").
 *
 * Scores every group of every selected chunk (skipping -1 entries) against
 * the same routing query as step 2 and keeps the kg best over all of them
 * (equal scores: lower global group id first).  A group is named by its global
 * id chunk * (C/g) + group-in-chunk; ids are written ascending, padded with -1.
 *
 *   chunk_idx  device int32 [B, Hkv, nblk, kc], ascending, as step 2 writes it;
 *              every entry must be a complete candidate chunk (checked on the
 *              device)
 *   group_sum  device float32 [B, Hkv, n_alloc/C, C/g, D]
 *   group_idx  device int32 [B, Hkv, nblk, kg] (output)
 *   group_score optional device float32 [B, Hkv, nblk, kg]; may be NULL
 * Limits: kc * C/g <= 8192.  No workspace.
 */
hga_status hga_route_groups(const hga_config* cfg, const void* q, int32_t q_len,
                            const int64_t* pos, const float* group_sum, int64_t n_alloc,
                            const int32_t* chunk_idx, int32_t* group_idx, float* group_score,
                            void* stream);

/*
 * Steps 2 and 3 in one launch (same passages as hga_route_chunks and
 * hga_route_groups).  Writes exactly what hga_route_chunks followed by
 * hga_route_groups writes - bit for bit - with the level-2 stage continuing
 * inside the level-1 kernel, so a decode step pays one launch for routing.
 * chunk_score and group_score may be NULL.
 */
hga_status hga_route(const hga_config* cfg, const void* q, int32_t q_len, const int64_t* pos,
                     const float* chunk_sum, const float* group_sum, int64_t n_alloc,
                     int32_t* chunk_idx, float* chunk_score, int32_t* group_idx,
                     float* group_score, void* stream);

/*
 * Host tier (HGA technical summary, "Architettura della Memoria": the hot tier
 * in VRAM holds the chunk summaries and the always-visible windows, the cold
 * tier in host RAM holds the whole K/V history; "Meccanismo Core", item 4: the
 * selected groups' original K/V are fetched from host RAM into VRAM for the
 * exact attention).
 *
 * With cfg->kv_loc == HGA_KV_HOST_PINNED the K/V cache [B, Hkv, n_alloc, D]
 * lives in pinned, device-mapped host memory.  The GPU keeps per (sequence, KV
 * head) a working buffer of hga_hot_rows() rows of D elements:
 *   [sink chunks | ring of local+1 chunks, chunk c at slot c mod (local+1) |
 *    kg routed groups, slot j holding entry j of group_idx]
 * Built for bf16, head_dim 128 decode.  hga_build_summaries accepts the host
 * cache as k (it reads it over the host link); hga_route* need no K/V.
 */
hga_status hga_hot_rows(const hga_config* cfg, int64_t* rows);

/*
 * Fills the working buffers for one decode step at pos (host tier): copies from
 * the pinned host cache the routed groups of group_idx (as hga_route_groups
 * or hga_route wrote it; the same groups hga_attend keeps) and window rows,
 * by refresh_window:
 *   0  the current chunk's rows up to pos (a decode loop that calls this at
 *      every consecutive position keeps the whole window current);
 *   1  those and the sink and local chunks (after a prefill, or after
 *      positions are skipped);
 *   2  the row at pos only: valid when the previous call for every sequence
 *      was at pos - 1 (a consecutive decode loop after one call with 1).
 * Any other value is HGA_ERR_INVALID_ARG.  The copy is a
 * kernel reading host memory directly (zero-copy 16-byte loads over the host
 * link); nothing is allocated.
 *   k_host, v_host  pinned host [B, Hkv, n_alloc, 128] bf16
 *   k_work, v_work  device [B, Hkv, hga_hot_rows(), 128] bf16 (caller-owned)
 */
hga_status hga_gather_host(const hga_config* cfg, const void* k_host, const void* v_host,
                           int64_t n_alloc, const int64_t* pos, const int32_t* group_idx,
                           void* k_work, void* v_work, int32_t refresh_window, void* stream);

/*
 * Warm tier (HGA technical summary, "Architettura della Memoria": a bounded
 * LRU cache in VRAM of recently routed spans, between the VRAM hot tier and
 * the host RAM history).  The cached unit is a routed group.  Per (sequence,
 * KV head) the working buffer's routed region holds warm_groups group slots
 * (topk_groups <= warm_groups <= 2048), described by a table in device memory:
 *   tags    int32 [B, Hkv, warm_groups]: group id held by each slot, -1 empty
 *   stamps  int32 [B, Hkv, warm_groups]: decode step of last use, 0 empty
 * A step's requests are the groups hga_attend keeps from group_idx (valid,
 * in a candidate chunk, strictly ascending).  The step clock of a (sequence,
 * KV head) is one more than its largest stamp; hits take it as stamp; the
 * misses, ascending, replace empty slots (by slot index) first, then the
 * least recently used (stamp, then group id, ascending), never a slot hit in
 * the same step.  A cached group's rows are copies of the host cache: when a
 * sequence's history changes (a new sequence in that batch slot, positions
 * moving backwards, K/V rewritten), reset its table.
 *
 * Rows per (sequence, KV head) of the warm working buffers:
 *   [sink chunks | ring of local+1 chunks | warm_groups cached groups].
 */
hga_status hga_warm_rows(const hga_config* cfg, int32_t warm_groups, int64_t* rows);

/*
 * Empties the warm tables of sequence seq (seq == -1: every sequence):
 * tags = -1, stamps = 0, with two memsets on stream.  Call once before the
 * first hga_gather_warm and whenever a sequence's history changes.
 */
hga_status hga_warm_reset(const hga_config* cfg, int32_t warm_groups, int32_t* tags,
                          int32_t* stamps, int32_t seq, void* stream);

/*
 * One decode step of the warm tier: for every (sequence, KV head), one CTA
 * looks its routed groups up in the table, assigns the misses their slots,
 * writes the table and slot_map, and copies from the pinned host cache only
 * the missed groups' rows, plus the window rows that refresh_window (0, 1 or
 * 2) names, as hga_gather_host does.
 *   k_host, v_host  pinned host [B, Hkv, n_alloc, 128] bf16
 *   group_idx       device int32 [B, Hkv, topk_groups] from the routing
 *   tags, stamps    the table above (read and written)
 *   slot_map        device int32 [B, Hkv, topk_groups], written: the slot of
 *                   every group_idx entry, -1 where the entry is not kept
 *   k_work, v_work  device [B, Hkv, hga_warm_rows(), 128] bf16; cached slots
 *                   keep their rows from step to step
 *   counters        optional device uint64 [2]: hits and misses added
 * Nothing is allocated.  Built for bf16, head_dim 128 decode.
 */
hga_status hga_gather_warm(const hga_config* cfg, const void* k_host, const void* v_host,
                           int64_t n_alloc, const int64_t* pos, const int32_t* group_idx,
                           int32_t warm_groups, int32_t* tags, int32_t* stamps, int32_t* slot_map,
                           void* k_work, void* v_work, int32_t refresh_window, uint64_t* counters,
                           void* stream);

/*
 * The exact attention of hga_attend (decode) over the warm working buffers:
 * routed entry j of group_idx is read from cached slot slot_map[j] (as
 * hga_gather_warm wrote it for the same group_idx).  Same units in the same
 * order as the device-resident and host-tier paths, so the same bits.  A kept
 * entry whose slot is outside [0, warm_groups) reads slot 0 and is flagged
 * (HGA_ERR_DEVICE_CHECK from hga_device_status).
 *   out  device [B, Hq, 1, 128] of cfg->out_dtype;  lse optional float32 [B, Hq, 1]
 */
hga_status hga_attend_warm(const hga_config* cfg, const void* q, const int64_t* pos,
                           const void* k_work, const void* v_work, int64_t n_alloc,
                           const int32_t* group_idx, const int32_t* slot_map, int32_t warm_groups,
                           void* out, float* lse, void* stream);

/*
 * Steps 4-5 - gather of the selected tokens' original K/V and exact softmax
 * attention over that bounded set (HGA technical summary, "Metodologia ->
 * Meccanismo Core", item 4 "Attenzione Esatta per Token"; "Contributi Chiave"
 * item 2: only retrieval is approximated, never the attention output).
 *
 * Each query at position p attends, with scale 1/sqrt(D), to: every token of
 * the sink chunks and of the local chunks, the tokens <= p of its own chunk,
 * and the g tokens of every group in its block's group_idx row.  No summary
 * value enters the output.
 *
 *   k, v       device [B, Hkv, n_alloc, D] (cfg->dtype); with kv_loc ==
 *              HGA_KV_HOST_PINNED, the device working buffers filled by
 *              hga_gather_host (decode only)
 *   group_idx  device int32 [B, Hkv, nblk, kg] from step 3; entries must be
 *              groups of candidate chunks (checked on the device; a bad entry
 *              is skipped and flagged)
 *   out        device [B, Hq, q_len, D] of cfg->out_dtype
 *   lse        optional device float32 [B, Hq, q_len]: natural-log
 *              log-sum-exp of the scaled scores; may be NULL
 *   workspace  device scratch of at least hga_workspace_size() bytes
 *              (may be NULL when that size is 0)
 */
hga_status hga_attend(const hga_config* cfg, const void* q, int32_t q_len, const int64_t* pos,
                      const void* k, const void* v, int64_t n_alloc, const int32_t* group_idx,
                      void* out, float* lse, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * One whole decode step: the summary append (HGA technical summary,
 * "Metodologia -> Meccanismo Core", item 3), level-1 and level-2 routing (item
 * 2), then the gather and exact attention of the chosen tokens (item 4).  It
 * writes what hga_build_summaries (per sequence, for the rows token pos[b]
 * closes), hga_route and hga_attend write: the summary rows bit for bit,
 * chunk_idx, group_idx and the scores bit for bit, out and lse up to the bf16
 * rounding of the softmax weights (the units are attended in another
 * grouping).
 *
 * With append != 0, for every sequence b the summary rows whose last token is
 * pos[b] (the group pos[b] ends, and its chunk when pos[b] ends that too) are
 * computed from k and stored in chunk_sum / group_sum; those rows belong to
 * the current chunk, which the step attends in full and never routes.  With
 * append == 0 the tables are only read.
 *
 * With topk_chunks <= 64 and topk_groups <= 128 the step is one launch: each
 * CTA works through (sequence, KV head) items, one at a time (one CTA per SM up
 * to one item per SM, two per SM above; when at most half the SMs would be
 * busy, each item is spread over a cluster of 2, 4 or 8 CTAs that scan slices
 * of the candidates, gather their selections in the first CTA and merge their
 * partials there); its warps stream the candidate chunk
 * summaries and the K/V of the always-visible chunks through shared-memory
 * rings, select the chunks and then the groups between barriers, attend the
 * routed groups and merge their partials, while another warp does the summary
 * append.  Wider routing gets the append, routing and attention kernels,
 * launched by this call (hga_decode_step_launches says which).  Decode only
 * (q_len is 1): bf16 K/V in device memory (kv_loc HGA_KV_DEVICE), head_dim 128,
 * group 16, at most 16 query heads per KV head, topk_groups <= 1024; other
 * shapes return HGA_ERR_UNSUPPORTED (use hga_route + hga_attend).  Arguments and layouts are those of hga_build_summaries,
 * hga_route and hga_attend; chunk_score, group_score and lse may be NULL.  No
 * workspace.
 */
hga_status hga_decode_step(const hga_config* cfg, const void* q, const int64_t* pos,
                           float* chunk_sum, float* group_sum, int64_t n_alloc, const void* k,
                           const void* v, int32_t* chunk_idx, float* chunk_score,
                           int32_t* group_idx, float* group_score, void* out, float* lse,
                           int32_t append, void* stream);

/*
 * How many kernel launches hga_decode_step makes for (cfg, n_alloc) on the
 * current device: 1 when it runs the one-launch kernel (routing and attention
 * of every (sequence, KV head) item in one grid), 2 when it launches the
 * routing kernel and then the attention kernel.  A pure host query (it reads
 * the device's SM count); no launch.  Returns HGA_ERR_UNSUPPORTED for shapes
 * hga_decode_step does not take.
 */
hga_status hga_decode_step_launches(const hga_config* cfg, int64_t n_alloc, int32_t* launches);

/*
 * Cold tier (HGA technical summary, "Architettura della Memoria": the whole K/V
 * history may live in host RAM or on NVMe; VRAM holds the summaries, the
 * windows and the warm LRU of routed groups).  The history lives in a file, K
 * then V, each [B, Hkv, n_alloc, 128] bf16 rows; a decode step with a cold
 * store runs
 *   hga_route -> hga_warm_plan -> (plan and counts to the host) ->
 *   hga_cold_stage -> hga_warm_fill -> hga_attend_warm,
 * so that only the warm tier's misses and the window rows are read from the
 * file, by a pool of host threads, into pinned staging the fill kernel reads
 * in place.  Staging per (sequence, KV head): [K | V][kg][16][128] of the
 * misses in plan order, then [K | V][(sink + local + 1) * C][128] of the
 * window rows (hga_cold_stage_bytes gives the whole size).
 */
typedef struct hga_cold_store hga_cold_store;

/* Opens the history file at path (create != 0: created, or grown, to
 * 2 * B * Hkv * n_alloc * 256 bytes).  A file shorter than that without create
 * is HGA_ERR_INVALID_ARG.  Close with hga_cold_close. */
hga_status hga_cold_open(const char* path, const hga_config* cfg, int64_t n_alloc,
                         int32_t create, hga_cold_store** store);
hga_status hga_cold_close(hga_cold_store* store);

/* Writes rows [t0, t1) of every (sequence, KV head) from host k, v
 * [B, Hkv, n_alloc, 128] bf16 (after a prefill; each decode step's new row
 * before that step), with up to `threads` host threads.  Synchronous. */
hga_status hga_cold_write(hga_cold_store* store, const void* k, const void* v, int64_t t0,
                          int64_t t1, int32_t threads);

/* Bytes of staging for one step of cfg's batch. */
hga_status hga_cold_stage_bytes(const hga_config* cfg, size_t* bytes);

/* The decision half of hga_gather_warm: the same table update and slot_map,
 * and per (sequence, KV head) its misses as (group, slot) int32 pairs in plan
 * [B, Hkv, kg, 2] with their count in n_plan [B, Hkv] (device); no row is
 * copied. */
hga_status hga_warm_plan(const hga_config* cfg, int64_t n_alloc, const int64_t* pos,
                         const int32_t* group_idx, int32_t warm_groups, int32_t* tags,
                         int32_t* stamps, int32_t* slot_map, int32_t* plan, int32_t* n_plan,
                         uint64_t* counters, void* stream);

/* Reads a step's rows from the file into staging (host memory, pinned for
 * hga_warm_fill): the missed groups of plan / n_plan (host copies of
 * hga_warm_plan's outputs) and the window rows of pos (host [B]) under
 * window_mode (0, 1, 2 as in hga_gather_host).  Synchronous, `threads` host
 * threads.  A group or position outside the history is HGA_ERR_INVALID_ARG. */
hga_status hga_cold_stage(hga_cold_store* store, const hga_config* cfg, const int64_t* pos,
                          const int32_t* plan, const int32_t* n_plan, int32_t window_mode,
                          void* staging, int32_t threads);

/* Copies the staged rows into the warm working buffers: the misses into the
 * slots plan names, the window rows into the window (device pos, plan and
 * n_plan; staging pinned host memory read in place over the host link). */
hga_status hga_warm_fill(const hga_config* cfg, int64_t n_alloc, const int64_t* pos,
                         const void* staging, const int32_t* plan, const int32_t* n_plan,
                         int32_t warm_groups, int32_t window_mode, void* k_work, void* v_work,
                         void* stream);

/*
 * Backward pass of a prefill call of hga_attend (HGA technical summary,
 * "Risultati Sperimentali": the method is trained and fine-tuned end to end;
 * "Metodologia -> Meccanismo Core", item 4: the output is an exact softmax
 * attention over the selected tokens).  The routing is a selection, so no
 * gradient flows through it or through the summaries: with the forward's token
 * sets held fixed (forced chunks, the block's own chunk causally, and the kept
 * groups of group_idx), for P = exp(S - lse), S = Q K^T / sqrt(D) and
 * Delta = rowsum(dO * O):
 *   dV = P^T dO,  dS = P * (dO V^T - Delta),  dQ = dS K / sqrt(D),
 *   dK = dS^T Q / sqrt(D),
 * accumulated over the G query heads of each KV head and every query row.
 *   q, d_out   device bf16 [B, Hq, q_len, 128]; q_len whole aligned chunks
 *              ending at pos[b] (as the forward)
 *   k, v       device bf16 [B, Hkv, n_alloc, 128]
 *   group_idx  the forward's routing, device int32 [B, Hkv, q_len / C, kg]
 *   out, lse   the forward's output (cfg->out_dtype) and natural-log LSE
 *   dq         device float32 [B, Hq, q_len, 128] (written)
 *   dk, dv     device float32 [B, Hkv, n_alloc, 128] (every row written; rows
 *              no query sees are zero)
 *   workspace  device scratch of hga_attend_backward_workspace_size() bytes
 * The sums run in a fixed order (no atomics): the result does not depend on
 * scheduling.  Built for bf16, head_dim 128, group 16, G <= 16,
 * topk_groups <= 128.
 */
hga_status hga_attend_backward_workspace_size(const hga_config* cfg, int64_t n_alloc,
                                              int32_t q_len, size_t* bytes);
hga_status hga_attend_backward(const hga_config* cfg, const void* q, int32_t q_len,
                               const int64_t* pos, const void* k, const void* v, int64_t n_alloc,
                               const int32_t* group_idx, const void* out, const float* lse,
                               const void* d_out, float* dq, float* dk, float* dv,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Ragged serving batch over a paged pool: hga_build_summaries for every
 * sequence b over its own tokens [0, seq_len[b]) (device int64 [B]), reading
 * k_pages through kv->block_table.  chunk_sum / group_sum are dense per
 * sequence, [B, Hkv, n_alloc / C, D] and [B, Hkv, n_alloc / C, C / g, D] with
 * n_alloc = kv->max_pages * kv->page_size (a multiple of C).  A block-table
 * entry the build needs that is not a page of the pool ([0, n_pages)) skips
 * its group (and chunk) and sets the device error word
 * (HGA_ERR_DEVICE_CHECK from hga_device_status).
 */
hga_status hga_build_summaries_paged(const hga_config* cfg, const void* k_pages,
                                     const hga_kv_pages* kv, const int64_t* seq_len,
                                     float* chunk_sum, float* group_sum, void* stream);

/*
 * hga_decode_step over a paged pool: the same routing and scores, bit for bit,
 * as hga_decode_step on a dense cache holding the same rows (per-sequence
 * positions pos[b] < n_alloc = kv->max_pages * kv->page_size; the summary
 * append reads the closed group's rows through the block table), and the same
 * output bits when both split the work alike.  (For a batch of at most half as
 * many items as SMs, a long block-table row can leave room for fewer CTAs per
 * item than the dense step takes; the output then differs by the bf16
 * rounding of the attention weights, a few 1e-5.)  One launch
 * of the decode-step kernel, which stages each sequence's block-table row in
 * shared memory; shapes it cannot take (hga_decode_step_launches would say 2,
 * or the block-table row does not fit beside the kernel's buffers) return
 * HGA_ERR_UNSUPPORTED.  An entry a step needs that is not a page of the pool
 * sets the device error word; its tiles read as zeros (never outside the pool).
 *   k_pages, v_pages  device bf16 pools [n_pages, Hkv, page_size, 128]
 */
hga_status hga_decode_step_paged(const hga_config* cfg, const void* q, const int64_t* pos,
                                 float* chunk_sum, float* group_sum, const void* k_pages,
                                 const void* v_pages, const hga_kv_pages* kv, int32_t* chunk_idx,
                                 float* chunk_score, int32_t* group_idx, float* group_score,
                                 void* out, float* lse, int32_t append, void* stream);

/*
 * hga_attend for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is a deployment convenience of this library.
 *
 * Some callers cannot provide the workspace hga_attend needs: frameworks that
 * own all device memory through their own pool and give an attention plugin
 * only its input and output buffers, and latency-critical loops where a
 * cudaMalloc / cudaFree (which may synchronise the device) is not allowed.
 * This call computes exactly what hga_attend computes, with the same
 * arguments minus the workspace: its split-K scratch lives in one fixed 8 MiB
 * array inside the library (present on every GPU that loads the library, until
 * the process exits).  It calls no allocator.
 *
 *  - Shapes whose hga_workspace_size() exceeds 8 MiB are rejected with
 *    HGA_ERR_WORKSPACE (use hga_attend with a caller workspace instead).
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - All calls on a device share the array, which keeps the last call's
 *    contents (nothing in it has to start at zero).  Calls whose kernels
 *    overlap on the GPU (other streams, other host threads) race on it and
 *    produce wrong results: serialise them.
 */
hga_status hga_attend_noalloc(const hga_config* cfg, const void* q, int32_t q_len,
                              const int64_t* pos, const void* k, const void* v, int64_t n_alloc,
                              const int32_t* group_idx, void* out, float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HGA_H_ */
