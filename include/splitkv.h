/*
 * splitkv.h -- C ABI of the Split-KV block-sparse anchor attention library
 * (libsplitkv.so, NVIDIA B200 / sm_100a).
 *
 * The method ("Split-KV: Efficient Context Parallelism for Training Diffusion
 * Drafters", paper digest page, Abstract; news page "Split-KV speeds diffusion
 * drafter training by keeping long-context data local"):
 *
 *   - anchors sampled from a packed context open blocks of block_size draft
 *     query tokens; block b attends to the preceding context of its own sample,
 *     keys [S_s, a_b), plus the block_size keys of its own block (news page,
 *     "Why short queries change the problem");
 *   - the context is cut into KV chunks; every chunk computes partial attention
 *     for each query block it touches and the partials are combined exactly with
 *     their normalisation statistics (news page, "Exchange the smaller side");
 *   - chunks are scheduled longest-processing-time-first by realised attention
 *     cost onto the least-loaded eligible worker (news page, "Balance actual
 *     attention work").  On one GPU a worker is a persistent CTA.
 *
 * Conventions for every entry point:
 *   - Return value: SPLITKV_OK (0) or a negative SPLITKV_ERR_* code; no C++
 *     exception crosses this boundary.  splitkv_error_string() names a code.
 *   - Tensors are caller-owned, contiguous DEVICE memory in these layouts
 *     (row-major, last index fastest), 16-byte aligned:
 *         q, dout      [Nq, Hq, d]   bfloat16 (raw 16-bit storage)
 *         k, v         [N, Hkv, d]   bfloat16
 *         kb, vb       [Nq, Hkv, d]  bfloat16  (the draft block's own keys/values,
 *                                                one row per draft token; unused
 *                                                and may be NULL under
 *                                                SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT)
 *         o            [Nq, Hq, d]   float32 or bfloat16 (see o_dtype)
 *         lse          [Nq, Hq]      float32, natural log
 *         dq           [Nq, Hq, d]   float32
 *         dk, dv       [N, Hkv, d]   float32
 *         dkb, dvb     [Nq, Hkv, d]  float32   (likewise)
 *     where N = sum of sample lengths, Nq = num_anchors * block_size, query
 *     token i belongs to block i / block_size, and query head h reads KV head
 *     h / (Hq / Hkv).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Attention calls are asynchronous on it.  splitkv_plan,
 *     splitkv_plan_update and the stats/export calls are host-only;
 *     splitkv_plan_upload enqueues a copy on the stream.
 *   - Workspaces are caller-allocated device memory of at least the size
 *     splitkv_workspace_size reports; the library allocates no per-call memory.
 *   - Calls that share a plan or a workspace must not run concurrently on
 *     different streams.  A plan's device memory holds the run-time claim
 *     cursors of its partial kernels (SPLITKV_FLAG_DYNAMIC_CLAIM: reset before,
 *     and advanced by, every launch) and its status words, so two launches of
 *     one plan in flight at once take items from each other's lists (items are
 *     skipped or run twice) even when their tensors and workspaces differ: give
 *     each concurrent stream its own plan.
 */
#ifndef SPLITKV_H_
#define SPLITKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes -------------------------------------------------------- */
#define SPLITKV_OK                        0
#define SPLITKV_ERR_INVALID_ARG          -1  /* bad pointer, size, layout or problem      */
#define SPLITKV_ERR_UNSUPPORTED          -2  /* valid problem outside the kernels' shapes */
#define SPLITKV_ERR_WORKSPACE_TOO_SMALL  -3
#define SPLITKV_ERR_CUDA                 -4  /* a CUDA runtime call failed                */
#define SPLITKV_ERR_TIMEOUT              -5  /* reserved: a bounded device wait gave up   */
#define SPLITKV_ERR_NOT_UPLOADED         -6  /* plan has no device copy yet               */
#define SPLITKV_ERR_NO_MEMORY            -7  /* host or device allocation failed          */

/* ---- plan flags -------------------------------------------------------------- */
/* Equal-count LPT (the pages' device rule: chunk counts kept equal).  Off by
 * default: CTAs have no memory limit, and plain LPT keeps Graham's bound. */
#define SPLITKV_FLAG_EQUAL_COUNT  1u
/* Reading B of the block keys (news page, "Why short queries change the
 * problem": every block also attends to "all tokens inside the block"): the
 * block's own tokens are the context positions after its anchor, so block b's
 * context interval is [S_s, min(a_b + bs, S_s + L_s)) and there are no
 * separate block keys.  Under this flag kb, vb (splitkv_merge,
 * splitkv_attn_fwd_static_scratch, splitkv_bwd_reduce, splitkv_attn_bwd) and
 * dkb, dvb may be NULL; they are neither read nor written.  Default (flag
 * clear, reading A): the block keys are the separate query-sized kb, vb. */
#define SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT  2u
/* bfloat16 partial records: the chunk outputs O_c of the forward workspace and
 * the dQ partials of the backward workspace are stored as bf16 (m_c, l_c and
 * every output stay float32).  Halves the record traffic of the partial
 * kernels, the merge and the dQ reduce, at one more bf16 rounding (relative
 * 2^-9) of each record element before the fp32 combine.  Served by the
 * tcgen05 kernels only (head_dim 128, G * bs a multiple of 8): attention calls
 * of other plans return SPLITKV_ERR_UNSUPPORTED. */
#define SPLITKV_FLAG_PARTIAL_BF16  4u
/* Tile cost for the backward LPT schedule: a (chunk, KV head) item of the
 * dK/dV kernel costs the work that kernel executes, in (row, key) pairs of
 * whole 128-row x 128-key tile steps -- for every 128-key tile of the chunk,
 * the query tiles that meet it -- instead of the allowed pairs (the pages'
 * "actual attention usage", the default).  Partly filled tiles then count as
 * what they cost, which evens out the measured per-CTA busy time of the dK/dV
 * kernel.  The forward schedule (used by the forward and dQ kernels), the
 * contiguous baseline and the pair counts keep the pair cost. */
#define SPLITKV_FLAG_TILE_COST  8u
/* Tile cost for the forward LPT schedule: a forward item (a chunk, or a slice of
 * q_slice query tiles, of one KV head) costs the work the forward kernel
 * executes on it, in (row, key) pairs of whole 128 x 128 tile steps.  That
 * kernel takes the item's query tiles two at a time, from the item's first
 * tile, and runs both over the 128-key tiles of their joint key range, so a
 * pair of tiles whose key ranges are [lo1, hi1) and [lo2, hi2) executes
 * 2 * ceil((max(hi) - min(lo)) / 128) steps (1 * ... for a last single tile).
 * The backward schedule, the contiguous baseline and the pair counts are not
 * affected (see SPLITKV_FLAG_TILE_COST for the backward schedule). */
#define SPLITKV_FLAG_FWD_TILE_COST  16u
/* Run-time claims: the LPT order of each schedule is kept, but instead of the
 * worker lists the CTAs of the forward, dK/dV and dQ kernels take the items of
 * that order one at a time, each CTA the next item as soon as it is free (an
 * atomic cursor per kernel in the plan's device memory, zeroed by every
 * launch).  This is LPT's "next item to the least-loaded worker" with the
 * loads the CTAs actually reach instead of the predicted costs, so per-SM speed
 * differences and cost-model error do not add to the makespan.  Results are
 * unchanged (every item writes only its own outputs); which CTA ran an item
 * varies from launch to launch.  The worker lists (SPLITKV_EXPORT_*_SCHEDULE)
 * and their loads are still computed: they are the static plan.  Served by the
 * tcgen05 kernels only (head_dim 128, G * bs a multiple of 8): attention calls
 * of other plans return SPLITKV_ERR_UNSUPPORTED.  Launches of one kernel on one
 * plan must not overlap (they share its cursor). */
#define SPLITKV_FLAG_DYNAMIC_CLAIM  32u
/* Contiguous schedules instead of LPT (the "unbalanced" baseline of the news page,
 * "Balance actual attention work", run on the kernels): each schedule keeps its
 * non-zero-cost items in (chunk, KV head, slice) order and gives item i of n to
 * worker floor(i W / n), whatever their costs.  Results are unchanged; the point is
 * to time what LPT saves.  Not combinable with SPLITKV_FLAG_EQUAL_COUNT or
 * SPLITKV_FLAG_DYNAMIC_CLAIM (INVALID_ARG).  The LPT-order exports then hold the
 * items in schedule order. */
#define SPLITKV_FLAG_CONTIGUOUS_SCHEDULE  64u
/* Rank plans (splitkv_plan_shard) only: chunks owned by ranks in order -- chunk c of n
 * to rank floor(c R / n) -- instead of by LPT (the news page's "unbalanced" device
 * baseline), to time what LPT ownership saves.  The CTA schedules inside a rank are
 * unaffected. */
#define SPLITKV_FLAG_CONTIGUOUS_RANKS  128u

/* ---- dtype codes (o) ------------------------------------------------------- */
#define SPLITKV_DTYPE_F32   0
#define SPLITKV_DTYPE_BF16  1

/* ---- workspace kinds --------------------------------------------------------- */
#define SPLITKV_WS_FWD  0
#define SPLITKV_WS_BWD  1
/* splitkv_read_cta_times only: the dQ kernel of the backward (tcgen05 path) */
#define SPLITKV_TIMES_DQ  2

/* ---- export selectors (splitkv_plan_export) ------------------------------- */
#define SPLITKV_EXPORT_ENTRIES        0  /* 4 per entry: chunk, block, lo, hi (record order)      */
#define SPLITKV_EXPORT_CHUNK_PAIRS    1  /* 1 per chunk: allowed (row, key) pairs per query head  */
#define SPLITKV_EXPORT_FWD_SCHEDULE   2  /* 5 per assigned item: worker, chunk, kv head, slice, cost */
#define SPLITKV_EXPORT_BWD_SCHEDULE   3  /* same, for the backward schedule (never sliced)        */
#define SPLITKV_EXPORT_FWD_LOADS      4  /* 1 per forward worker: summed cost                      */
#define SPLITKV_EXPORT_BWD_LOADS      5  /* 1 per backward worker                                  */
#define SPLITKV_EXPORT_CONTIG_LOADS   6  /* 1 per forward worker: the contiguous ("unbalanced")
                                            baseline                                               */
#define SPLITKV_EXPORT_FWD_LPT_ORDER  7  /* 4 per forward item, in LPT order: chunk, kv head,
                                            slice, cost (the order run-time claims take)         */
#define SPLITKV_EXPORT_BWD_LPT_ORDER  8  /* same, backward items                                 */
#define SPLITKV_EXPORT_CHUNK_OWNER    9  /* 1 per chunk: the rank that owns it (0 for a plain plan) */
#define SPLITKV_EXPORT_QUERY_SHARD   10  /* 4 values: rank, number of ranks, first block, end block
                                            of the blocks whose in-block term the plan adds      */

/* Largest number of ranks splitkv_combine_ranks / splitkv_sum_ranks take. */
#define SPLITKV_MAX_RANKS 4096

/* The problem, as the news page states it ("Why short queries change the
 * problem"): packed sample lengths, anchor positions, block size, and the
 * GQA head layout.  All pointers are HOST memory, read during the call only. */
typedef struct splitkv_problem {
  int32_t        num_samples;   /* S >= 1                                                  */
  const int32_t* sample_lens;   /* [S], every L_s >= 1; N = sum L_s < 2^31                 */
  int32_t        num_anchors;   /* A >= 1                                                  */
  const int32_t* anchors;       /* [A] global packed positions in [0, N); block b = anchors[b];
                                   any order, repeats allowed                                */
  int32_t        block_size;    /* bs >= 1                                                 */
  int32_t        num_q_heads;   /* Hq, a multiple of Hkv                                   */
  int32_t        num_kv_heads;  /* Hkv >= 1                                                */
  int32_t        head_dim;      /* d (the kernels take 64 or 128)                          */
  int32_t        kv_chunk;      /* C >= 1: chunk c covers keys [cC, min((c+1)C, N))         */
  int32_t        num_workers;   /* W >= 1: persistent CTAs of the forward partial kernel    */
  int32_t        num_bwd_workers; /* persistent CTAs of the backward partial kernel; 0 = W   */
  int32_t        q_slice;       /* 0 = one item per (chunk, KV head); k > 0 = items of at most
                                   k 128-row query tiles (forward schedule only)             */
  uint32_t       flags;         /* SPLITKV_FLAG_*                                          */
} splitkv_problem;

typedef struct splitkv_plan_s splitkv_plan_t;   /* opaque, owned by the library */

typedef struct splitkv_stats {
  int64_t  context_len;        /* N                                                        */
  int64_t  num_queries;        /* Nq                                                       */
  int32_t  num_chunks;
  int32_t  num_entries;        /* (chunk, block) pairs with a non-empty key interval        */
  int32_t  num_tiles;          /* 128-row query tiles over all chunks                       */
  int32_t  num_fwd_items;      /* non-zero-cost items of the forward schedule               */
  int32_t  num_bwd_items;
  int32_t  num_workers;
  int32_t  num_bwd_workers;
  uint64_t context_pairs;      /* sum over heads, rows and context keys of allowed pairs     */
  uint64_t block_pairs;        /* Hq * A * bs * bs (the in-block term)                      */
  uint64_t fwd_max_load;
  uint64_t bwd_max_load;
  double   fwd_imbalance;      /* max / mean - 1 over the W workers                         */
  double   bwd_imbalance;
  double   contig_imbalance;   /* same metric for the contiguous baseline                   */
  double   plan_us;            /* host time of the last splitkv_plan / splitkv_plan_update  */
} splitkv_stats;

/* Name of a status code (static string, never NULL). */
const char* splitkv_error_string(int status);

/* Build the mask metadata and both LPT schedules on the host (no CUDA call).
 * Metadata (news page, "Why short queries change the problem"; "Balance actual
 * attention work"): per block its context interval [S_s, a_b); per chunk the
 * blocks whose interval meets it, clipped to [lo, hi) and ordered by
 * (lo, hi, block) -- the "entries", whose order is also the order of partial
 * records in the workspace; 128-row query tiles of consecutive entries (a tile
 * holds 128 / (G * bs) blocks, G = Hq / Hkv, which must divide 128).
 * Schedule (digest Abstract; news page "Balance actual attention work"): items
 * (chunk, KV head[, slice]) of integer cost G * bs * sum(hi - lo); sorted by
 * cost descending, ties by (chunk, head, slice) ascending; each goes to the
 * eligible worker of least load, ties to the lowest id; zero-cost items are
 * dropped.  *out receives a plan the caller frees with splitkv_plan_destroy.
 * Errors: INVALID_ARG (NULL, non-positive sizes, an anchor outside [0, N),
 * Hq % Hkv != 0), UNSUPPORTED (128 % (G * bs) != 0), NO_MEMORY. */
int splitkv_plan(const splitkv_problem* problem, splitkv_plan_t** out);

/* One rank's plan of Split-KV over `num_ranks` ranks (news page, "Exchange the
 * smaller side": every device keeps its own share of the long context and
 * computes partial attention of all queries against it; "Balance actual
 * attention work": chunks go to devices by LPT on their cost with equal chunk
 * counts).  Ownership: every chunk, zero-cost ones included, is an item of cost
 * Hq * pairs_c (its realised (row, key) pairs over all query heads), sorted by
 * cost descending, ties by chunk ascending, each to the eligible rank of least
 * load (ties to the lowest rank); with n = q R + r chunks a rank is eligible while
 * it holds fewer than q chunks, or q while fewer than r ranks hold q + 1.  Query
 * side: rank r holds blocks [floor(r A / R), floor((r + 1) A / R)) -- their
 * queries, and their draft keys kb, vb (reading A) -- and adds their in-block
 * term.  The plan is splitkv_plan's over the chunks this rank owns: its entries
 * (and workspace), schedules and stats cover them only, and its chunk pairs are
 * 0 on other ranks' chunks.  Used with the same entry points:
 *   splitkv_attn_fwd + splitkv_merge give, for EVERY query row, the exact result
 *     over the keys this rank holds (O_r, LSE_r; O_r = 0 and LSE_r = -inf for a
 *     row that meets none of them); splitkv_combine_ranks merges the ranks'
 *     results of a row;
 *   splitkv_attn_bwd with the final o and lse gives every row's dq share (summed
 *     over ranks by splitkv_sum_ranks), complete dk, dv on the rows of this rank's
 *     chunks (rows of other ranks' chunks are not written) and complete dkb, dvb
 *     on the rows of its blocks (other rows not written).
 * q, dout, o and lse are full-size (every query row); k and v are addressed by
 * global position, and only the rows of this rank's chunks are read, except that
 * a 128-key tile starting in an owned chunk may read past the chunk end into rows
 * whose scores it masks (finite values are enough there: zero them once); kb and
 * vb are read on the rows of this rank's blocks only.  splitkv_plan_update keeps
 * the plan's rank.  Exports SPLITKV_EXPORT_CHUNK_OWNER and
 * SPLITKV_EXPORT_QUERY_SHARD give the assignment.
 * Errors: as splitkv_plan, and INVALID_ARG for num_ranks < 1 or rank outside
 * [0, num_ranks). */
int splitkv_plan_shard(const splitkv_problem* problem, int32_t num_ranks, int32_t rank,
                       splitkv_plan_t** out);

/* Rebuild `plan` in place for a new problem (same rules as splitkv_plan),
 * keeping its host and device buffers for reuse.  Blocks only until the
 * plan's previous upload has been consumed from its pinned staging buffer.
 * The device copy is stale until the next splitkv_plan_upload. */
int splitkv_plan_update(splitkv_plan_t* plan, const splitkv_problem* problem);

/* Copy the plan's tables to device memory owned by the plan (allocated or
 * grown on first need, which synchronises `stream`), through a pinned
 * staging buffer, asynchronously on `stream`.  Attention calls need it.
 * Errors: INVALID_ARG, CUDA, NO_MEMORY. */
int splitkv_plan_upload(splitkv_plan_t* plan, void* stream);

/* Free the plan and its host, pinned and device buffers (synchronises the
 * device if a device copy exists).  NULL is accepted. */
int splitkv_plan_destroy(splitkv_plan_t* plan);

/* Summary numbers of the plan (host only). */
int splitkv_plan_stats(const splitkv_plan_t* plan, splitkv_stats* out);

/* Copy one of the plan's host tables (SPLITKV_EXPORT_*) into out[0..capacity)
 * as int64 values; *count receives the number of values the table holds.
 * out may be NULL with capacity 0 to query the size.  Errors: INVALID_ARG,
 * WORKSPACE_TOO_SMALL (capacity < *count; *count is still set). */
int splitkv_plan_export(const splitkv_plan_t* plan, int what, int64_t* out,
                        int64_t capacity, int64_t* count);

/* Bytes of workspace an attention call needs (host only).
 *   SPLITKV_WS_FWD: the chunk partial records, as float32 (O_c as bfloat16
 *       under SPLITKV_FLAG_PARTIAL_BF16)
 *       O_c [E][bs][Hq][d], then m_c [E][bs][Hq], then l_c [E][bs][Hq]
 *     (E = number of entries, in entry order; each array starts on a 256-byte
 *     boundary).  m_c is the row's max of scale * q.k over the entry's keys
 *     (natural units), l_c = sum exp(s - m_c), O_c = sum exp(s - m_c) v / l_c.
 *   SPLITKV_WS_BWD: dQ partials float32 [E][bs][Hq][d] (bfloat16 under
 *       SPLITKV_FLAG_PARTIAL_BF16), then
 *     Delta = rowsum(dout * o) float32 [Nq][Hq]. */
int splitkv_workspace_size(const splitkv_plan_t* plan, int which, size_t* bytes);

/* Partial attention of every entry (news page, "Exchange the smaller side":
 * each shard evaluates all queries against its own keys).  For every entry
 * (chunk c, block b, [lo, hi)) and every query row of b and head h, over the
 * context keys j in [lo, hi) of KV head h / G: s = scale * q . k_j, and the
 * record (m_c, l_c, O_c) defined at splitkv_workspace_size is written to ws.
 * One persistent CTA per worker walks its forward schedule.  kb and vb are
 * not read here (the in-block term is formed by splitkv_merge).
 * Errors: INVALID_ARG (NULL/misaligned pointer, plan), NOT_UPLOADED,
 * UNSUPPORTED (d not 64 or 128), WORKSPACE_TOO_SMALL, CUDA (launch failure). */
int splitkv_attn_fwd(const splitkv_plan_t* plan, const void* q, const void* k,
                     const void* v, float scale, void* ws, size_t ws_bytes,
                     void* stream);

/* Exact combine (news page, "Exchange the smaller side"): for every query row
 * and head, the in-block term over the bs keys kb/vb of its own block gives a
 * record (m_b, l_b, O_b) (none under SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT, where
 * the block's keys are context keys); with the row's chunk records x (in chunk order),
 * M = max m_x, L = sum l_x exp(m_x - M), o = sum l_x exp(m_x - M) O_x / L,
 * lse = M + log L.  Records with l = 0 are skipped.  o is written as float32
 * or bfloat16 (o_dtype), lse as float32.  ws must hold a forward result of
 * the same plan.  Errors: as splitkv_attn_fwd. */
int splitkv_merge(const splitkv_plan_t* plan, const void* q, const void* kb,
                  const void* vb, float scale, const void* ws, size_t ws_bytes,
                  void* o, int o_dtype, float* lse, void* stream);

/* Backward with keys and values local to their chunk (news page, "Exchange
 * the smaller side": K/V stay local through forward and backward), recomputing
 * P = exp(s - lse) from the saved lse.  Per allowed (row i, key j):
 *   dv_j += P_ij dout_i;  dP_ij = dout_i . v_j;  dS_ij = P_ij (dP_ij - Delta_i);
 *   dk_j += scale dS_ij q_i;  dq_i += scale dS_ij k_j,
 * with Delta_i = dout_i . o_i.  dk/dv of a chunk are owned by the CTA of its
 * (chunk, KV head) item and summed over the G query heads; dq is written per
 * entry as a partial and reduced over chunks in ascending chunk order, then the
 * in-block term adds its dq and produces dkb/dvb (summed over the block's rows
 * and the G heads).  Keys no query reads get dk = dv = 0.  Deterministic.
 * o has dtype o_dtype.  Errors: as splitkv_attn_fwd. */
int splitkv_attn_bwd(const splitkv_plan_t* plan, const void* q, const void* k,
                     const void* v, const void* kb, const void* vb,
                     const void* o, int o_dtype, const float* lse,
                     const void* dout, float* dq, float* dk, float* dv,
                     float* dkb, float* dvb, float scale, void* ws,
                     size_t ws_bytes, void* stream);

/* The three launches of splitkv_attn_bwd, exposed so that callers can time or
 * overlap them; splitkv_attn_bwd is exactly these three in this order on one
 * stream, with the same arguments:
 *   splitkv_bwd_delta    Delta = rowsum(dout * o) into the backward workspace;
 *   splitkv_bwd_partial  the persistent chunk kernel: dk, dv (chunk-owned) and the
 *                        per-entry dq partials in the workspace;
 *   splitkv_bwd_reduce   dq = sum of the partials in ascending chunk order plus the
 *                        in-block term's dq; dkb, dvb of the in-block term.
 * Errors: as splitkv_attn_bwd. */
int splitkv_bwd_delta(const splitkv_plan_t* plan, const void* o, int o_dtype, const void* dout,
                      void* ws, size_t ws_bytes, void* stream);
int splitkv_bwd_partial(const splitkv_plan_t* plan, const void* q, const void* k, const void* v,
                        const float* lse, const void* dout, float* dk, float* dv, float scale,
                        void* ws, size_t ws_bytes, void* stream);
int splitkv_bwd_reduce(const splitkv_plan_t* plan, const void* q, const void* kb, const void* vb,
                       const float* lse, const void* dout, float* dq, float* dkb, float* dvb,
                       float scale, const void* ws, size_t ws_bytes, void* stream);

/* splitkv_bwd_partial is itself two launches on the tcgen05 path (head_dim
 * 128, G * bs a multiple of 8), exposed for timing: splitkv_bwd_dkdv (the
 * KV-stationary kernel: dk, dv) followed by splitkv_bwd_dq (the Q-stationary
 * kernel: the dq partials).  On other shapes one kernel produces all three and
 * runs in splitkv_bwd_dkdv; splitkv_bwd_dq then launches nothing.  Same
 * arguments and errors as splitkv_bwd_partial. */
int splitkv_bwd_dkdv(const splitkv_plan_t* plan, const void* q, const void* k, const void* v,
                     const float* lse, const void* dout, float* dk, float* dv, float scale,
                     void* ws, size_t ws_bytes, void* stream);
int splitkv_bwd_dq(const splitkv_plan_t* plan, const void* q, const void* k, const void* v,
                   const float* lse, const void* dout, float scale, void* ws, size_t ws_bytes,
                   void* stream);

/* Size of the library's static device scratch buffer (16 MiB): see
 * splitkv_attn_fwd_static_scratch. */
#define SPLITKV_STATIC_SCRATCH_BYTES (16u << 20)

/* Forward attention that allocates nothing: splitkv_attn_fwd followed by
 * splitkv_merge, with the partial records held in a buffer of
 * SPLITKV_STATIC_SCRATCH_BYTES that is a static array of the library's device
 * code (every GPU that loads the library keeps it until the process exits).
 * The pages have no counterpart to this call: it exists for callers that may
 * not call cudaMalloc per call (a framework whose caching allocator holds the
 * device memory, latency-critical loops that cannot take cudaMalloc's implicit
 * synchronisation, plug-ins handed raw pointers without an allocator).
 * The caller passes the inputs and outputs exactly as for splitkv_attn_fwd and
 * splitkv_merge; the plan must already have its device copy
 * (splitkv_plan_upload, a set-up step) in the CUDA context current at the
 * call.  The first call in a context looks up the buffer's device address
 * (cudaGetSymbolAddress; cached per context, keyed by the context's id, so a
 * caller's own driver-API context or a re-created primary context gets its
 * own lookup), so make that first call before any stream capture.  Every call
 * shares the one buffer, and calls whose kernels overlap on the GPU (different
 * streams, or different host threads) race on it: serialise them.  Each call
 * writes every record it reads, so left-over contents of an earlier call are
 * never used.
 * Errors: INVALID_ARG, NOT_UPLOADED and UNSUPPORTED as splitkv_merge;
 * WORKSPACE_TOO_SMALL when the problem's forward workspace
 * (splitkv_workspace_size, SPLITKV_WS_FWD) exceeds SPLITKV_STATIC_SCRATCH_BYTES
 * (checked before any CUDA call); CUDA when the current context cannot be
 * queried, the buffer's address cannot be looked up, or a launch fails. */
int splitkv_attn_fwd_static_scratch(const splitkv_plan_t* plan, const void* q, const void* k,
                                    const void* v, const void* kb, const void* vb, float scale,
                                    void* o, int o_dtype, float* lse, void* stream);

/* Time limit of the mbarrier waits inside this plan's tcgen05 kernels, in
 * nanoseconds of the device global timer (default 2e9, the limit of every
 * wait; 0 <= ns <= 6e10, else INVALID_ARG).  A wait that runs past it records
 * SPLITKV_ERR_TIMEOUT and its site in the plan's status words (read by
 * splitkv_plan_status), and the kernel winds down: every role stops, the copies
 * and products already in flight are awaited (with the default limit) and the
 * tensor memory is freed, so the context stays usable and the next launch runs
 * normally.  Takes effect from the next launch; host-only.  This is the failure
 * detection of the kernels made testable: a test sets a limit no wait can meet
 * and checks the status.  The pages have no counterpart to it. */
int splitkv_plan_set_wait_limit(splitkv_plan_t* plan, int64_t ns);

/* Device status of the plan's kernels: synchronises `stream`, returns
 * SPLITKV_OK, or the SPLITKV_ERR_* code a kernel recorded since the last call
 * (SPLITKV_ERR_TIMEOUT: a wait inside a kernel passed its 2-second limit and
 * the kernel wound down; its outputs are invalid), and clears the words.
 * If `site` is not NULL it receives the source site of the first wait that
 * timed out (0 if none).  Errors: INVALID_ARG, NOT_UPLOADED, CUDA. */
int splitkv_plan_status(const splitkv_plan_t* plan, void* stream, int32_t* site);

/* Self-test of the FMA-pipe exp2 the attention kernels use for part of their
 * exponentials (Cody-Waite range reduction and a fitted cubic): y[i] = 2^x[i]
 * for n device floats, asynchronously on `stream`.  Not part of the method;
 * it lets a test compare the approximation with CUDA's exp2f.
 * Errors: INVALID_ARG, CUDA. */
int splitkv_selftest_exp2(const float* x, float* y, int64_t n, void* stream);

/* splitkv_merge of a rank plan with the exchange of Split-KV over ranks fused in (news
 * page, "Exchange the smaller side"): instead of writing every query row's result to
 * local o, lse, the rows of block b go straight to the receive buffers of the rank that
 * owns b (blocks [floor(r A / R), floor((r + 1) A / R)) to rank r, as the plan's
 * SPLITKV_EXPORT_QUERY_SHARD): o_dest[r] float32 [R][rows_r][Hq][d] and lse_dest[r]
 * float32 [R][rows_r][Hq], rows_r = bs * (blocks of rank r), at slot `rank` -- the
 * layout splitkv_combine_ranks reads on rank r.  o_dest and lse_dest are DEVICE arrays of
 * R device pointers (8-byte aligned); entries may be another GPU's memory mapped into this
 * one (peer access), which the kernel writes with plain stores.  The caller orders the
 * owners' combine after every rank's merge (a collective or a barrier).  num_ranks and
 * rank must be the plan's (splitkv_plan_shard).  Errors: as splitkv_merge, INVALID_ARG
 * also for a rank mismatch or a NULL / misaligned pointer array. */
int splitkv_merge_to_owners(const splitkv_plan_t* plan, const void* q, const void* kb, const void* vb,
                            float scale, const void* ws, size_t ws_bytes, int32_t num_ranks, int32_t rank,
                            float* const* o_dest, float* const* lse_dest, void* stream);

/* splitkv_bwd_reduce of a rank plan with the dq exchange fused in: each block's dq rows
 * (this rank's share: its chunk partials, plus the in-block term for its own blocks) go
 * straight to the owner's receive buffer dq_dest[r] float32 [R][rows_r][Hq][d] at slot
 * `rank` (the layout splitkv_sum_ranks reads on rank r); dkb, dvb as splitkv_bwd_reduce
 * (rows of this rank's blocks).  dq_dest is a DEVICE array of R device pointers; as for
 * splitkv_merge_to_owners, entries may be peer-mapped and the caller orders the owners'
 * sums after every rank's call.  Errors: as splitkv_bwd_reduce, INVALID_ARG also for a
 * rank mismatch or a NULL / misaligned pointer array. */
int splitkv_bwd_reduce_to_owners(const splitkv_plan_t* plan, const void* q, const void* kb, const void* vb,
                                 const float* lse, const void* dout, float* dkb, float* dvb, float scale,
                                 const void* ws, size_t ws_bytes, int32_t num_ranks, int32_t rank,
                                 float* const* dq_dest, void* stream);

/* Let kernels on the current device read and write memory of `peer_device` (the receive
 * buffers of splitkv_merge_to_owners / splitkv_bwd_reduce_to_owners when they live on
 * another GPU, mapped here by CUDA IPC).  Already enabled counts as success.  Errors:
 * INVALID_ARG (no such device), UNSUPPORTED (the two GPUs have no peer path), CUDA. */
int splitkv_enable_peer_access(int32_t peer_device);

/* Exact combine of the ranks' results (news page, "Exchange the smaller side":
 * partials over disjoint key shares merged with their normalisation statistics).
 * o_parts [R][rows][head_dim] and lse_parts [R][rows] float32 (device; row =
 * query token x head, 16- and 4-byte aligned), rank r's exact result over its
 * keys (lse natural-log, -inf where rank r holds no key of the row).  For every
 * row: M = max_r lse_r, w_r = exp(lse_r - M), o = sum_r w_r o_r / sum_r w_r
 * (ranks in ascending order), lse = M + log(sum_r w_r); a row with no finite
 * lse_r gets o = 0, lse = -inf.  o is float32 (16-byte aligned) or bfloat16
 * (8-byte aligned) per o_dtype, [rows][head_dim]; lse [rows].  Asynchronous on
 * `stream`.  Errors: INVALID_ARG (num_ranks outside [1, SPLITKV_MAX_RANKS],
 * head_dim not a positive multiple of 4, NULL or misaligned pointer), CUDA. */
int splitkv_combine_ranks(int32_t num_ranks, int64_t rows, int32_t head_dim, const float* o_parts,
                          const float* lse_parts, void* o, int o_dtype, float* lse, void* stream);

/* Conversion of a finished float32 result array (o, dq, dk, dv, dkb, dvb) to
 * bfloat16, round to nearest even: dst[i] = bf16(src[i]) for i < n.  The pages
 * have no counterpart: the method's arithmetic is unchanged (it computes and
 * accumulates in fp32); this halves the bytes of results a caller keeps in bf16,
 * e.g. gradients copied back to the host.  src (float32) and dst (bfloat16, as
 * uint16) are DEVICE arrays of n elements owned by the caller, not overlapping;
 * 16-byte aligned pointers take the vector path, others an element-wise one.
 * Asynchronous on `stream`.  Errors: INVALID_ARG (n < 0 or above 2^42, NULL
 * pointer with n > 0), CUDA (launch failure). */
int splitkv_cast_bf16(int64_t n, const float* src, uint16_t* dst, void* stream);

/* Sum of the ranks' shares: out[i] = sum_r parts[r * n + i], ranks added in
 * ascending order (the dq of Split-KV over ranks: every rank's dq share of the
 * rows a rank owns).  parts [R][n] and out [n] float32, 16-byte aligned, n a
 * multiple of 4.  Asynchronous on `stream`.  Errors: INVALID_ARG, CUDA. */
int splitkv_sum_ranks(int32_t num_ranks, int64_t n, const float* parts, float* out, void* stream);

/* Self-test of the kernels' failure detection: one CTA waits, with the same bounded
 * mbarrier waits the attention kernels use, on a barrier nothing ever completes.  The
 * wait gives up after its time limit (2 s of the device global timer) and records
 * SPLITKV_ERR_TIMEOUT and its source site, which come back in status_out[0] and
 * status_out[1] (the kernel does not hang and the context stays usable).  Synchronises
 * `stream`; takes about two seconds.  Not part of the method.
 * Errors: INVALID_ARG, NO_MEMORY, CUDA. */
int splitkv_selftest_wait_timeout(int32_t* status_out, void* stream);

/* Per-CTA busy time of the last splitkv_attn_fwd (which = SPLITKV_WS_FWD), the
 * last dK/dV partial kernel (SPLITKV_WS_BWD; the single backward kernel of the
 * mma.sync path) or the last dQ partial kernel (SPLITKV_TIMES_DQ; tcgen05 path,
 * zeros before its first launch) on this plan: out_ns[w] = end - start of
 * worker w's CTA in nanoseconds (device global timer), for the schedule's
 * worker count (num_workers for the forward and dQ kernels).  Synchronises `stream`.  Errors: INVALID_ARG, NOT_UPLOADED,
 * WORKSPACE_TOO_SMALL (capacity below the worker count), CUDA. */
int splitkv_read_cta_times(const splitkv_plan_t* plan, int which, int64_t* out_ns,
                           int64_t capacity, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* SPLITKV_H_ */
