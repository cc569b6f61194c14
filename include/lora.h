/*
 * lora.h -- C ABI of the B200 multi-LoRA delta library (liblora_b200.so).
 *
 * What the library computes, for every row t of a mixed batch whose adapter
 * id a = ids[t] is not -1:
 *
 *     y[t, :] += (alpha_a / r_a) * B_a (A_a x[t, :])
 *
 * with A_a of shape r_a x d_in and B_a of shape d_out x r_a.  This is the
 * per-request adapter term of y = xW + (x A_i) B_i (alpha / r) from "Multi-LoRA
 * Serving: Why 100 Adapters Fit on One GPU" (section "Why can't you just merge
 * LoRA weights into the base model?"), with the adapter shapes of section "How
 * much memory does one LoRA adapter actually cost?" of the same page, and the
 * column form W.x + (B.A).x of "Serving Many LoRA Adapters From One Base
 * Model" (section "How it works").  xW is produced by the caller; the library
 * adds the delta in place.  All adapters of a batch are handled by one launch,
 * driven by an index vector (segmented gather, first page, section "How does
 * one batch run 30 different adapters at once?").  Adapters live in a paged
 * pool with a page table ("Multi-LoRA Serving: Sharing One GPU Across
 * Adapters", section "How S-LoRA Proved the Model").
 *
 * Conventions for every call:
 *  - Return value: LORA_OK (0) or one of the LORA_ERR_* codes below.  No C++
 *    exception crosses this boundary.
 *  - Pointers named "device" are device pointers owned by the caller (for
 *    example torch tensor storage); the library never frees them.
 *  - stream is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  Compute calls are asynchronous on that stream and never
 *    synchronise the host or allocate; those that take a workspace may be
 *    captured in a CUDA graph.
 *  - bf16 tensors are row-major with a leading dimension (ld*) counted in
 *    elements.  x, y, weights and workspace must be 16-byte aligned, and
 *    d_in, d_out, ldx and ldy must be multiples of 8, else LORA_ERR_ALIGNMENT.
 *  - x and y must not overlap.
 *  - Errors found on the device (bad adapter ids, timed-out waits) do not
 *    fault: the affected rows are left untouched and a sticky per-pool status
 *    word records the first error; read it with lora_get_error.
 */
#ifndef LORA_B200_H
#define LORA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */

enum {
    LORA_OK = 0,
    LORA_ERR_INVALID_ARG = 1,  /* null pointer, size out of range, bad enum   */
    LORA_ERR_ALIGNMENT = 2,    /* pointer / leading dimension alignment       */
    LORA_ERR_NO_PAGES = 3,     /* the page pool has too few free pages        */
    LORA_ERR_SLOT = 4,         /* slot index out of range                     */
    LORA_ERR_NOT_LOADED = 5,   /* slot holds no adapter (host check, or sticky
                                  device status when a batch names it)        */
    LORA_ERR_CUDA = 6,         /* a CUDA runtime call failed                  */
    LORA_ERR_BAD_ID = 7,       /* sticky device status: an id outside
                                  [-1, n_slots) or a malformed segment        */
    LORA_ERR_TIMEOUT = 8,      /* sticky device status: a bounded wait inside
                                  a kernel gave up                            */
    LORA_ERR_WORKSPACE = 9,    /* workspace smaller than lora_workspace_bytes */
    LORA_ERR_BOUNDS = 10       /* sticky device status, LORA_DEBUG builds only: an
                                  index or page outside its buffer was about to be
                                  used (the access was skipped or redirected) */
};

/* Human-readable name of a status code (static string, never NULL). */
LORA_API const char *lora_status_string(int status);

/* ------------------------------------------------------------- the pool */

/* Opaque pool handle; allocated by lora_pool_create, freed by
 * lora_pool_destroy.  It owns small device tables (page table, ranks, status
 * word) but not the page memory, which the caller provides. */
typedef struct lora_pool lora_pool;

/* One adapted weight matrix (a layer's projection): W is d_out x d_in. */
typedef struct {
    int d_in;
    int d_out;
} lora_target;

/*
 * Slot layout (the logical bytes of one adapter slot).  Targets follow one
 * another in order.  Target t holds A (r_max rows of d_in bf16; row j is
 * adapter row j) and then B transposed (r_max rows of d_out bf16; row j is
 * column j of B).  Each of these two blocks starts on a 256-byte boundary.
 * Rows rank..r_max-1 of both blocks are zero (rank padding, the static
 * max_lora_rank slot of "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU",
 * section "Where does multi-LoRA serving actually break?", item 2); kernels
 * read only the adapter's own rank.
 *
 * Inside a block of `width` columns the rows are stored in column tiles of
 * tc = 1024 columns (r_max <= 16), 512 (r_max <= 32) or 256 (r_max > 32),
 * so that r_max rows of a tile are 32 KiB: tile k
 * holds columns k*tc .. min((k+1)*tc, width)-1 of rows 0..r_max-1, row after
 * row (tw = that tile's width in 16-byte chunks of 8 columns), and starts at
 * byte k * r_max * tc * 2 of the block.  In a row of a tile, chunk c of every
 * complete group of eight chunks is stored at position c ^ (row % 8); a
 * trailing partial group keeps its order.  The first r rows of a tile are
 * thus one contiguous range (the decode kernel stages them with one copy),
 * and the rows of a staged tile fall in different shared-memory banks.
 *
 * Paging.  A slot's logical bytes are cut into pages of page_bytes; page p of
 * slot s lives at physical page page_table[s * pages_per_slot + p], i.e. at
 * byte pool_mem + page * page_bytes.  page_bytes == 0 means one page per slot
 * (a contiguous stacked pool [n_slots][slot_bytes rounded up to 256]).
 */

/* Bytes of page memory needed to hold every slot at once (0 on bad args).
 * page_bytes: 0, or a power of two >= 4096. */
LORA_API size_t lora_pool_bytes_required(const lora_target *targets, int n_targets,
                                int r_max, int n_slots, size_t page_bytes);

/*
 * Create a pool over caller-owned device memory.
 *   device        CUDA device ordinal the pool and all its calls use.
 *   targets       n_targets (1..4096) matrix shapes, copied.
 *   r_max         rank of a slot (1..64).
 *   n_slots       number of adapter slots (1..16384).
 *   page_bytes    0 (one page per slot) or a power of two >= 4096.
 *   pool_mem      device buffer of pool_bytes bytes, 256-byte aligned; it may
 *                 hold fewer pages than n_slots need (pages are taken from a
 *                 free list when a slot is first loaded: LORA_ERR_NO_PAGES when
 *                 it runs out).
 *   scatter_seed  0: free pages in ascending order; otherwise a seeded
 *                 permutation, so a slot's pages are scattered over the pool.
 * Returns LORA_OK and *out, or an error (nothing allocated).
 */
LORA_API int lora_pool_create(lora_pool **out, int device, const lora_target *targets,
                     int n_targets, int r_max, int n_slots, size_t page_bytes,
                     void *pool_mem, size_t pool_bytes, uint64_t scatter_seed);

/*
 * Copy one adapter matrix pair into a slot.
 *   rank   the adapter's rank on this target, 0..r_max (0 marks the target as
 *          not adapted: rows of this slot are then left untouched on it).
 *   A      bf16 [rank, d_in], row-major, dense.
 *   B      bf16 [d_out, rank], row-major, dense; stored transposed.
 *   src_is_device  1: A and B are device pointers (copies are asynchronous on
 *          stream); 0: host pointers (the call returns once the host data has
 *          been staged; the device copies complete in stream order).
 * The first load into an empty slot takes its pages from the free list.
 * Loading must not race with compute calls that read the same slot.
 */
LORA_API int lora_pool_load(lora_pool *pool, int slot, int target, int rank,
                   const void *A, const void *B, int src_is_device,
                   void *stream);

/*
 * Swap one adapter in from host memory for all targets at once, without the
 * host waiting: the adapter's weights move across the host link in one copy
 * into the caller's device staging area, then one kernel scatters them into
 * the slot's pages (A rows as given, B transposed, rank padding zeroed), all
 * in stream order.  The pages' home is the unified page pool ("Multi-LoRA
 * Serving: Sharing One GPU Across Adapters", section "How S-LoRA Proved the
 * Model": adapters move between host and GPU memory on demand).
 *   ranks    host int [n_targets]: the adapter's rank on each target (0 =
 *            not adapted there), each <= r_max
 *   src      host memory (pinned, for the copy to run asynchronously) of
 *            lora_swap_src_bytes(ranks) bytes: for each target t in order with
 *            ranks[t] > 0, A_t bf16 [rank, d_in] then B_t bf16 [d_out, rank],
 *            row-major, packed
 *   staging  device memory, 256-byte aligned, of at least
 *            lora_swap_staging_bytes(ranks) bytes; it must stay untouched
 *            until the stream has passed the call
 * The first load into an empty slot takes its pages from the free list.  The
 * call must not race with compute calls that read the same slot; compute on
 * other slots may run concurrently on other streams.  Errors: LORA_ERR_SLOT,
 * LORA_ERR_INVALID_ARG (rank out of range, src_bytes not the packed size),
 * LORA_ERR_ALIGNMENT, LORA_ERR_WORKSPACE (staging too small),
 * LORA_ERR_NO_PAGES, LORA_ERR_CUDA.
 */
LORA_API int lora_pool_swap_in(lora_pool *pool, int slot, const int *ranks, const void *src,
                      size_t src_bytes, void *staging, size_t staging_bytes, void *stream);

/* Bytes of the packed source of lora_pool_swap_in (0 for an invalid rank). */
LORA_API size_t lora_swap_src_bytes(const lora_pool *pool, const int *ranks);

/* Staging bytes lora_pool_swap_in needs (0 for an invalid rank). */
LORA_API size_t lora_swap_staging_bytes(const lora_pool *pool, const int *ranks);

/* Release a slot's pages to the free list and mark it empty (its rows then
 * raise LORA_ERR_NOT_LOADED).  Synchronous with respect to the device. */
LORA_API int lora_pool_unload(lora_pool *pool, int slot);

/* Free the pool's own device tables and the handle (not pool_mem).  Waits for
 * the device. */
LORA_API int lora_pool_destroy(lora_pool *pool);

/* Device pointer to the page table, int32 [n_slots][pages_per_slot]; -1 marks
 * a page that is not allocated.  Read-only; valid until destroy. */
LORA_API const int32_t *lora_pool_page_table(const lora_pool *pool);

/* Geometry of a pool, for callers that walk its memory (tests, tools). */
typedef struct {
    size_t slot_bytes;      /* logical bytes of one slot                     */
    size_t page_bytes;      /* physical page size (one slot when 0 was given) */
    int pages_per_slot;
    int n_pages;            /* physical pages in pool_mem                    */
    int free_pages;
    int n_slots, n_targets, r_max;
    int decode_ctas;        /* CTAs of the decode kernel that can be
                               resident at once on this device */
} lora_pool_info;

LORA_API int lora_pool_get_info(const lora_pool *pool, lora_pool_info *info);

/* Byte offsets inside a slot of target t's A block and B-transposed block. */
LORA_API int lora_pool_target_offsets(const lora_pool *pool, int target,
                             size_t *a_off, size_t *bt_off);

/* ---------------------------------------------------------- the workspace */

/*
 * Device workspace for calls on `target` with up to max_tokens rows (the
 * call's T): the plan (rows grouped by adapter, work items, tensor-core
 * tiles), then, where the tensor-core segment path can serve the target, the
 * fp32 partial V of each k-slice of d_in (T x slices x rank bound x 4 bytes).
 * A workspace shared by several targets takes the largest of their sizes.
 * Calls with a smaller workspace return LORA_ERR_WORKSPACE.  Its contents
 * need no initialisation; calls that overlap on the GPU need workspaces of
 * their own.
 */
LORA_API size_t lora_workspace_bytes(const lora_pool *pool, int target, int max_tokens);

/* Where each plan array lives inside a workspace sized for T rows (byte
 * offsets from the workspace base). */
typedef struct {
    size_t header;      /* int32[64]: [0] segments, [1] rows grouped,
                           [2] decode work items of the segments on the
                           decode path, [3] tensor-core tiles, [4] T,
                           [5] decode items when every segment takes the
                           decode path (long segments' items follow)     */
    size_t perm;        /* int32[T]: row indices grouped by segment        */
    size_t seg_start;   /* int32[S_max+1]: segment s = perm[seg_start[s] ..
                           seg_start[s+1])                                 */
    size_t seg_slot;    /* int32[S_max]: slot of segment s                 */
    size_t items;       /* int32[I_max][4]: decode items {slot, first perm
                           index, rows, segment}                            */
    size_t tiles;       /* int32[J_max][4]: tensor-core tiles {slot, first
                           row of x/y, rows, segment}                       */
    size_t total;
    int s_max, i_max, j_max;
} lora_plan_layout;

LORA_API int lora_plan_layout_get(const lora_pool *pool, int T, lora_plan_layout *out);

/* ---------------------------------------------------------------- plans */

/*
 * Build the plan of a batch from its index vector: rows grouped by adapter
 * (segments in ascending slot order, rows in ascending order inside a
 * segment), split into work items.  ids: device int32 [T], -1 = no adapter.
 * Rows with an invalid id (outside [-1, n_slots): LORA_ERR_BAD_ID; an empty
 * slot: LORA_ERR_NOT_LOADED) join no segment and set the sticky status.
 * A plan depends only on the batch, so one plan serves every target of a
 * forward step (lora_apply_plan).
 */
LORA_API int lora_plan_ids(lora_pool *pool, const int32_t *ids, int T, void *ws,
                  size_t ws_bytes, void *stream);

/*
 * Build the plan of a batch given as contiguous segments: rows
 * seg_offsets[s] .. seg_offsets[s+1]-1 use slot seg_slot[s].
 *   seg_offsets  device int32 [S+1], non-decreasing, within [0, T];
 *   seg_slot     device int32 [S]; -1 = the segment has no adapter.
 * Segments at least lora_mma_min_rows_for(S, T) long take the tensor-core
 * path (in 128-row tiles) when the target allows it (r_max <= 32 and the
 * slices fit in shared memory), the others the decode path.  Offsets that decrease or leave
 * [0, T] make the whole plan empty (LORA_ERR_BAD_ID); segments naming an
 * invalid slot are skipped (LORA_ERR_BAD_ID / LORA_ERR_NOT_LOADED).
 */
LORA_API int lora_plan_segments(lora_pool *pool, const int32_t *seg_offsets,
                       const int32_t *seg_slot, int S, int T, void *ws,
                       size_t ws_bytes, void *stream);

/* Segment length from which the tensor-core path is used in a batch of many
 * segments. */
LORA_API int lora_mma_min_rows(void);

/*
 * Segment length from which lora_plan_segments sends a segment to the
 * tensor-core path, for a batch of S segments over T rows: 1 (every segment)
 * when S <= 16 and the tiles fit the plan (floor(T / 128) + S tiles at most),
 * so that a prefill batch needs no decode launch for its short segments (a
 * segment of m rows is then one tile of m rows: the same adapter slices and
 * rows as on the decode path); lora_mma_min_rows() otherwise.  -1 for S < 0
 * or T outside [0, 2^20].
 */
LORA_API int lora_mma_min_rows_for(int S, int T);

/*
 * Apply a built plan to one target:  y[t] += scales[a] * B_a (A_a x[t]).
 *   x       device bf16 [T, ldx] (ldx >= d_in)
 *   y       device bf16 [T, ldy] (ldy >= d_out), updated in place: each
 *           adapted element becomes bf16_rn(y + scale * delta) computed in
 *           fp32; other rows are not touched.
 *   scales  device fp32 [n_slots]: alpha / r of each slot's adapter.
 *   T, ws, ws_bytes  as passed to the plan call.
 */
LORA_API int lora_apply_plan(lora_pool *pool, int target, const void *x, int ldx,
                    void *y, int ldy, const float *scales, int T,
                    const void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------- one-call entry */

/*
 * The heterogeneous-batch delta: for every row t with a = ids[t] != -1,
 *     y[t] += scales[a] * B_a (A_a x[t]),
 * the per-request term of y = xW + (x A) B (alpha / r) on "Multi-LoRA
 * Serving: Why 100 Adapters Fit on One GPU" (section "Why can't you just
 * merge LoRA weights into the base model?"; A_a here holds the rows of that
 * page's A transposed, so A_a x[t] is its x A), computed for every adapter of
 * the batch in one call from an index vector and the stacked pool, as the
 * same page's section "How does one batch run 30 different adapters at
 * once?" describes; xW is the caller's (y on entry).
 *   x, ldx   device bf16 [T, ldx], ldx >= d_in, a multiple of 8, 16-byte
 *            aligned; read only; must not overlap y
 *   y, ldy   device bf16 [T, ldy], ldy >= d_out, a multiple of 8, 16-byte
 *            aligned; each adapted element becomes bf16_rn(y + scale *
 *            delta) computed in fp32; rows with id -1 are not touched
 *   ids      device int32 [T]: slot of each row, -1 = no adapter
 *   scales   device fp32 [n_slots]: alpha / r of each slot's adapter
 *   ws       device workspace of at least lora_workspace_bytes(pool, target,
 *            T) bytes, 16-byte aligned (caller-owned)
 * Errors: host-checked arguments return LORA_ERR_INVALID_ARG /
 * LORA_ERR_ALIGNMENT / LORA_ERR_WORKSPACE with nothing launched; bad ids
 * and unloaded slots found on the device leave their rows untouched and set
 * the sticky status (lora_get_error).
 * Same result as lora_plan_ids followed by lora_apply_plan.  Batches
 * of at most 256 rows take one launch instead: the delta kernel groups the
 * rows itself (the same segments and items as lora_plan_ids), and ws is then
 * not written -- callers that reuse a plan across targets call lora_plan_ids
 * and lora_apply_plan.  ws / ws_bytes are checked the same way either way.
 */
LORA_API int lora_apply(lora_pool *pool, int target, const void *x, int ldx, void *y,
               int ldy, const int32_t *ids, const float *scales, int T,
               void *ws, size_t ws_bytes, void *stream);

/*
 * Several targets that read the same x -- the q, k and v projections of one
 * layer (the target modules of "Multi-LoRA Serving: Why 100 Adapters Fit on
 * One GPU", section "How much memory does one LoRA adapter actually cost?")
 * -- in one launch: for i < n_targets,
 *     y[t, y_cols[i] + n] += scales[a] * (B_a (A_a x[t]))[n],  a = ids[t],
 * with A_a, B_a the adapter's matrices on target targets[i].  Equal to
 * n_targets lora_apply calls on the column slices of y, bit for bit.
 *   n_targets  1 .. 4
 *   targets    host int [n_targets]: target indices, all with the same d_in
 *              and the same d_out
 *   y_cols     host int [n_targets]: first column of each target's slice of
 *              y, a multiple of 8; slices may not overlap and must end within
 *              ldy (e.g. 0, d_out, 2 d_out for a fused qkv output)
 *   x, ldx     device bf16 [T, ldx], shared by all the targets
 *   y, ldy     device bf16 [T, ldy], updated in place
 *   ids, scales, T, ws, ws_bytes, stream  as for lora_apply (ws sized for
 *              targets[0]); batches of at most 256 rows take one launch and
 *              leave ws unwritten.
 * Errors: LORA_ERR_INVALID_ARG for a bad count, target, shape mismatch,
 * overlapping or out-of-range slice; LORA_ERR_ALIGNMENT for a column not a
 * multiple of 8; device-side statuses as for lora_apply.
 */
LORA_API int lora_apply_multi(lora_pool *pool, int n_targets, const int *targets,
                     const void *x, int ldx, void *y, int ldy, const int *y_cols,
                     const int32_t *ids, const float *scales, int T, void *ws,
                     size_t ws_bytes, void *stream);

/* ------------------------------------------------ routed expert pairs */

/*
 * The delta inside expert routing (mixture-of-experts layers): each token t
 * is routed to top_k experts, and an adapted expert projection carries the
 * token's adapter's own shrink and expand for that expert ("Multi-LoRA
 * Serving: Sharing One GPU Across Adapters", section "MoE Models Raise the
 * Bar").  For every pair p = t * top_k + j:
 *     y[p] += scales[s] * B_s (A_s x[t]),  s = lora_ids[t] * n_experts + topk_ids[p],
 * with slot s of the pool holding adapter lora_ids[t]'s matrices for expert
 * topk_ids[p] on `target`.
 *   x, ldx     device bf16 [T, ldx]: one row per token
 *   y, ldy     device bf16 [T * top_k, ldy]: one row per pair (the expert
 *              output rows, in pair order), updated in place
 *   lora_ids   device int32 [T]: the token's adapter, -1 = none (its pairs'
 *              rows are untouched)
 *   topk_ids   device int32 [T * top_k]: the experts chosen for each token
 *   n_experts  experts per adapter (slots are adapter * n_experts + expert)
 *   scales, ws, ws_bytes, stream  as for lora_apply, with
 *              lora_moe_workspace_bytes(T * top_k)
 * Up to 256 pairs take one launch (the slots are formed and grouped inside
 * the delta kernel); beyond, three (pair slots, plan, delta).  A token's
 * adapter id below -1, an expert outside [0, n_experts) or a slot past the
 * pool raises the sticky LORA_ERR_BAD_ID and leaves that pair's row
 * untouched; an empty slot raises LORA_ERR_NOT_LOADED.  Equal, bit for bit,
 * to lora_apply on x with each token's row repeated top_k times and ids set
 * to the pairs' slots.
 */
LORA_API int lora_apply_moe(lora_pool *pool, int target, const void *x, int ldx, void *y,
                   int ldy, const int32_t *lora_ids, const int32_t *topk_ids, int T,
                   int top_k, int n_experts, const float *scales, void *ws,
                   size_t ws_bytes, void *stream);

/* Workspace of lora_apply_moe for up to max_pairs (T * top_k) pairs on
 * `target` (0 for bad arguments). */
LORA_API size_t lora_moe_workspace_bytes(const lora_pool *pool, int target, int max_pairs);

/* ------------------------------------------ the layer with its delta fused */

/*
 * The whole projection layer with each row's adapter, y written once:
 *     y[t, n] = bf16( sum_k W[n, k] x[t, k] + scales[a] * (B_a (A_a x[t]))[n] ),
 * a = ids[t]; rows with no adapter (id -1, a bad id, an empty slot, rank 0 on
 * this target) get the base term alone.  This is y = xW + (x A_i) B_i alpha/r
 * of "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU", section "Why
 * can't you just merge LoRA weights into the base model?", with W stored as
 * the d_out x d_in matrix of the column form W.x ("Serving Many LoRA Adapters
 * From One Base Model", section "How it works").  The delta is accumulated in
 * fp32 together with the base product and rounded once; unlike lora_apply, y
 * is only written.
 *   x, ldx     device bf16 [T, ldx], ldx >= d_in, multiple of 8
 *   W, ldw     device bf16 [d_out, ldw] row-major (one row per output
 *              feature), ldw >= d_in, multiple of 8; caller-owned, read only
 *   y, ldy     device bf16 [T, ldy], ldy >= d_out, multiple of 8; written;
 *              may overlap neither x nor W
 *   ids, scales, T, stream  as for lora_apply
 *   ws, ws_bytes  device workspace of at least lora_linear_workspace_bytes
 *              (the plan, then v = A_a x[t] in fp32)
 * Two launches for up to 256 rows (the shrink, then one tensor-core kernel
 * that streams W and adds the delta inside its accumulator), three beyond
 * (plan, shrink, that kernel).  Errors: as for lora_apply, and
 * LORA_ERR_INVALID_ARG for overlapping x / W / y.  The sticky device status
 * reports bad ids and empty slots as for lora_apply.
 */
LORA_API int lora_linear(lora_pool *pool, int target, const void *x, int ldx, const void *W,
                int ldw, void *y, int ldy, const int32_t *ids, const float *scales,
                int T, void *ws, size_t ws_bytes, void *stream);

/*
 * The second half of lora_linear for callers that keep v = A_a x[t] (from
 * lora_shrink): y[t] = bf16( W x[t] + scales[a] * B_a v[t, 0:r_a] ), one
 * launch, no workspace.  v, ldv as lora_expand takes them (device fp32
 * [T, ldv], ldv >= r_max, 4-byte aligned; rows without an adapter are not
 * read); the other arguments as for lora_linear.  lora_shrink followed by
 * lora_linear_expand gives y bit-identical to lora_linear.
 */
LORA_API int lora_linear_expand(lora_pool *pool, int target, const void *x, int ldx,
                       const void *W, int ldw, const float *v, int ldv, void *y,
                       int ldy, const int32_t *ids, const float *scales, int T,
                       void *stream);

/* Workspace of lora_linear for up to max_tokens rows on `target` (0 for bad
 * arguments). */
LORA_API size_t lora_linear_workspace_bytes(const lora_pool *pool, int target, int max_tokens);

/*
 * The delta for a batch given as contiguous segments (rows seg_offsets[s] ..
 * seg_offsets[s+1]-1 use slot seg_slot[s]): the segmented gather-and-multiply
 * of "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU", section "How does
 * one batch run 30 different adapters at once?", whose last paragraph notes
 * that prefill is compute-bound -- long segments therefore run on the tensor
 * cores, short ones on the decode kernel.  Arguments as lora_plan_segments
 * and lora_apply_plan; the result is that of lora_plan_segments followed by
 * lora_apply_plan.
 */
LORA_API int lora_apply_segments(lora_pool *pool, int target, const void *x, int ldx,
                        void *y, int ldy, const int32_t *seg_offsets,
                        const int32_t *seg_slot, int S, const float *scales,
                        int T, void *ws, size_t ws_bytes, void *stream);

/*
 * The two halves of the delta -- the adapter "shrink" (v = A_a x, rank r_a
 * out of d_in) and "expand" (y += scale B_a v) steps that "Multi-LoRA
 * Serving: Sharing One GPU Across Adapters" names in its section "MoE Models
 * Raise the Bar" -- for callers that keep v = A_a x[t]:
 *   lora_shrink writes v[t, 0:r_max] (fp32, device [T, ldv], ldv >= r_max;
 *   entries r_a..r_max-1 are written as 0) for every row with an adapter,
 *   and leaves other rows of v untouched.
 *   lora_expand adds scales[a] * B_a v[t, 0:r_a] to y[t] in place.
 * lora_shrink followed by lora_expand gives bit-identical y to lora_apply:
 * both use the same reduction order.  Like lora_apply, batches of at most
 * 256 rows are grouped inside the kernel and leave ws unwritten.
 */
LORA_API int lora_shrink(lora_pool *pool, int target, const void *x, int ldx,
                const int32_t *ids, int T, float *v, int ldv, void *ws,
                size_t ws_bytes, void *stream);

LORA_API int lora_expand(lora_pool *pool, int target, const float *v, int ldv, void *y,
                int ldy, const int32_t *ids, const float *scales, int T,
                void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------- no-allocation variant */

/* Largest batch (T) that lora_apply_noalloc accepts. */
#define LORA_NOALLOC_MAX_TOKENS 4096

/*
 * lora_apply for callers that cannot allocate device memory.  The web pages
 * this library follows have no counterpart of this call; it exists because
 * some callers cannot provide the plan workspace that lora_apply takes: their
 * device memory is owned by an allocator they must not go around (a
 * framework's caching allocator, a serving runtime that sizes every buffer up
 * front), or they run in a loop that cannot afford the device-wide
 * synchronisation that cudaMalloc / cudaFree may cause.
 *
 * The call computes exactly what lora_apply computes (bit for bit), with the
 * same arguments minus ws / ws_bytes.  Batches of at most 256 rows take one
 * launch that needs no plan, as in lora_apply.  Larger batches keep their
 * plan in one fixed array of device memory compiled into the library
 * (137,472 bytes, enough for LORA_NOALLOC_MAX_TOKENS rows); every GPU that loads
 * the library holds that array until the process exits.  The call itself
 * allocates nothing.
 *   - T > LORA_NOALLOC_MAX_TOKENS returns LORA_ERR_WORKSPACE (nothing runs).
 *   - The first call on a device looks up the array's device address (a
 *     runtime query, done with that device current, and again after a device
 *     reset or from another driver context).
 *   - All calls of more than 256 rows share the one array, which keeps the
 *     last call's plan.  No part of it needs clearing (each call rewrites
 *     everything it reads), but such calls that overlap on the GPU -- on
 *     different streams, or on different pools of the same device -- race on
 *     it and must be serialised by the caller.
 */
LORA_API int lora_apply_noalloc(lora_pool *pool, int target, const void *x, int ldx, void *y,
                                int ldy, const int32_t *ids, const float *scales, int T,
                                void *stream);

/* ------------------------------------------------------------ diagnostics */

/*
 * Synchronise stream, then read and clear the pool's sticky device status
 * (LORA_OK when no device-side error happened since the last read) into
 * *device_status.  The pages define no error channel; this one is the
 * library's own: device-side checks (an id outside [-1, n_slots), a slot
 * not loaded, a bounded wait that ran out) never fault, they record their
 * code here (the first one wins) and leave the affected rows untouched.
 * Returns LORA_ERR_INVALID_ARG for a null pool or device_status,
 * LORA_ERR_CUDA if the synchronisation fails.
 */
LORA_API int lora_get_error(lora_pool *pool, int *device_status, void *stream);

/* Number of kernels this library has launched in this process. */
LORA_API uint64_t lora_kernel_launches(void);

/*
 * Wall-clock limit of the decode kernel's bounded waits (for a stage of its
 * copy ring), in nanoseconds, for the launches that follow; 0 restores the default of one second.  A wait that
 * runs out sets LORA_ERR_TIMEOUT in the pool's sticky status, leaves the
 * rows that needed the data untouched and lets the kernel finish; it never
 * faults.  Tests lower it to reach that path quickly.
 */
LORA_API void lora_set_wait_limit_ns(uint64_t ns);

/*
 * Test of the bounded waits (no use outside tests).  Launches the decode
 * kernel of lora_apply for a batch of T <= 256 rows (arguments as for
 * lora_apply; no workspace) with its copy warp told to fill no stage, so
 * that the compute warps' first wait runs out after the limit set by
 * lora_set_wait_limit_ns.  Expected outcome: the launch completes,
 * lora_get_error then reads LORA_ERR_TIMEOUT, and y is left as it was.  No
 * copy is in flight when the wait gives up, and the CUDA context stays
 * usable.  Returns LORA_ERR_INVALID_ARG for T > 256.
 */
LORA_API int lora_selftest_stalled_apply(lora_pool *pool, int target, const void *x, int ldx,
                                void *y, int ldy, const int32_t *ids,
                                const float *scales, int T, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_B200_H */
