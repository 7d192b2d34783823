/*
 * lora_sgmv.h -- C ABI of the B200 (sm_100a) multi-LoRA delta library.
 *
 * What it computes.  "Serving several LoRAs, ControlNet and IP-Adapter"
 * (AI-infra handbook), section "LoRA: merged or alongside": a LoRA adds a
 * low-rank increment W' = W + B A to a weight (A is r x d, B is d x r, r from
 * 8 to 128); served unmerged, each adapted layer adds x A^T B^T to x W^T.
 * For a token row x[n] and an adapter a of rank r_a this library adds
 *
 *     y[n] += s * B[a] (A[a] x[n])          (shrink d_in -> r_a, expand r_a -> d_out)
 *
 * in place to y.  A mixed batch is grouped by adapter index, each group runs
 * its own low-rank product inside one kernel, and the results land back in the
 * original token order (same page, exercise 2's answer; the segmented
 * gather-matrix-vector kernels of Punica, "Punica: multi-tenant LoRA serving",
 * contribution 1).  Several LoRAs stacked on one request add their deltas
 * (same page, table row "Stacking several LoRAs"); the weight s of each is a
 * runtime scalar (same page: the LoRA weight may change every denoising step).
 *
 * Conventions common to every entry point
 * ---------------------------------------
 * - Types: activations and adapter weights are bf16 (passed as void*), the
 *   rank-r intermediate V is fp32, all sums are accumulated in fp32 and each
 *   output element of y is rounded to bf16 exactly once (round to nearest even).
 * - Memory: every pointer except `pool` itself and the ones documented as host
 *   pointers is DEVICE memory owned by the caller.  The library allocates
 *   nothing and keeps no state between calls; all scratch lives in the
 *   caller's workspace `ws` (see lora_workspace_size).
 * - Layout: X is [N, d_in] row-major with leading dimension ldx (elements),
 *   Y is [N, d_out] with ldy.  Adapter pool (lora_pool): adapter a's A is
 *   [rank[a], d_in] row-major starting at element A_off[a] of pool->A, its B is
 *   [d_out, rank[a]] row-major starting at element B_off[a] of pool->B; adapters
 *   may have different ranks and are never padded to the maximum rank.
 * - Requirements (checked on the host before anything is launched):
 *   d_in and d_out multiples of 8; 8 <= max_rank <= 128, max_rank % 8 == 0;
 *   1 <= n_adapters <= LORA_MAX_ADAPTERS; ldx >= d_in and ldy >= d_out, both
 *   multiples of 8; X, Y, pool->A, pool->B 16-byte aligned; ws 256-byte aligned
 *   and at least lora_workspace_size(...) bytes.  Violations return
 *   LORA_ERR_INVALID_ARG or LORA_ERR_UNSUPPORTED and launch nothing.
 * - Requirements checked on the device (the metadata lives in device memory):
 *   adapter ids in [0, n_adapters) (or -1 = no adapter where stated),
 *   rank[a] a multiple of 8 in [8, max_rank], A_off[a] and B_off[a]
 *   non-negative multiples of 8 whose matrices end inside A_elems / B_elems,
 *   segment/request offsets non-decreasing and
 *   within [0, N].  A violation sets a bit in the workspace's error word and
 *   skips the affected work (those rows keep their old y); it never traps.
 *   Read and clear the word with lora_get_error.
 * - Asynchrony: every compute entry point only enqueues kernels on `stream`
 *   (a cudaStream_t; NULL = the legacy default stream) and returns.  Calls
 *   that share one workspace must be ordered (same stream or events).
 * - Thread safety: the library is stateless; concurrent calls with distinct
 *   workspaces are safe.
 * - Overlap with the previous kernel: kernels are launched with programmatic
 *   dependent launch (environment variable LORA_SGMV_NO_PDL=1 turns it off),
 *   so one may start while the kernel before it on the stream finishes.  Each
 *   waits for that kernel before touching X, Y, V, W or the workspace; the
 *   decode kernel of lora_bgmv reads ids and the adapter pool before waiting.
 *   This matters only when the preceding kernel itself releases its dependents
 *   early (griddepcontrol.launch_dependents) -- such a kernel must not write
 *   ids or the pool.  Copies (cudaMemcpyAsync) and ordinary kernels before a
 *   call are always complete before it starts.
 */
#ifndef LORA_SGMV_H
#define LORA_SGMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

#define LORA_MAX_RANK 128
#define LORA_MAX_ADAPTERS 32768
#define LORA_MAX_ADS_PER_REQ 8
#define LORA_MAX_PROJ 4          /* projections sharing one input (lora_sgmv_shrink_proj, _apply_proj) */

/* Status codes.  Host-side codes are returned directly; device-side codes are
 * bits of the workspace error word returned by lora_get_error (OR-ed). */
typedef enum {
    LORA_OK = 0,
    LORA_ERR_INVALID_ARG = 1,   /* host: null pointer, negative size, bad leading dimension */
    LORA_ERR_UNSUPPORTED = 2,   /* host: shape, rank bound, alignment or limit not supported */
    LORA_ERR_BAD_ADAPTER = 4,   /* device: adapter id, rank or pool offset out of range */
    LORA_ERR_BAD_SEGMENT = 8,   /* device: segment/request offsets decreasing or outside [0, N] */
    LORA_ERR_CUDA = 16,         /* host: a CUDA runtime call (launch, copy) failed */
    LORA_ERR_WORKSPACE = 32,    /* host: workspace null, misaligned or too small */
    LORA_ERR_TIMEOUT = 64       /* device: a pipeline wait inside a kernel expired (work skipped) */
} lora_status;

/* One projection's resident adapter pool ("all LoRAs stay resident", same
 * page, section "Placement").  The struct itself is a HOST object read during
 * the call; every pointer in it is device memory. */
typedef struct lora_pool {
    const void *A;          /* bf16, packed A matrices                                  */
    const void *B;          /* bf16, packed B matrices                                  */
    const int64_t *A_off;   /* [n_adapters] element offset of adapter a's A in A        */
    const int64_t *B_off;   /* [n_adapters] element offset of adapter a's B in B        */
    const int32_t *rank;    /* [n_adapters] rank of adapter a                           */
    int64_t A_elems;        /* elements in A: adapter a must satisfy A_off[a] + rank[a]*d_in <= A_elems */
    int64_t B_elems;        /* elements in B: B_off[a] + d_out*rank[a] <= B_elems       */
    int32_t n_adapters;
    int32_t d_in;
    int32_t d_out;
    int32_t max_rank;       /* an upper bound of rank[a] over the pool (host-checked)   */
} lora_pool;

/* Operation codes for lora_workspace_size. */
typedef enum {
    LORA_OP_BGMV = 0,
    LORA_OP_SGMV_SHRINK = 1,
    LORA_OP_SGMV_EXPAND = 2,
    LORA_OP_APPLY_MULTI = 3,
    LORA_OP_ROUTE = 4,
    LORA_OP_MERGE = 5,
    LORA_OP_LINEAR = 6,
    LORA_OP_APPLY_PROJ = 7      /* max_rank = the projections' max_rank summed */
} lora_op;

/* Bytes of workspace `op` needs for N token rows.  n_items = n_seg for the
 * SGMV ops, n_req for lora_apply_multi, ignored otherwise; max_ads_per_req is
 * used by lora_apply_multi only.  For LORA_OP_MERGE, N = d_out (the rows of
 * the weight being merged into).  Pure host function, no CUDA call.  Returns
 * 0 for arguments the corresponding entry point would reject. */
LORA_API size_t lora_workspace_size(int op, int32_t N, int32_t n_adapters, int32_t d_in, int32_t d_out,
                           int32_t max_rank, int32_t n_items, int32_t max_ads_per_req);

/* Number of kernels one call of `op` launches for these sizes (pure host
 * function): lets a caller budget a CUDA graph or count launches.  0 for
 * arguments the entry point would reject or that launch nothing (N == 0), and
 * for LORA_OP_APPLY_PROJ, whose count depends on the pools (see
 * lora_sgmv_apply_proj). */
LORA_API int lora_kernel_launches(int op, int32_t N, int32_t n_adapters, int32_t d_in, int32_t n_items);

/* Clear the workspace's error word (cudaMemsetAsync of its 256-byte header on
 * `stream`).  Call once on a fresh workspace. */
LORA_API lora_status lora_workspace_init(void *ws, void *stream);

/* Synchronise `stream`, read the workspace's error word, clear it, and return
 * the device-side status bits (LORA_ERR_BAD_ADAPTER | LORA_ERR_BAD_SEGMENT) or
 * LORA_OK; LORA_ERR_CUDA if the copy itself fails. */
LORA_API int lora_get_error(void *ws, void *stream);

/*
 * lora_route -- group an unsorted batch by adapter index (exercise 2's answer
 * on the handbook page: group the activations by LoRA index, then put the
 * results back in the original order).  A stable counting sort:
 *   perm[0..n_valid)   token indices grouped by adapter (ascending id), in
 *                      original order within a group; tokens with id -1 are
 *                      left out;
 *   seg_ad[0..n_seg)   the distinct adapters present, ascending;
 *   seg_off[0..n_seg]  group bounds in perm (seg_off[0] = 0);
 *   *n_seg_out         n_seg (device int32).
 * Capacities: perm >= N, seg_off >= min(N, n_adapters) + 1, seg_ad >=
 * min(N, n_adapters).  ids: device int32 [N], -1 = no adapter; any other id
 * outside [0, n_adapters) sets LORA_ERR_BAD_ADAPTER and is left out.
 */
LORA_API lora_status lora_route(const int32_t *ids, int32_t N, int32_t n_adapters, int32_t *perm,
                       int32_t *seg_off, int32_t *seg_ad, int32_t *n_seg_out,
                       void *ws, size_t ws_bytes, void *stream);

/*
 * lora_bgmv -- decode: one token per request, each with its own adapter.
 *   Y[n] += scale * B[ids[n]] A[ids[n]] X[n]   for ids[n] != -1
 * ids: device int32 [N], unsorted, -1 = no adapter (row untouched).  The
 * grouping runs inside the call: tokens are sorted stably by adapter and cut
 * into items of up to 16 tokens, and each item's A and B rows cross HBM once
 * (the items of one adapter re-read them from L2).  For N <= 8192,
 * n_adapters <= 8192 and d_in <= 32768 (and a grouping that fits the kernel's
 * shared memory) the whole call is one kernel launch (thread-block clusters of
 * 8 CTAs; only the workspace's error word is used); larger calls take a
 * three-kernel path through the workspace.
 */
LORA_API lora_status lora_bgmv(const void *X, int64_t ldx, void *Y, int64_t ldy, const lora_pool *pool,
                      const int32_t *ids, int32_t N, float scale,
                      void *ws, size_t ws_bytes, void *stream);

/*
 * lora_sgmv_shrink -- prefill, tokens already grouped into segments:
 *   V[n][j] = sum_i A[a][j][i] X[n][i],  j < rank[a],  a = seg_ad[k],
 *   for seg_off[k] <= n < seg_off[k+1].
 * V: device fp32 [N, ldv], ldv >= max_rank.  Entries j >= rank[a] and rows
 * outside every segment are not written.  seg_off: device int32 [n_seg+1],
 * non-decreasing, within [0, N]; empty segments are allowed.  seg_ad: device
 * int32 [n_seg].
 */
LORA_API lora_status lora_sgmv_shrink(const void *X, int64_t ldx, float *V, int64_t ldv,
                             const lora_pool *pool, const int32_t *seg_off, const int32_t *seg_ad,
                             int32_t n_seg, int32_t N, void *ws, size_t ws_bytes, void *stream);

/*
 * lora_sgmv_shrink_proj -- the shrinks of several projections that read the
 * same input (attention's Q, K and V; an MLP's gate and up), done as one
 * shrink over their A rows stacked along the rank axis, so X is read once
 * ("Serving several LoRAs, ControlNet and IP-Adapter", self-test answer 1:
 * a LoRA attaches to the Q, K, V and O projections, sometimes the MLP):
 *   V[n][c_p + j] = sum_i A_p[a][j][i] X[n][i],  j < rank_p[a],  a = seg_ad[k],
 * for seg_off[k] <= n < seg_off[k+1] and every projection p < n_proj, where
 * A_p is pools[p]'s A and c_p = pools[0].max_rank + ... + pools[p-1].max_rank.
 * Projection p's expand is then lora_sgmv_expand(V + c_p, ldv, Y_p, ...,
 * &pools[p], ...).
 * pools: host array of n_proj (1 .. LORA_MAX_PROJ) pools with one d_in and
 * one n_adapters (adapter a of every pool belongs to the same fine-tune);
 * their d_out, ranks and storage may differ.  V: device fp32 [N, ldv],
 * ldv >= sum of the pools' max_rank; entries past an adapter's rank and rows
 * outside every segment are not written.  Segment arguments and workspace
 * (LORA_OP_SGMV_SHRINK, sized with any of the pools' max_rank) as for
 * lora_sgmv_shrink.  Long segments take one plan launch plus one tensor-core
 * launch per group of consecutive projections whose max_ranks sum to at most
 * 256; short ones take the plan plus one CUDA-core shrink per projection.
 * A bad adapter id is reported once per projection pool it fails in.
 */
LORA_API lora_status lora_sgmv_shrink_proj(const void *X, int64_t ldx, float *V, int64_t ldv,
                             const lora_pool *pools, int32_t n_proj, const int32_t *seg_off,
                             const int32_t *seg_ad, int32_t n_seg, int32_t N,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * lora_sgmv_apply_proj -- the whole delta of projections that share their input
 * (the shrink of lora_sgmv_shrink_proj, then every projection's expand):
 *   Y_p[n] += scale[p] * B_p[a] (A_p[a] X[n]),  a = seg_ad[k], seg_off[k] <= n < seg_off[k+1],
 * for p < n_proj.  One plan serves the shrink and all the expands, and the
 * intermediate stays in the workspace: 1 + (tensor-core shrink launches) + 1
 * kernels on the tensor-core path (long segments: every projection's expand runs
 * in one launch, the GPU's CTAs split among the projections in proportion to
 * their outputs), 1 + 2 n_proj on the CUDA-core path.  Y, ldy, scale: HOST arrays of n_proj entries (Y[p] a device
 * bf16 [N, ldy[p]] matrix, ldy[p] >= pools[p].d_out).  Pools and segments as
 * in lora_sgmv_shrink_proj.  Workspace: lora_workspace_size(LORA_OP_APPLY_PROJ,
 * N, n_adapters, d_in, 0, sum of the pools' max_rank, n_seg, 0).
 */
LORA_API lora_status lora_sgmv_apply_proj(const void *X, int64_t ldx, void *const *Y, const int64_t *ldy,
                             const lora_pool *pools, int32_t n_proj, const int32_t *seg_off,
                             const int32_t *seg_ad, int32_t n_seg, int32_t N, const float *scale,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * lora_linear_sgmv -- an adapted projection computed unmerged in one pass of
 * the tensor cores ("Serving several LoRAs, ControlNet and IP-Adapter",
 * section "LoRA: merged or alongside": served unmerged, the layer adds the
 * low-rank x A^T B^T to x W^T):
 *   Y[n][o] = sum_i W[o][i] X[n][i] + scale * sum_{j < rank[a]} B[a][o][j] V[n][j],
 *   V[n][j] = sum_i A[a][j][i] X[n][i],
 * for seg_off[k] <= n < seg_off[k+1], a = seg_ad[k]; seg_ad[k] = -1 means no
 * adapter (Y = W X only).  Rows outside every segment are not written.  Y is
 * OUTPUT ONLY (overwritten, not accumulated), rounded to bf16 once.
 * W: device bf16 [d_out, d_in] row-major (a torch Linear weight), leading
 * dimension ldw >= d_in, multiple of 8, 16-byte aligned; X [N, ldx] and
 * Y [N, ldy] as elsewhere; pool->d_in / d_out give the projection's shape.
 * Adapters may have any rank the pool allows (a multiple of 8 up to
 * max_rank): B is read through a tensor map when the rank is 16, 32, 64 or 128
 * and B_off[a] a multiple of it, and gathered with 16-byte copies otherwise.
 * A segment whose adapter fails the usual device checks gets Y = W X and sets
 * LORA_ERR_BAD_ADAPTER.  Workspace: lora_workspace_size(LORA_OP_LINEAR, N,
 * n_adapters, d_in, d_out, max_rank, n_seg, 0) (it holds s V).  Launches
 * three kernels (plan, tcgen05 shrink, tcgen05 projection).  Needs the
 * tensor-core path (B200): LORA_ERR_UNSUPPORTED where tensor maps cannot be
 * built for the given pointers and strides.
 */
LORA_API lora_status lora_linear_sgmv(const void *X, int64_t ldx, const void *W, int64_t ldw, void *Y, int64_t ldy,
                             const lora_pool *pool, const int32_t *seg_off, const int32_t *seg_ad,
                             int32_t n_seg, int32_t N, float scale, void *ws, size_t ws_bytes, void *stream);

/*
 * lora_sgmv_expand -- the second half of the segmented product:
 *   Y[n][o] += scale * sum_{j < rank[a]} B[a][o][j] V[n][j]
 * for every row n inside segment k (a = seg_ad[k]); other rows untouched.
 * Same segment arguments as lora_sgmv_shrink.
 */
LORA_API lora_status lora_sgmv_expand(const float *V, int64_t ldv, void *Y, int64_t ldy,
                             const lora_pool *pool, const int32_t *seg_off, const int32_t *seg_ad,
                             int32_t n_seg, int32_t N, float scale,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * lora_apply_multi -- requests that stack several co-occurring adapters
 * ("Co-occurrence Patterns of LoRA Adapters in Production Diffusion Model
 * Inference Services", abstract: multi-adapter requests; handbook table row
 * "Stacking several LoRAs"):
 *   Y[n] += sum_{p in ad_off[q]..ad_off[q+1]} ad_scale[p] * B[ad_id[p]] A[ad_id[p]] X[n]
 * for req_off[q] <= n < req_off[q+1].  All of a row's deltas are summed in
 * fp32 before the single bf16 rounding of y.  req_off, ad_off: device int32
 * [n_req+1], non-decreasing; ad_id: device int32; ad_scale: device fp32.
 * A request may list at most max_ads_per_req (<= LORA_MAX_ADS_PER_REQ)
 * adapters (device-checked: LORA_ERR_BAD_SEGMENT); an adapter listed twice
 * counts twice.
 */
LORA_API lora_status lora_apply_multi(const void *X, int64_t ldx, void *Y, int64_t ldy,
                             const lora_pool *pool, const int32_t *req_off, const int32_t *ad_off,
                             const int32_t *ad_id, const float *ad_scale, int32_t n_req, int32_t N,
                             int32_t max_ads_per_req, void *ws, size_t ws_bytes, void *stream);

/*
 * lora_apply_multi_static -- lora_apply_multi without a caller workspace.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory: code inside a region captured into a
 * CUDA graph where allocation is not allowed, a process whose device memory
 * belongs to another allocator, or a plugin that is handed only its input and
 * output buffers.  It computes exactly what lora_apply_multi computes (same
 * arguments minus the workspace, same kernels) and allocates nothing: no
 * cudaMalloc, cudaFree or allocating library call.
 *
 * Its scratch (the work-group list, the error word and the fp32 rank-r
 * intermediate, N * max_ads_per_req * max_rank floats plus a few KB) lives in
 * one array of LORA_STATIC_SCRATCH_BYTES compiled into the library; every GPU
 * that loads the library holds those bytes until the process exits.  Calls
 * whose scratch would not fit return LORA_ERR_WORKSPACE and launch nothing
 * (use lora_apply_multi with a workspace instead).
 *
 * All calls share the one array and it keeps the last call's contents: each
 * call first clears the error word on `stream`, so calls that overlap on the
 * GPU (different streams without ordering, or several host threads) race on
 * the scratch and must not be issued.  The first call on a device looks up
 * the array's device address (cudaGetSymbolAddress, once per device, with the
 * device current); make that first call before any stream capture.
 *
 * err_out: optional device uint32; when non-null the call's device-side status
 * bits (as lora_get_error would return them) are copied there on `stream`.
 */
#define LORA_STATIC_SCRATCH_BYTES (32u << 20)
LORA_API lora_status lora_apply_multi_static(const void *X, int64_t ldx, void *Y, int64_t ldy,
                                             const lora_pool *pool, const int32_t *req_off,
                                             const int32_t *ad_off, const int32_t *ad_id,
                                             const float *ad_scale, int32_t n_req, int32_t N,
                                             int32_t max_ads_per_req, uint32_t *err_out, void *stream);

/* Library version string (host). */
/*
 * lora_merge -- fold an adapter into a base weight, or take it out again.
 *
 * "Serving several LoRAs, ControlNet and IP-Adapter", section "LoRA: merged or
 * alongside": a merged LoRA is W' = W + B A in the weight itself (no per-token
 * cost), and switching adapters means unmerging one and merging another.  For
 * the base weight W [pool->d_out, pool->d_in] (bf16, row-major, leading
 * dimension ldw, a multiple of 8; 16-byte aligned; updated in place) and
 * adapter `adapter` of the pool:
 *     W[o][i] <- bf16( W[o][i] + scale * sum_j B[a][o][j] * A[a][j][i] )
 * accumulated in fp32 with one bf16 rounding per element.  Unmerging is the
 * same call with -scale; as W is rounded each time, merge then unmerge
 * restores W to within bf16 rounding, not bit for bit.
 *
 * ws: at least lora_workspace_size(LORA_OP_MERGE, pool->d_out, ...) bytes
 * (the error word sits at its start, as for the other ops).  Errors: the
 * host checks of the other entry points, and `adapter` outside
 * [0, n_adapters) -> LORA_ERR_INVALID_ARG; an adapter whose device metadata is
 * invalid leaves W unchanged and sets LORA_ERR_BAD_ADAPTER in the error word.
 * Launches two kernels (adapter preparation, the tensor-core expand over W's
 * tiles), or three on the CUDA-core path (d_out < 128: preparation, tiling,
 * expand).
 */
LORA_API lora_status lora_merge(void *W, int64_t ldw, const lora_pool *pool, int32_t adapter, float scale,
                                void *ws, size_t ws_bytes, void *stream);

/*
 * Resident adapter pool with on-demand loads -- the system layer around the ops.
 *
 * "Serving several LoRAs, ControlNet and IP-Adapter", section "Placement": the
 * adapters in use stay resident on the GPU; the rest wait in host memory and are
 * brought in when a batch needs them.  The caller owns the pool's device storage:
 * a lora_pool `storage` of n_slots = storage->n_adapters fixed-size slots, with
 * A_elems >= n_slots * max_rank * d_in, B_elems >= n_slots * d_out * max_rank and
 * A_off, B_off (int64) and rank (int32) arrays of n_slots.  Slot s holds one
 * adapter at A_off[s] = s * max_rank * d_in, B_off[s] = s * d_out * max_rank; an
 * empty slot has rank 0 (the ops reject it).  `storage` itself, with its slots as
 * adapter indices, is the pool the ops take.
 *
 * lora_pm_create: host state for `storage` (n_slots <= LORA_MAX_ADAPTERS); writes
 *   the offsets and empties every slot, on `stream`.  Free with lora_pm_destroy
 *   (host state only; the storage stays the caller's).
 * lora_pm_register: the host copy of adapter `key` (>= 0): A [rank, d_in] and
 *   B [d_out, rank] bf16, row-major, in host memory that stays valid while a copy
 *   of it may be in flight (pinned memory makes the copies asynchronous).
 *   Registering a key again replaces its copy and marks it for reloading.
 * lora_pm_acquire: makes keys[0..n) resident and writes each one's slot to
 *   slots[i] (NULL allowed: preloading).  A resident key keeps its slot; a
 *   missing one takes a free slot, else the least recently used slot that no key
 *   of this call occupies; its A and B are copied in and its rank set, all on
 *   `stream`, so later work on that stream sees them (work on other streams must
 *   synchronise with it; a slot being replaced must not be in use there).
 *   *n_loaded (optional) = adapters copied.  Unregistered key ->
 *   LORA_ERR_INVALID_ARG, more distinct keys than slots -> LORA_ERR_UNSUPPORTED,
 *   both before anything changes.  Calls on one manager are serialised.
 */
typedef struct lora_pool_mgr lora_pool_mgr;
LORA_API lora_status lora_pm_create(const lora_pool *storage, void *stream, lora_pool_mgr **out);
LORA_API void lora_pm_destroy(lora_pool_mgr *m);
LORA_API lora_status lora_pm_register(lora_pool_mgr *m, int64_t key, const void *A_host, const void *B_host,
                                      int32_t rank);
LORA_API lora_status lora_pm_acquire(lora_pool_mgr *m, const int64_t *keys, int32_t n, int32_t *slots,
                                     int32_t *n_loaded, void *stream);

/*
 * Co-occurrence preloading ("Co-occurrence Patterns of LoRA Adapters in
 * Production Diffusion Model Inference Services", abstract: requests that
 * combine adapters do so in recurring patterns, and preloading the top-k
 * co-occurring adapters covers most of them).
 *
 * lora_pm_observe: records one request's adapter keys[0..n) (duplicates count
 *   once): every pair of distinct keys in it co-occurred once more.  Host only.
 * lora_pm_set_preload: top_k > 0 makes every later lora_pm_acquire, after the
 *   batch's own keys, also bring in the top_k partners of each batch key (most
 *   requests in common first, ties to the smaller key) that are registered, not
 *   resident and not in the batch -- into free slots, else least recently used
 *   slots that no key of this acquire holds, until none is left; the copies go
 *   on the acquire's stream like the batch's own.  0 (the default) turns it off.
 * lora_pm_preloaded: adapters the last acquire preloaded (-1 for a NULL manager).
 */
LORA_API lora_status lora_pm_observe(lora_pool_mgr *m, const int64_t *keys, int32_t n);
LORA_API lora_status lora_pm_set_preload(lora_pool_mgr *m, int32_t top_k);
LORA_API int32_t lora_pm_preloaded(lora_pool_mgr *m);

/*
 * lora_test_stall -- testing hook for the timeout path (no counterpart on the
 * pages).  While `stall` is non-zero, the kernels that stream their operands
 * through a load pipeline (the tensor-core kernels of the SGMV, multi-adapter,
 * projection and merge calls) issue no loads
 * at all, and every wait inside a kernel gives up after `wait_seconds`
 * (clamped to [1 us, 2 s]): such a call changes none of its outputs, reports
 * LORA_ERR_TIMEOUT through lora_get_error, and leaves the device ready for the
 * next call.  stall = 0 restores normal operation (waits bounded by 2 s).
 * Process-wide; not for production use.
 */
LORA_API void lora_test_stall(int stall, double wait_seconds);

LORA_API const char *lora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LORA_SGMV_H */
