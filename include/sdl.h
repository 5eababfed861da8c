/*
 * sdl.h -- C ABI of libsdl, block-sparse attention for diffusion-LLM
 * denoising steps on NVIDIA B200 (sm_100a).
 *
 * The operations follow "Step-dLLM: Adaptive Step-aware Sparse Attention for
 * Efficient Diffusion LLM Inference" (mlinfo.pages.dev, abstract): at anchor
 * steps of the denoising trajectory a block-sparse mask is rebuilt under one
 * head-adaptive global budget, it is reused until the next anchor, and a
 * fused block-sparse attention kernel evaluates bidirectional attention on
 * the kept blocks only; dense FlashAttention is the baseline.  The abstract
 * does not define the block score or the selection rule; the readings this
 * library implements are stated at each call.
 *
 * Conventions for every call:
 *   - All pointers named q, k, v, o, lse, scores, row_ptr, col_idx, mask_u8
 *     and workspace are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory per call.  Its own device state is static:
 *     one status word, the fixed scratch array of sdl_select_mask_noalloc,
 *     and a ring of 64 tile counters for the attention kernels (each launch
 *     takes the next one and its last CTA resets it, so at most 64 attention
 *     launches may be in flight on one device at a time; a launch that found
 *     its counter shared is reported as SDL_ERR_OVERLAP by
 *     sdl_last_device_status).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).  Argument errors are returned
 *     before anything is launched; a launch failure returns SDL_ERR_CUDA and
 *     sdl_last_cuda_error() gives the cudaError_t.
 *   - Q is [B, L, H, d], K and V are [B, L, H_kv, d] and O is [B, L, H, d],
 *     each addressed through element strides (b, t, h) with d contiguous.
 *   - bf16 tensors must start on 16-byte boundaries and have strides that are
 *     multiples of 8 elements (the tensor-memory-access unit's rule); a zero
 *     stride (a broadcast view) is refused on any axis with more than one
 *     index (SDL_ERR_INVALID_ARG).
 *   - No exception or abort crosses the ABI.
 */
#ifndef SDL_H
#define SDL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SDL_OK = 0,
  SDL_ERR_INVALID_ARG = 1, /* null pointer, bad size or stride, bad sparsity */
  SDL_ERR_UNSUPPORTED = 2, /* valid but not implemented: d, block, L % block */
  SDL_ERR_CAPACITY = 3,    /* col_capacity below the budget */
  SDL_ERR_WORKSPACE = 4,   /* workspace null or smaller than required */
  SDL_ERR_CUDA = 5,        /* a CUDA call failed; see sdl_last_cuda_error() */
  SDL_ERR_TIMEOUT = 6,     /* a kernel's bounded wait ran out (device status) */
  SDL_ERR_BAD_MASK = 7,    /* a col_idx entry out of range or out of order */
  SDL_ERR_OVERLAP = 8      /* two attention launches in flight shared a tile counter
                              (device status; their outputs are not trustworthy) */
} sdl_status;

typedef enum { SDL_BF16 = 0, SDL_FP32 = 1 } sdl_dtype;

typedef struct {
  int32_t B;     /* batch (independent sequences) */
  int32_t H;     /* query heads */
  int32_t H_kv;  /* key/value heads; H % H_kv == 0, query head h reads KV head h / (H / H_kv) */
  int32_t L;     /* tokens per sequence; L % block == 0 */
  int32_t d;     /* head dimension: 64 or 128 */
  int32_t block; /* block size in tokens: 64 or 128 */
  int32_t dtype; /* sdl_dtype of q, k, v, o */
  int32_t reserved;
  int64_t q_strides[3]; /* element strides of the (b, t, h) axes */
  int64_t k_strides[3];
  int64_t v_strides[3];
  int64_t o_strides[3];
} sdl_shape;

/* Blocks kept for the whole call: B * floor((1 - sparsity) * H * nb^2 + 0.5),
 * nb = L / block.  The budget is per batch element (each sequence is its own
 * problem) and counts the H * nb diagonal blocks that are always kept.
 * Returns -1 for a bad shape, sparsity outside [0, 1), or a per-sequence
 * budget below H * nb.  Host-only; launches nothing. */
int64_t sdl_mask_budget(const sdl_shape* shape, double sparsity);

/* Workspace bytes that sdl_block_scores / sdl_select_mask need (0 on a bad shape). */
size_t sdl_scores_workspace_bytes(const sdl_shape* shape);
size_t sdl_select_workspace_bytes(const sdl_shape* shape);

/* Block scores (anchor steps).  The Step-dLLM abstract refreshes the mask at
 * anchor steps but leaves the block-importance estimate open; this call
 * implements mean pooling of Q and K over each block, the pooled product and
 * a row softmax:
 *   Qbar[b,h,i,:] = mean_{t in block i} Q[b,t,h,:],  Kbar likewise per KV head,
 *   scores[b,h,i,j] = softmax_j(scale * Qbar[b,h,i,:] . Kbar[b,h/g,j,:]).
 * scores: fp32 [B, H, nb, nb] row-major.  scale <= 0 means 1/sqrt(d).
 * workspace: at least sdl_scores_workspace_bytes(shape) bytes (pooled Q, K). */
sdl_status sdl_block_scores(const void* q, const void* k, const sdl_shape* shape, float scale,
                            float* scores, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Mask selection (anchor steps): the head-adaptive global budget of the
 * Step-dLLM abstract.  Per batch element, every diagonal block (i, i) of every
 * head is kept, and the rest of the budget goes to the largest off-diagonal
 * scores of ALL heads together (ties: lower flat index (h*nb + i)*nb + j
 * first), so heads whose mass is concentrated in few blocks keep few blocks.
 * Output is CSR over query-block rows r = (b*H + h)*nb + i:
 *   row_ptr: int32 [B*H*nb + 1], col_idx: int32 [budget], ascending j per row.
 * col_capacity must be >= sdl_mask_budget() (else SDL_ERR_CAPACITY).
 * mask_u8 (nullable): uint8 [B, H, nb, nb], 1 = kept.
 * workspace: at least sdl_select_workspace_bytes(shape) bytes; its contents
 * on entry do not matter.  Only shape->B, H, L, block are read. */
sdl_status sdl_select_mask(const float* scores, const sdl_shape* shape, double sparsity,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                           uint8_t* mask_u8, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Scope of the mask budget.  SDL_BUDGET_SEQUENCE is the Step-dLLM abstract's
 * head-adaptive global budget (sdl_select_mask).  SDL_BUDGET_HEAD is the uniform
 * per-head budget of the prior methods the abstract compares against (SparseD
 * abstract): every head keeps floor((1 - s) * nb^2 + 0.5) blocks of its own. */
typedef enum { SDL_BUDGET_SEQUENCE = 0, SDL_BUDGET_HEAD = 1 } sdl_budget_scope;

/* Total kept blocks of a call under `scope` (the sum over sequences or heads),
 * or -1 when sparsity is outside [0, 1) or a budget is below its diagonal. */
int64_t sdl_mask_budget_scoped(const sdl_shape* shape, double sparsity, int scope);

/* Workspace bytes sdl_select_mask_scoped needs under `scope` (0 on a bad shape
 * or scope); for SDL_BUDGET_SEQUENCE it equals sdl_select_workspace_bytes. */
size_t sdl_select_workspace_bytes_scoped(const sdl_shape* shape, int scope);

/* sdl_select_mask with the budget taken per `scope`: for SDL_BUDGET_HEAD each
 * head's largest scores are taken among that head's own entries (the same rule
 * as sdl_select_mask applied to every head alone); outputs as sdl_select_mask,
 * with sdl_mask_budget_scoped entries, and a workspace of
 * sdl_select_workspace_bytes_scoped bytes. */
sdl_status sdl_select_mask_scoped(const float* scores, const sdl_shape* shape, double sparsity,
                                  int scope, int32_t* row_ptr, int32_t* col_idx,
                                  int64_t col_capacity, uint8_t* mask_u8, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ---- Column-sparse attention (the PulseCol abstract) ------------------------
 * Every query head keeps a set of key tokens ("columns") for all of its query
 * rows; the set is chosen at refresh steps and reused between them.  The
 * abstract gives no estimator or budget; this library's reading:
 *   sdl_col_scores:  S[b,h,u] = (1/nb) sum over query blocks i of
 *                    softmax over u of (scale * Qbar[b,h,i,:] . k[b,u,h/g,:]),
 *                    fp32 [B, H, L], Qbar the block means of Q (block = shape
 *                    block); workspace sdl_col_scores_workspace_bytes
 *   sdl_col_budget:  Lc = 64 * floor((1 - s) * L / 64 + 0.5) columns per head,
 *                    at least 64 and at most L (-1 on bad arguments)
 *   sdl_col_select:  cols int32 [B, H, Lc]: each head's Lc largest S, ties to
 *                    the lower u, ascending (col_capacity elements of room, at
 *                    least B*H*Lc, else SDL_ERR_CAPACITY)
 *   sdl_col_gather:  k_cols[b,c,h,:] = k[b, cols[b,h,c], h/g, :] and likewise
 *                    v, contiguous [B, Lc, H, d] of the shape's dtype (K/V
 *                    duplicated per query head under GQA)
 *   sdl_col_sparse_attn: O[b,t,h,:] = sum over c of softmax_c(scale * q_t .
 *                    k_cols[b,c,h,:]) v_cols[b,c,h,:] for every query token t,
 *                    optional LSE [B,H,L]; Lc a multiple of 64.  Q and O as in
 *                    sdl_dense_attn (the shape's k/v strides are ignored).
 * All asynchronous on `stream`; errors as the block-sparse calls. */
int64_t sdl_col_budget(const sdl_shape* shape, double sparsity);
size_t sdl_col_scores_workspace_bytes(const sdl_shape* shape);
sdl_status sdl_col_scores(const void* q, const void* k, const sdl_shape* shape, float scale,
                          float* col_scores, void* workspace, size_t workspace_bytes,
                          void* stream);
sdl_status sdl_col_select(const float* col_scores, const sdl_shape* shape, double sparsity,
                          int32_t* cols, int64_t col_capacity, void* stream);
sdl_status sdl_col_gather(const void* k, const void* v, const sdl_shape* shape,
                          const int32_t* cols, int32_t Lc, void* k_cols, void* v_cols,
                          void* stream);
sdl_status sdl_col_sparse_attn(const void* q, const void* k_cols, const void* v_cols,
                               const sdl_shape* shape, int32_t Lc, float scale, void* o,
                               float* lse, void* stream);

/* ---- Fused anchor step ------------------------------------------------------
 * sdl_block_scores, then sdl_select_mask (global budget per sequence, no
 * mask_u8), then, when `plan` is not NULL (64-token blocks only),
 * sdl_tile_plan, as one launch: the mask refresh of the Step-dLLM abstract's
 * anchor steps.  Outputs are bit for bit those of the three calls.  `scores`
 * (fp32 [B,H,nb,nb]) is written as well.  Arguments and errors as the three
 * calls; one caller-owned workspace of sdl_anchor_workspace_bytes bytes.  The
 * launch is cooperative (all its blocks resident at once); its grid barriers
 * are bounded and a timeout raises SDL_ERR_TIMEOUT in sdl_last_device_status. */
size_t sdl_anchor_workspace_bytes(const sdl_shape* shape);
sdl_status sdl_anchor_refresh(const void* q, const void* k, const sdl_shape* shape, float scale,
                              double sparsity, float* scores, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, int32_t* plan,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ---- Whole anchor step, one call --------------------------------------------
 * Everything an anchor step of the Step-dLLM abstract (the mask refresh at
 * steps 0, K, 2K, ...) produces for the attention calls that follow it, with
 * every launch issued from here back to back and no return to the caller in
 * between: the fused block scores and selection of sdl_anchor_refresh, then
 * sdl_tile_plan, sdl_tile_order and (when `lists` is not NULL)
 * sdl_tile_lists.  The paper describes the refresh, not this scheduling
 * aid.  Outputs are bit for bit those of the separate calls: scores fp32
 * [B,H,nb,nb], row_ptr int32 [B*H*nb + 1], col_idx int32 (col_capacity >=
 * sdl_mask_budget), plan int32 [B,H,ceil(nb/2),2], order int32
 * [B*H*ceil(nb/2)], lists (16-byte aligned, lists_bytes >=
 * sdl_tile_lists_bytes) for sdl_sparse_attn_listed.  64-token blocks only
 * (else SDL_ERR_UNSUPPORTED); plan and order must not be NULL
 * (SDL_ERR_INVALID_ARG).  Workspace as sdl_anchor_refresh
 * (sdl_anchor_workspace_bytes).  All buffers are device memory owned by the
 * caller.  Arguments are validated before the first launch, so an error
 * return launches nothing; a launch failure returns SDL_ERR_CUDA and stops
 * the sequence there. */
sdl_status sdl_anchor_step(const void* q, const void* k, const sdl_shape* shape, float scale,
                           double sparsity, float* scores, int32_t* row_ptr, int32_t* col_idx,
                           int64_t col_capacity, int32_t* plan, int32_t* order, void* lists,
                           size_t lists_bytes, void* workspace, size_t workspace_bytes,
                           void* stream);

/* ---- Mask selection with the heads of a sequence split over ranks ----------
 * The global budget of the Step-dLLM abstract (and the rule of sdl_select_mask)
 * when rank r of W holds the contiguous head range [h_r, h_r + H_local) of
 * every sequence (ranks in head order, so flat index order is rank order), as
 * when attention is sharded over GPUs by heads.  `local` describes this
 * rank's part (H = H_local heads; its scores are fp32 [B, H_local, nb, nb]);
 * `heads_total` is the sequence's head count, the budget is
 * floor((1 - sparsity) * heads_total * nb^2 + 0.5) per sequence.  Steps, every
 * rank in the same order:
 *   1. for pass p = 0, 1, ..., SDL_SELECT_PASSES - 1:
 *        sdl_select_shard_pass(p); then sum the pass-p histogram over ranks in
 *        place (int32, `count` elements at `offset_bytes` into the workspace,
 *        from sdl_select_shard_hist), e.g. one all-reduce;
 *   2. sdl_select_shard_count: writes int64 totals[2 b] (keys above the
 *      threshold on this rank) and totals[2 b + 1] (keys equal to it);
 *   3. gather the totals of all ranks and pass offsets[2 b] = the sum over all
 *      ranks of totals[2 b], offsets[2 b + 1] = the sum of totals[2 b + 1] over
 *      the ranks before this one;
 *   4. sdl_select_shard_finish: this rank's CSR (row_ptr over its B * H_local * nb
 *      rows, starting at 0; col_idx ascending per row; optional mask_u8), its
 *      part of the global selection exactly.
 * The workspace (caller-owned, sdl_select_shard_workspace_bytes) must persist
 * across the steps; offsets must stay valid until finish has run on the stream.
 * col_capacity must be at least sdl_select_shard_capacity (an upper bound on
 * this rank's kept blocks).  Errors as sdl_select_mask; SDL_ERR_INVALID_ARG also
 * when heads_total < H_local. */
#define SDL_SELECT_PASSES 3
size_t sdl_select_shard_workspace_bytes(const sdl_shape* local);
sdl_status sdl_select_shard_hist(const sdl_shape* local, int pass, size_t* offset_bytes,
                                 size_t* count);
int64_t sdl_select_shard_capacity(const sdl_shape* local, int32_t heads_total, double sparsity);
sdl_status sdl_select_shard_pass(const float* scores, const sdl_shape* local, int32_t heads_total,
                                 double sparsity, int pass, void* workspace,
                                 size_t workspace_bytes, void* stream);
sdl_status sdl_select_shard_count(const float* scores, const sdl_shape* local, int32_t heads_total,
                                  double sparsity, void* workspace, size_t workspace_bytes,
                                  int64_t* totals, void* stream);
sdl_status sdl_select_shard_finish(const float* scores, const sdl_shape* local,
                                   int32_t heads_total, double sparsity, const int64_t* offsets,
                                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                   uint8_t* mask_u8, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* Allocation-free variant of sdl_select_mask (no counterpart in the paper; it
 * exists for callers that cannot allocate device memory, such as code running
 * inside a device-memory pool's own callbacks or a serving process that reserves
 * all of its memory at start-up and forbids cudaMalloc afterwards).
 * Same arguments and results as sdl_select_mask minus the workspace: the
 * scratch is a fixed 2 MiB array inside libsdl (held by every GPU that loads the
 * library until exit).  Problems needing more scratch than that
 * (sdl_select_workspace_bytes > 2 MiB) return SDL_ERR_WORKSPACE without launching.
 * The first call on each device looks up the array's device address; make it
 * before any stream capture.  The array used is the one of the current device:
 * `stream` must belong to the device that is current when the call is made.
 * The looked-up address is kept for the life of the process, so it is not
 * valid after a cudaDeviceReset (the same holds for the device status word
 * behind sdl_last_device_status).  Nothing is allocated by any call.  All calls
 * share the array: calls that may overlap on the GPU (other streams, other
 * threads) race and must be serialized by the caller. */
sdl_status sdl_select_mask_noalloc(const float* scores, const sdl_shape* shape, double sparsity,
                                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                   uint8_t* mask_u8, void* stream);

/* Block-sparse attention (every step), the fused kernel of the Step-dLLM
 * abstract: for token t of query block i of head h,
 *   O[b,t,h,:] = sum_u softmax_u(scale * q_t . k_u) v_u
 * over the tokens u of the blocks col_idx[row_ptr[r] .. row_ptr[r+1]) of row
 * r = (b*H + h)*nb + i, non-causal, K and V read from KV head h / (H/H_kv).
 * Lists must be ascending with entries in [0, nb); a bad entry is skipped and
 * reported as SDL_ERR_BAD_MASK by sdl_last_device_status().
 * lse (nullable): fp32 [B, H, L], natural-log sum of exp of the logits.
 * scale <= 0 means 1/sqrt(d).  bf16 runs on tcgen05 tensor cores (fp32
 * accumulation, output rounded to nearest even); fp32 runs on CUDA cores.
 * Tile counter: each bf16 launch of this and the other attention calls takes
 * its tiles from one of 64 device counters, used in turn across launches,
 * and the launch's last CTA resets it.  So at most 64 bf16 attention launches
 * may be in flight at once.  A CUDA graph that captures one keeps the counter
 * it was captured with, so such a graph must not run concurrently with itself. */
sdl_status sdl_sparse_attn(const void* q, const void* k, const void* v, const sdl_shape* shape,
                           const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o,
                           float* lse, void* stream);

/* Tile plan for 64-token blocks (a scheduling aid with no counterpart in the
 * abstract): the attention kernels run 128-row tensor-core tiles, each holding
 * two query blocks and walking the union of their kept lists, so pairing
 * blocks whose lists overlap saves work.  Writes plan, int32
 * [B, H, ceil(nb/2), 2] (device, caller-owned): tile p of head (b, h) holds
 * query blocks plan[..., p, 0] and plan[..., p, 1] (-1 for the single block
 * left when nb is odd).  Per head, blocks are taken in order of descending
 * list length (ties: lower index) and each unpaired block is paired with the
 * unpaired block whose kept list shares the most entries (ties: lower index).
 * Heads with more than 256 blocks get adjacent pairs.  Only block == 64;
 * other block sizes return SDL_ERR_UNSUPPORTED. */
sdl_status sdl_tile_plan(const int32_t* row_ptr, const int32_t* col_idx, const sdl_shape* shape,
                         int32_t* plan, void* stream);

/* sdl_sparse_attn with a tile plan from sdl_tile_plan (NULL: adjacent pairs,
 * which is what sdl_sparse_attn uses).  Same results up to fp32 summation
 * order.  The plan must pair every query block of every head exactly once;
 * entries outside [0, nb) are skipped and reported as SDL_ERR_BAD_MASK.  Used
 * for bf16 with block == 64 only (fp32 and 128-token blocks ignore it). */
sdl_status sdl_sparse_attn_planned(const void* q, const void* k, const void* v,
                                   const sdl_shape* shape, const int32_t* row_ptr,
                                   const int32_t* col_idx, const int32_t* plan, float scale,
                                   void* o, float* lse, void* stream);

/* Order in which the attention kernel takes the tiles of a plan, costliest
 * first (a scheduling aid): tiles are taken from a global counter by
 * persistent CTAs, and when the longest tiles come last (as with heads that
 * keep many blocks at the end of the head order) the other SMs sit idle while
 * they finish.  Writes order, int32 [B * H * ceil(nb/2)]: a permutation of the
 * tile indices (b * H + h) * ceil(nb/2) + p, sorted by the sum of the tile's two
 * query blocks' list lengths, descending (ties in any order).  Only block ==
 * 64 (SDL_ERR_UNSUPPORTED otherwise). */
sdl_status sdl_tile_order(const int32_t* row_ptr, const int32_t* plan, const sdl_shape* shape,
                          int32_t* order, void* stream);

/* sdl_sparse_attn_planned taking the plan's tiles in `order` (from
 * sdl_tile_order, or any permutation of the tile indices).  Results are those
 * of sdl_sparse_attn_planned bit for bit (a tile's result does not depend on
 * which CTA runs it or when); entries outside the tile range are skipped and
 * reported as SDL_ERR_BAD_MASK. */
sdl_status sdl_sparse_attn_scheduled(const void* q, const void* k, const void* v,
                                     const sdl_shape* shape, const int32_t* row_ptr,
                                     const int32_t* col_idx, const int32_t* plan,
                                     const int32_t* order, float scale, void* o, float* lse,
                                     void* stream);

/* Tile lists built once per mask (a scheduling aid, like the plan and the
 * order): for every position r of `order` (NULL: the plan's tile order;
 * `plan` NULL: adjacent query blocks paired) the tile's identity, its two
 * query blocks' first tokens and the ascending union
 * of their kept 64-token key blocks with a keep bit per query block -- exactly
 * the list the attention kernel would otherwise build when it takes the tile.
 * `lists` (16-byte aligned, caller-owned) must hold sdl_tile_lists_bytes
 * bytes (else SDL_ERR_WORKSPACE): per position a record of 8 int32 {tile,
 * list length, first token of each half (L: half unused), 0, 0, 0, 0}, then
 * per position a row of 16-bit entries (key block | keep bits << 14), rows
 * padded to a multiple of 8 entries.  64-token blocks only
 * (SDL_ERR_UNSUPPORTED otherwise); plan entries outside the block range are
 * reported as SDL_ERR_BAD_MASK, as in the attention calls.
 * sdl_sparse_attn_listed: sdl_sparse_attn_scheduled reading the tiles and
 * their lists from `lists` (taken in record order) instead of building each
 * list from the CSR when the tile is taken; results are those of
 * sdl_sparse_attn_scheduled with the same plan and order, bit for bit.
 * Records or entries out of range are skipped or zeroed and reported as
 * SDL_ERR_BAD_MASK.  bf16 and 64-token blocks only (SDL_ERR_UNSUPPORTED
 * otherwise).  The lists depend on the mask, plan and
 * order alone (not on Q, K, V): rebuild them whenever one of those changes. */
size_t sdl_tile_lists_bytes(const sdl_shape* shape);
sdl_status sdl_tile_lists(const int32_t* row_ptr, const int32_t* col_idx, const int32_t* plan,
                          const int32_t* order, const sdl_shape* shape, void* lists,
                          size_t lists_bytes, void* stream);
sdl_status sdl_sparse_attn_listed(const void* q, const void* k, const void* v,
                                  const sdl_shape* shape, const void* lists, float scale, void* o,
                                  float* lse, void* stream);

/* Dense bidirectional attention, the baseline of the same abstract: the
 * sparse call with every block of every row kept. */
sdl_status sdl_dense_attn(const void* q, const void* k, const void* v, const sdl_shape* shape,
                          float scale, void* o, float* lse, void* stream);

/* Synchronizes `stream`, then reports and clears the device status word set by
 * kernels: SDL_ERR_TIMEOUT if a bounded wait ran out, SDL_ERR_BAD_MASK if a
 * list entry was rejected, SDL_ERR_OVERLAP if more bf16 attention launches
 * were in flight at once than there are tile counters (the last CTA of each
 * launch checks its counter's final count), SDL_OK otherwise; the first of
 * these in that order when several bits are set. */
sdl_status sdl_last_device_status(void* stream);

/* Where the bad-mask report behind the last sdl_last_device_status of this
 * thread came from: 0 if it reported none, else site << 24 | the low 24 bits
 * of the offending value, for the first report since the read before it.
 * Sites: 1 a tile-plan entry outside [-1, nb) (value: the tile); 2 a CSR
 * entry out of range or not ascending (the entry); 3 a tile-lists record's
 * tile or length (the tile); 4 a record's first tokens (t0); 5 a list entry's
 * key sub-block (the entry); 6 a take-order entry read by the attention kernel
 * (the entry); 7 one read by sdl_tile_lists (the entry); 8 a CSR entry in the
 * fp32 kernel (the entry).  A diagnostic: the pages describe no such word. */
int sdl_last_device_detail(void);

/* Self-check of the failure path: launches one warp that waits, through the
 * same bounded wait every kernel of the library uses, on an mbarrier phase
 * that nothing completes, giving up after `limit_ns` (1 us .. 1 s, else
 * SDL_ERR_INVALID_ARG).  The next sdl_last_device_status then returns
 * SDL_ERR_TIMEOUT, and the context stays usable. */
sdl_status sdl_wait_selfcheck(uint64_t limit_ns, void* stream);

/* cudaError_t of the last failed CUDA call in this thread (0 if none). */
int sdl_last_cuda_error(void);

/* Static description of a status code. */
const char* sdl_status_string(sdl_status status);

#ifdef __cplusplus
}
#endif

#endif /* SDL_H */
