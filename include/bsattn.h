/*
 * bsattn.h - C ABI of libbsattn.so: block-sparse softmax attention over video
 * tokens laid out as a [t,h,w] latent grid, for NVIDIA B200 (sm_100a).
 *
 * The operations follow two methods described on the web:
 *  - "LVSA: Training-Free Sparse Attention for Long Video Diffusion",
 *    section 2 "Methodology", "Core mechanism": each query frame t attends
 *    the frame set A(t) = G_s U W(t) (rotating global anchors G_s plus an
 *    extended local window W(t)), with |A(t)| = C; "Complexity": the cost is
 *    T*C*P^2*d, linear in the number of frames T.
 *  - The Draft Attention article ("科学家提出视频扩散模型加速方法，在H100实现
 *    一倍以上端到端加速", 163.com): tokens are reshaped to [t,h,w]; Q and K are
 *    average-pooled over pool_h x pool_w tiles into a low-resolution draft
 *    attention map, which yields a sparse block mask (pool_h*pool_w equals
 *    the block size) guiding full-resolution block-sparse attention; a reorder
 *    makes the selected blocks contiguous in memory.
 *
 * Conventions common to every entry point
 *  - Tensors are owned by the caller: device pointers, contiguous, 16-byte
 *    aligned, and at least as large as the plan's geometry implies (given
 *    with each entry point).  The library sees only pointers and cannot
 *    check sizes; the Python binding checks them before every call.
 *    Nothing is allocated per call; a plan owns only small index data and a
 *    device status word, allocated by bsa_plan_create on the device that is
 *    current at that time.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and returns after enqueueing its kernel(s).  Argument
 *    errors are detected on the host before anything is enqueued and
 *    reported as a status code; bsa_last_error() then describes the error.
 *  - Errors found on the device (a block list naming a block out of range,
 *    a bounded wait that ran out) are recorded in the plan's status word and
 *    reported by bsa_poll_status().  Kernels never trap.
 *  - Natural layout: [B, N, Hh, D] bf16, token n = (t*H + y)*W + x.
 *    Slot layout: [B, Hh, Npad, D] bf16 (Npad = bsa_padded_tokens()); the
 *    token -> slot map is set by the plan's layout (below).  Slots that hold
 *    no token are "empty"; attention never reads them as keys.
 *  - Supported head dims: D = 64 or 128.  Block size: a divisor of 128.
 */
#ifndef BSATTN_H_
#define BSATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,    /* bad sizes, null pointer, inconsistent plan      */
  BSA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. D = 96)         */
  BSA_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned                */
  BSA_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed               */
  BSA_ERR_TIMEOUT = 5,        /* a bounded device wait ran out (see poll)        */
  BSA_ERR_BAD_BLOCKLIST = 6   /* a block list named a block out of range, or a
                                 row_ptr decreased, or (block < 128) a row was
                                 not ascending; offending entries were skipped   */
} bsa_status;

/* Token -> slot maps (Draft Attention article, the reorder paragraph and its
 * figure "Full Map" vs "Reordered Full Map").
 *  BSA_LAYOUT_FRAME: each frame padded to nbf = ceil(H*W/block) whole blocks;
 *      token (t,y,x) -> slot t*nbf*block + y*W + x.  Used by the LVSA mask.
 *  BSA_LAYOUT_TILE:  each pool_h x pool_w tile of a frame is one block
 *      (block = pool_h*pool_w); with TH = ceil(H/pool_h), TW = ceil(W/pool_w),
 *      token (t, i*pool_h+a, j*pool_w+b) -> slot
 *      ((t*TH + i)*TW + j)*block + a*pool_w + b.  Used by the draft mask.
 * In both, Npad is the block count times block, rounded up to a multiple of
 * 128 (the attention tile); slots past the last block are empty. */
typedef enum { BSA_LAYOUT_FRAME = 0, BSA_LAYOUT_TILE = 1 } bsa_layout;

/* LVSA mask variants (bsa_plan_set_lvsa_variant). */
typedef enum {
  BSA_ANCHORS_ROTATING = 0, /* G_s = {f : (f - s) mod T_per == 0} (LVSA)       */
  BSA_ANCHORS_FIXED = 1,    /* G = {f : f mod T_per == 0} at every step         */
  BSA_ANCHORS_NONE = 2      /* no global frames: the sliding window alone       */
} bsa_anchor_mode;
typedef enum {
  BSA_WINDOW_DISTANCE = 0,  /* grow t+1, t-1, t+2, t-2, ...                     */
  BSA_WINDOW_ALTERNATE = 1  /* right and left pointers take turns, right first
                               (default)                                        */
} bsa_window_order;

/* Draft pooling (bsa_plan_set_draft_pooling). */
typedef enum { BSA_POOL_MEAN = 0, BSA_POOL_MAX = 1 } bsa_pooling;

/* Empty slots written by bsa_reorder_fwd (bsa_plan_set_reorder_pads). */
typedef enum { BSA_PADS_WRITE = 0, BSA_PADS_KEEP = 1 } bsa_reorder_pads;

/* Precision of the draft logits (bsa_plan_set_draft_precision). */
typedef enum { BSA_DRAFT_FP64 = 0, BSA_DRAFT_FP32 = 1 } bsa_draft_precision;

typedef struct bsa_plan_s* bsa_plan_t;

/* Create a plan for batch B, Hh heads, head dim D, latent grid T x H x W.
 * layout FRAME: `block` tokens per block (pool_h, pool_w ignored).
 * layout TILE:  block must equal pool_h*pool_w.
 * Allocates the plan's device data (per-128-slot validity masks, status
 * word) on the current device.  On error *plan is set to NULL. */
bsa_status bsa_plan_create(bsa_plan_t* plan, int B, int Hh, int D, int T, int H, int W,
                           int layout, int pool_h, int pool_w, int block);

/* Free the plan and its device data.  No call using it may be in flight. */
bsa_status bsa_plan_destroy(bsa_plan_t plan);

/* Choose the LVSA mask variant used by bsa_lvsa_mask and bsa_lvsa_attn_fwd
 * with this plan (default ROTATING, ALTERNATE).  "LVSA", section 2 "Core
 * mechanism", contrasts its rotating anchors with fixed-grid global frames,
 * and the page's introduction lists plain sliding windows; FIXED and NONE
 * give those patterns under the same budget C.  The page leaves the growth
 * order of the extended window open: ALTERNATE lets a right and a left
 * pointer take turns (right first), each moving past frames already present
 * (the anchors); a side that runs off [0, T) stops and the other continues.
 * That is the window "extended alternately right then left, skipping anchors,
 * clamped at the edges" of the workloads these kernels are measured on, and
 * the default.  DISTANCE adds the nearest frame not yet present (ties to the
 * right).  Takes effect for calls issued after it; returns
 * BSA_ERR_INVALID_ARG for unknown values. */
bsa_status bsa_plan_set_lvsa_variant(bsa_plan_t plan, int anchors, int window_order);

/* Choose the pooling of bsa_draft_mask, bsa_draft_mask_noalloc and
 * bsa_draft_mask_natural with this plan (default MEAN).  MAX takes the channel-wise maximum over the tile's
 * tokens inside the grid: the Draft Attention article reports trying max
 * pooling first and preferring the average at high sparsity. */
bsa_status bsa_plan_set_draft_pooling(bsa_plan_t plan, int pooling);

/* Choose the precision of the draft logits of bsa_draft_mask,
 * bsa_draft_mask_noalloc and bsa_draft_mask_natural(_e4m3) with this plan
 * (default FP64).  The Draft Attention article fixes none.  FP64: the pooled
 * values and the logits in fp64.  FP32: the pooled values (still summed in
 * fp64) rounded once to fp32 and the logits' products and sums rounded to
 * fp32, about twice as fast to score; the block lists can differ from FP64
 * where two logits agree to fp32 precision.  Either way the evaluation order
 * is fixed (below), so the lists are reproducible bit for bit.  The
 * workspace size (bsa_draft_workspace_bytes) follows the precision.  Takes
 * effect for calls issued after it; BSA_ERR_INVALID_ARG for unknown values. */
bsa_status bsa_plan_set_draft_precision(bsa_plan_t plan, int precision);

/* Geometry queries (return -1 for a NULL plan). */
int64_t bsa_padded_tokens(bsa_plan_t plan);   /* Npad                          */
int64_t bsa_num_blocks(bsa_plan_t plan);      /* blocks per (b, head): Nb      */
int     bsa_block_size(bsa_plan_t plan);

/* LVSA frame mask for denoising step s ("LVSA", section 2, "Rotating global
 * anchors" and "Extended adaptive window").
 *   G_s = {f in [0,T) : (f - s) mod T_per == 0};
 *   A(t) = G_s U {t}, then grown until |A(t)| = C by a right and a left
 *   pointer taking turns, right first, each skipping frames already present;
 *   a side that runs off [0,T) stops and the other continues.
 * (Other anchor grids and growth orders: bsa_plan_set_lvsa_variant.)
 * Requires a FRAME plan, 1 <= T_per, C <= T and |G_s U {t}| <= C for every t.
 * Outputs (device):
 *   frame_sets int32[T*C] (may be NULL): row t = A(t) ascending;
 *   row_ptr    int32[Nb+1]: row r = query block r, r*C*nbf entries before it;
 *   col_idx    int32[Nb*C*nbf]: for query block r in frame t = r / nbf, every
 *              block f*nbf + i of every frame f in A(t), ascending.
 * The block list is the same for every batch and head (per_head_lists = 0). */
bsa_status bsa_lvsa_mask(bsa_plan_t plan, int C, int T_per, int s, int32_t* frame_sets,
                         int32_t* row_ptr, int32_t* col_idx, void* stream);

/* Number of col_idx entries bsa_lvsa_mask writes (Nb*C*nbf), or -1. */
int64_t bsa_lvsa_nnz(bsa_plan_t plan, int C);

/* Blocks kept per query-block row at `sparsity_pct` percent sparsity:
 * k = ceil(Nb*(100 - sparsity_pct)/100), i.e. never sparser than asked. */
int bsa_draft_keep_count(bsa_plan_t plan, int sparsity_pct);

/* Scratch bytes bsa_draft_mask needs (the pooled Q and K in the plan's
 * draft precision: 2*B*Hh*Nb*D*8 bytes for FP64, *4 for FP32). */
size_t bsa_draft_workspace_bytes(bsa_plan_t plan);

/* Draft mask (Draft Attention article: average pooling of Q and K over each
 * pool_h x pool_w tile, low-resolution map softmax(Qbar Kbar^T / sqrt(D)),
 * sparse mask keeping the important blocks at the stated sparsity).
 * Requires a TILE plan.  q_slots, k_slots: slot layout (output of
 * bsa_reorder_fwd).  For every (b, head, query block i):
 *   qbar_i, kbar_j = mean over the tile's tokens inside the grid (fp64
 *     sequential sum in row-major tile order, one IEEE division; rounded
 *     once to fp32 in FP32 precision), or their maximum with
 *     bsa_plan_set_draft_pooling(BSA_POOL_MAX);
 *   L[i][j] = sum_c qbar_i[c]*kbar_j[c], sequential over c, each product and
 *     sum rounded to the plan's draft precision (fp64 by default; no fused
 *     multiply-add);
 *   keep the k = bsa_draft_keep_count() blocks j with the largest L[i][j],
 *     ties to the lower j, written ascending.
 * Outputs (device): kv_idx int32[B*Hh*Nb*k]; row_ptr int32[B*Hh*Nb+1] (may be
 * NULL; row r starts at r*k); draft_map float[B*Hh*Nb*Nb] (may be NULL) =
 * softmax_j(L[i][j]/sqrt(D)).  Use with bsa_attn_fwd(per_head_lists = 1).
 * workspace: device scratch of at least bsa_draft_workspace_bytes(); its
 * contents on entry do not matter. */
bsa_status bsa_draft_mask(bsa_plan_t plan, const void* q_slots, const void* k_slots,
                          int sparsity_pct, int32_t* row_ptr, int32_t* kv_idx,
                          float* draft_map, void* workspace, size_t workspace_bytes,
                          void* stream);

/* bsa_draft_mask for callers that cannot allocate device memory (the paper
 * has no counterpart; this is a convenience of this library).  Examples: a
 * plugin inside a host program that owns every device allocation and passes
 * only input and output buffers, or a caller held to a fixed memory budget
 * where an extra allocation could fail or stall the device mid-step.
 * Same arguments, outputs and results as bsa_draft_mask, minus the workspace:
 * the scratch lives in a 48 MiB array inside the library
 * (bsa_draft_noalloc_max_scratch_bytes()), held by every GPU that loads the
 * library until the process exits.  Problems needing more scratch than that
 * (bsa_draft_workspace_bytes) return BSA_ERR_UNSUPPORTED.  The first call made on a
 * device looks up that array's device address (one cudaGetSymbolAddress);
 * make that first call before any stream capture.  All calls on a device
 * share the array: calls whose kernels overlap on the GPU race on it, calls
 * in order on one stream do not.  Nothing in it needs clearing between calls.
 * The current device must be the plan's device (BSA_ERR_INVALID_ARG
 * otherwise).  The address is cached for the life of the process: after
 * cudaDeviceReset on a device, do not call this entry point again in that
 * process. */
bsa_status bsa_draft_mask_noalloc(bsa_plan_t plan, const void* q_slots, const void* k_slots,
                                  int sparsity_pct, int32_t* row_ptr, int32_t* kv_idx,
                                  float* draft_map, void* stream);

/* Scratch capacity of bsa_draft_mask_noalloc, in bytes (48 MiB). */
size_t bsa_draft_noalloc_max_scratch_bytes(void);

/* Reorder (Draft Attention article, reorder paragraph): gather natural-layout
 * tensors x [B, N, Hh, D] into the plan's slot layout y [B, Hh, Npad, D]
 * (2-byte elements, copied bit for bit); empty slots are written as zero.
 * Up to three tensors in one launch: x1/y1 and x2/y2 may be NULL (both of a
 * pair), x2/y2 only together with x1/y1; otherwise BSA_ERR_INVALID_ARG. */
bsa_status bsa_reorder_fwd(bsa_plan_t plan, const void* x0, void* y0, const void* x1,
                           void* y1, const void* x2, void* y2, void* stream);

/* Whether bsa_reorder_fwd with this plan writes the empty slots (default
 * WRITE: zeros).  KEEP leaves them untouched and writes only the slots that
 * hold tokens: for callers whose slot buffers already hold zeros there, for
 * example buffers that an earlier call with WRITE filled and that nothing
 * has written since (the other entry points only read the empty slots).
 * The attention reads empty key slots, masked, so they must hold finite
 * values.  Takes effect for calls issued after it; BSA_ERR_INVALID_ARG for
 * unknown values. */
bsa_status bsa_plan_set_reorder_pads(bsa_plan_t plan, int pads);

/* Inverse reorder: slot layout [B, Hh, Npad, D] -> natural layout
 * [B, N, Hh, D], bit for bit; empty slots are dropped. */
bsa_status bsa_reorder_inv(bsa_plan_t plan, const void* x_slots, void* x_nat, void* stream);

/* Block-sparse attention forward (LVSA section 2 and the Draft Attention
 * article: softmax attention restricted to the allowed blocks).
 * q, k, v, o: slot layout [B, Hh, Npad, D] bf16.  lse: float[B*Hh*Npad] or
 * NULL.  Block list: one CSR with rows r = list*Nb + qb, list = b*Hh + h if
 * per_head_lists else 0; row r lists the key blocks (index < Nb) that query
 * block qb may attend, without repeats (ascending when block < 128).
 * For every non-empty query slot q:
 *   O[q] = sum_k softmax_k(scale * <q, k>) v_k over the non-empty slots k of
 *   the allowed blocks; LSE[q] = log sum_k exp(scale * <q, k>).
 * fp32 accumulation; probabilities rounded to bf16 before the PV product.
 * Empty query slots, and queries with no allowed key, get O = 0 and
 * LSE = -inf.  Block lists are not modified. */
bsa_status bsa_attn_fwd(bsa_plan_t plan, const void* q, const void* k, const void* v,
                        const int32_t* row_ptr, const int32_t* col_idx, int per_head_lists,
                        float scale, void* o, float* lse, void* stream);

/* Draft-path attention on the natural layout: bsa_attn_fwd with the reorder
 * of the Draft Attention article fused into the tile loads and the stores.
 * Requires a TILE plan with pool_h * pool_w = 128 (one pooling tile per
 * 128-slot tile; otherwise BSA_ERR_UNSUPPORTED).  q, k, v, o: natural layout
 * [B, N, Hh, D] bf16; block i of (b, head) is the pool_h x pool_w tile
 * (t, i_h, i_w), read through a 5-D tensor map whose part past the grid edge
 * reads as zero; o is written for every token (nothing else).  lse:
 * float[B*Hh*N] at (b*Hh + h)*N + n, or NULL.  Block lists, per_head_lists
 * and scale as for bsa_attn_fwd; the result equals bsa_reorder_fwd +
 * bsa_attn_fwd + bsa_reorder_inv bit for bit. */
bsa_status bsa_attn_fwd_natural(bsa_plan_t plan, const void* q, const void* k, const void* v,
                                const int32_t* row_ptr, const int32_t* col_idx, int per_head_lists,
                                float scale, void* o, float* lse, void* stream);

/* bsa_draft_mask on natural-layout q, k [B, N, Hh, D] bf16 (no reorder
 * first): the pooling reads each tile's tokens in place, in the same order,
 * so every output is identical to bsa_draft_mask on the reordered tensors.
 * Requires a TILE plan; workspace as for bsa_draft_mask. */
bsa_status bsa_draft_mask_natural(bsa_plan_t plan, const void* q, const void* k, int sparsity_pct,
                                  int32_t* row_ptr, int32_t* kv_idx, float* draft_map,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* e4m3 quantization for the 8-bit draft attention (the Draft Attention
 * article names quantization as its next step without fixing a format; this
 * is the reading taken).  q, k, v: natural layout [B, N, Hh, D] bf16; q8, k8,
 * v8: the same layout, one e4m3 byte per element; scales: float[3*B*Hh],
 * entry (t*B + b)*Hh + h for tensor t = 0 (Q), 1 (K), 2 (V):
 *   scale = fp32(max |x| over the head) / 448 (1 for an all-zero head),
 *   code  = e4m3 nearest to x / scale (fp32 division), ties to even,
 *           saturating at +-448.
 * Uses a small buffer owned by the plan: calls on one plan must not overlap. */
bsa_status bsa_quantize_e4m3(bsa_plan_t plan, const void* q, const void* k, const void* v, void* q8,
                             void* k8, void* v8, float* scales, void* stream);

/* The front half of the 8-bit draft pipeline in one call: the draft mask of
 * bsa_draft_mask_natural and the quantization of bsa_quantize_e4m3, with the
 * same outputs bit for bit (arguments as there).  The pooling pass that
 * reads Q and K for the draft map also takes their per-head maxima, so the
 * quantization reads only V once more before converting all three tensors.
 * Uses the plan's buffer as bsa_quantize_e4m3 does. */
bsa_status bsa_draft_mask_natural_e4m3(bsa_plan_t plan, const void* q, const void* k, const void* v,
                                       int sparsity_pct, int32_t* row_ptr, int32_t* kv_idx,
                                       float* draft_map, void* workspace, size_t workspace_bytes,
                                       void* q8, void* k8, void* v8, float* scales, void* stream);

/* bsa_attn_fwd_natural on e4m3 inputs (from bsa_quantize_e4m3): the QK and
 * PV products are 8-bit tensor-core MMAs (kind::f8f6f4) with fp32
 * accumulation; the scores are S * sq * sk; P is rounded to e4m3 (it stays
 * below 2^8); O is multiplied by sv.  Requires D = 128 and a TILE plan with
 * pool_h * pool_w = 128.  o: bf16 natural layout; lse as for
 * bsa_attn_fwd_natural, of the scores scale * S * sq * sk (the dequantized
 * inputs; P's rounding does not enter it).  Result within the e4m3 rounding
 * of Q, K, V and P of the exact attention (see the tests for the bound
 * used). */
bsa_status bsa_attn_fwd_natural_e4m3(bsa_plan_t plan, const void* q8, const void* k8,
                                     const void* v8, const float* scales, const int32_t* row_ptr,
                                     const int32_t* col_idx, int per_head_lists, float scale,
                                     void* o, float* lse, void* stream);

/* LVSA attention in one pass on the natural layout ("LVSA", section 2 "Core
 * mechanism"; the reorder of the Draft Attention article is fused into the
 * tile loads, so no padded copies are made).
 * Requires a FRAME plan (its block size is not used), D = 64 or 128,
 * T <= 4096 and H*W >= 37; C, T_per and s as for bsa_lvsa_mask.
 * q, k, v, o: natural layout [B, N, Hh, D] bf16, o written for every token.
 * lse: float[B*Hh*N] at (b*Hh + h)*N + n, or NULL.
 * Every query token of frame t attends exactly the key tokens of the frames
 * in A(t):  O[n] = sum_m softmax_m(scale * <q_n, k_m>) v_m over those keys;
 * LSE[n] = log sum_m exp(scale * <q_n, k_m>).  The result is that of
 * bsa_lvsa_mask + bsa_reorder_fwd + bsa_attn_fwd + bsa_reorder_inv, up to the
 * order of fp32 summation.  fp32 accumulation; probabilities rounded to bf16
 * before the PV product. */
bsa_status bsa_lvsa_attn_fwd(bsa_plan_t plan, int C, int T_per, int s, const void* q,
                             const void* k, const void* v, float scale, void* o, float* lse,
                             void* stream);

/* Synchronize `stream`, read and clear the plan's device status word.
 * Returns BSA_OK, BSA_ERR_BAD_BLOCKLIST, BSA_ERR_TIMEOUT or BSA_ERR_CUDA.
 * A recorded timeout is sticky: until this call clears it, every later
 * kernel of the plan sees it at start and returns at once without writing
 * its outputs (so a plan whose wait ran out stops working instead of
 * waiting again).  Callers that do not poll after each step get stale
 * outputs in that state; poll at least once per step to detect it. */
bsa_status bsa_poll_status(bsa_plan_t plan, void* stream);

/* Set the limit, in nanoseconds, of every bounded wait inside the plan's
 * kernels (default 2e9).  A wait that runs out records BSA_ERR_TIMEOUT. */
bsa_status bsa_set_wait_limit_ns(bsa_plan_t plan, uint64_t ns);

/* Failure-detection self test: launches one CTA that waits on a barrier no
 * one arrives on, for at most `limit_ns`; the wait runs out, the kernel
 * records BSA_ERR_TIMEOUT in the plan's status word and returns normally. */
bsa_status bsa_selftest_timeout(bsa_plan_t plan, uint64_t limit_ns, void* stream);

/* Message describing the last error of the calling thread ("" if none). */
const char* bsa_last_error(void);

/* Library version string. */
const char* bsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSATTN_H_ */
