/*
 * moe.h -- C ABI of the B200 (sm_100a) fused MoE expert layer.
 *
 * What the layer computes (per token t, top-k slots j = 0..k-1, e = topk_idx[t,j]):
 *
 *   xh      = E4M3(x[t]) * UE8M0(x_scales[t, c/128])                  (1x128 blocks)
 *   h       = xh @ W1[e]^T,  W1[e] = [2I, H]: rows [0,I) gate, [I,2I) up
 *   a       = min(g,L) * sigmoid(alpha*min(g,L)) * (clamp(u,-L,L) + up_bias)
 *   q, sq   = FP8 E4M3 requantisation of a with one UE8M0 scale per 1x128 block
 *   y[t,j]  = (q * sq) @ W2[e]^T,  W2[e] = [H, I]
 *   out[t]  = bf16( sum_j topk_w[t,j] * y[t,j] )     (fp32 sum, j ascending)
 *
 * with W1, W2 in E4M3 (128x128 UE8M0 blocks) or E2M1 (1x32 UE8M0 blocks).  The
 * BF16 variant (MOE_W_BF16) takes bf16 x and weights without scales and passes
 * a to FC2 rounded to bf16 instead of q * sq.
 *
 * Sources (web pages, by title and section):
 *   - DeepGEMM PR #445 "fix(sm90): support parameterized SwiGLU in FP8 MegaMoE",
 *     Summary / Compatibility: the activation and its parameters (defaults
 *     alpha = 1, up_bias = 0 give SiLU(gate) * up; the clamp is optional).
 *   - DeepGEMM PR #386 "Optimize sm100 version with token-aware BM240 tiling,
 *     native UE8M0, and direct combine", title / Description: UE8M0 block
 *     scales consumed natively and the direct weighted combine to token order.
 *   - fw-ai/DeepGEMM PR #16 "Sync upstream through PR #441: fix Mega MoE
 *     scheduler ordering", Overview: the persistent tile scheduler's task-info
 *     slots and their release ordering (used inside moe_fc1 / moe_fc2 /
 *     moe_fc1_fc2), and the BF16 / FP8 / FP4 Mega MoE variants.
 *   - TensorRT-LLM PR #16346 "DSV4 o_proj: fuse fp8/UE8M0 quantize ...",
 *     Description: BF16/FP32 -> FP8 + 1x128 UE8M0 quantisation fused into a
 *     GEMM epilogue (the FC1 epilogue here).
 *
 * Conventions for every entry point:
 *   - Tensors are row-major and contiguous unless a layout call says otherwise
 *     (moe_plan_set_weight_layout); device pointers must be 16-byte aligned
 *     (MXFP4 weight codes 32-byte, their scales 4-byte, or 16-byte when
 *     chunked).
 *   - Ownership: the caller owns every buffer, host or device.  The library
 *     never allocates or frees device memory; a plan is a small host object.
 *   - Errors are returned as moe_status; nothing is thrown across the ABI.
 *     Argument validation happens before anything is enqueued: a call that
 *     returns an error has launched nothing.
 *   - Masked slots: topk_idx = -1 marks a slot that is not routed (it
 *     contributes nothing to its token's output); this is not an error.
 *   - Device-side problems (an expert id >= E or < -1, a bounded wait that ran
 *     out) are recorded in an error word inside the workspace; read it with
 *     moe_check_device_error().  A slot with such an id is not routed either.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) unless stated otherwise.  Calls with different plans or
 *     different workspaces may run concurrently; two calls sharing one
 *     workspace must be ordered on one stream.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* null pointer, bad size, k > E, ...           */
  MOE_ERR_UNSUPPORTED = 2,    /* shape the kernels do not handle (H % 128 ...) */
  MOE_ERR_ALIGNMENT = 3,      /* pointer not 16 B (MXFP4 weights: 32 B) aligned */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime call failed                     */
  MOE_ERR_DEVICE_TIMEOUT = 5, /* a bounded device wait ran out (see error word) */
  MOE_ERR_BAD_ROUTING = 6     /* a topk_idx entry was outside [0, E)            */
} moe_status;

/* Weight formats.  With the two block-scaled formats the activations x are
 * E4M3 with one UE8M0 per 1x128 and the FC1 activation is requantised to that
 * format.  MOE_W_BF16 is the BF16 variant the pages name next to FP8/FP4
 * (fw-ai/DeepGEMM PR #16, Overview): x is bf16 [T,H] and x_scales is unused
 * (may be NULL), W1 bf16 [E,2I,H] and W2 bf16 [E,H,I] with no scales (NULL
 * allowed), and the FC1 activation goes to FC2 as bf16 (round to nearest
 * even), fp32 accumulation throughout.                                       */
typedef enum {
  MOE_W_E4M3_UE8M0_128x128 = 0, /* W1 u8 [E,2I,H], scales u8 [E,2I/128,H/128]  */
  MOE_W_E2M1_UE8M0_1x32 = 1,    /* W1 u8 [E,2I,H/2] (two E2M1 codes per byte,
                                   element 2i in the low nibble),
                                   scales u8 [E,2I,H/32]; W2 likewise [E,H,I/2],
                                   [E,H,I/32]                                   */
  MOE_W_BF16 = 2                /* W1 bf16 [E,2I,H], W2 bf16 [E,H,I], no scales */
} moe_wdtype;

typedef struct {
  int w_dtype; /* a moe_wdtype */
} moe_dtypes;

typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_SWIGLU_OAI = 1 } moe_act_kind;

/* Activation parameters (DeepGEMM PR #445, Summary).  For MOE_ACT_SWIGLU the
 * other fields are ignored (alpha = 1, up_bias = 0, no clamp).  For
 * MOE_ACT_SWIGLU_OAI, limit > 0 (+INFINITY = no clamp).                      */
typedef struct {
  int kind; /* a moe_act_kind */
  float alpha;
  float up_bias;
  float limit;
} moe_act_params;

typedef struct moe_plan_s *moe_plan_t;

/* Build a plan for T tokens, hidden size H, expert intermediate size I, E
 * experts and top-k.  Host only; enqueues nothing and allocates no device
 * memory.  Requirements: T >= 1; H % 256 == 0 (FC2 output tiles are 256
 * columns wide); I % 128 == 0; 1 <= k <= E <= 256; T*k < 2^31.  Returns
 * MOE_ERR_INVALID_ARG (sizes, k > E, activation parameters) or
 * MOE_ERR_UNSUPPORTED (H, I or E outside what the kernels handle) otherwise.
 * Source: the layer's sizes and variants as the Mega MoE pages name them
 * (fw-ai/DeepGEMM PR #16, Overview; DeepGEMM PR #445, Summary, for the
 * activation parameters).
 */
moe_status moe_plan(int T, int H, int I, int E, int k, moe_dtypes dtypes,
                    moe_act_params act, moe_plan_t *out);

/* Release a plan (NULL is allowed).
 * No counterpart on the pages.
 */
void moe_plan_destroy(moe_plan_t plan);

/* Size in bytes of the device workspace moe_forward and the step calls need
 * (256-byte aligned pointer required).  0 for a NULL plan.
 * No counterpart on the pages.
 */
size_t moe_workspace_bytes(moe_plan_t plan);

/* The whole layer: route -> gather -> FC1 (+ activation + FP8 requant) -> FC2
 * -> combine, enqueued on `stream`.
 *   x          u8 [T,H]      E4M3 codes of the activations (MOE_W_BF16: bf16 [T,H])
 *   x_scales   u8 [T,H/128]  UE8M0 scale bytes (MOE_W_BF16: unused, may be NULL)
 *   topk_idx   i32 [T,k]     expert ids
 *   topk_w     f32 [T,k]     combine weights
 *   w1, w1_scales, w2, w2_scales   weights in the plan's moe_wdtype layout
 *   out        bf16 [T,H]    written entirely
 *   workspace  moe_workspace_bytes(plan) bytes, device, 256-B aligned.
 * All pointers are device pointers.
 * Sources: those of the steps below (moe_route ... moe_combine).
 */
moe_status moe_forward(moe_plan_t plan, const void *x, const uint8_t *x_scales,
                       const int32_t *topk_idx, const float *topk_w,
                       const void *w1, const uint8_t *w1_scales, const void *w2,
                       const uint8_t *w2_scales, void *out, void *workspace,
                       moe_stream_t stream);

/* moe_forward with the per-step activations on the HOST: x, x_scales,
 * topk_idx and topk_w are host pointers (pinned memory gives asynchronous
 * copies), the weights and the workspace are device pointers, and out_host is
 * a host bf16 [T,H] buffer.  The host-to-device copies, the layer and the
 * device-to-host copy of the output are enqueued on `stream`; the output is
 * valid after the stream has been synchronised.
 * No counterpart on the pages (a host-buffer convenience around
 * moe_forward).
 */
moe_status moe_forward_hostio(moe_plan_t plan, const void *x_host,
                              const uint8_t *x_scales_host,
                              const int32_t *topk_idx_host,
                              const float *topk_w_host, const void *w1,
                              const uint8_t *w1_scales, const void *w2,
                              const uint8_t *w2_scales, void *out_host,
                              void *workspace, moe_stream_t stream);

/* n_batches consecutive layers with their activations on the HOST, pipelined:
 * batch i's inputs (x_host[i], x_scales_host[i], topk_idx_host[i],
 * topk_w_host[i]; the layouts of moe_forward) are copied in while batch i-1
 * computes, and batch i's output (out_host[i], bf16 [T,H]) is copied back while
 * batch i+1 computes.  The copies run on two streams the plan creates on its
 * first such call on a device (released by moe_plan_destroy); the layers run
 * on `stream`, in order.  Work enqueued on `stream` before the call comes
 * first, and `stream` completes only after every output has landed: the
 * outputs are valid once `stream` has been synchronised.  Host buffers should
 * be pinned (pageable memory works, without overlap); out_host entries may
 * repeat (each batch's copy lands after the previous one).  The workspace
 * holds two staging sets, so consecutive batches never wait for one another's
 * copies.  Two calls with the same plan must be ordered on one stream.
 * Results are byte-identical to moe_forward on the same inputs.
 * Errors: MOE_ERR_INVALID_ARG for n_batches < 1 or a NULL array or entry
 * (x_scales_host may be NULL for MOE_W_BF16), checked before anything is
 * enqueued; MOE_ERR_CUDA if creating the copy streams or an enqueue fails --
 * then the batches enqueued before the failure stay enqueued (synchronise
 * `stream` and the device before reusing the buffers).
 * No counterpart on the pages (a host-buffer serving loop around
 * moe_forward).
 */
moe_status moe_forward_hostio_batches(moe_plan_t plan, int n_batches,
                                      const void *const *x_host,
                                      const uint8_t *const *x_scales_host,
                                      const int32_t *const *topk_idx_host,
                                      const float *const *topk_w_host, const void *w1,
                                      const uint8_t *w1_scales, const void *w2,
                                      const uint8_t *w2_scales, void *const *out_host,
                                      void *workspace, moe_stream_t stream);

/* ---- The steps of moe_forward, callable one by one (same workspace). ---- */

/* Step 1, routing: per-expert histogram, exclusive scan and stable scatter of
 * the T*k slots (slot s = t*k + j).  Results live in the workspace and are
 * exposed by moe_workspace_view(): counts i32[E], offsets i32[E+1], perm i32[S]
 * (position -> slot, ascending slot order within an expert, -1 past the
 * routed slots) and inv i32[S] (slot -> position, -1 for an unrouted slot).
 * Sources: DeepGEMM PR #386 Description (tokens grouped per expert).        */
moe_status moe_route(moe_plan_t plan, const int32_t *topk_idx, void *workspace,
                     moe_stream_t stream);

/* Step 2, gather: copies the x rows (and their scale bytes) of every routed
 * slot into expert order inside the workspace, each expert's block starting
 * at a multiple of 128 rows.  Needs moe_route() first.
 * Source: DeepGEMM PR #386 Description (tokens grouped per expert before the
 * expert GEMMs).
 */
moe_status moe_gather(moe_plan_t plan, const void *x, const uint8_t *x_scales,
                      void *workspace, moe_stream_t stream);

/* Steps 1 and 2 together: the same results as moe_route() followed by
 * moe_gather() (every workspace byte except the multi-block routing scratch).
 * Up to 4096 slots this is one launch in which each block repeats the
 * counting sort in shared memory and then copies its share of rows; above
 * that it enqueues the separate launches.  moe_forward() uses it.  Same
 * argument rules as the two calls.
 * Sources: those of moe_route and moe_gather.
 */
moe_status moe_route_gather(moe_plan_t plan, const int32_t *topk_idx, const void *x,
                            const uint8_t *x_scales, void *workspace, moe_stream_t stream);

/* Step 3, FC1: the FC1 grouped GEMM on the 5th-generation tensor cores with
 * the block scales applied in hardware, the fused (OAI-)SwiGLU, and the FP8
 * E4M3 + UE8M0 1x128 requantisation of the activation, all in one kernel.
 * Needs moe_gather() first.
 * Sources: DeepGEMM PR #445 "Environment" (FP8 E4M3 weights) and Summary
 * (the activation); DeepGEMM PR #386 title (native UE8M0 scales); TensorRT-
 * LLM PR #16346 Description (FP8 + 1x128 UE8M0 requantisation in a GEMM
 * epilogue).
 */
moe_status moe_fc1(moe_plan_t plan, const void *w1, const uint8_t *w1_scales,
                   void *workspace, moe_stream_t stream);

/* Step 4, FC2: grouped GEMM of the requantised activation with W2; bf16 rows
 * written in slot order (y[s], s = t*k + j).  Needs moe_fc1() first.
 * Source: DeepGEMM PR #386 title ("direct combine": rows land where the
 * combine reads them).
 */
moe_status moe_fc2(moe_plan_t plan, const void *w2, const uint8_t *w2_scales,
                   void *workspace, moe_stream_t stream);

/* Steps 3 + 4 in one persistent launch (what moe_forward uses): FC1 tiles and
 * FC2 tiles are handed out by one dynamic tile counter, all FC1 tiles first;
 * an FC2 tile of an m-tile starts once every FC1 tile of that m-tile has
 * published its activation rows.  Same results as moe_fc1() then moe_fc2().
 * Needs moe_gather() first (and moe_route() before it, which resets the
 * launch's counters).
 * Source: fw-ai/DeepGEMM PR #16 Overview (the persistent scheduler and its
 * task-slot release ordering).
 */
moe_status moe_fc1_fc2(moe_plan_t plan, const void *w1, const uint8_t *w1_scales,
                       const void *w2, const uint8_t *w2_scales, void *workspace,
                       moe_stream_t stream);

/* Step 5, combine: out[t] = bf16(sum_j topk_w[t,j] * y[t*k+j]) in fp32, j
 * ascending; unrouted slots are skipped.  Needs moe_fc2() first.
 * Sources: DeepGEMM PR #386 title ("direct combine").                        */
moe_status moe_combine(moe_plan_t plan, const float *topk_w, void *out,
                       void *workspace, moe_stream_t stream);

/* The step before the layer: quantise bf16 activations x_bf16 [T,H] (device)
 * to the layer's input format -- E4M3 codes x_codes u8 [T,H] and one UE8M0
 * scale byte per 1x128 block x_scales u8 [T,H/128] -- with the rule the FC1
 * epilogue uses for the activation: n = smallest integer with
 * max(amax, 1e-4) <= 448 * 2^n, codes = round-to-nearest-even saturating E4M3
 * of x / 2^n, scale byte n + 127 (TensorRT-LLM PR #16346 "DSV4 o_proj: fuse
 * fp8/UE8M0 quantize ...", Description).  Inputs must be finite.  H % 128 == 0,
 * x_bf16 16-byte and x_codes 8-byte aligned.  Needs no plan or workspace.   */
moe_status moe_quantize_act(const void *x_bf16, int T, int H, uint8_t *x_codes,
                            uint8_t *x_scales, moe_stream_t stream);

/* Allocation-free routing.  The pages have no counterpart of this entry point.
 *
 * Same result as moe_route() (counts i32[E], offsets i32[E+1], perm i32[S],
 * inv i32[S], all device pointers owned by the caller, 4-byte aligned), but
 * it needs no workspace and allocates nothing: its
 * scratch (per-block histograms, tile offsets, an error word) is a ~515 KiB
 * array in the library's static device memory, which every GPU that loads the
 * library keeps until the process exits.  It is meant for callers that cannot
 * allocate device memory where they route -- e.g. a runtime whose pooled
 * allocator owns the device's whole budget, or a latency-critical loop where
 * an allocation could synchronise the device.
 *   - Sizes: S = T*k <= MOE_ROUTE_STATIC_MAX_SLOTS and E <= 256; larger
 *     requests return MOE_ERR_UNSUPPORTED and enqueue nothing.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     the call clears what must start at zero.  Calls that overlap on the GPU
 *     (different streams, no ordering between them) race on the array and
 *     must not be issued.
 *   - Expert ids outside [0, E) are handled as moe_route() handles them (the
 *     slot is not routed: inv[s] = -1, -1 is a masked slot), but an id other
 *     than -1 is NOT reported: this entry point has no workspace error word
 *     for moe_check_device_error() to read, and reading its own would need a
 *     device synchronisation.  Callers that must detect bad ids check
 *     counts (sum < T*k) or inv themselves.
 *   - Returns MOE_ERR_CUDA only for a failure of its own launches or copies;
 *     an error left by an earlier, unrelated launch is neither reported nor
 *     cleared.                                                              */
#define MOE_ROUTE_STATIC_MAX_SLOTS (1 << 20)
moe_status moe_route_static(const int32_t *topk_idx, int T, int k, int E,
                            int32_t *counts, int32_t *offsets, int32_t *perm,
                            int32_t *inv, moe_stream_t stream);

/* Device pointers (inside `workspace`) of the intermediate results, for
 * inspection.  Rows of act / act_f32 are in expert order with every expert's
 * block starting at a multiple of 128 rows: expert e's rows are
 * pad_offsets[e] .. pad_offsets[e]+counts[e]-1.                              */
typedef struct {
  int32_t *counts;      /* [E]                                        */
  int32_t *offsets;     /* [E+1]                                      */
  int32_t *perm;        /* [S]                                        */
  int32_t *inv;         /* [S]                                        */
  int32_t *pad_offsets; /* [E+1]  row offsets, multiples of 128       */
  uint8_t *act;         /* FC1 output activation (E4M3, or bf16 for
                           MOE_W_BF16), tiled: read it row-major with
                           moe_copy_act()                             */
  float *act_f32;       /* [rows, I]  the activation before requant,
                           written only when debug capture is on      */
  uint16_t *y;          /* [S, H] bf16, slot order (FC2 output)       */
  uint32_t *error_word; /* bit set = moe_status code seen on device   */
  int64_t rows;         /* capacity of the padded row space           */
} moe_workspace_view_t;

moe_status moe_workspace_view(moe_plan_t plan, void *workspace,
                              moe_workspace_view_t *view);

/* FP8 scale bytes of the activation (FC1 output) for padded row r and block
 * b = column / 128 are stored inside the workspace in the layout the FC2
 * tensor cores read; this copies them out as a plain u8 [rows, I/128] array
 * (device pointer `dst`), enqueued on `stream`.  MOE_ERR_UNSUPPORTED for
 * MOE_W_BF16 plans (no scales).
 * No counterpart on the pages (inspection).
 */
moe_status moe_copy_act_scales(moe_plan_t plan, const void *workspace,
                               uint8_t *dst, moe_stream_t stream);

/* Weight layout.  MOE_WEIGHTS_ROW_MAJOR (default): W1/W2 as described at
 * moe_forward, read by 2-D TMA tiles.  MOE_WEIGHTS_TILED: W1/W2 are the output
 * of moe_prepack_weights() -- the same bytes rearranged into 128 x 128-byte
 * tiles that the tensor cores consume directly, streamed by linear bulk copies
 * (faster; FP8 and BF16 weights, MOE_ERR_UNSUPPORTED for MXFP4).  Weight
 * scales keep their layout in both cases.                                   */
typedef enum {
  MOE_WEIGHTS_ROW_MAJOR = 0,
  MOE_WEIGHTS_TILED = 1,
  /* MXFP4 only: the E2M1 codes stay row-major (read by TMA, which widens them),
   * w1_scales / w2_scales are the output of moe_prepack_weight_scales(),
   * 16-byte aligned.                                                          */
  MOE_WEIGHTS_SCALES_CHUNKED = 2,
  /* MXFP4 only: the E2M1 codes are the output of moe_prepack_weights() (8 KB
   * tiles, one contiguous stream per k-block of 128 weight rows) and the
   * scales that of moe_prepack_weight_scales().  The fastest MXFP4 layout.   */
  MOE_WEIGHTS_TILED_SCALES_CHUNKED = 3
} moe_weight_layout;
moe_status moe_plan_set_weight_layout(moe_plan_t plan, int layout);

/* Rearrange MXFP4 weight scales w1_scales u8 [E,2I,H/32] and w2_scales u8
 * [E,H,I/32] (device, 4-byte aligned) into 512-byte chunks (outputs: device
 * buffers of the same sizes, 16-byte aligned, not overlapping the inputs):
 * with K the row length (H, or I) and rows counted across experts, the chunk
 * of row block b (rows 128b..128b+127) and k-block kb (elements 128kb..+127) is
 * at (b * K/128 + kb) * 512 and holds row r's four scale bytes at
 * (r % 32) * 16 + (r / 32) * 4 -- the layout the tensor core's scale copy
 * reads, so a pipeline stage needs two contiguous 512-byte copies instead of
 * 256 scattered 4-byte reads.  Done once per weight set, on `stream`.
 * MOE_ERR_UNSUPPORTED for other weight formats.
 * No counterpart on the pages (a storage layout for this library's tensor-
 * core kernels).
 */
moe_status moe_prepack_weight_scales(moe_plan_t plan, const uint8_t *w1_scales,
                                     const uint8_t *w2_scales, uint8_t *w1_scales_chunked,
                                     uint8_t *w2_scales_chunked, moe_stream_t stream);

/* GEMM variant for moe_fc1_fc2 / moe_forward.  With tiled FP8 weights the two
 * GEMMs can run on CTA pairs with the 2-SM tensor-core MMA (each pair computes
 * 256 x 256 tiles; each SM loads half of the weight tile).  mode 0: automatic
 * (currently the single-CTA kernel, which measured as fast at every size
 * tried), 1: never, 2: always (MOE_ERR_UNSUPPORTED without tiled FP8
 * weights; set the weight layout first).  Results are the same bytes either
 * way.  On pairs,
 * moe_fc1_fc2 enqueues two kernels: the weight scales (w1_scales, w2_scales)
 * are first expanded into a workspace region, then the GEMMs run.
 * No counterpart on the pages (the B200's 2-SM MMA).
 */
moe_status moe_plan_set_cta_pairs(moe_plan_t plan, int mode);

/* 1 if moe_fc1_fc2 / moe_forward run the GEMMs on CTA pairs with the plan's
 * current settings, 0 if not (or plan is NULL).
 * No counterpart on the pages.
 */
int moe_plan_cta_pairs_active(moe_plan_t plan);

/* Token-major ("swap AB") GEMM tiles, the swapAB variant of the Mega MoE
 * kernels (DeepGEMM PR #445, Summary and its calc_diff table).  The
 * tensor-core MMAs used here have M = 128; a tile with few token rows (an
 * expert's last, ragged tile; every tile at decode sizes) is mostly padding.
 * With swap AB each 128-row weight block is the A operand and the tile's
 * tokens are B, with N = their count rounded up to 16, so the tensor work
 * follows the tokens.  mode 0: automatic, tile by tile (token-major for tiles
 * of at most 96 tokens), 1: never, 2: every tile.  All weight formats; not
 * combined with CTA pairs.  Results agree with token-row tiles within rounding
 * (the sums run in a different order inside the MMA) and are deterministic. */
moe_status moe_plan_set_swap_ab(moe_plan_t plan, int mode);

/* 0: the GEMMs use token-row tiles only; 1: token-major tiles throughout;
 * 2: chosen tile by tile (automatic mode).
 * Source: as moe_plan_set_swap_ab.
 */
int moe_plan_swap_ab_active(moe_plan_t plan);

/* Wide token-major tiles: the token-aware tiling of DeepGEMM PR #386
 * ("Optimize sm100 version with token-aware BM240 tiling, native UE8M0, and
 * direct combine", title).  The tokens of two consecutive 128-row tiles of
 * one expert, up to 240 of them, become one token-major tile (the MMA's N),
 * so an expert with 129..240 tokens streams its weights once instead of
 * twice; two accumulators of 128 weight rows x 240 tokens fill TMEM columns
 * 0..479.  The GEMM launch with wide tiles keeps three pipeline stages (its
 * stages hold two token tiles).  mode 0: automatic (wide tiles for MXFP4
 * weights when the layer has 96 < T*k/E <= 224 slots per expert, where they
 * measured faster; FP8 and BF16 weights measured slower with them), 1: never,
 * 2: always.  Needs
 * token-major tiles (not with moe_plan_set_swap_ab mode 1 or CTA pairs).
 * Results agree with the other tilings within rounding (the MMA's N and the
 * sum order inside it change) and are deterministic.                       */
moe_status moe_plan_set_wide_tiles(moe_plan_t plan, int mode);

/* 1 if moe_fc1_fc2 / moe_forward run the GEMM with wide token-major tiles with
 * the plan's current settings, 0 if not (or plan is NULL).
 * Source: as moe_plan_set_wide_tiles.
 */
int moe_plan_wide_tiles_active(moe_plan_t plan);

/* Rearrange row-major FP8 or BF16 weights w1 [E,2I,H] and w2 [E,H,I] (device)
 * into the tiled layout (w1_tiled, w2_tiled: device buffers of the same sizes,
 * 16-byte aligned; must not overlap the inputs).  With KB = the bytes of one
 * row (K for FP8, 2K for BF16), tile (b, kb) -- rows 128b..128b+127 of the
 * [E*2I, H] (or [E*H, I]) matrix, bytes 128kb..128kb+127 of each row -- is
 * 16384 bytes at offset (b * KB/128 + kb) * 16384, and byte c of tile row r
 * lies at r*128 + ((c/16) XOR (r%8))*16 + c%16.  MXFP4 plans: the packed E2M1
 * codes w1 u8 [E,2I,H/2], w2 u8 [E,H,I/2] go to 8192-byte tiles of 128 rows x
 * 64 bytes (128 codes): with KB = K/2, tile (b, kb) at (b * KB/64 + kb) * 8192
 * holds byte c of row r (bytes 64kb..64kb+63 of the row) at r*64 + c, no
 * swizzle (layout MOE_WEIGHTS_TILED_SCALES_CHUNKED).  Done once per weight set
 * (e.g. at model load), enqueued on `stream`.
 * No counterpart on the pages (a storage layout for this library's tensor-
 * core kernels).
 */
moe_status moe_prepack_weights(moe_plan_t plan, const void *w1, const void *w2,
                               void *w1_tiled, void *w2_tiled, moe_stream_t stream);

/* Copy the FC1 activation codes out of the workspace as a row-major u8
 * [rows, I] array (MOE_W_BF16: bf16 [rows, I]; device pointer `dst`, 16-byte
 * aligned), enqueued on `stream`; inside the workspace they are kept in the
 * tiled layout.
 * No counterpart on the pages (inspection).
 */
moe_status moe_copy_act(moe_plan_t plan, const void *workspace, uint8_t *dst,
                        moe_stream_t stream);

/* Debug flags (0 by default).  Bit 0: FC1 also writes the fp32 activation
 * before requantisation to act_f32 (costs bandwidth); that buffer is placed at
 * the end of the workspace, so setting or clearing bit 0 changes
 * moe_workspace_bytes() (query it again and allocate at least that much
 * before the next call) but moves no other buffer.  Bit 1: test hook for
 * the failure path -- in the fused FC1+FC2 launch (moe_fc1_fc2, moe_forward
 * without CTA pairs) every FC2 tile waits for one FC1 completion more than its
 * m-tile can provide, so that bounded wait runs out (about 2 s): the launch
 * stops, the error word gets MOE_ERR_DEVICE_TIMEOUT, nothing traps or hangs,
 * and the output is undefined.  Other bits: MOE_ERR_INVALID_ARG.
 * No counterpart on the pages.
 */
moe_status moe_plan_set_debug(moe_plan_t plan, int flags);

/* Zero the workspace's device error word (enqueued on `stream`).
 * No counterpart on the pages.
 */
moe_status moe_clear_device_error(moe_plan_t plan, void *workspace,
                                  moe_stream_t stream);

/* Synchronises `stream`, reads the device error word and returns MOE_OK or
 * the most severe recorded status (timeout before bad routing).
 * No counterpart on the pages.
 */
moe_status moe_check_device_error(moe_plan_t plan, const void *workspace,
                                  moe_stream_t stream);

/* Human-readable name of a status code (static string).
 * No counterpart on the pages.
 */
const char *moe_status_str(moe_status status);

/* Kernel launches one moe_forward enqueues for this plan.
 * No counterpart on the pages.
 */
int moe_forward_launch_count(moe_plan_t plan);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
