/*
 * dmoe.h -- C ABI of libdmoe.so, the dropless mixture-of-experts (dMoE) expert layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (MegaBlocks walkthrough "02 · dropless MoE 与 block-sparse 重构", sections 2-4;
 * Fast-LLM issue #56 "[feat] Support sparse copy for a large number of experts", error log):
 *   1. route each token to its top-k experts (top-k of the softmax over E logits);
 *   2. build the sparse map: per-expert histogram, stable sort of (token, slot) entries by
 *      expert, bins, padded_bins rounded up to 128 rows so that every 128-row block belongs
 *      to exactly one expert (walkthrough section 2, section 4.1);
 *   3. padded_gather: copy each token row to its padded row (section 4.2);
 *   4. gated-SiLU expert FFN on the non-empty 128-row blocks only:
 *        H = silu(X_pad W1_e^T) * (X_pad W3_e^T),  Y_pad = H W2_e^T
 *      (block-sparse view of sections 2-3; gated SiLU of the issue's config);
 *   5. padded_scatter: y_t = sum_s w_ts * Y_pad[dest_row[t*k+s]] (section 4.2);
 *   6. backward: gather and scatter swap roles, plus the routing-weight gradient
 *      (section 4.2); the activation is recomputed from the saved pre-activations
 *      (section 4.4).  Only X_pad, A and Bm are kept for it: the routing-weight gradient
 *      <dy_t, Y_ts> is formed as <dy_t W2_e, H_ts> inside the dH GEMM, so neither H nor
 *      Y_pad has to outlive the forward (the activation-memory saving of SonicMoE, abstract).
 *
 * Conventions (all entry points)
 *   - The caller owns and allocates ALL device memory, including workspaces; the library
 *     never allocates, frees or synchronises.  Query sizes with dmoe_workspace_bytes and
 *     dmoe_saved_bytes.
 *   - Every launch is asynchronous on `stream` (a cudaStream_t, passed as void*; NULL is
 *     the legacy default stream).  No call reads device memory on the host, so the whole
 *     layer can run without a host synchronisation, and a whole step can be captured in a
 *     CUDA graph.  Kernels are launched with programmatic dependent launch: a kernel may
 *     start before the previous kernel on the stream has finished, but it waits for all
 *     earlier work of the stream before its first access to global memory, so stream
 *     ordering is exactly as for plain launches, also with the caller's own kernels.
 *   - Every call returns an int: DMOE_OK (0) or a negative DMOE_ERR_* detected on the host
 *     BEFORE any launch (nothing is launched then), or DMOE_ERR_LAUNCH if a launch failed.
 *   - Conditions only the device can see set bits in the caller's int32 status word
 *     (dmoe_map.status); read it after synchronising and decode with dmoe_status_string.
 *     No kernel traps; every wait in a kernel is bounded and sets DMOE_STATUS_TIMEOUT when
 *     it gives up.
 *   - All device pointers must be 16-byte aligned.
 *   - bf16 = IEEE bfloat16 stored as uint16; all matrices row-major, C-contiguous.
 *   - Weights use the (out, in) layout: W1, W3 are [E, ffn, hidden] (W1 = gate, W3 = up),
 *     W2 is [E, hidden, ffn].
 *   - Entries are flattened j = t*k + s (token t, slot s); this is the flattening implied by
 *     the gather rule "source row = index_a // TOP_K" (walkthrough section 4.2).
 *   - Blocking is fixed at 128 rows ("self.blocking = 128", walkthrough section 2).
 *   - Requires an sm_100 device (B200); other devices get DMOE_ERR_DEVICE.
 */
#ifndef DMOE_H
#define DMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols exported from libdmoe.so (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define DMOE_API __attribute__((visibility("default")))
#else
#define DMOE_API
#endif

#define DMOE_BLOCKING 128
#define DMOE_MAX_EXPERTS 1024
#define DMOE_MAX_TOP_K 32

/* Error codes (returned). */
#define DMOE_OK 0
#define DMOE_ERR_NULL (-1)             /* a required pointer is NULL */
#define DMOE_ERR_SHAPE (-2)            /* ffn % 128 != 0 (walkthrough section 5: the topology
                                          rejects it), hidden % 128 != 0, T < 1, top_k < 1,
                                          top_k > E, top_k > DMOE_MAX_TOP_K */
#define DMOE_ERR_TOO_MANY_EXPERTS (-3) /* E < 1 or E > DMOE_MAX_EXPERTS: a documented limit,
                                          never an opaque resource failure (the issue's
                                          OutOfResources at E = 64) */
#define DMOE_ERR_WORKSPACE (-4)        /* workspace smaller than dmoe_workspace_bytes */
#define DMOE_ERR_ALIGN (-5)            /* a pointer is not 16-byte aligned */
#define DMOE_ERR_LAUNCH (-6)           /* a CUDA launch or runtime call failed */
#define DMOE_ERR_DEVICE (-7)           /* current device is not sm_100 */
#define DMOE_ERR_TOO_LARGE (-8)        /* T*top_k or the padded row bound exceeds 2^31-1 */

/* Device status bits (OR-ed into dmoe_map.status by the kernels). */
#define DMOE_STATUS_NONFINITE_LOGITS 0x1   /* a NaN or +-inf logit was routed on */
#define DMOE_STATUS_EXPERT_OUT_OF_RANGE 0x2 /* caller-given top_experts outside [0, E) */
#define DMOE_STATUS_DUPLICATE_EXPERT 0x4   /* caller-given top_experts repeat within a token */
#define DMOE_STATUS_TIMEOUT 0x8            /* a bounded in-kernel wait gave up */

/* Problem shape.  T tokens, hidden size h, ffn size f (per expert), E experts, top_k, and
 * the variant flags: 0 (the default: weights are the softmax over all E logits at the chosen
 * experts, and the forward saves X_pad, A and Bm for the backward) or an OR of
 * DMOE_ROUTE_RENORMALIZE or DMOE_ROUTE_TOKEN_ROUNDING (not both), DMOE_FUSED_COMBINE and
 * DMOE_SAVE_X_ONLY.  Other bits are rejected.  Every call of one layer instance must see the
 * same flags. */
typedef struct {
  int32_t T, hidden, ffn, num_experts, top_k;
  int32_t flags;
} dmoe_dims;

/* Routing variant: the k weights of a token are the softmax over its k chosen logits only,
 * so they sum to 1 (the top-k renormalisation some MoE layers use; the pages' default does
 * not renormalise).  Read by dmoe_sparse_map (weights) and the router backward (dlogits). */
#define DMOE_ROUTE_RENORMALIZE 0x1

/* Block floating point of the padded expert outputs (Y_pad of dmoe_expert_down, dX_pad of
 * dmoe_bwd_dx): fp16 values [P_max, h] and fp32 scales [P_max, 4 * ceil(h / 512)] (ceil(h/128)
 * scales per row, the row padded to a multiple of 4); the value of row r, column c is
 * fp16[r][c] * |scale[r][c / DMOE_SCALE_COLS]|.  Each scale is a power of two chosen from the
 * largest magnitude m of its 128 columns: the one that puts m into [2^13, 2^14), except that
 * for m < 2^-11 it stops at 2^24 (the largest power of two fp16 holds; m then still lands on a
 * normal fp16 down to m = 2^-38), and 1 for an all-zero group.  The sign bit of a scale is set
 * when fp16 cannot hold the scale itself (m < 2^-38 or m >= 2^29) and for a group holding an
 * inf or NaN (magnitude 1, values unscaled); the combine sums the other groups with the
 * mixed-precision fma (fp16 value times fp16 scale into fp32) and converts these.  Every value
 * keeps fp16's 11 significant bits at bf16's size.  Scale pointers are 16-byte aligned like
 * every other pointer.  The k rows of a token are summed afterwards in fp32; rounding each to
 * bf16 first (8 bits) would put k roundings into every output element (measured at full
 * size: 5.2-5.4 % of the output's RMS at the largest element, against 3.1-3.3 % this way). */
#define DMOE_SCALE_COLS 128

/* Routing variant: tile-aware token rounding (SonicMoE abstract: the routing is rounded so that
 * every expert's token count is a multiple of the GEMM tile, and the grouped GEMMs compute no
 * padding rows).  The abstract gives the method in one sentence; this library's reading: for
 * every expert e whose top-k count c_e has r = c_e mod 128 != 0, when r >= 64 and at least
 * 128 - r tokens are not routed to e, the 128 - r best-ranked such tokens are added to e
 * (round up); otherwise e's r worst-ranked entries are dropped (round down).  A token ranks
 * for expert e by its logit l[t][e], larger first, equal logits by the lower token index.  A
 * token keeps its surviving slots in slot order, then its added experts in increasing expert
 * order; every entry's weight is the softmax over all E logits at its expert.
 *   The map then holds a token-major entry list of N' <= dmoe_entries_max(dims) = T*k + 64*E
 *   entries: map->entry_offsets [T+1] (token t owns entries [offsets[t], offsets[t+1])),
 *   top_experts / weights [entries_max] (expert and weight of each entry; past N': -1 and 0),
 *   indices / bin_ids / dest_row [entries_max] over those entries (dest_row -1 past N'), and
 *   tokens_per_expert / bins / padded_bins of the rounded counts (padded_bins == bins).
 *   Forward, backward and the step calls follow the list (dweights per entry).  The router
 *   calls, dmoe_expert_glu_gather and dmoe_sparse_map_noalloc reject the flag
 *   (DMOE_ERR_SHAPE), as does T > 2^20; dmoe_sparse_map needs the logits. */
#define DMOE_ROUTE_TOKEN_ROUNDING 0x2

/* Forward variant: the weighted combine fused into the down GEMM (the walkthrough's padded
 * scatter, section 4.2, done by the GEMM's epilogue; the SonicMoE abstract's IO overlap).  The
 * epilogue multiplies each real padded row's fp32 result by its routing weight and adds it,
 * with vector reductions, into an fp32 token-major accumulator; a last pass rounds it to
 * bf16.  Y_pad is never written or read.  The additions of a token's k rows happen in any
 * order: bit-for-bit reproducible for top_k <= 2 (a + b = b + a from zero), reproducible to
 * fp32 rounding otherwise.  dmoe_forward then runs dmoe_padded_gather, dmoe_expert_glu and
 * dmoe_expert_down_combine.  Not combined with DMOE_ROUTE_TOKEN_ROUNDING (DMOE_ERR_SHAPE). */
#define DMOE_FUSED_COMBINE 0x8

/* Memory variant (walkthrough section 4.4's MemoryOptimizedMLP; the SonicMoE abstract's
 * activation-memory saving): the training forward saves only X_pad (dmoe_saved_bytes shrinks
 * from (2h + 4f) to 2h bytes per padded row) and dmoe_backward recomputes A and Bm with one
 * more GLU GEMM (4*N*h*f FLOP) into its workspace (DMOE_WS_BACKWARD grows by 4f bytes per
 * padded row).  Every result is bit-identical to the default variant's. */
#define DMOE_SAVE_X_ONLY 0x4

/* The sparse map.  All device pointers, caller-owned; N = T*top_k entries (with
 * DMOE_ROUTE_TOKEN_ROUNDING: dmoe_entries_max(dims) and the token-major layout described
 * there), P_max = dmoe_padded_rows_max(dims).  Meaning (walkthrough sections 4.1-4.3):
 *   top_experts [T, k] int32   expert of entry t*k+s, slot s = s-th pick in descending
 *                              logit order, ties to the lower expert index.  Output of
 *                              dmoe_sparse_map when logits are given, else its INPUT.
 *   weights     [T, k] fp32    softmax over all E logits at the chosen expert (no
 *                              renormalisation over the k picks; with DMOE_ROUTE_RENORMALIZE,
 *                              the softmax over the k chosen logits).  Output when logits are
 *                              given; otherwise caller-provided and only read by forward.
 *   tokens_per_expert [E]      histogram of top_experts
 *   bins [E]                   inclusive cumsum of tokens_per_expert
 *   padded_bins [E]            inclusive cumsum of round_up(tokens_per_expert, 128)
 *   indices [N]                entries stably sorted by expert: flattened entry index
 *   bin_ids [N]                expert of the i-th sorted entry
 *   dest_row [N]               padded row of entry j: (i - bins[e-1]) + padded_bins[e-1],
 *                              i its sorted position, e its expert, bins[-1] = 0
 *   block_expert [P_max/128]   expert owning 128-row block b; -1 for b >= num_blocks
 *   num_blocks [1]             padded_bins[E-1] / 128
 *   status [1]                 device status bits; dmoe_sparse_map overwrites it with its own */
typedef struct {
  int32_t *top_experts;
  float *weights;
  int32_t *tokens_per_expert;
  int32_t *bins;
  int32_t *padded_bins;
  int32_t *indices;
  int32_t *bin_ids;
  int32_t *dest_row;
  int32_t *block_expert;
  int32_t *num_blocks;
  int32_t *status;
  int32_t *entry_offsets; /* [T+1], DMOE_ROUTE_TOKEN_ROUNDING only (may be NULL otherwise) */
} dmoe_map;

/* Workspace kinds for dmoe_workspace_bytes. */
#define DMOE_WS_MAP 0      /* dmoe_sparse_map */
#define DMOE_WS_FORWARD 1        /* dmoe_forward with saved == NULL (inference) */
#define DMOE_WS_BACKWARD 2       /* dmoe_backward */
#define DMOE_WS_FORWARD_TRAIN 3  /* dmoe_forward with saved != NULL (training) */
#define DMOE_WS_ROUTER_BACKWARD 4 /* dmoe_router_backward */

/* Columns per routing-weight partial sum of the dH GEMM: dmoe_bwd_dglu's partials have
 * ceil(ffn / DMOE_DGLU_TILE_COLS) columns per row. */
#define DMOE_DGLU_TILE_COLS 128

/* Static bound on the padded row count: floor((T*k + 127*E)/128)*128.  Every padded
 * buffer is sized from it, so no call needs the data-dependent size on the host (the
 * walkthrough's padded_gather reads padded_bins[-1] on the host, section 4.2; this library
 * does not). Returns 0 for invalid dims. */
DMOE_API size_t dmoe_padded_rows_max(const dmoe_dims *dims);

/* Entries of the map: T*top_k, or with DMOE_ROUTE_TOKEN_ROUNDING the bound T*top_k + 64*E on
 * the rounded entry list (0 for invalid dims).  P_max is computed from it. */
DMOE_API size_t dmoe_entries_max(const dmoe_dims *dims);

/* Bytes of workspace the call `kind` needs (0 for invalid dims). */
DMOE_API size_t dmoe_workspace_bytes(const dmoe_dims *dims, int kind);

/* Bytes of the activations dmoe_forward saves for dmoe_backward, and their byte offsets
 * inside that buffer: offsets[0] X_pad [P_max,h], [1] A = X_pad W1^T [P_max,f],
 * [2] Bm = X_pad W3^T [P_max,f], all bf16 (H and Y_pad are not kept: the backward recomputes
 * the activation from A and Bm and never needs Y_pad).  With DMOE_SAVE_X_ONLY only X_pad is
 * kept (offsets[1] = offsets[2] = 0).  offsets may be NULL.  Returns 0 for invalid dims. */
DMOE_API size_t dmoe_saved_bytes(const dmoe_dims *dims, size_t offsets[3]);

/* Routing + sparse map (walkthrough section 4.1; the Fast-LLM get_sparse_map step).
 *   logits: [T, E] bf16 device pointer, or NULL to take map->top_experts as given (then
 *           map->weights is not written; out-of-range or duplicate experts set status bits
 *           and such entries are dropped from the map).
 *   map:    caller-owned outputs (see dmoe_map); map->status is overwritten with the map's
 *           own bits (later calls OR theirs in).
 *   ws:     workspace of dmoe_workspace_bytes(dims, DMOE_WS_MAP) bytes.
 * Shared memory per CTA is O(E) and independent of T (the issue's kernel needed 262144 B
 * at E = 64, top-8, 2 x 2048 tokens).  Three kernels, no global atomics but one completion
 * ticket, no host sync; results are deterministic. */
DMOE_API int dmoe_sparse_map(const dmoe_dims *dims, const void *logits, const dmoe_map *map, void *ws,
                    size_t ws_bytes, void *stream);

/* Forward of the expert layer (walkthrough section 4.5 schematic, gated SiLU).
 *   x [T,h], w1 [E,f,h], w3 [E,f,h], w2 [E,h,f]: bf16 inputs.  map: from dmoe_sparse_map.
 *   y [T,h] bf16 output.
 *   saved: NULL for inference, else a buffer of dmoe_saved_bytes(dims) bytes that receives
 *          X_pad, A, Bm for dmoe_backward.
 *   ws: dmoe_workspace_bytes(dims, DMOE_WS_FORWARD) bytes when saved == NULL, else
 *       dmoe_workspace_bytes(dims, DMOE_WS_FORWARD_TRAIN) bytes (H and Y_pad, dead after the
 *       call returns on the stream).
 * Runs padded_gather, the GLU GEMM, the down GEMM and the weighted padded_scatter. */
DMOE_API int dmoe_forward(const dmoe_dims *dims, const void *x, const void *w1, const void *w3,
                 const void *w2, const dmoe_map *map, void *y, void *saved, void *ws,
                 size_t ws_bytes, void *stream);

/* Backward (walkthrough section 4.2: the gradient of padded_scatter is padded_gather plus a
 * routing-weight gradient, the gradient of padded_gather is padded_scatter; section 4.4:
 * the activation is recomputed from the saved pre-activations).
 *   dy [T,h] bf16; w1, w3, w2 as in dmoe_forward; map from dmoe_sparse_map; saved from
 *   dmoe_forward(saved != NULL).
 *   Outputs: dx [T,h] bf16; dw1, dw3 [E,f,h] fp32; dw2 [E,h,f] fp32 (the weight gradients
 *   of a mixed-precision step are kept in fp32; experts that receive no token get exact
 *   zeros); dweights [T,k] fp32 = <dy_t, Y_ts>, where Y_ts = H_ts W2_e^T is the expert's
 *   unweighted output row, computed as <dy_t W2_e, H_ts>.  All results are deterministic.
 *   ws: dmoe_workspace_bytes(dims, DMOE_WS_BACKWARD) bytes.
 *   Runs dmoe_padded_gather(dy), dmoe_bwd_dglu, dmoe_bwd_wgrad, dmoe_bwd_dx and
 *   dmoe_bwd_scatter in that order. */
DMOE_API int dmoe_backward(const dmoe_dims *dims, const void *dy, const void *w1, const void *w3,
                  const void *w2, const dmoe_map *map, const void *saved, void *dx, float *dw1,
                  float *dw3, float *dw2, float *dweights, void *ws, size_t ws_bytes,
                  void *stream);

/* Allocation-free variant of dmoe_sparse_map.  The pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory when they build the map, e.g.
 * a plugin whose host application owns every device allocation, or a loop that must not
 * call cudaMalloc (it can synchronise the device and its cost is unbounded), and therefore
 * cannot provide the DMOE_WS_MAP workspace.
 *   Same arguments, results and status bits as dmoe_sparse_map, without ws / ws_bytes.
 *   Scratch: a static array of DMOE_NOALLOC_SCRATCH_BYTES in device global memory inside
 *     libdmoe.so; every GPU that loads the library holds it until the process exits.  The
 *     call needs (ceil(T/64) * (num_experts + 1) + 1 + ceil(T/32768) * num_experts) * 4
 *     bytes of it and returns DMOE_ERR_WORKSPACE, before any launch, when that exceeds the
 *     limit (e.g. T > 65152 at E = 256).
 *   The call performs no allocation (no cudaMalloc, no cudaFree, no allocating library
 *     routine).  Its first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (once per device, with that device current); make that first call
 *     before any stream capture.  The address stays cached for the life of the process: after
 *     cudaDeviceReset (or anything else that destroys and re-creates the device's primary
 *     context) the array may move, so such a caller must unload and reload libdmoe.so before
 *     calling this entry point again.
 *   Every call on a device shares the one array and leaves its contents behind; each call
 *     rewrites all of the scratch it reads before reading it, so stale contents never leak
 *     into a result.  Calls whose executions overlap on the GPU (different streams, or
 *     different host threads without ordering) race on the array: serialise them. */
#define DMOE_NOALLOC_SCRATCH_BYTES (1u << 20)
DMOE_API int dmoe_sparse_map_noalloc(const dmoe_dims *dims, const void *logits,
                                     const dmoe_map *map, void *stream);

/* ---- Step entry points (each one kernel; dmoe_forward is exactly this sequence). ---- */

/* padded_gather (walkthrough section 4.2, A_TO_B direction): x_pad[dest_row[t*k+s]] = x[t]
 * for every slot s; the padding rows of every expert's last block are written as zeros
 * (section 5: padding rows hold zeros).  x [T,h] bf16 -> x_pad [P_max,h] bf16; rows at or
 * beyond num_blocks*128 are not touched. */
DMOE_API int dmoe_padded_gather(const dmoe_dims *dims, const void *x, const dmoe_map *map, void *x_pad,
                       void *stream);

/* GLU GEMM over the non-empty row blocks: for every block b < num_blocks with expert
 * e = block_expert[b], A = X_pad[b] W1_e^T, Bm = X_pad[b] W3_e^T (fp32 accumulation in
 * tensor memory) and H[b] = bf16(silu(A) * Bm).  a_out / b_out (both or neither) receive
 * bf16(A), bf16(Bm); h_out may be NULL when they are given (the recompute of
 * DMOE_SAVE_X_ONLY).  x_pad [P_max,h] -> h_out, a_out, b_out [P_max,f], all bf16. */
DMOE_API int dmoe_expert_glu(const dmoe_dims *dims, const void *x_pad, const void *w1, const void *w3,
                    const dmoe_map *map, void *h_out, void *a_out, void *b_out, void *stream);

/* GLU GEMM with the padded gather fused into its operand load (walkthrough section 4.2's
 * gather, out[index_b] = x[index_a // TOP_K], done by the GEMM's TMA row gathers, four rows
 * per instruction): the same results as dmoe_padded_gather followed by dmoe_expert_glu, bit
 * for bit, and X_pad is never written or read.  x [T,h] bf16 -> h_out (a_out, b_out: both or
 * neither) [P_max,f] bf16.  Measured on B200 it is about 3x slower than the gather kernel +
 * dmoe_expert_glu (the row-gather instruction rate cannot feed the MMAs), so dmoe_forward
 * does not use it; it serves callers that cannot hold the X_pad buffer. */
DMOE_API int dmoe_expert_glu_gather(const dmoe_dims *dims, const void *x, const void *w1,
                                    const void *w3, const dmoe_map *map, void *h_out, void *a_out,
                                    void *b_out, void *stream);

/* Down GEMM: Y_pad[b] = w * (H[b] W2_e^T) for every block b < num_blocks, fp32
 * accumulation, each row times the routing weight w of its entry (map->weights; 0 for a
 * padding row: the walkthrough's section 4.2 scatter weight, applied here so that the combine
 * sums unweighted rows), stored in block floating point (see DMOE_SCALE_COLS).
 * h_in [P_max,f] bf16 -> y_pad [P_max,h] fp16, y_scale [P_max, 4*ceil(h/512)] fp32. */
DMOE_API int dmoe_expert_down(const dmoe_dims *dims, const void *h_in, const void *w2,
                              const dmoe_map *map, void *y_pad, float *y_scale, void *stream);

/* Down GEMM and weighted combine in one (DMOE_FUSED_COMBINE): y_t = bf16(sum over the
 * token's entries of w_ts * (H W2_e^T) row), the sum in fp32 in y_acc by vector reductions
 * from the GEMM's epilogue.  h_in [P_max,f] bf16, map->weights -> y [T,h] bf16; y_acc: T*h
 * fp32 of caller workspace (zeroed by the call).  Three launches: zero, GEMM, rounding. */
DMOE_API int dmoe_expert_down_combine(const dmoe_dims *dims, const void *h_in, const void *w2,
                                      const dmoe_map *map, void *y, float *y_acc, void *stream);

/* Weighted padded_scatter (walkthrough section 4.2, B_TO_A direction, times the routing
 * weight): y_t = bf16(sum_{s=0..k-1} w_ts * Y_pad[dest_row[t*k+s]]), summed in fp32 in
 * slot order (each entry one fused multiply-add), no atomics.  weights == NULL means w = 1:
 * the rows of dmoe_expert_down, which already carry their routing weight, and the backward's
 * gather gradient, dx_t = sum_s dX_pad[dest_row[t*k+s]].  Row format: y_scale == NULL:
 * y_pad [P_max,h] bf16; otherwise block floating point (see DMOE_SCALE_COLS: y_pad fp16,
 * y_scale [P_max, 4*ceil(h/512)]).  -> y [T,h] bf16. */
DMOE_API int dmoe_padded_scatter(const dmoe_dims *dims, const void *y_pad, const float *y_scale,
                                 const dmoe_map *map, const float *weights, void *y,
                                 void *stream);

/* ---- Backward step entry points (each one kernel).  dmoe_backward is: dy_pad =
 * dmoe_padded_gather(dy) (the gradient of the weighted scatter is a gather, walkthrough
 * section 4.2; the weight is applied inside the dH GEMM), then dglu, wgrad, dx, scatter. ---- */

/* dH GEMM with the gated-SiLU gradient and the routing-weight gradient fused into its
 * epilogue (walkthrough section 4.4: the activation is recomputed from the saved
 * pre-activations instead of being stored; section 4.2: the routing-weight gradient).
 * For every row block b < num_blocks of expert e, with G = dY_pad[b] W2_e (fp32; dY_pad holds
 * the unweighted rows of dy), s = sigmoid(A), h = A*s*Bm and w the routing weight of the row
 * (0 for a padding row):
 *   da = bf16(w*G*Bm*s*(1 + A(1-s))),  dbm = bf16(w*G*A*s),  hw = bf16(w*h)   [P_max,f];
 *   dw_part[r * nt + n] = sum over the columns c of group n of G[r,c]*h[r,c]   (fp32,
 *     nt = ceil(f / DMOE_DGLU_TILE_COLS) groups of 128 columns; since G h^T = dy (H W2_e^T)^T,
 *     the groups of a row sum to the routing-weight gradient <dy_t, Y_ts>).
 * map->weights is read.  a_saved, bm_saved: bf16 A, Bm of dmoe_forward; dy_pad [P_max,h]. */
DMOE_API int dmoe_bwd_dglu(const dmoe_dims *dims, const void *dy_pad, const void *w2,
                           const void *a_saved, const void *bm_saved, const dmoe_map *map,
                           void *da, void *dbm, void *hw, float *dw_part, void *stream);

/* dX GEMM: dX_pad[b] = dA[b] W1_e + dBm[b] W3_e, one fp32 accumulator over both K passes,
 * stored in block floating point (see DMOE_SCALE_COLS): the k rows of a token are summed by
 * dmoe_bwd_scatter, and rounding each of them to bf16 first would put k bf16 roundings into
 * every element of dx.
 * da, dbm [P_max,f] bf16 -> dx_pad [P_max,h] fp16, dx_scale [P_max, 4*ceil(h/512)] fp32. */
DMOE_API int dmoe_bwd_dx(const dmoe_dims *dims, const void *da, const void *dbm, const void *w1,
                         const void *w3, const dmoe_map *map, void *dx_pad, float *dx_scale,
                         void *stream);

/* Weight gradients, per expert e over its padded rows r in [padded_bins[e-1], padded_bins[e])
 * (padding rows are zero, so they add nothing; the walkthrough's stk path needs a transposed
 * topology for this, section 4.3; here each output tile walks its expert's rows directly):
 *   dW1_e = sum_r dA_r^T X_pad_r,  dW3_e = sum_r dBm_r^T X_pad_r  ([f,h] each),
 *   dW2_e = sum_r dY_pad_r^T Hw_r  ([h,f]; dY_pad unweighted, Hw = w*H from dmoe_bwd_dglu);
 * fp32 accumulation and fp32 output (dw1, dw3, dw2 are float*), no split-K, so the result is
 * deterministic; experts without rows get exact zeros. */
DMOE_API int dmoe_bwd_wgrad(const dmoe_dims *dims, const void *x_pad, const void *hw,
                            const void *dy_pad, const void *da, const void *dbm,
                            const dmoe_map *map, float *dw1, float *dw3, float *dw2, void *stream);

/* Scatter-sum of the backward plus the routing-weight gradient (walkthrough section 4.2: the
 * gradient of padded_gather is padded_scatter with w = 1):
 *   dx_t = bf16(sum_s dX_pad[dest_row[t*k+s]])  (fp32 sum in slot order),
 *   dweights[t*k+s] = sum_{n < nt} dw_part[dest_row[t*k+s] * nt + n]  (fp32, tile order; 0 for
 *   an entry dropped from the map).
 * dx_pad, dx_scale from dmoe_bwd_dx (each row's values are fp16 * scale, exact in fp32),
 * dw_part from dmoe_bwd_dglu -> dx [T,h] bf16, dweights [T,k] fp32. */
DMOE_API int dmoe_bwd_scatter(const dmoe_dims *dims, const void *dx_pad, const float *dx_scale,
                              const float *dw_part, const dmoe_map *map, void *dx,
                              float *dweights, void *stream);

/* ---- The linear router (the steps on either side of the routing). ----
 * The pages fix only the router's output, (scores, top_experts) (issue #56 error log;
 * "router(x)" in the walkthrough's schematic forward, section 4.5).  These calls implement
 * the plainest reading: a linear router without bias, logits = x W_r^T with W_r [E, h] bf16
 * in the (out, in) layout, whose bf16 logits feed dmoe_sparse_map.  They require
 * num_experts % 8 == 0 (DMOE_ERR_SHAPE otherwise: the [T, E] rows must be multiples of 16
 * bytes). */

/* logits [T, E] = bf16(x W_r^T), fp32 accumulation on the tensor cores.  x [T, h] bf16.
 * status: the int32 device status word that a bounded wait that gives up marks with
 * DMOE_STATUS_TIMEOUT (e.g. map->status). */
DMOE_API int dmoe_router_forward(const dmoe_dims *dims, const void *x, const void *w_router,
                                 void *logits, int32_t *status, void *stream);

/* Gradient of the routing weights with respect to the logits: with p_t = softmax(logits_t)
 * over all E (fp32; with DMOE_ROUTE_RENORMALIZE over the k chosen experts, zero elsewhere)
 * and j_s = map->top_experts[t][s],
 *   dlogits[t][i] = sum_s dweights[t][s] * p_t[j_s] * ([i == j_s] - p_t[i])
 * (the expert choice itself carries no gradient).  logits [T, E] bf16 (the ones routed),
 * dweights [T, k] fp32 (from dmoe_backward) -> dlogits [T, E] bf16. */
DMOE_API int dmoe_router_dlogits(const dmoe_dims *dims, const void *logits, const dmoe_map *map,
                                 const float *dweights, void *dlogits, void *stream);

/* Backward of the router: dlogits as in dmoe_router_dlogits, then
 *   dx [T, h] bf16 += dlogits W_r    (in place: dx holds the expert path's input gradient from
 *                                     dmoe_backward; the sum is formed in fp32, rounded once),
 *   dw_router [E, h] fp32 = dlogits^T x   (overwritten; split over the tokens into fp32
 *                                     partials that are summed in a fixed order, so the result
 *                                     is deterministic).
 * ws: dmoe_workspace_bytes(dims, DMOE_WS_ROUTER_BACKWARD) bytes (dlogits and the partials).
 * map: from dmoe_sparse_map (top_experts; status receives timeout bits). */
DMOE_API int dmoe_router_backward(const dmoe_dims *dims, const void *x, const void *w_router,
                                  const void *logits, const dmoe_map *map, const float *dweights,
                                  void *dx, float *dw_router, void *ws, size_t ws_bytes,
                                  void *stream);

/* ---- Diagnostics. ---- */
DMOE_API const char *dmoe_error_string(int code);
/* Human-readable list of the bits set in a host copy of the status word. */
DMOE_API const char *dmoe_status_string(int32_t status);
/* Library version, e.g. "dmoe-b200 0.1". */
DMOE_API const char *dmoe_version(void);

/* Test-only fault injection (no counterpart on the pages; it exercises the library's own
 * failure path).  With enable != 0, the NEXT grouped-GEMM launch of this process (any GEMM
 * step) runs with a wait budget of ~10^7 cycles and its pair leaders withhold their first
 * operand stage: the MMA's bounded wait on that stage expires, the kernel sets
 * DMOE_STATUS_TIMEOUT in map->status, every role of every CTA leaves through its own
 * bounded waits, and the launch returns normally with that launch's results invalid.  No
 * trap, no fault; the context stays usable.  The switch clears itself on that launch. */
DMOE_API int dmoe_debug_inject_stall(int enable);

#ifdef __cplusplus
}
#endif

#endif /* DMOE_H */
