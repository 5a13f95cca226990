// kernels.h -- host-side launchers of the dMoE kernels (internal to libdmoe.so).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dmoe {

// Tokens per map tile: one CTA of the routing/histogram kernel and of the stable-scatter
// kernel handles this many tokens (kMapTokTile * top_k entries).
constexpr int kMapTokTile = 64;

inline int map_tiles(int T) { return (T + kMapTokTile - 1) / kMapTokTile; }

// The scan covers the tiles in segments of kScanSeg (32 warps x kScanCache tiles in registers).
constexpr int kScanCache = 16;
constexpr int kScanSeg = 32 * kScanCache;
inline int map_segments(int T) { return (map_tiles(T) + kScanSeg - 1) / kScanSeg; }

// Map workspace: per-tile histograms [map_tiles(T), E] int32, one ticket counter, one status
// word per tile, then the per-segment expert totals (later prefixes) [map_segments(T), E].
inline size_t map_workspace_ints(int T, int E) {
  return (size_t)map_tiles(T) * E + 1 + (size_t)map_tiles(T) + (size_t)map_segments(T) * E;
}
inline unsigned int *map_ticket(int32_t *tile_hist, int T, int E) {
  return reinterpret_cast<unsigned int *>(tile_hist + (size_t)map_tiles(T) * E);
}
inline int32_t *map_flags(int32_t *tile_hist, int T, int E) {
  return tile_hist + (size_t)map_tiles(T) * E + 1;
}
inline int32_t *map_segs(int32_t *tile_hist, int T, int E) {
  return tile_hist + (size_t)map_tiles(T) * E + 1 + (size_t)map_tiles(T);
}

// Map: routing + per-tile histogram (logits given) or histogram of given top_experts
// (absent_ok: an expert id of -1 marks an absent entry, left out without a status bit).
cudaError_t launch_route_hist(const uint16_t *logits, int T, int E, int k, bool renorm, int32_t *top,
                              float *weights, int32_t *tile_hist, cudaStream_t st,
                              bool absent_ok = false);
// Map: scan over tiles and experts; bins, padded_bins, num_blocks and the status word
// (overwritten with the call's bits, or OR-ed into with or_status).
cudaError_t launch_map_scan(int T, int E, int32_t *tile_hist, int32_t *tokens_per_expert,
                            int32_t *bins, int32_t *padded_bins, int32_t *num_blocks,
                            int32_t *status, cudaStream_t st, bool or_status = false);
// Map: stable scatter of entries to sorted order (indices, bin_ids, dest_row) and the
// block -> expert table.
cudaError_t launch_map_scatter(int T, int E, int k, int nblk_cap, const int32_t *top,
                               const int32_t *tile_off, const int32_t *bins,
                               const int32_t *padded_bins, int32_t *indices, int32_t *bin_ids,
                               int32_t *dest_row, int32_t *block_expert, cudaStream_t st);

// Tile-aware token rounding (round.cu): scratch of the rounding kernels and the launcher.
// The routing's top [T,k] / weights [T,k] and the counts of the top-k routing go in; the
// rounded routing comes out as a token-major entry list: entry_offsets [T+1], experts and
// weights [cap] (entries past the list's end: expert -1, weight 0).
constexpr int kRoundMaxT = 1 << 20;  // the selection keeps a bitmap of T bits per CTA
constexpr size_t kRoundMaxSelectSmem = kRoundMaxT / 8;
// Row stride of the rank images: T rounded up to whole 32-token groups.
inline int round_img_stride(int T) { return (T + 31) / 32 * 32; }
struct RoundScratch {
  uint16_t *img;       // [E][round_img_stride(T)] rank images of the logits, a row per expert
  int32_t *param;      // [3E] per expert: mode, threshold image, threshold token
  int32_t *tok_count;  // [T]
  int32_t *tile_sum;   // [map_tiles(T)]
  int32_t *tile_off;   // [map_tiles(T) + 1]
};
// counts, bins, indices: the top-k routing's map (its sorted entries find each expert's tokens).
cudaError_t launch_round_tokens(const uint16_t *logits, const int32_t *top, const float *weights,
                                const int32_t *counts, const int32_t *bins,
                                const int32_t *indices, int T, int E, int k, const RoundScratch &s,
                                int32_t *entry_offsets, int32_t *out_expert, float *out_weight,
                                long long cap, cudaStream_t st);

// Entries of token t: [t*k, t*k + k), or with a token-major entry list (offsets != NULL, the
// rounded routing) [offsets[t], offsets[t+1]).
// Token-major padded gather with zero-filled padding rows.
cudaError_t launch_gather(int T, int h, int k, int E, const void *x, const int32_t *dest_row,
                          const int32_t *counts, const int32_t *padded_bins, void *x_pad,
                          cudaStream_t st, const int32_t *offsets = nullptr);
// Token-major weighted combine (weights may be NULL: w = 1) of bf16 rows (y_scale NULL) or of
// block-floating-point rows (fp16 values, y_scale [P_max, dmoe_scale_stride(h)]).
cudaError_t launch_combine(int T, int h, int k, const void *y_pad, const float *y_scale,
                           const int32_t *dest_row, const float *weights, void *y,
                           cudaStream_t st, const int32_t *offsets = nullptr);

// Backward scatter: dx_t = bf16(sum_s dX_pad[dest_row[t*k+s]]) over the block-floating-point
// rows of launch_dx_gemm (value = fp16 * scale, summed in fp32) and, from the DGLU GEMM's
// partial sums part [P_max, nt], dweights[t*k+s] = sum_n part[dest_row[t*k+s]][n].
cudaError_t launch_bwd_scatter(int T, int h, int k, const void *dx_pad, const float *dx_scale,
                               const int32_t *dest_row,
                               const float *part, int nt, void *dx, float *dweights,
                               cudaStream_t st, const int32_t *offsets = nullptr);

// Shape and map pointers shared by the grouped GEMM launchers.
struct GemmProblem {
  int h, f, E, nblk_cap;
  int T, k;
  const int32_t *num_blocks;
  const int32_t *block_expert;
  const int32_t *padded_bins;
  const int32_t *bins;
  const int32_t *indices;
  const float *weights;
  int32_t *status;
};

// Grouped tcgen05 GEMMs over the non-empty row blocks (forward) ...
cudaError_t launch_glu_gemm(const GemmProblem &g, const void *x_pad, const void *w1,
                            const void *w3, void *h_out, void *a_out, void *b_out,
                            cudaStream_t st);
cudaError_t launch_glu_gather_gemm(const GemmProblem &g, const void *x, const void *w1,
                                   const void *w3, void *h_out, void *a_out, void *b_out,
                                   cudaStream_t st);
// Y_pad [P_max,h] in block floating point: fp16 values, y_scale [P_max, dmoe_scale_stride(h)]
// fp32, one power-of-two scale per row and DMOE_SCALE_COLS columns (value = fp16 * scale), 11
// significant bits per value at bf16's size (the k rows of a token are summed by the combine; a bf16
// rounding of each would put k roundings into every output element).
cudaError_t launch_down_gemm(const GemmProblem &g, const void *h_in, const void *w2, void *y_pad,
                             float *y_scale, cudaStream_t st);
// ... and the backward: dH with the fused dGLU epilogue, dX, and the weight gradients.
// Columns per routing-weight partial of the DGLU epilogue (part has ceil(f / kDgluTileCols)
// columns).
constexpr int kDgluTileCols = DMOE_DGLU_TILE_COLS;
// Down GEMM with the weighted combine fused into its epilogue: y_acc[t] += w_ts * (H W2_e^T)
// row of each real padded row (fp32 vector reductions into y_acc [T, h]; no Y_pad).
cudaError_t launch_down_red_gemm(const GemmProblem &g, const void *h_in, const void *w2,
                                 float *y_acc, cudaStream_t st);
// n (a multiple of 8) fp32 accumulator values: zeroed / rounded to bf16.
cudaError_t launch_acc_zero(long long n, float *acc, cudaStream_t st);
cudaError_t launch_acc_round(long long n, const float *acc, void *y, cudaStream_t st);
cudaError_t launch_dglu_gemm(const GemmProblem &g, const void *dy_pad, const void *w2,
                             const void *a_in, const void *b_in, void *da_out, void *db_out,
                             void *hw_out, float *part, cudaStream_t st);
// dX_pad [P_max,h] fp16 with dx_scale [P_max, ceil(h/DMOE_SCALE_COLS)] fp32 (block floating
// point, as Y_pad of the down GEMM).
cudaError_t launch_dx_gemm(const GemmProblem &g, const void *da, const void *db, const void *w1,
                           const void *w3, void *dx_pad, float *dx_scale, cudaStream_t st);
cudaError_t launch_wgrad_gemm(const GemmProblem &g, const void *x_pad, const void *h_in,
                              const void *dy_pad, const void *da, const void *db, float *dw1,
                              float *dw3, float *dw2, cudaStream_t st);

// The linear router (dense rows over T tokens; E % 8 == 0):
//   logits = bf16(x W_r^T);  dx += dlogits W_r;  partial dW_r of each K split (fp32 slabs of
//   round_up(E, 128) rows), summed by launch_router_wgrad_reduce;  dlogits from the routing
//   weights' gradient.
constexpr int kRouterMaxSplits = 16;
cudaError_t launch_router_gemm(int T, int h, int E, const void *x, const void *wr, void *logits,
                               int32_t *status, cudaStream_t st);
cudaError_t launch_router_dx_gemm(int T, int h, int E, const void *dlogits, const void *wr, void *dx,
                                  int32_t *status, cudaStream_t st);
int router_wgrad_splits(int T, int h, int E);
cudaError_t launch_router_wgrad_gemm(int T, int h, int E, const void *dlogits, const void *x,
                                     float *partials, int splits, int32_t *status,
                                     cudaStream_t st);
cudaError_t launch_router_wgrad_reduce(int h, int E, int splits, const float *partials,
                                       float *dw_router, cudaStream_t st);
cudaError_t launch_router_dlogits(int T, int E, int k, bool renorm, const uint16_t *logits,
                                  const int32_t *top, const float *dweights, uint16_t *dlogits,
                                  cudaStream_t st);

int device_sm_count();

// Test-only: make the next grouped-GEMM launch stall on purpose (see dmoe_debug_inject_stall).
void set_inject_stall(int on);

}  // namespace dmoe
