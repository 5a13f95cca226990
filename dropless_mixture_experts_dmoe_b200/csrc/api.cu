// api.cu -- the C ABI of libdmoe.so (declared in include/dmoe.h): argument checks, workspace
// layout and the launch sequence of each entry point.  Every check runs on the host before
// the first launch of a call; nothing here reads device memory or synchronises.
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

using namespace dmoe;

namespace {

constexpr size_t kAlign = 256;

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool rounding(const dmoe_dims *d) { return (d->flags & DMOE_ROUTE_TOKEN_ROUNDING) != 0; }

// Entries of the map: T*k, plus up to 64 added per expert with token rounding (an expert
// rounds up only from a remainder of at least 64, adding at most 64).
long long entries_of(const dmoe_dims *d) {
  return (long long)d->T * d->top_k +
         (rounding(d) ? (long long)(DMOE_BLOCKING / 2) * d->num_experts : 0);
}

// Shape validation shared by all entry points.
int check_dims(const dmoe_dims *d) {
  if (!d) return DMOE_ERR_NULL;
  if (d->num_experts < 1 || d->num_experts > DMOE_MAX_EXPERTS) return DMOE_ERR_TOO_MANY_EXPERTS;
  if (d->T < 1 || d->top_k < 1 || d->top_k > d->num_experts || d->top_k > DMOE_MAX_TOP_K)
    return DMOE_ERR_SHAPE;
  if (d->ffn < DMOE_BLOCKING || d->ffn % DMOE_BLOCKING != 0) return DMOE_ERR_SHAPE;
  if (d->hidden < DMOE_BLOCKING || d->hidden % DMOE_BLOCKING != 0) return DMOE_ERR_SHAPE;
  if (d->flags & ~(DMOE_ROUTE_RENORMALIZE | DMOE_ROUTE_TOKEN_ROUNDING | DMOE_SAVE_X_ONLY |
                   DMOE_FUSED_COMBINE))
    return DMOE_ERR_SHAPE;
  if (rounding(d) && ((d->flags & (DMOE_ROUTE_RENORMALIZE | DMOE_FUSED_COMBINE)) ||
                      d->T > kRoundMaxT))
    return DMOE_ERR_SHAPE;
  const long long n = entries_of(d);
  const long long pmax =
      (n + (long long)(DMOE_BLOCKING - 1) * d->num_experts) / DMOE_BLOCKING * DMOE_BLOCKING;
  if (n > 0x7FFFFFFFLL || pmax > 0x7FFFFFFFLL) return DMOE_ERR_TOO_LARGE;
  return DMOE_OK;
}

long long pmax_of(const dmoe_dims *d) {
  const long long n = entries_of(d);
  return (n + (long long)(DMOE_BLOCKING - 1) * d->num_experts) / DMOE_BLOCKING * DMOE_BLOCKING;
}

// The current device must be an sm_100 part.  The answer is cached per device ordinal (a
// process may see GPUs of several kinds); ordinals past the cache are checked on every call.
constexpr int kDeviceCache = 64;
std::atomic<int> g_device_ok[kDeviceCache];  // 0 unknown, 1 sm_100, 2 other

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return DMOE_ERR_DEVICE;
  int known = (dev < kDeviceCache) ? g_device_ok[dev].load(std::memory_order_relaxed) : 0;
  if (known == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return DMOE_ERR_DEVICE;
    known = (major == 10) ? 1 : 2;
    if (dev < kDeviceCache) g_device_ok[dev].store(known, std::memory_order_relaxed);
  }
  return known == 1 ? DMOE_OK : DMOE_ERR_DEVICE;
}

int check_map(const dmoe_map *m, bool need_weights, const dmoe_dims *d = nullptr) {
  if (!m || !m->top_experts || !m->tokens_per_expert || !m->bins || !m->padded_bins ||
      !m->indices || !m->bin_ids || !m->dest_row || !m->block_expert || !m->num_blocks ||
      !m->status)
    return DMOE_ERR_NULL;
  if (need_weights && !m->weights) return DMOE_ERR_NULL;
  if (d && rounding(d) && !m->entry_offsets) return DMOE_ERR_NULL;
  return DMOE_OK;
}

// The token-major entry list's row offsets (token rounding), else NULL (t*k + s).
inline const int32_t *entry_offsets_of(const dmoe_dims *d, const dmoe_map *m) {
  return rounding(d) ? m->entry_offsets : nullptr;
}

// Map workspace.  Plain routing: the map kernels' scratch for (T, E).  Token rounding: that
// scratch sized for the larger of the two maps it builds (T tokens x k, then the entry list
// as entries_of(d) single entries) | the top-k routing top [T,k] int32, weights [T,k] fp32 |
// rank images [E][T rounded up to 32] u16 | per-expert thresholds [3E] | per-token counts
// [T] | tile totals [tiles] | tile offsets [tiles + 1].
struct MapLayout {
  size_t top, w, img, param, tokc, tsum, toff, total;
};
MapLayout map_layout(const dmoe_dims *d) {
  MapLayout l = {};
  size_t hist = sizeof(int32_t) * map_workspace_ints(d->T, d->num_experts);
  if (!rounding(d)) {
    l.total = align_up(hist);
    return l;
  }
  const size_t hist2 = sizeof(int32_t) * map_workspace_ints((int)entries_of(d), d->num_experts);
  if (hist2 > hist) hist = hist2;
  const size_t T = (size_t)d->T, Tk = T * d->top_k, E = (size_t)d->num_experts;
  const size_t tiles = (size_t)map_tiles(d->T);
  l.top = align_up(hist);
  l.w = align_up(l.top + Tk * 4);
  l.img = align_up(l.w + Tk * 4);
  l.param = align_up(l.img + E * (size_t)round_img_stride((int)T) * 2);
  l.tokc = align_up(l.param + 3 * E * 4);
  l.tsum = align_up(l.tokc + T * 4);
  l.toff = align_up(l.tsum + tiles * 4);
  l.total = align_up(l.toff + (tiles + 1) * 4);
  return l;
}

inline int launch_rc(cudaError_t e) { return e == cudaSuccess ? DMOE_OK : DMOE_ERR_LAUNCH; }

GemmProblem problem_of(const dmoe_dims *d, const dmoe_map *m) {
  GemmProblem g;
  g.h = d->hidden;
  g.f = d->ffn;
  g.E = d->num_experts;
  g.nblk_cap = (int)(pmax_of(d) / DMOE_BLOCKING);
  g.T = d->T;
  g.k = d->top_k;
  g.bins = m->bins;
  g.indices = m->indices;
  g.weights = m->weights;
  g.num_blocks = m->num_blocks;
  g.block_expert = m->block_expert;
  g.padded_bins = m->padded_bins;
  g.status = m->status;
  return g;
}

inline int dglu_tiles(const dmoe_dims *d) { return (d->ffn + kDgluTileCols - 1) / kDgluTileCols; }


inline int scale_cols(const dmoe_dims *d) { return dmoe_scale_stride(d->hidden); }

inline bool save_x_only(const dmoe_dims *d) { return (d->flags & DMOE_SAVE_X_ONLY) != 0; }

// Backward workspace layout: dY_pad [P,h] bf16, whose region is reused for dX_pad [P,h] fp16
// once the weight gradients have read dY_pad | dA [P,f] | dBm [P,f] | Hw [P,f] | routing-weight
// partials [P, ceil(f/256)] fp32 | dX_pad scales [P, dmoe_scale_stride(h)] fp32 | with
// DMOE_SAVE_X_ONLY the recomputed A [P,f] and Bm [P,f]
struct BwdLayout {
  size_t dy, da, db, hw, part, dxs, a, bm, total;
};
BwdLayout bwd_layout(const dmoe_dims *d) {
  const size_t P = (size_t)pmax_of(d);
  BwdLayout l;
  l.dy = 0;
  l.da = align_up(l.dy + P * d->hidden * 2);
  l.db = align_up(l.da + P * d->ffn * 2);
  l.hw = align_up(l.db + P * d->ffn * 2);
  l.part = align_up(l.hw + P * d->ffn * 2);
  l.dxs = align_up(l.part + P * dglu_tiles(d) * sizeof(float));
  l.a = l.bm = l.total = align_up(l.dxs + P * scale_cols(d) * sizeof(float));
  if (save_x_only(d)) {
    l.bm = align_up(l.a + P * d->ffn * 2);
    l.total = align_up(l.bm + P * d->ffn * 2);
  }
  return l;
}

inline bool fused_combine(const dmoe_dims *d) { return (d->flags & DMOE_FUSED_COMBINE) != 0; }

// Forward workspace layout: H [P,f] | Y_pad [P,h] fp16 | Y_pad scales [P, dmoe_scale_stride(h)]
// fp32 (with DMOE_FUSED_COMBINE instead the token accumulator y_acc [T,h] fp32) | X_pad [P,h].
// A training forward keeps X_pad in the saved buffer and uses only the first part (`train`).
struct FwdLayout {
  size_t h, ypad, yscale, yacc, xpad, train, total;
};
FwdLayout fwd_layout(const dmoe_dims *d) {
  const size_t P = (size_t)pmax_of(d);
  FwdLayout l;
  l.h = 0;
  l.ypad = l.yscale = l.yacc = align_up(l.h + P * d->ffn * 2);
  if (fused_combine(d)) {
    l.xpad = align_up(l.yacc + (size_t)d->T * d->hidden * sizeof(float));
  } else {
    l.yscale = align_up(l.ypad + P * d->hidden * 2);
    l.xpad = align_up(l.yscale + P * scale_cols(d) * sizeof(float));
  }
  l.train = l.xpad;
  l.total = align_up(l.xpad + P * d->hidden * 2);
  return l;
}

// Router backward workspace: dlogits [T,E] bf16 | split-K partials of dW_r
// [kRouterMaxSplits, round_up(E,128), h] fp32
struct RouterLayout {
  size_t dlogits, part, total;
};
RouterLayout router_layout(const dmoe_dims *d) {
  RouterLayout l;
  const size_t Ep = (size_t)(d->num_experts + DMOE_BLOCKING - 1) / DMOE_BLOCKING * DMOE_BLOCKING;
  l.dlogits = 0;
  l.part = align_up(l.dlogits + (size_t)d->T * d->num_experts * 2);
  l.total = align_up(l.part + (size_t)kRouterMaxSplits * Ep * d->hidden * sizeof(float));
  return l;
}

// The router's tensors have E columns; a TMA row must be a multiple of 16 bytes.  Its
// gradient is defined for the top-k routing only (not for the rounded one).
inline int check_router_dims(const dmoe_dims *d) {
  int rc = check_dims(d);
  if (rc) return rc;
  return (d->num_experts % 8 == 0 && !rounding(d)) ? DMOE_OK : DMOE_ERR_SHAPE;
}

// Saved activations: X_pad [P,h] | A [P,f] | Bm [P,f]; X_pad only with DMOE_SAVE_X_ONLY
// (offsets of A and Bm reported as 0)
void saved_layout(const dmoe_dims *d, size_t off[3], size_t *total) {
  const size_t P = (size_t)pmax_of(d);
  off[0] = 0;
  if (save_x_only(d)) {
    off[1] = off[2] = 0;
    *total = align_up(P * d->hidden * 2);
    return;
  }
  off[1] = align_up(off[0] + P * d->hidden * 2);
  off[2] = align_up(off[1] + P * d->ffn * 2);
  *total = align_up(off[2] + P * d->ffn * 2);
}

}  // namespace

extern "C" {

size_t dmoe_entries_max(const dmoe_dims *dims) {
  if (check_dims(dims) != DMOE_OK) return 0;
  return (size_t)entries_of(dims);
}

size_t dmoe_padded_rows_max(const dmoe_dims *dims) {
  if (check_dims(dims) != DMOE_OK) return 0;
  return (size_t)pmax_of(dims);
}

size_t dmoe_workspace_bytes(const dmoe_dims *dims, int kind) {
  if (check_dims(dims) != DMOE_OK) return 0;
  switch (kind) {
    case DMOE_WS_MAP:
      return map_layout(dims).total;
    case DMOE_WS_FORWARD:
      return fwd_layout(dims).total;
    case DMOE_WS_FORWARD_TRAIN:
      return fwd_layout(dims).train;
    case DMOE_WS_ROUTER_BACKWARD:
      return router_layout(dims).total;
    case DMOE_WS_BACKWARD:
      return bwd_layout(dims).total;
    default:
      return 0;
  }
}

size_t dmoe_saved_bytes(const dmoe_dims *dims, size_t offsets[3]) {
  if (check_dims(dims) != DMOE_OK) return 0;
  size_t off[3], total;
  saved_layout(dims, off, &total);
  if (offsets)
    for (int i = 0; i < 3; ++i) offsets[i] = off[i];
  return total;
}

int dmoe_sparse_map(const dmoe_dims *dims, const void *logits, const dmoe_map *map, void *ws,
                    size_t ws_bytes, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, logits != nullptr || rounding(dims), dims))) return rc;
  if (!ws || (rounding(dims) && !logits)) return DMOE_ERR_NULL;  // rounding ranks by logit
  if (ws_bytes < dmoe_workspace_bytes(dims, DMOE_WS_MAP)) return DMOE_ERR_WORKSPACE;
  if ((logits && !aligned16(logits)) || !aligned16(ws) || !aligned16(map->top_experts) ||
      (logits && !aligned16(map->weights)))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = dims->T, E = dims->num_experts, k = dims->top_k;
  const int nblk_cap = (int)(pmax_of(dims) / DMOE_BLOCKING);
  int32_t *tile_hist = static_cast<int32_t *>(ws);
  const bool renorm = (dims->flags & DMOE_ROUTE_RENORMALIZE) != 0;
  if (rounding(dims)) {
    // top-k routing and its map (in the map's arrays, rebuilt below), the rounding into the
    // token-major entry list, then the map of that list (one entry per "token"; absent
    // entries past its end are left out)
    const MapLayout l = map_layout(dims);
    uint8_t *w = static_cast<uint8_t *>(ws);
    int32_t *top = reinterpret_cast<int32_t *>(w + l.top);
    float *wts = reinterpret_cast<float *>(w + l.w);
    RoundScratch s;
    s.img = reinterpret_cast<uint16_t *>(w + l.img);
    s.param = reinterpret_cast<int32_t *>(w + l.param);
    s.tok_count = reinterpret_cast<int32_t *>(w + l.tokc);
    s.tile_sum = reinterpret_cast<int32_t *>(w + l.tsum);
    s.tile_off = reinterpret_cast<int32_t *>(w + l.toff);
    const int N = (int)entries_of(dims);
    const uint16_t *lg = static_cast<const uint16_t *>(logits);
    if ((rc = launch_rc(launch_route_hist(lg, T, E, k, false, top, wts, tile_hist, st)))) return rc;
    if ((rc = launch_rc(launch_map_scan(T, E, tile_hist, map->tokens_per_expert, map->bins,
                                        map->padded_bins, map->num_blocks, map->status, st))))
      return rc;
    if ((rc = launch_rc(launch_map_scatter(T, E, k, nblk_cap, top, tile_hist, map->bins,
                                           map->padded_bins, map->indices, map->bin_ids,
                                           map->dest_row, map->block_expert, st))))
      return rc;
    if ((rc = launch_rc(launch_round_tokens(lg, top, wts, map->tokens_per_expert, map->bins,
                                            map->indices, T, E, k, s, map->entry_offsets,
                                            map->top_experts, map->weights, N, st))))
      return rc;
    if ((rc = launch_rc(launch_route_hist(nullptr, N, E, 1, false, map->top_experts, nullptr,
                                          tile_hist, st, /*absent_ok=*/true))))
      return rc;
    if ((rc = launch_rc(launch_map_scan(N, E, tile_hist, map->tokens_per_expert, map->bins,
                                        map->padded_bins, map->num_blocks, map->status, st,
                                        /*or_status=*/true))))
      return rc;
    return launch_rc(launch_map_scatter(N, E, 1, nblk_cap, map->top_experts, tile_hist, map->bins,
                                        map->padded_bins, map->indices, map->bin_ids,
                                        map->dest_row, map->block_expert, st));
  }
  if ((rc = launch_rc(launch_route_hist(static_cast<const uint16_t *>(logits), T, E, k, renorm,
                                        map->top_experts, map->weights, tile_hist, st))))
    return rc;
  if ((rc = launch_rc(launch_map_scan(T, E, tile_hist, map->tokens_per_expert, map->bins,
                                      map->padded_bins, map->num_blocks, map->status, st))))
    return rc;
  return launch_rc(launch_map_scatter(T, E, k, nblk_cap, map->top_experts, tile_hist, map->bins,
                                      map->padded_bins, map->indices, map->bin_ids,
                                      map->dest_row, map->block_expert, st));
}

int dmoe_padded_gather(const dmoe_dims *dims, const void *x, const dmoe_map *map, void *x_pad,
                       void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, false, dims))) return rc;
  if (!x || !x_pad) return DMOE_ERR_NULL;
  if (!aligned16(x) || !aligned16(x_pad)) return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_gather(dims->T, dims->hidden, dims->top_k, dims->num_experts, x,
                                 map->dest_row, map->tokens_per_expert, map->padded_bins, x_pad,
                                 static_cast<cudaStream_t>(stream), entry_offsets_of(dims, map)));
}

int dmoe_expert_glu(const dmoe_dims *dims, const void *x_pad, const void *w1, const void *w3,
                    const dmoe_map *map, void *h_out, void *a_out, void *b_out, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, false))) return rc;
  if (!x_pad || !w1 || !w3 || (a_out == nullptr) != (b_out == nullptr) || (!h_out && !a_out))
    return DMOE_ERR_NULL;
  if (!aligned16(x_pad) || !aligned16(w1) || !aligned16(w3) || (h_out && !aligned16(h_out)) ||
      (a_out && !aligned16(a_out)) || (b_out && !aligned16(b_out)))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_glu_gemm(problem_of(dims, map), x_pad, w1, w3, h_out, a_out, b_out,
                                   static_cast<cudaStream_t>(stream)));
}

int dmoe_expert_glu_gather(const dmoe_dims *dims, const void *x, const void *w1, const void *w3,
                           const dmoe_map *map, void *h_out, void *a_out, void *b_out,
                           void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (rounding(dims)) return DMOE_ERR_SHAPE;  // its row gathers assume t*k + s entries
  if ((rc = check_map(map, false))) return rc;
  if (!x || !w1 || !w3 || !h_out) return DMOE_ERR_NULL;
  if ((a_out == nullptr) != (b_out == nullptr)) return DMOE_ERR_NULL;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w3) || !aligned16(h_out) ||
      (a_out && !aligned16(a_out)) || (b_out && !aligned16(b_out)))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_glu_gather_gemm(problem_of(dims, map), x, w1, w3, h_out, a_out, b_out,
                                          static_cast<cudaStream_t>(stream)));
}

int dmoe_expert_down(const dmoe_dims *dims, const void *h_in, const void *w2,
                     const dmoe_map *map, void *y_pad, float *y_scale, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, true))) return rc;  // the rows go out weighted
  if (!h_in || !w2 || !y_pad || !y_scale) return DMOE_ERR_NULL;
  if (!aligned16(h_in) || !aligned16(w2) || !aligned16(y_pad) || !aligned16(y_scale))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_down_gemm(problem_of(dims, map), h_in, w2, y_pad, y_scale,
                                    static_cast<cudaStream_t>(stream)));
}

int dmoe_expert_down_combine(const dmoe_dims *dims, const void *h_in, const void *w2,
                             const dmoe_map *map, void *y, float *y_acc, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (rounding(dims)) return DMOE_ERR_SHAPE;  // the epilogue finds a row's token as j / k
  if ((rc = check_map(map, true))) return rc;
  if (!h_in || !w2 || !y || !y_acc) return DMOE_ERR_NULL;
  if (!aligned16(h_in) || !aligned16(w2) || !aligned16(y) || !aligned16(y_acc) ||
      !aligned16(map->weights))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long n = (long long)dims->T * dims->hidden;
  if ((rc = launch_rc(launch_acc_zero(n, y_acc, st)))) return rc;
  if ((rc = launch_rc(launch_down_red_gemm(problem_of(dims, map), h_in, w2, y_acc, st)))) return rc;
  return launch_rc(launch_acc_round(n, y_acc, y, st));
}

int dmoe_padded_scatter(const dmoe_dims *dims, const void *y_pad, const float *y_scale,
                        const dmoe_map *map, const float *weights, void *y, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, false, dims))) return rc;
  if (!y_pad || !y) return DMOE_ERR_NULL;
  if (!aligned16(y_pad) || !aligned16(y) || !aligned16(y_scale)) return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_combine(dims->T, dims->hidden, dims->top_k, y_pad, y_scale,
                                  map->dest_row, weights, y, static_cast<cudaStream_t>(stream),
                                  entry_offsets_of(dims, map)));
}

int dmoe_forward(const dmoe_dims *dims, const void *x, const void *w1, const void *w3,
                 const void *w2, const dmoe_map *map, void *y, void *saved, void *ws,
                 size_t ws_bytes, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, true))) return rc;
  if (!x || !w1 || !w3 || !w2 || !y) return DMOE_ERR_NULL;
  if (!ws) return DMOE_ERR_NULL;
  const FwdLayout l = fwd_layout(dims);
  if (ws_bytes < (saved ? l.train : l.total)) return DMOE_ERR_WORKSPACE;
  uint8_t *w = static_cast<uint8_t *>(ws);
  float *yscale = reinterpret_cast<float *>(w + l.yscale);
  float *yacc = reinterpret_cast<float *>(w + l.yacc);
  uint8_t *xpad = w + l.xpad, *hbuf = w + l.h, *ypad = w + l.ypad, *abuf = nullptr,
          *bbuf = nullptr;
  if (saved) {
    size_t off[3], total;
    saved_layout(dims, off, &total);
    uint8_t *s = static_cast<uint8_t *>(saved);
    xpad = s + off[0];
    if (!save_x_only(dims)) {  // else the backward recomputes A and Bm from X_pad
      abuf = s + off[1];
      bbuf = s + off[2];
    }
  }
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w3) || !aligned16(w2) || !aligned16(y) ||
      !aligned16(ws) || !aligned16(xpad) || !aligned16(map->weights))
    return DMOE_ERR_ALIGN;
  // The separate token-major gather (about 80 % of HBM bandwidth) is faster than feeding the
  // GLU GEMM through TMA row gathers, whose instruction rate cannot keep up with the MMAs.
  if ((rc = dmoe_padded_gather(dims, x, map, xpad, stream))) return rc;
  if ((rc = dmoe_expert_glu(dims, xpad, w1, w3, map, hbuf, abuf, bbuf, stream))) return rc;
  if (fused_combine(dims)) return dmoe_expert_down_combine(dims, hbuf, w2, map, y, yacc, stream);
  if ((rc = dmoe_expert_down(dims, hbuf, w2, map, ypad, yscale, stream))) return rc;
  return dmoe_padded_scatter(dims, ypad, yscale, map, nullptr, y, stream);  // rows weighted
}

int dmoe_bwd_dglu(const dmoe_dims *dims, const void *dy_pad, const void *w2, const void *a_saved,
                  const void *bm_saved, const dmoe_map *map, void *da, void *dbm, void *hw,
                  float *dw_part, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, true))) return rc;
  if (!dy_pad || !w2 || !a_saved || !bm_saved || !da || !dbm || !hw || !dw_part)
    return DMOE_ERR_NULL;
  if (!aligned16(dy_pad) || !aligned16(w2) || !aligned16(a_saved) || !aligned16(bm_saved) ||
      !aligned16(da) || !aligned16(dbm) || !aligned16(hw) || !aligned16(dw_part))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_dglu_gemm(problem_of(dims, map), dy_pad, w2, a_saved, bm_saved, da, dbm,
                                    hw, dw_part, static_cast<cudaStream_t>(stream)));
}

int dmoe_bwd_scatter(const dmoe_dims *dims, const void *dx_pad, const float *dx_scale,
                     const float *dw_part, const dmoe_map *map, void *dx, float *dweights,
                     void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, false, dims))) return rc;
  if (!dx_pad || !dx_scale || !dw_part || !dx || !dweights) return DMOE_ERR_NULL;
  if (!aligned16(dx_pad) || !aligned16(dx) || !aligned16(dx_scale)) return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_bwd_scatter(dims->T, dims->hidden, dims->top_k, dx_pad, dx_scale,
                                      map->dest_row, dw_part, dglu_tiles(dims), dx, dweights,
                                      static_cast<cudaStream_t>(stream),
                                      entry_offsets_of(dims, map)));
}

int dmoe_bwd_dx(const dmoe_dims *dims, const void *da, const void *dbm, const void *w1,
                const void *w3, const dmoe_map *map, void *dx_pad, float *dx_scale,
                void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, false))) return rc;
  if (!da || !dbm || !w1 || !w3 || !dx_pad || !dx_scale) return DMOE_ERR_NULL;
  if (!aligned16(da) || !aligned16(dbm) || !aligned16(w1) || !aligned16(w3) ||
      !aligned16(dx_pad) || !aligned16(dx_scale))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(
      launch_dx_gemm(problem_of(dims, map), da, dbm, w1, w3, dx_pad, dx_scale,
                     static_cast<cudaStream_t>(stream)));
}

int dmoe_bwd_wgrad(const dmoe_dims *dims, const void *x_pad, const void *hw,
                   const void *dy_pad, const void *da, const void *dbm, const dmoe_map *map,
                   float *dw1, float *dw3, float *dw2, void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, false))) return rc;
  if (!x_pad || !hw || !dy_pad || !da || !dbm || !dw1 || !dw3 || !dw2) return DMOE_ERR_NULL;
  if (!aligned16(x_pad) || !aligned16(hw) || !aligned16(dy_pad) || !aligned16(da) ||
      !aligned16(dbm) || !aligned16(dw1) || !aligned16(dw3) || !aligned16(dw2))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_wgrad_gemm(problem_of(dims, map), x_pad, hw, dy_pad, da, dbm, dw1,
                                     dw3, dw2, static_cast<cudaStream_t>(stream)));
}

int dmoe_backward(const dmoe_dims *dims, const void *dy, const void *w1, const void *w3,
                  const void *w2, const dmoe_map *map, const void *saved, void *dx, float *dw1,
                  float *dw3, float *dw2, float *dweights, void *ws, size_t ws_bytes,
                  void *stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_map(map, true))) return rc;
  if (!dy || !w1 || !w3 || !w2 || !saved || !dx || !dw1 || !dw3 || !dw2 || !dweights || !ws)
    return DMOE_ERR_NULL;
  const BwdLayout l = bwd_layout(dims);
  if (ws_bytes < l.total) return DMOE_ERR_WORKSPACE;
  if (!aligned16(saved) || !aligned16(ws) || !aligned16(dx)) return DMOE_ERR_ALIGN;
  size_t off[3], total;
  saved_layout(dims, off, &total);
  const uint8_t *sv = static_cast<const uint8_t *>(saved);
  const void *xpad = sv + off[0], *abuf = sv + off[1], *bbuf = sv + off[2];
  uint8_t *w = static_cast<uint8_t *>(ws);
  void *dypad = w + l.dy, *da = w + l.da, *db = w + l.db, *hw = w + l.hw;
  if (save_x_only(dims)) {  // A and Bm again, from the saved X_pad: the forward's exact bits
    abuf = w + l.a;
    bbuf = w + l.bm;
    if ((rc = dmoe_expert_glu(dims, xpad, w1, w3, map, nullptr, w + l.a, w + l.bm, stream)))
      return rc;
  }
  float *part = reinterpret_cast<float *>(w + l.part);
  float *dxs = reinterpret_cast<float *>(w + l.dxs);
  void *dxpad = dypad;  // dY_pad is dead once the weight gradients have read it
  if ((rc = dmoe_padded_gather(dims, dy, map, dypad, stream))) return rc;
  if ((rc = dmoe_bwd_dglu(dims, dypad, w2, abuf, bbuf, map, da, db, hw, part, stream))) return rc;
  if ((rc = dmoe_bwd_wgrad(dims, xpad, hw, dypad, da, db, map, dw1, dw3, dw2, stream))) return rc;
  if ((rc = dmoe_bwd_dx(dims, da, db, w1, w3, map, dxpad, dxs, stream))) return rc;
  return dmoe_bwd_scatter(dims, dxpad, dxs, part, map, dx, dweights, stream);
}

int dmoe_router_forward(const dmoe_dims *dims, const void *x, const void *w_router, void *logits,
                        int32_t *status, void *stream) {
  int rc = check_router_dims(dims);
  if (rc) return rc;
  if (!x || !w_router || !logits || !status) return DMOE_ERR_NULL;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits)) return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_router_gemm(dims->T, dims->hidden, dims->num_experts, x, w_router,
                                      logits, status, static_cast<cudaStream_t>(stream)));
}

int dmoe_router_dlogits(const dmoe_dims *dims, const void *logits, const dmoe_map *map,
                        const float *dweights, void *dlogits, void *stream) {
  int rc = check_router_dims(dims);
  if (rc) return rc;
  if (!logits || !map || !map->top_experts || !dweights || !dlogits) return DMOE_ERR_NULL;
  if (!aligned16(logits) || !aligned16(dlogits)) return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return launch_rc(launch_router_dlogits(dims->T, dims->num_experts, dims->top_k,
                                         (dims->flags & DMOE_ROUTE_RENORMALIZE) != 0,
                                         static_cast<const uint16_t *>(logits), map->top_experts,
                                         dweights, static_cast<uint16_t *>(dlogits),
                                         static_cast<cudaStream_t>(stream)));
}

int dmoe_router_backward(const dmoe_dims *dims, const void *x, const void *w_router,
                         const void *logits, const dmoe_map *map, const float *dweights,
                         void *dx, float *dw_router, void *ws, size_t ws_bytes, void *stream) {
  int rc = check_router_dims(dims);
  if (rc) return rc;
  if (!x || !w_router || !logits || !map || !map->top_experts || !map->status || !dweights ||
      !dx || !dw_router || !ws)
    return DMOE_ERR_NULL;
  const RouterLayout l = router_layout(dims);
  if (ws_bytes < l.total) return DMOE_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits) || !aligned16(dx) ||
      !aligned16(dw_router) || !aligned16(ws))
    return DMOE_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = dims->T, h = dims->hidden, E = dims->num_experts;
  uint8_t *w = static_cast<uint8_t *>(ws);
  void *dl = w + l.dlogits;
  float *part = reinterpret_cast<float *>(w + l.part);
  if ((rc = dmoe_router_dlogits(dims, logits, map, dweights, dl, stream))) return rc;
  if ((rc = launch_rc(launch_router_dx_gemm(T, h, E, dl, w_router, dx, map->status, st))))
    return rc;
  const int splits = router_wgrad_splits(T, h, E);
  if ((rc = launch_rc(launch_router_wgrad_gemm(T, h, E, dl, x, part, splits, map->status, st))))
    return rc;
  return launch_rc(launch_router_wgrad_reduce(h, E, splits, part, dw_router, st));
}

const char *dmoe_error_string(int code) {
  switch (code) {
    case DMOE_OK:
      return "ok";
    case DMOE_ERR_NULL:
      return "a required pointer is NULL";
    case DMOE_ERR_SHAPE:
      return "invalid shape (ffn and hidden must be multiples of 128; 1 <= top_k <= min(E, 32); T >= 1)";
    case DMOE_ERR_TOO_MANY_EXPERTS:
      return "number of experts outside [1, 1024]";
    case DMOE_ERR_WORKSPACE:
      return "workspace too small";
    case DMOE_ERR_ALIGN:
      return "a pointer is not 16-byte aligned";
    case DMOE_ERR_LAUNCH:
      return "a CUDA launch failed";
    case DMOE_ERR_DEVICE:
      return "current device is not sm_100 (B200)";
    case DMOE_ERR_TOO_LARGE:
      return "T*top_k or the padded row bound exceeds 2^31-1";
    default:
      return "unknown error";
  }
}

const char *dmoe_status_string(int32_t status) {
  static thread_local char buf[160];
  buf[0] = 0;
  if (status == 0) return "ok";
  if (status & DMOE_STATUS_NONFINITE_LOGITS) strcat(buf, "nonfinite_logits ");
  if (status & DMOE_STATUS_EXPERT_OUT_OF_RANGE) strcat(buf, "expert_out_of_range ");
  if (status & DMOE_STATUS_DUPLICATE_EXPERT) strcat(buf, "duplicate_expert ");
  if (status & DMOE_STATUS_TIMEOUT) strcat(buf, "timeout ");
  return buf;
}

const char *dmoe_version(void) { return "dmoe-b200 0.1"; }

int dmoe_debug_inject_stall(int enable) {
  set_inject_stall(enable);
  return DMOE_OK;
}

}  // extern "C"
