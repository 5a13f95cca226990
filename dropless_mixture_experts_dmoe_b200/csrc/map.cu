// map.cu -- routing and sparse-map construction (MegaBlocks walkthrough "02 · dropless MoE 与
// block-sparse 重构", sections 4.1-4.3; Fast-LLM issue #56 get_sparse_map).
//
// Three kernels, no spin-waits, deterministic results (the only global atomic is the scan's
// completion ticket):
//   k_route_hist   one warp per token: top-k by integer max over order-preserving keys
//                  (ties -> lower expert index), fp32 softmax weights, per-tile histogram in
//                  shared memory (O(E) bytes, independent of T).
//   k_map_scan     one CTA per 32 experts: per-expert exclusive offsets of every tile; the
//                  last CTA to finish (a ticket counter, no waiting) computes bins,
//                  padded_bins (round_up to 128), num_blocks and the block -> expert table.
//   k_map_scatter  one CTA per tile: stable rank of every entry inside its expert (warp
//                  histograms + __match_any_sync ranks in entry order), then indices,
//                  bin_ids and dest_row from the index math of section 4.2.
#include "common.cuh"
#include "kernels.h"

namespace dmoe {

constexpr int kMapThreads = 256;
constexpr int kMapWarps = kMapThreads / 32;

__device__ __forceinline__ bool bf16_nonfinite(uint16_t b) { return (b & 0x7F80u) == 0x7F80u; }

// ---- routing + histogram ---------------------------------------------------------------------

// KPL = logits per lane (E <= 32*KPL).
template <int KPL>
__global__ void __launch_bounds__(kMapThreads) k_route_hist(const uint16_t *__restrict__ logits,
                                                            int T, int E, int k, int renorm,
                                                            int32_t *__restrict__ top,
                                                            float *__restrict__ weights,
                                                            int32_t *__restrict__ tile_hist,
                                                            int32_t *status,
                                                            unsigned int *__restrict__ done) {
  extern __shared__ int hist[];  // [E]
  if (blockIdx.x == 0 && threadIdx.x == 0) *done = 0u;  // ticket counter of k_map_scan
  for (int e = threadIdx.x; e < E; e += kMapThreads) hist[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kMapTokTile;
  bool bad = false;
  // this warp's tokens are t0 + warp, t0 + warp + 8, ...; the next token's logits are loaded
  // while the current token is ranked
  uint16_t nxt[KPL];
  auto load_row = [&](int t) {
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const int e = lane + 32 * i;
      nxt[i] = (t < T && e < E) ? __ldg(logits + (size_t)t * E + e) : (uint16_t)0;
    }
  };
  load_row(t0 + warp);
  for (int tt = warp; tt < kMapTokTile; tt += kMapWarps) {
    const int t = t0 + tt;
    if (t >= T) break;
    uint16_t cur[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) cur[i] = nxt[i];
    if (tt + kMapWarps < kMapTokTile) load_row(t + kMapWarps);
    uint32_t key[KPL];
    float val[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const int e = lane + 32 * i;
      key[i] = 0u;
      val[i] = 0.0f;
      if (e < E) {
        const uint16_t b = cur[i];
        bad |= bf16_nonfinite(b);
        key[i] = (bf16_order(b) << 16) | (0xFFFFu - (uint32_t)e);
        val[i] = __uint_as_float((uint32_t)b << 16);
      }
    }
    // k rounds of a warp-wide integer max; the winner's lane clears the key.
    int my_e = 0;
    uint32_t my_key = 0, top_key = 0;
    for (int s = 0; s < k; ++s) {
      uint32_t best = 0;
#pragma unroll
      for (int i = 0; i < KPL; ++i) best = max(best, key[i]);
      const uint32_t wb = __reduce_max_sync(0xFFFFFFFFu, best);
      const int e = 0xFFFF - (int)(wb & 0xFFFFu);
      if (s == 0) top_key = wb;
      if ((e & 31) == lane) {
#pragma unroll
        for (int i = 0; i < KPL; ++i)
          if (i == (e >> 5)) key[i] = 0u;
      }
      if (lane == s) {
        my_e = e;
        my_key = wb;
      }
    }
    // softmax over all E logits (or, renormalised, over the k picks), max = the first pick.
    const float m = ((top_key >> 16) == 0u) ? __uint_as_float(0x7FC00000u)
                                           : bf16_from_order(top_key >> 16);
    const float v = (lane < k) ? (((my_key >> 16) == 0u) ? __uint_as_float(0x7FC00000u)
                                                         : bf16_from_order(my_key >> 16))
                               : 0.0f;
    float sum = 0.0f;
    if (renorm) {
      if (lane < k) sum = expf(v - m);
    } else {
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        if (lane + 32 * i < E) sum += expf(val[i] - m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    if (lane < k) {
      top[(size_t)t * k + lane] = my_e;
      weights[(size_t)t * k + lane] = expf(v - m) / sum;
      atomicAdd(&hist[my_e], 1);
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) set_status(status, DMOE_STATUS_NONFINITE_LOGITS);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kMapThreads)
    tile_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

// Histogram of caller-given top_experts; invalid ids are reported and left out of the map.
__global__ void __launch_bounds__(kMapThreads) k_given_hist(const int32_t *__restrict__ top,
                                                            int T, int E, int k,
                                                            int32_t *__restrict__ tile_hist,
                                                            int32_t *status,
                                                            unsigned int *__restrict__ done) {
  extern __shared__ int hist[];
  if (blockIdx.x == 0 && threadIdx.x == 0) *done = 0u;  // ticket counter of k_map_scan
  for (int e = threadIdx.x; e < E; e += kMapThreads) hist[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kMapTokTile;
  int flags = 0;
  for (int tt = warp; tt < kMapTokTile; tt += kMapWarps) {
    const int t = t0 + tt;
    if (t >= T) break;
    int e = -1 - lane;  // distinct sentinels for lanes >= k
    if (lane < k) {
      e = top[(size_t)t * k + lane];
      if (e < 0 || e >= E) {
        flags |= DMOE_STATUS_EXPERT_OUT_OF_RANGE;
        e = -1 - lane;
      }
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    if (e >= 0) {
      if (__popc(peers) > 1) flags |= DMOE_STATUS_DUPLICATE_EXPERT;
      atomicAdd(&hist[e], 1);
    }
  }
  flags = __reduce_or_sync(0xFFFFFFFFu, flags);
  if (flags && lane == 0) set_status(status, flags);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kMapThreads)
    tile_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

// ---- scan ------------------------------------------------------------------------------------

constexpr int kScanThreads = 1024;

// Inclusive block-wide scan of one int per thread (1024 threads).
__device__ __forceinline__ int block_incl_scan(int v, int *warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xFFFFFFFFu, v, off);
    if (lane >= off) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += n;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += warp_tot[warp - 1];
  __syncthreads();
  return v;
}

// Per-tile exclusive offsets inside each expert, then (in the last CTA to finish) bins,
// padded_bins, num_blocks and the block -> expert table.  Grid: one CTA per 32 experts; warp c
// of a CTA owns tile chunk c (32 chunks), lane l owns expert 32*blockIdx.x + l, so every load
// of a tile's histogram row is one coalesced 128-byte access.  No CTA waits for another: the
// CTA that takes the last ticket of `done` (zeroed by the routing kernel) does the final part.
__global__ void __launch_bounds__(kScanThreads) k_map_scan(int n_tiles, int E, int nblk_cap,
                                                           int32_t *__restrict__ tile_hist,
                                                           int32_t *__restrict__ tokens_per_expert,
                                                           int32_t *__restrict__ bins,
                                                           int32_t *__restrict__ padded_bins,
                                                           int32_t *__restrict__ block_expert,
                                                           int32_t *__restrict__ num_blocks,
                                                           unsigned int *__restrict__ done) {
  __shared__ int chunk[32][33];
  __shared__ int s_pb[DMOE_MAX_EXPERTS];
  __shared__ int warp_tot[32];
  __shared__ bool is_last;
  const int c = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + lane;
  const int tpc = (n_tiles + 31) / 32;
  const int tb = c * tpc, te = min(n_tiles, tb + tpc);
  int sum = 0;
  if (e < E) {
    int t = tb;
    for (; t + 4 <= te; t += 4) {  // independent loads in flight
      const int v0 = tile_hist[(size_t)t * E + e], v1 = tile_hist[(size_t)(t + 1) * E + e];
      const int v2 = tile_hist[(size_t)(t + 2) * E + e], v3 = tile_hist[(size_t)(t + 3) * E + e];
      sum += v0 + v1 + v2 + v3;
    }
    for (; t < te; ++t) sum += tile_hist[(size_t)t * E + e];
  }
  chunk[c][lane] = sum;
  __syncthreads();
  if (c == 0) {  // exclusive scan over the 32 chunks of this lane's expert
    int run = 0;
    for (int cc = 0; cc < 32; ++cc) {
      const int v = chunk[cc][lane];
      chunk[cc][lane] = run;
      run += v;
    }
    if (e < E) tokens_per_expert[e] = run;
  }
  __syncthreads();
  if (e < E) {  // counts -> exclusive offsets inside the expert
    int run = chunk[c][lane];
    for (int t = tb; t < te; ++t) {
      const int v = tile_hist[(size_t)t * E + e];
      tile_hist[(size_t)t * E + e] = run;
      run += v;
    }
  }
  // ---- last CTA: bins, padded_bins, block table ----
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int tid = threadIdx.x;
  const int cnt = (tid < E) ? *((volatile int32_t *)tokens_per_expert + tid) : 0;
  const int pad = ((cnt + kBlock - 1) / kBlock) * kBlock;
  const int incl = block_incl_scan(cnt, warp_tot);
  const int pincl = block_incl_scan(pad, warp_tot);
  if (tid < E) {
    bins[tid] = incl;
    padded_bins[tid] = pincl;
    s_pb[tid] = pincl;
  }
  __syncthreads();
  const int nb = s_pb[E - 1] / kBlock;
  if (tid == 0) {
    *num_blocks = nb;
    *done = 0u;  // ready for the next call
  }
  for (int b = tid; b < nblk_cap; b += kScanThreads) {
    int owner = -1;
    if (b < nb) {  // smallest e with padded_bins[e] > b*128
      int lo = 0, hi = E - 1;
      const int row = b * kBlock;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_pb[mid] > row)
          hi = mid;
        else
          lo = mid + 1;
      }
      owner = lo;
    }
    block_expert[b] = owner;
  }
}

// ---- stable scatter --------------------------------------------------------------------------

__global__ void __launch_bounds__(kMapThreads) k_map_scatter(int T, int E, int k,
                                                             const int32_t *__restrict__ top,
                                                             const int32_t *__restrict__ tile_off,
                                                             const int32_t *__restrict__ bins,
                                                             const int32_t *__restrict__ padded_bins,
                                                             int32_t *__restrict__ indices,
                                                             int32_t *__restrict__ bin_ids,
                                                             int32_t *__restrict__ dest_row) {
  extern __shared__ int wh[];  // [kMapWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long N = (long long)T * k;
  const long long j0 = (long long)blockIdx.x * kMapTokTile * k;
  const long long j1 = min(N, j0 + (long long)kMapTokTile * k);
  const int n = (int)(j1 - j0);
  const int per_warp = (((n + kMapWarps - 1) / kMapWarps) + 31) & ~31;
  const long long wb = j0 + (long long)warp * per_warp;
  const long long we = min(j1, wb + per_warp);
  for (int i = threadIdx.x; i < kMapWarps * E; i += kMapThreads) wh[i] = 0;
  __syncthreads();
  int *my = wh + warp * E;
  const unsigned lt_mask = (1u << lane) - 1u;
  // pass 1: per-warp histogram of its contiguous entry range
  for (long long base = wb; base < we; base += 32) {
    const long long j = base + lane;
    int e = -1 - lane;
    if (j < we) {
      const int v = top[j];
      if (v >= 0 && v < E) e = v;
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive offsets per (warp, expert): expert start + tile offset + earlier warps
  for (int e = threadIdx.x; e < E; e += kMapThreads) {
    int run = ((e > 0) ? bins[e - 1] : 0) + tile_off[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < kMapWarps; ++w) {
      const int v = wh[w * E + e];
      wh[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  // pass 2: sorted position of every entry, in entry order within each expert
  for (long long base = wb; base < we; base += 32) {
    const long long j = base + lane;
    int e = -1 - lane;
    if (j < we) {
      const int v = top[j];
      if (v >= 0 && v < E) e = v;
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    if (e >= 0) {
      const int i = my[e] + __popc(peers & lt_mask);
      const int bins_prev = (e > 0) ? bins[e - 1] : 0;
      const int pbins_prev = (e > 0) ? padded_bins[e - 1] : 0;
      indices[i] = (int32_t)j;
      bin_ids[i] = e;
      dest_row[j] = (i - bins_prev) + pbins_prev;  // offset_in_bin + padded_bins[e-1]
    } else if (j < we) {
      dest_row[j] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
    __syncwarp();
  }
}

// ---- launchers -------------------------------------------------------------------------------

cudaError_t launch_route_hist(const uint16_t *logits, int T, int E, int k, bool renorm, int32_t *top,
                              float *weights, int32_t *tile_hist, int32_t *status,
                              cudaStream_t st) {
  const int tiles = map_tiles(T);
  const size_t smem = sizeof(int) * (size_t)E;
  unsigned int *done = map_ticket(tile_hist, T, E);
  if (!logits) {
    k_given_hist<<<tiles, kMapThreads, smem, st>>>(top, T, E, k, tile_hist, status, done);
    return cudaGetLastError();
  }
#define DMOE_ROUTE(KPL)                                                                      \
  k_route_hist<KPL><<<tiles, kMapThreads, smem, st>>>(logits, T, E, k, renorm ? 1 : 0, top,    \
                                                      weights, tile_hist,                      \
                                                      status, done)
  if (E <= 32)
    DMOE_ROUTE(1);
  else if (E <= 64)
    DMOE_ROUTE(2);
  else if (E <= 128)
    DMOE_ROUTE(4);
  else if (E <= 256)
    DMOE_ROUTE(8);
  else if (E <= 512)
    DMOE_ROUTE(16);
  else
    DMOE_ROUTE(32);
#undef DMOE_ROUTE
  return cudaGetLastError();
}

cudaError_t launch_map_scan(int T, int E, int nblk_cap, int32_t *tile_hist,
                            int32_t *tokens_per_expert, int32_t *bins, int32_t *padded_bins,
                            int32_t *block_expert, int32_t *num_blocks, cudaStream_t st) {
  k_map_scan<<<(E + 31) / 32, kScanThreads, 0, st>>>(map_tiles(T), E, nblk_cap, tile_hist,
                                                      tokens_per_expert, bins, padded_bins,
                                                      block_expert, num_blocks,
                                                      map_ticket(tile_hist, T, E));
  return cudaGetLastError();
}

cudaError_t launch_map_scatter(int T, int E, int k, const int32_t *top, const int32_t *tile_off,
                               const int32_t *bins, const int32_t *padded_bins, int32_t *indices,
                               int32_t *bin_ids, int32_t *dest_row, cudaStream_t st) {
  const size_t smem = sizeof(int) * (size_t)kMapWarps * E;
  k_map_scatter<<<map_tiles(T), kMapThreads, smem, st>>>(T, E, k, top, tile_off, bins,
                                                         padded_bins, indices, bin_ids, dest_row);
  return cudaGetLastError();
}

}  // namespace dmoe
