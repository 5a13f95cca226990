// round.cu -- tile-aware token rounding of the routing (SonicMoE abstract: the routing is
// adjusted so that every expert's token count is a multiple of the GEMM tile, 128 rows here,
// and the grouped GEMMs compute no padding rows).
//
// The abstract describes the method in one sentence.  This library reads it as: start from
// the top-k routing; for every expert e whose count c_e is not a multiple of 128, with
// r = c_e mod 128, either add the 128 - r best-ranked tokens that are not routed to e
// (round up, when r >= 64 and enough such tokens exist) or drop e's r worst-ranked entries
// (round down).  A token ranks for expert e by its logit l[t][e] (larger first), equal logits
// by the lower token index.  A token keeps its surviving slots in slot order, followed by its
// added experts in increasing expert order, and every entry's weight is the softmax over all E
// logits at its expert.  The result is a variable number of entries per token, stored as a
// token-major entry list with row offsets (CSR): entry_offsets [T+1], experts and weights
// [N'].  The padded map of that list (built by the map kernels with one entry per "token") has
// no padding rows.
//
// Kernels, all without inter-CTA waiting:
//   k_round_images   the logits' rank images transposed to one contiguous row per expert
//                    (64 x 64 tiles through shared memory, coalesced on both sides).
//   k_round_select   one CTA per expert: decides round up / down and finds the rank threshold
//                    (logit image v*, token t*) with two 8-bit histogram passes over the
//                    candidates' logit images and one ordered pass over the tied tokens, each
//                    thread taking groups of 32 consecutive tokens.
//   k_round_apply    one CTA per 64-token tile, warp per token: applies the thresholds; the
//                    count pass writes per-token counts and tile totals, the write pass the
//                    token's entries at its row offset.
//   k_round_offsets  one CTA: exclusive scan of the tile totals (the list's length N').
#include "common.cuh"
#include "kernels.h"

namespace dmoe {

namespace {

constexpr int kSelThreads = 512;
constexpr int kApplyThreads = 512;
constexpr int kApplyWarps = kApplyThreads / 32;

// Rank image of a bf16 logit: order-preserving 16-bit value (-0 taken as +0), NaN lowest (0).
__device__ __forceinline__ uint32_t rank_image(uint16_t b) {
  if ((b & 0x7FFFu) > 0x7F80u) return 0u;  // NaN ranks last
  if (b == 0x8000u) b = 0;                  // -0 ties with +0
  return (b & 0x8000u) ? (uint32_t)(~b & 0xFFFFu) : (uint32_t)(b | 0x8000u);
}


// Block-wide sum of one int per thread (kSelThreads threads).
__device__ __forceinline__ int block_sum(int v, int *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_add_sync(0xFFFFFFFFu, v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int s = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) s += red[w];
  return s;
}

}  // namespace

// img[e][t] = rank_image(logits[t][e]) (row stride Tp): 64 tokens x 64 experts per CTA
// through shared memory.
__global__ void __launch_bounds__(256) k_round_images(const uint16_t *__restrict__ logits, int T,
                                                      int Tp, int E, uint16_t *__restrict__ img) {
  __shared__ uint16_t tile[64][66];
  pdl_wait();
  pdl_trigger();
  const int e0 = blockIdx.x * 64, t0 = blockIdx.y * 64;
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int tt = i / 64, ee = i % 64;  // read along a token's row
    const int t = t0 + tt, e = e0 + ee;
    tile[tt][ee] = (t < T && e < E) ? (uint16_t)rank_image(logits[(size_t)t * E + e]) : 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int ee = i / 64, tt = i % 64;  // write along an expert's column
    const int t = t0 + tt, e = e0 + ee;
    if (t < T && e < E) img[(size_t)e * Tp + t] = tile[tt][ee];
  }
}

// One CTA per expert e.  Candidates: for round down, the tokens routed to e (drop the r worst
// ranked); for round up, the tokens not routed to e (add the 128 - r best ranked).  Finds the
// rank threshold so that exactly m = r (down) or 128 - r (up) candidates are on the chosen side:
//   up:    t added   iff image > v*, or image == v* and t <= t*
//   down:  t dropped iff image < v*, or image == v* and t >= t*
// param[3e..3e+2] = {mode (0 none, 1 down, 2 up), v*, t*}.  img [E][Tp]: the rank images, one
// row per expert, Tp = T rounded up to 32.  The tokens routed to e are its entries of the
// top-k routing's sorted order (indices[bins[e-1] .. bins[e]), entry j of token j / k);
// routed_bits: this CTA's bitmap of them (dynamic shared memory, T bits).  A thread takes
// groups of 32 consecutive tokens (one bitmap word, four 16-byte loads of images), so every
// pass is one load round followed by shared-memory work.
struct SelGroup {
  uint32_t cand;    // bit j: token 32g + j is a candidate
  uint16_t v[32];   // the tokens' rank images
};

__device__ __forceinline__ SelGroup sel_group(const uint32_t *routed_bits,
                                              const uint16_t *col, int g, int T, bool up) {
  SelGroup q;
  const int t0 = g * 32;
  const uint32_t routed = routed_bits[g];
  const uint32_t valid = (T - t0 >= 32) ? 0xFFFFFFFFu : ((1u << (T - t0)) - 1u);
  q.cand = (up ? ~routed : routed) & valid;
  const uint4 *src = reinterpret_cast<const uint4 *>(col + t0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = __ldg(src + i);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      q.v[8 * i + 2 * j] = (uint16_t)(ww[j] & 0xFFFFu);
      q.v[8 * i + 2 * j + 1] = (uint16_t)(ww[j] >> 16);
    }
  }
  return q;
}

// Exclusive prefix over the block (kSelThreads threads) of one int per thread; *total gets
// the block's sum.
__device__ __forceinline__ int block_excl_scan(int v, int *red, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xFFFFFFFFu, x, off);
    if (lane >= off) x += n;
  }
  __syncthreads();
  if (lane == 31) red[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) {
    if (w < warp) before += red[w];
    all += red[w];
  }
  *total = all;
  return before + x - v;
}

__global__ void __launch_bounds__(kSelThreads) k_round_select(const int32_t *__restrict__ indices,
                                                              const int32_t *__restrict__ bins,
                                                              const int32_t *__restrict__ counts,
                                                              int T, int Tp, int E, int k,
                                                              const uint16_t *__restrict__ img,
                                                              int32_t *__restrict__ param) {
  extern __shared__ uint32_t routed_bits[];  // [ceil(T/32)]
  __shared__ int hist[256];
  __shared__ int red[kSelThreads / 32];
  __shared__ int s_sel[2];
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  const int c = counts[e];
  const int r = c % kBlock;
  const bool up = (2 * r >= kBlock) && (T - c >= kBlock - r);
  if (r == 0) {
    if (threadIdx.x == 0) {
      param[3 * e] = 0;
      param[3 * e + 1] = 0;
      param[3 * e + 2] = 0;
    }
    return;
  }
  const int m = up ? kBlock - r : r;  // candidates to take
  const uint16_t *col = img + (size_t)e * Tp;
  const int words = (T + 31) / 32;
  for (int i = threadIdx.x; i < words; i += kSelThreads) routed_bits[i] = 0u;
  for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0;
  __syncthreads();
  const int b0 = (e > 0) ? bins[e - 1] : 0;
  for (int i = b0 + threadIdx.x; i < b0 + c; i += kSelThreads) {
    const int t = indices[i] / k;
    atomicOr(&routed_bits[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  // pass A: histogram of the candidates' high bytes
  for (int g = threadIdx.x; g < words; g += kSelThreads) {
    const SelGroup q = sel_group(routed_bits, col, g, T, up);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if ((q.cand >> j) & 1u) atomicAdd(&hist[q.v[j] >> 8], 1);
  }
  __syncthreads();
  // the high byte H holding the m-th candidate on the chosen side (from the top for round
  // up, from the bottom for round down), and the candidates strictly beyond it
  if (threadIdx.x == 0) {
    int acc = 0, sel = 0;
    for (int i = 0; i < 256; ++i) {
      const int b = up ? 255 - i : i;
      if (acc + hist[b] >= m) {
        sel = b;
        break;
      }
      acc += hist[b];
    }
    s_sel[0] = sel;
    s_sel[1] = acc;
  }
  __syncthreads();
  const uint32_t H = (uint32_t)s_sel[0];
  const int beyond_h = s_sel[1];
  for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0;
  __syncthreads();
  // pass B: low bytes of the candidates whose high byte is H
  for (int g = threadIdx.x; g < words; g += kSelThreads) {
    const SelGroup q = sel_group(routed_bits, col, g, T, up);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (((q.cand >> j) & 1u) && (uint32_t)(q.v[j] >> 8) == H) atomicAdd(&hist[q.v[j] & 0xFFu], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = beyond_h, sel = 0;
    for (int i = 0; i < 256; ++i) {
      const int b = up ? 255 - i : i;
      if (acc + hist[b] >= m) {
        sel = b;
        break;
      }
      acc += hist[b];
    }
    s_sel[0] = sel;
    s_sel[1] = acc;
  }
  __syncthreads();
  const uint32_t vstar = (H << 8) | (uint32_t)s_sel[0];
  const int beyond = s_sel[1];  // candidates strictly better (up) / worse (down) than v*
  // the tied candidates (image v*), group by group in token order: round up takes the ties
  // with the lowest token indices (the q-th lowest tied token, q = m - beyond); round down
  // drops those with the highest (the (ties - q + 1)-th lowest)
  int ties = 0;
  for (int g = threadIdx.x; g < words; g += kSelThreads) {
    const SelGroup q = sel_group(routed_bits, col, g, T, up);
#pragma unroll
    for (int j = 0; j < 32; ++j) ties += (((q.cand >> j) & 1u) && q.v[j] == vstar) ? 1 : 0;
  }
  ties = block_sum(ties, red);
  const int qn = m - beyond;
  const int want = up ? qn : ties - qn + 1;  // 1-based rank among the tied tokens, in t order
  if (threadIdx.x == 0) s_sel[0] = -1;
  __syncthreads();
  int seen = 0;
  for (int g0 = 0; g0 < words; g0 += kSelThreads) {  // rounds of kSelThreads groups
    const int g = g0 + threadIdx.x;
    uint32_t tiebits = 0u;
    if (g < words) {
      const SelGroup q = sel_group(routed_bits, col, g, T, up);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        tiebits |= (((q.cand >> j) & 1u) && q.v[j] == vstar) ? (1u << j) : 0u;
    }
    int total;
    const int before = seen + block_excl_scan(__popc(tiebits), red, &total);
    const int need = want - before;  // this thread's group holds it when 1 <= need <= popc
    if (need >= 1 && need <= __popc(tiebits)) {
      uint32_t b = tiebits;
      for (int i = 1; i < need; ++i) b &= b - 1u;  // drop the lower ties
      s_sel[0] = g * 32 + (__ffs(b) - 1);
    }
    seen += total;
    if (seen >= want) break;  // uniform: every thread has the same `seen`
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    param[3 * e] = up ? 2 : 1;
    param[3 * e + 1] = (int32_t)vstar;
    param[3 * e + 2] = s_sel[0];
  }
}

// Token-major application of the thresholds.  WRITE == false: per-token entry counts into
// tok_count and the tile's total into tile_sum.  WRITE == true: the token's entries at
// tile_off[tile] + (its offset inside the tile): experts, weights, the row offsets, and (the
// last tile) entry_offsets[T]; every CTA also fills a slice of the unused tail of the list
// (expert -1, weight 0) up to cap.
template <bool WRITE>
__global__ void __launch_bounds__(kApplyThreads) k_round_apply(
    const uint16_t *__restrict__ logits, const int32_t *__restrict__ top,
    const float *__restrict__ weights, const int32_t *__restrict__ param, int T, int E, int k,
    int32_t *__restrict__ tok_count, int32_t *__restrict__ tile_sum,
    const int32_t *__restrict__ tile_off, int32_t *__restrict__ entry_offsets,
    int32_t *__restrict__ out_expert, float *__restrict__ out_weight, long long cap) {
  // dynamic shared memory: the thresholds param[3E], then [kApplyWarps][ceil(E/32)]
  // routed-expert bitmaps
  extern __shared__ int32_t sm_apply[];
  __shared__ int s_cnt[kMapTokTile];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ew = (E + 31) / 32;
  int32_t *sp = sm_apply;
  uint32_t *bits = reinterpret_cast<uint32_t *>(sm_apply + 3 * E) + warp * ew;
  for (int i = threadIdx.x; i < 3 * E; i += kApplyThreads) sp[i] = param[i];
  __syncthreads();
  const int t_first = blockIdx.x * kMapTokTile;
  if (WRITE) {  // offsets of this tile's tokens: an exclusive scan of their counts
    if (threadIdx.x < kMapTokTile) {
      const int t = t_first + threadIdx.x;
      s_cnt[threadIdx.x] = (t < T) ? tok_count[t] : 0;
    }
    __syncthreads();
    if (warp == 0) {
      int run = tile_off[blockIdx.x];
      for (int base = 0; base < kMapTokTile; base += 32) {
        int v = s_cnt[base + lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int n = __shfl_up_sync(0xFFFFFFFFu, v, off);
          if (lane >= off) v += n;
        }
        const int excl = run + v - s_cnt[base + lane];
        run += __shfl_sync(0xFFFFFFFFu, v, 31);
        __syncwarp();
        s_cnt[base + lane] = excl;
      }
    }
    __syncthreads();
  }
  int tile_total = 0;
  for (int tt = warp; tt < kMapTokTile; tt += kApplyWarps) {
    const int t = t_first + tt;
    if (t >= T) break;
    for (int i = lane; i < ew; i += 32) bits[i] = 0u;
    __syncwarp();
    const uint16_t *row = logits + (size_t)t * E;
    int e_s = -1;
    float w_s = 0.0f;
    bool keep = false;
    if (lane < k) {
      e_s = top[(size_t)t * k + lane];
      w_s = weights[(size_t)t * k + lane];
      atomicOr(&bits[e_s >> 5], 1u << (e_s & 31));
      keep = true;
      if (sp[3 * e_s] == 1) {  // round down: dropped below the threshold
        const uint32_t v = rank_image(row[e_s]);
        const uint32_t vs = (uint32_t)sp[3 * e_s + 1];
        keep = !(v < vs || (v == vs && t >= sp[3 * e_s + 2]));
      }
    }
    __syncwarp();
    // the token's softmax: its largest logit is its first pick (weight w0 = 1 / sum)
    const int e0 = __shfl_sync(0xFFFFFFFFu, e_s, 0);
    const float w0 = __shfl_sync(0xFFFFFFFFu, w_s, 0);
    const float m = __uint_as_float((uint32_t)row[e0] << 16);
    const unsigned kept = __ballot_sync(0xFFFFFFFFu, keep);
    int n = __popc(kept);
    const int base = WRITE ? s_cnt[tt] : 0;
    if (WRITE && keep) {
      const int pos = base + __popc(kept & ((1u << lane) - 1u));
      out_expert[pos] = e_s;
      out_weight[pos] = w_s;
    }
    // added experts, in increasing expert order
    for (int e0b = 0; e0b < E; e0b += 32) {
      const int e = e0b + lane;
      bool add = false;
      if (e < E && sp[3 * e] == 2 && !((bits[e >> 5] >> (e & 31)) & 1u)) {
        const uint32_t v = rank_image(row[e]);
        const uint32_t vs = (uint32_t)sp[3 * e + 1];
        add = v > vs || (v == vs && t <= sp[3 * e + 2]);
      }
      const unsigned am = __ballot_sync(0xFFFFFFFFu, add);
      if (WRITE && add) {
        const int pos = base + n + __popc(am & ((1u << lane) - 1u));
        const float l = __uint_as_float((uint32_t)row[e] << 16);
        out_expert[pos] = e;
        out_weight[pos] = __fmul_rn(exp2f(__fmul_rn(__fsub_rn(l, m), 1.4426950408889634f)), w0);
      }
      n += __popc(am);
    }
    if (lane == 0) {
      if (WRITE) {
        entry_offsets[t] = base;
        if (t == T - 1) entry_offsets[T] = base + n;
      } else {
        tok_count[t] = n;
      }
    }
    tile_total += n;
    __syncwarp();
  }
  if (!WRITE) {
    __syncthreads();
    if (lane == 0) s_cnt[warp] = tile_total;
    __syncthreads();
    if (threadIdx.x == 0) {
      int s = 0;
      for (int w = 0; w < kApplyWarps; ++w) s += s_cnt[w];
      tile_sum[blockIdx.x] = s;
    }
  } else {  // the unused tail of the list: absent entries
    const long long total = tile_off[gridDim.x];
    for (long long j = total + (long long)blockIdx.x * kApplyThreads + threadIdx.x; j < cap;
         j += (long long)gridDim.x * kApplyThreads) {
      out_expert[j] = -1;
      out_weight[j] = 0.0f;
    }
  }
}

// Exclusive scan of the tile totals into tile_off[0..tiles] (tile_off[tiles] = N').
__global__ void __launch_bounds__(1024) k_round_offsets(const int32_t *__restrict__ tile_sum,
                                                        int tiles,
                                                        int32_t *__restrict__ tile_off) {
  __shared__ int warp_tot[32];
  __shared__ int s_carry;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < tiles; base += 1024) {
    const int i = base + threadIdx.x;
    const int v0 = (i < tiles) ? tile_sum[i] : 0;
    int v = v0;
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
    const int incl = v + ((warp > 0) ? warp_tot[warp - 1] : 0) + s_carry;
    if (i < tiles) tile_off[i] = incl - v0;
    __syncthreads();
    if (threadIdx.x == 1023) s_carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) tile_off[tiles] = s_carry;
}

cudaError_t launch_round_tokens(const uint16_t *logits, const int32_t *top, const float *weights,
                                const int32_t *counts, const int32_t *bins,
                                const int32_t *indices, int T, int E, int k, const RoundScratch &s,
                                int32_t *entry_offsets, int32_t *out_expert, float *out_weight,
                                long long cap, cudaStream_t st) {
  const size_t sel_smem = sizeof(uint32_t) * (size_t)((T + 31) / 32);
  cudaError_t err = cudaSuccess;
  static cudaError_t attr = cudaFuncSetAttribute(
      k_round_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRoundMaxSelectSmem);
  if (attr != cudaSuccess) return attr;
  const int Tp = round_img_stride(T);
  if ((err = launch_pdl(k_round_images, dim3((E + 63) / 64, (T + 63) / 64), 256, 0, st, logits, T,
                        Tp, E, s.img)) != cudaSuccess)
    return err;
  if ((err = launch_pdl(k_round_select, E, kSelThreads, sel_smem, st, indices, bins, counts, T, Tp,
                        E, k, (const uint16_t *)s.img, s.param)) != cudaSuccess)
    return err;
  const int tiles = map_tiles(T);
  const size_t ap_smem = sizeof(int32_t) * (3 * (size_t)E + (size_t)kApplyWarps * ((E + 31) / 32));
  if ((err = launch_pdl(k_round_apply<false>, tiles, kApplyThreads, ap_smem, st, logits, top,
                        weights, s.param, T, E, k, s.tok_count, s.tile_sum, s.tile_off,
                        entry_offsets, out_expert, out_weight, cap)) != cudaSuccess)
    return err;
  if ((err = launch_pdl(k_round_offsets, 1, 1024, 0, st, s.tile_sum, tiles, s.tile_off)) !=
      cudaSuccess)
    return err;
  return launch_pdl(k_round_apply<true>, tiles, kApplyThreads, ap_smem, st, logits, top, weights,
                    s.param, T, E, k, s.tok_count, s.tile_sum, s.tile_off, entry_offsets,
                    out_expert, out_weight, cap);
}

}  // namespace dmoe
