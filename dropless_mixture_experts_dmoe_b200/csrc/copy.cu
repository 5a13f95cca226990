// copy.cu -- padded_gather and the weighted padded_scatter (MegaBlocks walkthrough "02 ·
// dropless MoE 与 block-sparse 重构", section 4.2: one pair of copy kernels, gather
// out[index_b] = x[index_a // TOP_K], scatter in reverse times the routing weight).
//
// Both kernels are token-major rather than one program per sorted entry: a warp reads a
// token row once with 16-byte vector loads and writes (or reads) its k padded rows, so x is
// read once in the gather and y is written once, without atomics, in the scatter.  Both are
// HBM-bound; the grid is a multiple of the SM count and every warp walks work items with a
// grid stride.
#include "common.cuh"
#include "kernels.h"

namespace dmoe {

constexpr int kCopyThreads = 256;
constexpr int kCopyWarps = kCopyThreads / 32;
constexpr int kGatherVPL = 8;   // 16-byte vectors in flight per lane (gather)
constexpr int kCombineVPL = 2;  // 16-byte vectors per lane per slot (combine)
constexpr int kCombineSlots = 8;

__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// A row slice is 32 * kGatherVPL 16-byte vectors (4 KB); a token's row is split into
// ceil(vpr / slice) slices so that short-T workloads still keep many warps busy.
constexpr int kSliceVecs = 32 * kGatherVPL;

// Work items: [0, T*S) token slices (S slices per row); then 128*E padding rows (expert e,
// row r of its last block).
__global__ void __launch_bounds__(kCopyThreads) k_gather(int T, int h, int k, int E,
                                                         const uint4 *__restrict__ x,
                                                         const int32_t *__restrict__ dest_row,
                                                         const int32_t *__restrict__ counts,
                                                         const int32_t *__restrict__ padded_bins,
                                                         uint4 *__restrict__ x_pad) {
  const int lane = threadIdx.x & 31;
  const int vpr = h >> 3;  // 16-byte vectors per row
  const int S = (vpr + kSliceVecs - 1) / kSliceVecs;
  const long long ntok = (long long)T * S;
  const long long items = ntok + (long long)kBlock * E;
  const long long nw = (long long)gridDim.x * kCopyWarps;
  for (long long it = (long long)blockIdx.x * kCopyWarps + (threadIdx.x >> 5); it < items;
       it += nw) {
    if (it < ntok) {
      const int t = (int)(it / S);
      const int v0 = (int)(it - (long long)t * S) * kSliceVecs;
      const int d = (lane < k) ? dest_row[(size_t)t * k + lane] : -1;
      const uint4 *src = x + (size_t)t * vpr;
      uint4 buf[kGatherVPL];
#pragma unroll
      for (int u = 0; u < kGatherVPL; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vpr) buf[u] = ld_nc_v4(src + v);
      }
      for (int s = 0; s < k; ++s) {
        const int r = __shfl_sync(0xFFFFFFFFu, d, s);
        if (r < 0) continue;
        uint4 *dst = x_pad + (size_t)r * vpr;
#pragma unroll
        for (int u = 0; u < kGatherVPL; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < vpr) dst[v] = buf[u];
        }
      }
    } else {
      const long long p = it - ntok;
      const int e = (int)(p / kBlock), r = (int)(p % kBlock);
      const int c = counts[e];
      const int pend = padded_bins[e];
      const int first_pad = ((e > 0) ? padded_bins[e - 1] : 0) + c;
      const int row = first_pad + r;
      if (row < pend) {  // padding rows of the expert's last block are zero
        uint4 *dst = x_pad + (size_t)row * vpr;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        for (int v = lane; v < vpr; v += 32) dst[v] = z;
      }
    }
  }
}

// y_t = sum_{s<k} w_ts * Y_pad[dest_row[t*k+s]]: fp32, slot order, one fused multiply-add per
// slot and element, rounded once to bf16.  weights == NULL: w = 1.
__global__ void __launch_bounds__(kCopyThreads) k_combine(int T, int h, int k,
                                                          const uint4 *__restrict__ y_pad,
                                                          const int32_t *__restrict__ dest_row,
                                                          const float *__restrict__ weights,
                                                          uint4 *__restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int vpr = h >> 3;
  const int S = (vpr + kSliceVecs - 1) / kSliceVecs;
  const long long items = (long long)T * S;
  const long long nw = (long long)gridDim.x * kCopyWarps;
  for (long long it = (long long)blockIdx.x * kCopyWarps + (threadIdx.x >> 5); it < items;
       it += nw) {
    const int t = (int)(it / S);
    const int vs = (int)(it - (long long)t * S) * kSliceVecs;
    const int ve = min(vpr, vs + kSliceVecs);
    const int d = (lane < k) ? dest_row[(size_t)t * k + lane] : -1;
    const float wl = (lane < k) ? (weights ? weights[(size_t)t * k + lane] : 1.0f) : 0.0f;
    for (int v0 = vs; v0 < ve; v0 += 32 * kCombineVPL) {
      float acc[kCombineVPL][8];
#pragma unroll
      for (int u = 0; u < kCombineVPL; ++u)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
      for (int s0 = 0; s0 < k; s0 += kCombineSlots) {
        uint4 buf[kCombineSlots][kCombineVPL];
#pragma unroll
        for (int ss = 0; ss < kCombineSlots; ++ss) {
          const int s = s0 + ss;
          const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
          if (s < k && r >= 0) {
#pragma unroll
            for (int u = 0; u < kCombineVPL; ++u) {
              const int v = v0 + u * 32 + lane;
              if (v < ve) buf[ss][u] = ld_nc_v4(y_pad + (size_t)r * vpr + v);
            }
          }
        }
#pragma unroll
        for (int ss = 0; ss < kCombineSlots; ++ss) {
          const int s = s0 + ss;
          const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
          const float ws = __shfl_sync(0xFFFFFFFFu, wl, s & 31);
          if (s < k && r >= 0) {
#pragma unroll
            for (int u = 0; u < kCombineVPL; ++u) {
              const uint32_t *q = reinterpret_cast<const uint32_t *>(&buf[ss][u]);
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                acc[u][2 * p] = fmaf(ws, bf16_lo(q[p]), acc[u][2 * p]);
                acc[u][2 * p + 1] = fmaf(ws, bf16_hi(q[p]), acc[u][2 * p + 1]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kCombineVPL; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < ve) {
          uint4 o;
          o.x = pack_bf16x2(acc[u][0], acc[u][1]);
          o.y = pack_bf16x2(acc[u][2], acc[u][3]);
          o.z = pack_bf16x2(acc[u][4], acc[u][5]);
          o.w = pack_bf16x2(acc[u][6], acc[u][7]);
          y[(size_t)t * vpr + v] = o;
        }
      }
    }
  }
}

// Backward of the weighted scatter (walkthrough section 4.2: its gradient is a gather plus the
// routing-weight gradient).  Warp per token: for each slot s with padded row r,
//   dY_pad[r] = bf16(w_ts * dy_t)   and   dweights[t*k+s] = <dy_t, Y_pad[r]> (fp32 dot,
// fixed lane order).  Work items past T zero the padding rows of every expert's last block,
// like the forward gather, so the weight gradients never see stale rows.
__global__ void __launch_bounds__(kCopyThreads) k_dy_gather(int T, int h, int k, int E,
                                                            const uint4 *__restrict__ dy,
                                                            const int32_t *__restrict__ dest_row,
                                                            const float *__restrict__ weights,
                                                            const int32_t *__restrict__ counts,
                                                            const int32_t *__restrict__ padded_bins,
                                                            const uint4 *__restrict__ y_pad,
                                                            uint4 *__restrict__ dy_pad,
                                                            float *__restrict__ dweights) {
  const int lane = threadIdx.x & 31;
  const int vpr = h >> 3;
  const long long items = (long long)T + (long long)kBlock * E;
  const long long nw = (long long)gridDim.x * kCopyWarps;
  for (long long it = (long long)blockIdx.x * kCopyWarps + (threadIdx.x >> 5); it < items;
       it += nw) {
    if (it < T) {
      const int t = (int)it;
      const int d = (lane < k) ? dest_row[(size_t)t * k + lane] : -1;
      const float wl = (lane < k) ? weights[(size_t)t * k + lane] : 0.0f;
      const uint4 *src = dy + (size_t)t * vpr;
      for (int s = 0; s < k; ++s) {
        const int r = __shfl_sync(0xFFFFFFFFu, d, s);
        const float ws = __shfl_sync(0xFFFFFFFFu, wl, s);
        float dot = 0.0f;
        if (r >= 0) {
          const uint4 *yrow = y_pad + (size_t)r * vpr;
          uint4 *orow = dy_pad + (size_t)r * vpr;
          for (int v0 = 0; v0 < vpr; v0 += 32 * kGatherVPL) {
            uint4 g[kGatherVPL], yv[kGatherVPL];
#pragma unroll
            for (int u = 0; u < kGatherVPL; ++u) {
              const int v = v0 + u * 32 + lane;
              if (v < vpr) {
                g[u] = __ldg(src + v);
                yv[u] = ld_nc_v4(yrow + v);
              }
            }
#pragma unroll
            for (int u = 0; u < kGatherVPL; ++u) {
              const int v = v0 + u * 32 + lane;
              if (v < vpr) {
                const uint32_t *gq = reinterpret_cast<const uint32_t *>(&g[u]);
                const uint32_t *yq = reinterpret_cast<const uint32_t *>(&yv[u]);
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float g0 = bf16_lo(gq[q]), g1 = bf16_hi(gq[q]);
                  dot = fmaf(g0, bf16_lo(yq[q]), dot);
                  dot = fmaf(g1, bf16_hi(yq[q]), dot);
                  o[q] = pack_bf16x2(ws * g0, ws * g1);
                }
                orow[v] = make_uint4(o[0], o[1], o[2], o[3]);
              }
            }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
        if (lane == 0) dweights[(size_t)t * k + s] = dot;
      }
    } else {
      const long long q = it - T;
      const int e = (int)(q / kBlock), r = (int)(q % kBlock);
      const int row = ((e > 0) ? padded_bins[e - 1] : 0) + counts[e] + r;
      if (row < padded_bins[e]) {
        uint4 *dst = dy_pad + (size_t)row * vpr;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        for (int v = lane; v < vpr; v += 32) dst[v] = z;
      }
    }
  }
}

static int copy_grid(long long items) {
  const long long per_cta = kCopyWarps;
  long long want = (items + per_cta - 1) / per_cta;
  const long long cap = (long long)device_sm_count() * 8;  // 8 resident CTAs per SM
  if (want > cap) want = cap;
  return (int)(want < 1 ? 1 : want);
}

static long long slices(int h) { return ((h >> 3) + kSliceVecs - 1) / kSliceVecs; }

cudaError_t launch_gather(int T, int h, int k, int E, const void *x, const int32_t *dest_row,
                          const int32_t *counts, const int32_t *padded_bins, void *x_pad,
                          cudaStream_t st) {
  const long long items = (long long)T * slices(h) + (long long)kBlock * E;
  k_gather<<<copy_grid(items), kCopyThreads, 0, st>>>(
      T, h, k, E, static_cast<const uint4 *>(x), dest_row, counts, padded_bins,
      static_cast<uint4 *>(x_pad));
  return cudaGetLastError();
}

cudaError_t launch_combine(int T, int h, int k, const void *y_pad, const int32_t *dest_row,
                           const float *weights, void *y, cudaStream_t st) {
  k_combine<<<copy_grid((long long)T * slices(h)), kCopyThreads, 0, st>>>(
      T, h, k, static_cast<const uint4 *>(y_pad),
                                                   dest_row, weights, static_cast<uint4 *>(y));
  return cudaGetLastError();
}

}  // namespace dmoe

namespace dmoe {

cudaError_t launch_dy_gather(int T, int h, int k, int E, const void *dy, const int32_t *dest_row,
                             const float *weights, const int32_t *counts,
                             const int32_t *padded_bins, const void *y_pad, void *dy_pad,
                             float *dweights, cudaStream_t st) {
  const long long items = (long long)T + (long long)kBlock * E;
  k_dy_gather<<<copy_grid(items), kCopyThreads, 0, st>>>(
      T, h, k, E, static_cast<const uint4 *>(dy), dest_row, weights, counts, padded_bins,
      static_cast<const uint4 *>(y_pad), static_cast<uint4 *>(dy_pad), dweights);
  return cudaGetLastError();
}

}  // namespace dmoe
