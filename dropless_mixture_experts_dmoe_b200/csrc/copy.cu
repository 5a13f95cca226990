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
  pdl_wait();
  pdl_trigger();
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
// VPL 16-byte vectors per lane for each of SLOTS slots are loaded before any is consumed
// (VPL * SLOTS = 16 loads in flight per lane): few slots (small top_k) take wide row pieces.
template <int VPL, int SLOTS>
__global__ void __launch_bounds__(kCopyThreads) k_combine(int T, int h, int k,
                                                          const uint4 *__restrict__ y_pad,
                                                          const int32_t *__restrict__ dest_row,
                                                          const float *__restrict__ weights,
                                                          uint4 *__restrict__ y) {
  pdl_wait();
  pdl_trigger();
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
    for (int v0 = vs; v0 < ve; v0 += 32 * VPL) {
      float acc[VPL][8];
#pragma unroll
      for (int u = 0; u < VPL; ++u)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
      for (int s0 = 0; s0 < k; s0 += SLOTS) {
        uint4 buf[SLOTS][VPL];
#pragma unroll
        for (int ss = 0; ss < SLOTS; ++ss) {
          const int s = s0 + ss;
          const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
          if (s < k && r >= 0) {
#pragma unroll
            for (int u = 0; u < VPL; ++u) {
              const int v = v0 + u * 32 + lane;
              if (v < ve) buf[ss][u] = ld_nc_v4(y_pad + (size_t)r * vpr + v);
            }
          }
        }
#pragma unroll
        for (int ss = 0; ss < SLOTS; ++ss) {
          const int s = s0 + ss;
          const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
          const float ws = __shfl_sync(0xFFFFFFFFu, wl, s & 31);
          if (s < k && r >= 0) {
#pragma unroll
            for (int u = 0; u < VPL; ++u) {
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
      for (int u = 0; u < VPL; ++u) {
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

// Backward scatter-sum (the gradient of the gather, walkthrough section 4.2): dx_t =
// bf16(sum_{s<k} dX_pad[dest_row[t*k+s]]) in fp32, slot order, rounded once.  dX_pad rows are
// block floating point: fp16 values times a power-of-two scale per row and 256-column tile
// (scale[r * nsc + c / 256]); fp16 * scale is exact in fp32, so each slot adds its value with
// one fused multiply-add.  With it the routing-weight gradient dweights[t*k+s] =
// sum_{n<nt} part[dest_row[t*k+s] * nt + n] in column-tile order.  A lane covers 8 consecutive
// columns (one 16-byte vector) per slot; VPL such vectors per lane and SLOTS slots are loaded
// before any is consumed.
template <int VPL, int SLOTS>
__global__ void __launch_bounds__(kCopyThreads, 2) k_scatter_sum(int T, int h, int k,
                                                              const uint4 *__restrict__ dx_pad,
                                                              const float *__restrict__ scale,
                                                              const int32_t *__restrict__ dest_row,
                                                              uint4 *__restrict__ dx,
                                                              const float *__restrict__ part,
                                                              int nt,
                                                              float *__restrict__ dweights) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int vpr = h >> 3;      // 16-byte vectors (8 columns) per row
  const int nsc = (h + 255) >> 8;  // scales per row
  constexpr int kSlice = 32 * VPL;
  const int S = (vpr + kSlice - 1) / kSlice;
  const long long items = (long long)T * S;
  const long long nw = (long long)gridDim.x * kCopyWarps;
  for (long long it = (long long)blockIdx.x * kCopyWarps + (threadIdx.x >> 5); it < items;
       it += nw) {
    const int t = (int)(it / S);
    const int v0 = (int)(it - (long long)t * S) * kSlice;
    const int d = (lane < k) ? dest_row[(size_t)t * k + lane] : -1;
    if (v0 == 0 && lane < k) {
      float g = 0.0f;
      if (d >= 0)
        for (int n = 0; n < nt; ++n) g += __ldg(part + (size_t)d * nt + n);
      dweights[(size_t)t * k + lane] = g;  // 0 for an entry dropped from the map
    }
    float acc[VPL][8];
#pragma unroll
    for (int u = 0; u < VPL; ++u)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
    for (int s0 = 0; s0 < k; s0 += SLOTS) {
      uint4 buf[SLOTS][VPL];
      float sc[SLOTS][VPL];
#pragma unroll
      for (int ss = 0; ss < SLOTS; ++ss) {
        const int s = s0 + ss;
        const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
        if (s < k && r >= 0) {
#pragma unroll
          for (int u = 0; u < VPL; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < vpr) {
              buf[ss][u] = ld_nc_v4(dx_pad + (size_t)r * vpr + v);
              sc[ss][u] = __ldg(scale + (size_t)r * nsc + (v >> 5));
            }
          }
        }
      }
#pragma unroll
      for (int ss = 0; ss < SLOTS; ++ss) {
        const int s = s0 + ss;
        const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
        if (s < k && r >= 0) {
#pragma unroll
          for (int u = 0; u < VPL; ++u) {
            const uint32_t *q = reinterpret_cast<const uint32_t *>(&buf[ss][u]);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              acc[u][2 * p] = fmaf(f16_lo(q[p]), sc[ss][u], acc[u][2 * p]);
              acc[u][2 * p + 1] = fmaf(f16_hi(q[p]), sc[ss][u], acc[u][2 * p + 1]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vpr) {
        uint4 o;
        o.x = pack_bf16x2(acc[u][0], acc[u][1]);
        o.y = pack_bf16x2(acc[u][2], acc[u][3]);
        o.z = pack_bf16x2(acc[u][4], acc[u][5]);
        o.w = pack_bf16x2(acc[u][6], acc[u][7]);
        dx[(size_t)t * vpr + v] = o;
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
  return launch_pdl(k_gather, copy_grid(items), kCopyThreads, 0, st, T, h, k, E,
                    static_cast<const uint4 *>(x), dest_row, counts, padded_bins,
                    static_cast<uint4 *>(x_pad));
}

cudaError_t launch_combine(int T, int h, int k, const void *y_pad, const int32_t *dest_row,
                           const float *weights, void *y, cudaStream_t st) {
  const int grid = copy_grid((long long)T * slices(h));
  const uint4 *src = static_cast<const uint4 *>(y_pad);
  uint4 *dst = static_cast<uint4 *>(y);
  auto kernel = (k <= 2) ? k_combine<8, 2> : (k <= 4) ? k_combine<4, 4> : k_combine<2, 8>;
  return launch_pdl(kernel, grid, kCopyThreads, 0, st, T, h, k, src, dest_row, weights, dst);
}

cudaError_t launch_bwd_scatter(int T, int h, int k, const void *dx_pad, const float *dx_scale,
                               const int32_t *dest_row, const float *part, int nt, void *dx,
                               float *dweights, cudaStream_t st) {
  // 16-byte vectors per lane and slot: at most 16 loads in flight per lane within 128
  // registers (two CTAs per SM)
  const int vpl = (k <= 2) ? 4 : 2;
  auto kernel = (k <= 2) ? k_scatter_sum<4, 2> : (k <= 4) ? k_scatter_sum<2, 4>
                                                          : k_scatter_sum<2, 8>;
  const long long items = (long long)T * (((h >> 3) + 32 * vpl - 1) / (32 * vpl));
  return launch_pdl(kernel, copy_grid(items), kCopyThreads, 0, st, T, h, k,
                    static_cast<const uint4 *>(dx_pad), dx_scale, dest_row,
                    static_cast<uint4 *>(dx), part, nt, dweights);
}

}  // namespace dmoe
