// copy.cu -- padded_gather and the weighted padded_scatter (MegaBlocks walkthrough "02 ·
// dropless MoE 与 block-sparse 重构", section 4.2: one pair of copy kernels, gather
// out[index_b] = x[index_a // TOP_K], scatter in reverse times the routing weight).
//
// Both kernels are token-major rather than one program per sorted entry: a warp reads a
// token row once with 16-byte vector loads and writes (or reads) its k padded rows, so x is
// read once in the gather and y is written once, without atomics, in the scatter.  Both are
// HBM-bound; the grid is a multiple of the SM count and every warp walks work items with a
// grid stride.
#include <mutex>

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

// The entries of token t: [t*k, t*k + k), or [offsets[t], offsets[t+1]) for a token-major
// entry list (the rounded routing, where tokens have different entry counts).
__device__ __forceinline__ void token_entries(const int32_t *__restrict__ offsets, int t, int k,
                                              long long &base, int &cnt) {
  if (offsets) {
    base = offsets[t];
    cnt = offsets[t + 1] - (int)base;
  } else {
    base = (long long)t * k;
    cnt = k;
  }
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
                                                         uint4 *__restrict__ x_pad,
                                                         const int32_t *__restrict__ offsets) {
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
      long long base;
      int cnt;
      token_entries(offsets, t, k, base, cnt);
      const uint4 *src = x + (size_t)t * vpr;
      uint4 buf[kGatherVPL];
#pragma unroll
      for (int u = 0; u < kGatherVPL; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vpr) buf[u] = ld_nc_v4(src + v);
      }
      for (int c0 = 0; c0 < cnt; c0 += 32) {  // one pass of up to 32 entries (k <= 32)
        const int nc = min(32, cnt - c0);
        const int d = (lane < nc) ? dest_row[base + c0 + lane] : -1;
        for (int s = 0; s < nc; ++s) {
          const int r = __shfl_sync(0xFFFFFFFFu, d, s);
          if (r < 0) continue;
          uint4 *dst = x_pad + (size_t)r * vpr;
#pragma unroll
          for (int u = 0; u < kGatherVPL; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < vpr) dst[v] = buf[u];
          }
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

// Token-major sum of each token's padded rows, the padded_scatter of walkthrough section 4.2:
//   out_t = bf16(sum_s c_s * rows[dest_row[e_s]])   over the token's entries e_s in order,
// fp32 accumulation rounded once, no atomics.  Forward combine: c_s = w_s, the routing weight
// (weights != NULL).  Backward (the gradient of the gather, section 4.2): c_s = 1 and, with
// dweights != NULL, the routing-weight gradient dweights[e] = sum_{n<nt} part[dest_row[e]*nt + n]
// in column-tile order.  Row format: bf16 (scale == NULL) or block floating point, fp16 values
// times a power-of-two scale per row and DMOE_SCALE_COLS columns (scale[r * nsc + c / 128]),
// which is exact in fp32, so each entry adds c_s * scale * value with one rounding.
// A lane covers 8 consecutive columns (one 16-byte vector) per entry; VPL vectors per lane
// and SLOTS entries are loaded before any is consumed.
template <int VPL, int SLOTS, bool F16S>
__global__ void __launch_bounds__(kCopyThreads, 4)
    k_combine(int T, int h, int k, const uint4 *__restrict__ rows,
              const float *__restrict__ scale, const int32_t *__restrict__ dest_row,
              const float *__restrict__ weights, uint4 *__restrict__ out,
              const float *__restrict__ part, int nt, float *__restrict__ dweights,
              const int32_t *__restrict__ offsets) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int vpr = h >> 3;                                      // 16-byte vectors per row
  const int nsc = dmoe_scale_stride(h);  // scales per row (padded to a multiple of 4)
  constexpr int kVecPerScale = DMOE_SCALE_COLS / 8;
  static_assert(VPL % 2 == 0, "scales are loaded for pairs of vectors");
  const int S = (vpr + kSliceVecs - 1) / kSliceVecs;  // 4 KB row slices per token
  const long long items = (long long)T * S;
  const long long nw = (long long)gridDim.x * kCopyWarps;
  const long long first = (long long)blockIdx.x * kCopyWarps + (threadIdx.x >> 5);
  // The first 32 entries of the warp's next item (dest rows, weights) are loaded while the
  // current item's rows are summed, so an item starts with its row loads.
  long long nbase = 0;
  int ncnt = 0, nd = -1;
  float nwt = 1.0f;
  auto fetch = [&](long long item) {
    token_entries(offsets, (int)(item / S), k, nbase, ncnt);
    const int kk = max(0, min(32, ncnt));
    nd = (lane < kk) ? dest_row[nbase + lane] : -1;
    nwt = (lane < kk && weights) ? weights[nbase + lane] : 1.0f;
  };
  if (first < items) fetch(first);
  for (long long it = first; it < items; it += nw) {
    const int t = (int)(it / S);
    const int vs = (int)(it - (long long)t * S) * kSliceVecs;
    const int ve = min(vpr, vs + kSliceVecs);
    const long long base = nbase;
    const int cnt = ncnt, d_first = nd;
    const float w_first = nwt;
    if (it + nw < items) fetch(it + nw);
    // the token's entries (up to 32 per pass; more only with the rounded routing), loaded
    // once per slice and reused by its row pieces
    for (int c0 = 0; c0 == 0 || c0 < cnt; c0 += 32) {
      const int kk = max(0, min(32, cnt - c0));
      const int d = (c0 == 0) ? d_first : ((lane < kk) ? dest_row[base + c0 + lane] : -1);
      const float wl =
          (c0 == 0) ? w_first : ((lane < kk && weights) ? weights[base + c0 + lane] : 1.0f);
      if (dweights && vs == 0 && lane < kk) {
        float g = 0.0f;
        if (d >= 0)
          for (int n = 0; n < nt; ++n) g += __ldg(part + (size_t)d * nt + n);
        dweights[base + c0 + lane] = g;  // 0 for an entry dropped from the map
      }
      for (int v0 = vs; v0 < ve; v0 += 32 * VPL) {
        float acc[VPL][8];
        if (c0 == 0) {
#pragma unroll
          for (int u = 0; u < VPL; ++u)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
        } else {  // a later pass of a token with more than 32 entries: continue the sum
#pragma unroll
          for (int u = 0; u < VPL; ++u) {
            const int v = v0 + u * 32 + lane;
            const uint4 o = (v < ve) ? out[(size_t)t * vpr + v] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t *q = reinterpret_cast<const uint32_t *>(&o);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              acc[u][2 * p] = bf16_lo(q[p]);
              acc[u][2 * p + 1] = bf16_hi(q[p]);
            }
          }
        }
        for (int s0 = 0; s0 < kk; s0 += SLOTS) {
          uint4 buf[SLOTS][VPL];
          float cf[SLOTS][VPL];
          uint32_t slow = 0;  // F16S: (slot, vector) pairs that take the converting path
#pragma unroll
          for (int ss = 0; ss < SLOTS; ++ss) {
            const int s = s0 + ss;
            const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
            const float ws = __shfl_sync(0xFFFFFFFFu, wl, s & 31);
            if (s < kk && r >= 0) {
#pragma unroll
              for (int u = 0; u < VPL; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < ve) buf[ss][u] = ld_nc_v4(rows + (size_t)r * vpr + v);
                cf[ss][u] = ws;
              }
              if (F16S) {
                // The scales of this lane's vectors: vector v lies in group v / 16, and v0 is a
                // multiple of 64 vectors (4 groups), so one 16-byte load serves two vectors
                // (lanes 0-15 take groups 0 and 2 of it, lanes 16-31 groups 1 and 3).  Scale
                // rows are padded to a multiple of 4 groups, so the load stays in the row.
                // Unweighted rows whose scale fp16 holds exactly take the fp16 path (the
                // coefficient kept as fp16 bits); the others are converted (coefficient
                // w * |scale| in fp32).
#pragma unroll
                for (int u2 = 0; u2 < VPL / 2; ++u2) {
                  if (v0 + u2 * 64 < ve) {
                    const float4 s4 = __ldg(reinterpret_cast<const float4 *>(
                        scale + (size_t)r * nsc + v0 / kVecPerScale + 4 * u2));
                    const float sa = (lane < 16) ? s4.x : s4.y, sb = (lane < 16) ? s4.z : s4.w;
                    const bool pa = !weights && scale_fits_f16(sa);
                    const bool pb = !weights && scale_fits_f16(sb);
                    cf[ss][2 * u2] = pa ? __uint_as_float(__half_as_ushort(__float2half_rn(sa)))
                                        : ws * fabsf(sa);
                    cf[ss][2 * u2 + 1] =
                        pb ? __uint_as_float(__half_as_ushort(__float2half_rn(sb))) : ws * fabsf(sb);
                    slow |= (pa ? 0u : 1u) << (ss * VPL + 2 * u2);
                    slow |= (pb ? 0u : 1u) << (ss * VPL + 2 * u2 + 1);
                  }
                }
              }
            }
          }
#pragma unroll
          for (int ss = 0; ss < SLOTS; ++ss) {
            const int s = s0 + ss;
            const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
            if (s < kk && r >= 0) {
#pragma unroll
              for (int u = 0; u < VPL; ++u) {
                const uint32_t *q = reinterpret_cast<const uint32_t *>(&buf[ss][u]);
                const float c = cf[ss][u];
                if (F16S && !((slow >> (ss * VPL + u)) & 1u)) {
                  const uint16_t c16 = (uint16_t)__float_as_uint(c);
#pragma unroll
                  for (int p = 0; p < 4; ++p)
                    fma2_f16_f32(acc[u][2 * p], acc[u][2 * p + 1], q[p], c16);
                } else {
#pragma unroll
                  for (int p = 0; p < 4; ++p) {
                    const float lo = F16S ? f16_lo(q[p]) : bf16_lo(q[p]);
                    const float hi = F16S ? f16_hi(q[p]) : bf16_hi(q[p]);
                    acc[u][2 * p] = fmaf(c, lo, acc[u][2 * p]);
                    acc[u][2 * p + 1] = fmaf(c, hi, acc[u][2 * p + 1]);
                  }
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
            out[(size_t)t * vpr + v] = o;
          }
        }
      }
    }
  }
}

// Fused combine helpers: zero the fp32 token accumulator before the down GEMM reduces into
// it, and round it to the bf16 output afterwards (8 columns per thread and step).
__global__ void __launch_bounds__(kCopyThreads) k_acc_zero(long long n8, float4 *__restrict__ acc) {
  pdl_wait();
  pdl_trigger();
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long i = (long long)blockIdx.x * kCopyThreads + threadIdx.x; i < n8;
       i += (long long)gridDim.x * kCopyThreads) {
    acc[2 * i] = z;
    acc[2 * i + 1] = z;
  }
}

__global__ void __launch_bounds__(kCopyThreads) k_acc_round(long long n8,
                                                            const float4 *__restrict__ acc,
                                                            uint4 *__restrict__ y) {
  pdl_wait();
  pdl_trigger();
  for (long long i = (long long)blockIdx.x * kCopyThreads + threadIdx.x; i < n8;
       i += (long long)gridDim.x * kCopyThreads) {
    const float4 a = acc[2 * i], b = acc[2 * i + 1];
    y[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                      pack_bf16x2(b.z, b.w));
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
                          cudaStream_t st, const int32_t *offsets) {
  const long long items = (long long)T * slices(h) + (long long)kBlock * E;
  return launch_pdl(k_gather, copy_grid(items), kCopyThreads, 0, st, T, h, k, E,
                    static_cast<const uint4 *>(x), dest_row, counts, padded_bins,
                    static_cast<uint4 *>(x_pad), offsets);
}

// Shape of the combine: work items of one token's 4 KB row slice, 4 row loads in flight per
// lane within 64 registers and four CTAs (32 warps) per SM (measured 13 % faster at top-8 and
// 17 % at top-2 than 8 loads per lane at two CTAs per SM).
static cudaError_t combine(int T, int h, int k, const void *rows, const float *scale,
                           const int32_t *dest_row, const float *weights, void *out,
                           const float *part, int nt, float *dweights, const int32_t *offsets,
                           cudaStream_t st) {
  auto kernel = scale ? k_combine<2, 2, true> : k_combine<2, 2, false>;
  const long long items = (long long)T * slices(h);
  return launch_pdl(kernel, copy_grid(items), kCopyThreads, 0, st, T, h, k,
                    static_cast<const uint4 *>(rows), scale, dest_row, weights,
                    static_cast<uint4 *>(out), part, nt, dweights, offsets);
}

cudaError_t launch_acc_zero(long long n, float *acc, cudaStream_t st) {
  const int grid = copy_grid((n / 8 + 31) / 32);
  return launch_pdl(k_acc_zero, grid, kCopyThreads, 0, st, n / 8, reinterpret_cast<float4 *>(acc));
}

cudaError_t launch_acc_round(long long n, const float *acc, void *y, cudaStream_t st) {
  const int grid = copy_grid((n / 8 + 31) / 32);
  return launch_pdl(k_acc_round, grid, kCopyThreads, 0, st, n / 8,
                    reinterpret_cast<const float4 *>(acc), static_cast<uint4 *>(y));
}

cudaError_t launch_combine(int T, int h, int k, const void *y_pad, const float *y_scale,
                           const int32_t *dest_row, const float *weights, void *y,
                           cudaStream_t st, const int32_t *offsets) {
  return combine(T, h, k, y_pad, y_scale, dest_row, weights, y, nullptr, 0, nullptr, offsets,
                 st);
}

cudaError_t launch_bwd_scatter(int T, int h, int k, const void *dx_pad, const float *dx_scale,
                               const int32_t *dest_row, const float *part, int nt, void *dx,
                               float *dweights, cudaStream_t st, const int32_t *offsets) {
  return combine(T, h, k, dx_pad, dx_scale, dest_row, nullptr, dx, part, nt, dweights, offsets,
                 st);
}

}  // namespace dmoe
