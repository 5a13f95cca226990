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
__global__ void __launch_bounds__(kCopyThreads, 2) k_combine(int T, int h, int k,
                                                          const uint4 *__restrict__ rows,
                                                          const float *__restrict__ scale,
                                                          const int32_t *__restrict__ dest_row,
                                                          const float *__restrict__ weights,
                                                          uint4 *__restrict__ out,
                                                          const float *__restrict__ part, int nt,
                                                          float *__restrict__ dweights,
                                                          const int32_t *__restrict__ offsets) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int vpr = h >> 3;                                      // 16-byte vectors per row
  const int nsc = dmoe_scale_stride(h);  // scales per row (padded to a multiple of 4)
  constexpr int kVecPerScale = DMOE_SCALE_COLS / 8;
  const int S = (vpr + kSliceVecs - 1) / kSliceVecs;  // 4 KB row slices per token
  const long long items = (long long)T * S;
  const long long nw = (long long)gridDim.x * kCopyWarps;
  for (long long it = (long long)blockIdx.x * kCopyWarps + (threadIdx.x >> 5); it < items;
       it += nw) {
    const int t = (int)(it / S);
    const int vs = (int)(it - (long long)t * S) * kSliceVecs;
    const int ve = min(vpr, vs + kSliceVecs);
    long long base;
    int cnt;
    token_entries(offsets, t, k, base, cnt);
    // the token's entries (up to 32 per pass; more only with the rounded routing), loaded
    // once per slice and reused by its row pieces
    for (int c0 = 0; c0 == 0 || c0 < cnt; c0 += 32) {
      const int kk = max(0, min(32, cnt - c0));
      const int d = (lane < kk) ? dest_row[base + c0 + lane] : -1;
      const float wl = (lane < kk && weights) ? weights[base + c0 + lane] : 1.0f;
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
#pragma unroll
          for (int ss = 0; ss < SLOTS; ++ss) {
            const int s = s0 + ss;
            const int r = __shfl_sync(0xFFFFFFFFu, d, s & 31);
            const float ws = __shfl_sync(0xFFFFFFFFu, wl, s & 31);
            if (s < kk && r >= 0) {
#pragma unroll
              for (int u = 0; u < VPL; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < ve) {
                  buf[ss][u] = ld_nc_v4(rows + (size_t)r * vpr + v);
                  cf[ss][u] = F16S ? ws * __ldg(scale + (size_t)r * nsc + v / kVecPerScale) : ws;
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

// The combine with its rows staged in shared memory by bulk copies (the common case: the
// fixed t*k + s layout, k <= 8).  Each warp walks its items -- (token, row slice of W bytes) --
// with two stages: while it sums item i from shared memory, the k bulk copies of item i+1 (its
// rows' slices, and with block floating point their scales) are in flight, so the data in
// flight costs no registers and each warp keeps a whole item ahead.  Same sums as k_combine:
// fp32, slot order, one fused multiply-add per entry, rounded once.
// Shared memory per warp: 2 stages of k * (W + W/64) bytes, then 2 mbarriers.
template <bool F16S>
__global__ void __launch_bounds__(256, 1) k_combine_staged(
    int T, int h, int k, int W, const uint8_t *__restrict__ rows, const float *__restrict__ scale,
    const int32_t *__restrict__ dest_row, const float *__restrict__ weights,
    uint4 *__restrict__ out, const float *__restrict__ part, int nt, float *__restrict__ dweights,
    int32_t *status, long long wait_cycles) {
  extern __shared__ __align__(128) uint8_t smem_st[];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, wpc = blockDim.x >> 5;
  const int row_bytes = h * 2;
  const int sbytes = W / 64;                           // scale bytes of one row slice
  const int stage_bytes = k * (W + sbytes);
  uint8_t *my = smem_st + (size_t)warp * 2 * stage_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem_st + (size_t)wpc * 2 * stage_bytes) + 2 * warp;
  const int S = (row_bytes + W - 1) / W;               // slices per token row
  const int nsc = dmoe_scale_stride(h);
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const long long gw = (long long)blockIdx.x * wpc + warp, nw = (long long)gridDim.x * wpc;
  const long long n_items_total = (long long)T * S;
  // this warp's items: it = gw + i * nw
  auto issue = [&](long long it, int stg, int d) {
    const int t = (int)(it / S), sl = (int)(it - (long long)t * S);
    const int c0 = sl * W;
    const int wb = min(W, row_bytes - c0);             // bytes of this slice (multiple of 256)
    const unsigned live = __ballot_sync(0xFFFFFFFFu, lane < k && d >= 0);
    const uint32_t bar = smem_u32(&bars[stg]);
    uint8_t *st = my + (size_t)stg * stage_bytes;
    // the slice's scales (one per DMOE_SCALE_COLS columns = 256 bytes of row), whole 16-byte
    // pieces: the scale rows are padded to a multiple of 4 and slices start at multiples of 4
    const int sb = F16S ? ((wb / 256 + 3) / 4) * 16 : 0;
    if (lane == 0) mbar_arrive_expect_tx(&bars[stg], (uint32_t)(__popc(live) * (wb + sb)));
    __syncwarp();
    if (lane < k && d >= 0) {
      fence_async_smem();  // this stage's earlier reads come before the copies' writes
      bulk_load(smem_u32(st + lane * W), rows + (size_t)d * row_bytes + c0, (uint32_t)wb, bar);
      if (F16S)
        bulk_load(smem_u32(st + k * W + lane * sbytes), scale + (size_t)d * nsc + c0 / 256,
                  (uint32_t)sb, bar);
    }
  };
  // items of this warp, with each item's dest rows / weights loaded one item ahead
  long long it = gw;
  int d_cur = -1, d_nxt = -1;
  float w_cur = 0.f, w_nxt = 0.f;
  if (it < n_items_total) {
    const int t = (int)(it / S);
    d_cur = (lane < k) ? dest_row[(size_t)t * k + lane] : -1;
    w_cur = (lane < k && weights) ? weights[(size_t)t * k + lane] : 1.0f;
    issue(it, 0, d_cur);
  }
  uint32_t phase0 = 0, phase1 = 0;
  for (int i = 0; it < n_items_total; ++i, it += nw) {
    const int stg = i & 1;
    const long long nx = it + nw;
    if (nx < n_items_total) {  // the next item: its rows (the token's or the next token's)
      const int t = (int)(nx / S), tc = (int)(it / S);
      if (t != tc) {
        d_nxt = (lane < k) ? dest_row[(size_t)t * k + lane] : -1;
        w_nxt = (lane < k && weights) ? weights[(size_t)t * k + lane] : 1.0f;
      } else {
        d_nxt = d_cur;
        w_nxt = w_cur;
      }
      issue(nx, stg ^ 1, d_nxt);
    }
    const int t = (int)(it / S), sl = (int)(it - (long long)t * S);
    const int c0 = sl * W;
    const int wb = min(W, row_bytes - c0);
    if (dweights && sl == 0 && lane < k) {
      float g = 0.0f;
      if (d_cur >= 0)
        for (int n = 0; n < nt; ++n) g += __ldg(part + (size_t)d_cur * nt + n);
      dweights[(size_t)t * k + lane] = g;  // 0 for an entry dropped from the map
    }
    int ok = 1;
    if (lane == 0) {
      volatile int no_abort = 0;  // the warps of this kernel wait on their own copies only
      ok = mbar_wait(&bars[stg], stg ? phase1 : phase0, status, &no_abort, wait_cycles) ? 1 : 0;
    }
    if (stg) phase1 ^= 1u; else phase0 ^= 1u;
    if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;  // a copy never landed: status says TIMEOUT
    const uint8_t *st = my + (size_t)stg * stage_bytes;
    for (int v = lane; v < wb / 16; v += 32) {
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
      for (int s = 0; s < k; ++s) {
        const int ds = __shfl_sync(0xFFFFFFFFu, d_cur, s);
        const float ws = __shfl_sync(0xFFFFFFFFu, w_cur, s);
        if (ds < 0) continue;
        const uint4 qv = *reinterpret_cast<const uint4 *>(st + s * W + v * 16);
        float c = ws;
        if (F16S) c *= reinterpret_cast<const float *>(st + k * W + s * sbytes)[v / 16];
        const uint32_t *qq = reinterpret_cast<const uint32_t *>(&qv);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float lo = F16S ? f16_lo(qq[p]) : bf16_lo(qq[p]);
          const float hi = F16S ? f16_hi(qq[p]) : bf16_hi(qq[p]);
          acc[2 * p] = fmaf(c, lo, acc[2 * p]);
          acc[2 * p + 1] = fmaf(c, hi, acc[2 * p + 1]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      out[((size_t)t * row_bytes + c0) / 16 + v] = o;
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
    d_cur = d_nxt;
    w_cur = w_nxt;
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

// Shape of the combine: work items of one token's 4 KB row slice; 8 row loads in flight per
// lane within 128 registers (two CTAs per SM); few entries take wide row pieces.
static cudaError_t combine(int T, int h, int k, const void *rows, const float *scale,
                           const int32_t *dest_row, const float *weights, void *out,
                           const float *part, int nt, float *dweights, const int32_t *offsets,
                           int32_t *status, cudaStream_t st) {
  if (!offsets && k <= 8) {  // rows staged in shared memory by bulk copies
    const int row_bytes = h * 2;
    int W = ((32768 / k) / 1024) * 1024;                  // a stage holds <= 32 KB of rows
    W = min(W, (row_bytes + 1023) / 1024 * 1024);
    const int stage = k * (W + W / 64);
    const int wpc = max(1, min(8, (96 * 1024) / stage));  // warps per CTA
    const size_t smem = (size_t)wpc * 2 * stage + (size_t)wpc * 2 * sizeof(uint64_t);
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
      attr = cudaFuncSetAttribute(k_combine_staged<true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
      if (attr == cudaSuccess)
        attr = cudaFuncSetAttribute(k_combine_staged<false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    });
    if (attr != cudaSuccess) return attr;
    const int per_sm = max(1, (int)((227 * 1024) / smem));
    const long long items = (long long)T * ((row_bytes + W - 1) / W);
    long long grid = (long long)device_sm_count() * per_sm;
    grid = min(grid, (items + wpc - 1) / wpc);
    auto kernel = scale ? k_combine_staged<true> : k_combine_staged<false>;
    return launch_pdl(kernel, (int)max(grid, 1LL), 32 * wpc, smem, st, T, h, k, W,
                      static_cast<const uint8_t *>(rows), scale, dest_row, weights,
                      static_cast<uint4 *>(out), part, nt, dweights, status, kWaitCycles);
  }
  auto kernel = scale ? ((k <= 2) ? k_combine<4, 2, true> : k_combine<2, 4, true>)
                      : ((k <= 2) ? k_combine<4, 2, false> : k_combine<2, 4, false>);
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
                           int32_t *status, cudaStream_t st, const int32_t *offsets) {
  return combine(T, h, k, y_pad, y_scale, dest_row, weights, y, nullptr, 0, nullptr, offsets,
                 status, st);
}

cudaError_t launch_bwd_scatter(int T, int h, int k, const void *dx_pad, const float *dx_scale,
                               const int32_t *dest_row, const float *part, int nt, void *dx,
                               float *dweights, int32_t *status, cudaStream_t st,
                               const int32_t *offsets) {
  return combine(T, h, k, dx_pad, dx_scale, dest_row, nullptr, dx, part, nt, dweights, offsets,
                 status, st);
}

}  // namespace dmoe
