// router.cu -- the element-wise and reduction kernels of the linear router's backward.
//
// The router's output is the (scores, top_experts) pair of the Fast-LLM issue #56 error log
// ("router(x)" in the MegaBlocks walkthrough's schematic forward, section 4.5); the routing
// weight of slot s is w_ts = p_t[j_s], p_t = softmax over all E logits, without
// renormalisation.  Its gradient flows back through that softmax:
//   dlogits[t][i] = sum_s dw_ts * p_t[j_s] * ([i == j_s] - p_t[i]) = p_t[i] * (g_ti - c_t),
//   g_ti = dw_ts if expert i is the pick of slot s (else 0),  c_t = sum_s dw_ts * p_t[j_s].
// With the renormalised routing variant p_t is the softmax over the k chosen logits (zero at
// the other experts), and the same formula applies.
// The router GEMMs themselves (logits, dx += dlogits W_r, dW_r = dlogits^T x) are modes of the
// grouped tcgen05 kernel in gemm.cu; dW_r is split over the token dimension there, and the
// fp32 partials are summed here in split order, so the result is deterministic.
#include "common.cuh"
#include "kernels.h"

namespace dmoe {

constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;

// One warp per token (grid-stride).  Lane l owns the groups of 8 consecutive experts
// g = l + 32 i (i < GPL, E <= 256 * GPL), read and written as 16-byte vectors (E % 8 == 0);
// the next token's row is loaded while the current one is processed.
template <int GPL>
__global__ void __launch_bounds__(kRouterThreads)
    k_router_dlogits(int T, int E, int k, int renorm, const uint16_t *__restrict__ logits,
                     const int32_t *__restrict__ top, const float *__restrict__ dweights,
                     uint16_t *__restrict__ dlogits) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int groups = E >> 3;
  const long long nw = (long long)gridDim.x * kRouterWarps;
  long long t = (long long)blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  uint4 nxt[GPL];
#pragma unroll
  for (int i = 0; i < GPL; ++i)
    nxt[i] = (t < T && lane + 32 * i < groups)
                 ? __ldg(reinterpret_cast<const uint4 *>(logits + (size_t)t * E) + lane + 32 * i)
                 : make_uint4(0u, 0u, 0u, 0u);
  for (; t < T; t += nw) {
    uint4 cur[GPL];
#pragma unroll
    for (int i = 0; i < GPL; ++i) cur[i] = nxt[i];
    const int jl = (lane < k) ? __ldg(top + (size_t)t * k + lane) : -1;
    const float dl = (lane < k) ? __ldg(dweights + (size_t)t * k + lane) : 0.0f;
    const long long tn = t + nw;  // the next token of this warp
#pragma unroll
    for (int i = 0; i < GPL; ++i)
      nxt[i] = (tn < T && lane + 32 * i < groups)
                   ? __ldg(reinterpret_cast<const uint4 *>(logits + (size_t)tn * E) + lane + 32 * i)
                   : make_uint4(0u, 0u, 0u, 0u);
    float g[GPL][8];   // dweights scattered to the chosen experts
    bool sel[GPL][8];  // chosen experts
#pragma unroll
    for (int i = 0; i < GPL; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        g[i][j] = 0.0f;
        sel[i][j] = false;
      }
    for (int s = 0; s < k; ++s) {
      const int e = __shfl_sync(0xFFFFFFFFu, jl, s);
      const float d = __shfl_sync(0xFFFFFFFFu, dl, s);
#pragma unroll
      for (int i = 0; i < GPL; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const bool hit = (e == 8 * (lane + 32 * i) + j);
          g[i][j] += hit ? d : 0.0f;
          sel[i][j] |= hit;
        }
    }
    float p[GPL][8];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < GPL; ++i) {
      const uint32_t *q = reinterpret_cast<const uint32_t *>(&cur[i]);
      const bool live = lane + 32 * i < groups;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        p[i][2 * j] = live ? bf16_lo(q[j]) : -INFINITY;
        p[i][2 * j + 1] = live ? bf16_hi(q[j]) : -INFINITY;
        m = fmaxf(m, fmaxf(p[i][2 * j], p[i][2 * j + 1]));
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < GPL; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool in = (lane + 32 * i < groups) && (!renorm || sel[i][j]);
        p[i][j] = in ? __expf(p[i][j] - m) : 0.0f;
        z += p[i][j];
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, off);
    const float rz = 1.0f / z;
#pragma unroll
    for (int i = 0; i < GPL; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) p[i][j] *= rz;
    float c = 0.0f;  // sum_s dw_ts p_t[j_s]
#pragma unroll
    for (int i = 0; i < GPL; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) c += g[i][j] * p[i][j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, off);
    uint4 *out = reinterpret_cast<uint4 *>(dlogits + (size_t)t * E);
#pragma unroll
    for (int i = 0; i < GPL; ++i) {
      const int gi = lane + 32 * i;
      if (gi < groups) {
        uint4 o;
        o.x = pack_bf16x2(p[i][0] * (g[i][0] - c), p[i][1] * (g[i][1] - c));
        o.y = pack_bf16x2(p[i][2] * (g[i][2] - c), p[i][3] * (g[i][3] - c));
        o.z = pack_bf16x2(p[i][4] * (g[i][4] - c), p[i][5] * (g[i][5] - c));
        o.w = pack_bf16x2(p[i][6] * (g[i][6] - c), p[i][7] * (g[i][7] - c));
        out[gi] = o;
      }
    }
  }
}

// dW_r[e][c] = sum over splits s (in order) of partials[(s * Ep + e) * h + c]; 4 columns per
// thread, grid-stride.
__global__ void __launch_bounds__(kRouterThreads)
    k_router_wgrad_reduce(int h, int E, int Ep, int splits, const float4 *__restrict__ partials,
                          float4 *__restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int hv = h >> 2;
  const long long n = (long long)E * hv;
  const size_t slab = (size_t)Ep * hv;
  for (long long i = (long long)blockIdx.x * kRouterThreads + threadIdx.x; i < n;
       i += (long long)gridDim.x * kRouterThreads) {
    float4 a = __ldg(partials + i);
    for (int s = 1; s < splits; ++s) {
      const float4 b = __ldg(partials + (size_t)s * slab + i);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    out[i] = a;
  }
}

static int grid_for(long long items, long long per_cta) {
  long long g = (items + per_cta - 1) / per_cta;
  const long long cap = (long long)device_sm_count() * 8;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_router_dlogits(int T, int E, int k, bool renorm, const uint16_t *logits,
                                  const int32_t *top, const float *dweights, uint16_t *dlogits,
                                  cudaStream_t st) {
  const int grid = grid_for(T, kRouterWarps);
  auto kernel = (E <= 256) ? k_router_dlogits<1> : (E <= 512) ? k_router_dlogits<2>
                                                              : k_router_dlogits<4>;
  return launch_pdl(kernel, grid, kRouterThreads, 0, st, T, E, k, renorm ? 1 : 0, logits, top,
                    dweights, dlogits);
}

cudaError_t launch_router_wgrad_reduce(int h, int E, int splits, const float *partials,
                                       float *dw_router, cudaStream_t st) {
  const int Ep = (E + kBlock - 1) / kBlock * kBlock;
  const long long n = (long long)E * (h >> 2);
  return launch_pdl(k_router_wgrad_reduce, grid_for(n, kRouterThreads), kRouterThreads, 0, st, h,
                    E, Ep, splits, reinterpret_cast<const float4 *>(partials),
                    reinterpret_cast<float4 *>(dw_router));
}

}  // namespace dmoe
