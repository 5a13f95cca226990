// gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The walkthrough ("02 · dropless MoE 与 block-sparse 重构", sections 2-3) views the expert
// FFN as a block-sparse product in which 128-row block i of the padded activations only
// meets the ffn/128 column blocks of its own expert.  Here that non-zero set is enumerated
// directly: a tile is (row block b, output column tile n) and its B operand is the weight
// slab of expert block_expert[b].  The tile list is read on the device from num_blocks, so no
// host synchronisation is needed and no tile past the real padded size is ever issued.  The
// backward's weight gradients (section 4.2's role swap, section 4.3's transposed topology)
// are a tile per (expert, output tile) whose K loop walks that expert's row blocks.
//
// Kernel structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile (128 x 64 bf16) and B tile (256 x 64 bf16) per stage,
//               4-stage ring, 128-byte swizzle, completion on an mbarrier (expect-tx).
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma (M=128, N=256,
//               K=16; bf16 in, fp32 accumulate) and tcgen05.commit to release smem stages and
//               to hand a finished accumulator to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp its 32-lane TMEM
//               sub-partition), fused element-wise work, bf16 stores.
// Two accumulators (2 x 256 columns) let the epilogue of tile i overlap the MMAs of i+1.
//
// Modes (operand majors: K = K-major, MN = M/N-major; weights are (out, in) = [E, f, h] for
// W1/W3 and [E, h, f] for W2):
//   GLU   A = X_pad (K)      B = [W1_e ; W3_e] rows of 128 f-columns each (K)
//         out H = bf16(silu(gate) * up); optionally bf16(gate), bf16(up) for the backward
//   DOWN  A = H (K)          B = W2_e (K)                 out Y_pad
//   DGLU  A = dY_pad (K)     B = W2_e^T (MN)              dH; epilogue recomputes the
//         activation from the saved A, Bm: dA = dH*Bm*s*(1+A(1-s)), dBm = dH*A*s, s = sigmoid(A)
//   DX    A = dA then dBm (K), B = W1_e then W3_e (MN), one accumulator over both K passes
//   WGRAD per expert e and output tile: dW1_e = dA^T X_pad, dW3_e = dBm^T X_pad,
//         dW2_e = dY^T H, K = the expert's padded rows (both operands MN-major); fp32
//         outputs; experts without rows get exact zeros.
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dmoe {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int CHUNK_BYTES = 64 * BK * 2;  // one 64 x 64 MN-major box: 8 KB
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;
constexpr int GEMM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr int RASTER_GROUP = 16;  // row blocks per raster group
constexpr size_t GEMM_SMEM = (size_t)STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

enum GemmMode { MODE_GLU = 0, MODE_DOWN = 1, MODE_DGLU = 2, MODE_DX = 3, MODE_WGRAD = 4 };

template <int MODE>
struct ModeTraits {
  static constexpr int a_mn = (MODE == MODE_WGRAD) ? 1 : 0;
  static constexpr int b_mn = (MODE == MODE_DGLU || MODE == MODE_DX || MODE == MODE_WGRAD) ? 1 : 0;
};

struct GemmParams {
  CUtensorMap tm[5];
  const int32_t *num_blocks;
  const int32_t *block_expert;
  const int32_t *padded_bins;
  int E, h, f;
  int n_tiles;  // row-block modes: column tiles per row block
  int k_iters;  // row-block modes: 64-wide K steps per tile
  __nv_bfloat16 *out0, *out1, *out2;
  float *fout0, *fout1, *fout2;  // WGRAD: fp32 dW1, dW3, dW2
  const __nv_bfloat16 *in0, *in1;
  int32_t *status;
};

struct Tile {
  int b, n, e, m, which, row0, kit;
};

// Row-block modes: tile t -> (row block b, column tile n).  Groups of RASTER_GROUP row blocks;
// inside a group the row block varies fastest, so CTAs running together share B tiles.
__device__ __forceinline__ void rowblock_coords(int t, int nb, int n_tiles, int &b, int &n) {
  const int per_group = RASTER_GROUP * n_tiles;
  const int g = t / per_group;
  const int local = t - g * per_group;
  const int gb0 = g * RASTER_GROUP;
  const int gsz = min(RASTER_GROUP, nb - gb0);
  n = local / gsz;
  b = gb0 + (local - n * gsz);
}

// Weight-gradient tiles per expert: dW1 and dW3 are [f, h] (f/128 x ceil(h/256) tiles), dW2 is
// [h, f] (h/128 x ceil(f/256) tiles).
__device__ __forceinline__ int wg_tiles13(const GemmParams &p) {
  return (p.f / BM) * ((p.h + BN - 1) / BN);
}
__device__ __forceinline__ int wg_tiles2(const GemmParams &p) {
  return (p.h / BM) * ((p.f + BN - 1) / BN);
}

template <int MODE>
__device__ __forceinline__ int total_tiles(const GemmParams &p, int nb) {
  if (MODE == MODE_WGRAD) return p.E * (2 * wg_tiles13(p) + wg_tiles2(p));
  return nb * p.n_tiles;
}

template <int MODE>
__device__ __forceinline__ Tile decode(const GemmParams &p, int t, int nb) {
  Tile tl;
  if (MODE == MODE_WGRAD) {
    const int t13 = wg_tiles13(p), t2 = wg_tiles2(p);
    const int tpe = 2 * t13 + t2;
    tl.e = t / tpe;
    int r = t - tl.e * tpe;
    int ncols;
    if (r < 2 * t13) {
      tl.which = r / t13;
      r -= tl.which * t13;
      ncols = (p.h + BN - 1) / BN;
    } else {
      tl.which = 2;
      r -= 2 * t13;
      ncols = (p.f + BN - 1) / BN;
    }
    tl.m = r / ncols;
    tl.n = r - tl.m * ncols;
    const int start = (tl.e > 0) ? p.padded_bins[tl.e - 1] : 0;
    const int end = p.padded_bins[tl.e];
    tl.row0 = start;
    tl.kit = (end - start) / BK;
    tl.b = 0;
  } else {
    rowblock_coords(t, nb, p.n_tiles, tl.b, tl.n);
    tl.e = p.block_expert[tl.b];
    tl.m = 0;
    tl.which = 0;
    tl.row0 = tl.b * BM;
    tl.kit = p.k_iters;
  }
  return tl;
}

// Issue the TMA loads of K step kb of tile tl into stage buffers sa (A) and sb (B).
template <int MODE>
__device__ __forceinline__ void load_stage(const GemmParams &p, const Tile &tl, int kb, uint8_t *sa,
                                           uint8_t *sb, uint64_t *bar) {
  if (MODE == MODE_GLU) {
    const int brow = tl.e * p.f + tl.n * (BN / 2);
    tma_load_2d(sa, &p.tm[0], bar, kb * BK, tl.row0);
    tma_load_2d(sb, &p.tm[1], bar, kb * BK, brow);
    tma_load_2d(sb + B_BYTES / 2, &p.tm[2], bar, kb * BK, brow);
  } else if (MODE == MODE_DOWN) {
    tma_load_2d(sa, &p.tm[0], bar, kb * BK, tl.row0);
    tma_load_2d(sb, &p.tm[1], bar, kb * BK, tl.e * p.h + tl.n * BN);
  } else if (MODE == MODE_DGLU) {
    tma_load_2d(sa, &p.tm[0], bar, kb * BK, tl.row0);
#pragma unroll
    for (int c = 0; c < BN / 64; ++c)
      tma_load_2d(sb + c * CHUNK_BYTES, &p.tm[1], bar, tl.n * BN + c * 64, tl.e * p.h + kb * BK);
  } else if (MODE == MODE_DX) {
    const int kf = p.f / BK;
    const int pass = (kb < kf) ? 0 : 1;
    const int kk = kb - pass * kf;
    tma_load_2d(sa, &p.tm[pass], bar, kk * BK, tl.row0);
#pragma unroll
    for (int c = 0; c < BN / 64; ++c)
      tma_load_2d(sb + c * CHUNK_BYTES, &p.tm[2 + pass], bar, tl.n * BN + c * 64,
                  tl.e * p.f + kk * BK);
  } else {  // MODE_WGRAD
    const int ya = tl.row0 + kb * BK;
    const CUtensorMap *ta = &p.tm[tl.which];             // dA, dBm, dY_pad
    const CUtensorMap *tb = &p.tm[tl.which == 2 ? 4 : 3];  // X_pad, X_pad, H
#pragma unroll
    for (int c = 0; c < BM / 64; ++c) tma_load_2d(sa + c * CHUNK_BYTES, ta, bar, tl.m * BM + c * 64, ya);
#pragma unroll
    for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * CHUNK_BYTES, tb, bar, tl.n * BN + c * 64, ya);
  }
}

__device__ __forceinline__ void store16_bf16(__nv_bfloat16 *dst, const float *v) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  st_global_v4(dst, p[0], p[1], p[2], p[3]);
  st_global_v4(dst + 8, p[4], p[5], p[6], p[7]);
}

__device__ __forceinline__ void store16_f32(float *dst, const float *v) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    st_global_v4(dst + 4 * i, __float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                 __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3]));
}

__device__ __forceinline__ void load16_bf16(const __nv_bfloat16 *src, float *v) {
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
  const uint4 q0 = s[0], q1 = s[1];
  const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_lo(w[i]);
    v[2 * i + 1] = bf16_hi(w[i]);
  }
}

// Epilogue of one tile for the thread that owns accumulator row `r` (TMEM lane).
template <int MODE>
__device__ __forceinline__ void epilogue_tile(const GemmParams &p, const Tile &tl, uint32_t tb,
                                              int r) {
  if (MODE == MODE_GLU) {
    const size_t grow = (size_t)tl.row0 + r;
    const int n0 = tl.n * (BN / 2);
    const size_t off = grow * p.f + n0;
    for (int c = 0; c < BN / 2; c += 16) {
      uint32_t g[16], u[16];
      tmem_ld16(tb + c, g);
      tmem_ld16(tb + BN / 2 + c, u);
      tmem_ld_wait();
      float hv[16], gv[16], uv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        gv[i] = __uint_as_float(g[i]);
        uv[i] = __uint_as_float(u[i]);
        hv[i] = silu_f(gv[i]) * uv[i];
      }
      store16_bf16(p.out0 + off + c, hv);
      if (p.out1) store16_bf16(p.out1 + off + c, gv);
      if (p.out2) store16_bf16(p.out2 + off + c, uv);
    }
  } else if (MODE == MODE_DOWN || MODE == MODE_DX) {
    const size_t grow = (size_t)tl.row0 + r;
    const int n0 = tl.n * BN;
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= p.h) break;  // uniform across the warp
      uint32_t v[16];
      tmem_ld16(tb + c, v);
      tmem_ld_wait();
      float fv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) fv[i] = __uint_as_float(v[i]);
      store16_bf16(p.out0 + grow * p.h + n0 + c, fv);
    }
  } else if (MODE == MODE_DGLU) {
    const size_t grow = (size_t)tl.row0 + r;
    const int n0 = tl.n * BN;
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= p.f) break;
      uint32_t v[16];
      tmem_ld16(tb + c, v);
      const size_t off = grow * p.f + n0 + c;
      float a[16], bm[16], da[16], db[16];
      load16_bf16(p.in0 + off, a);
      load16_bf16(p.in1 + off, bm);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float dh = __uint_as_float(v[i]);
        const float s = 1.0f / (1.0f + __expf(-a[i]));
        da[i] = dh * bm[i] * s * (1.0f + a[i] * (1.0f - s));
        db[i] = dh * a[i] * s;
      }
      store16_bf16(p.out0 + off, da);
      store16_bf16(p.out1 + off, db);
    }
  } else {  // MODE_WGRAD
    const int rows = (tl.which == 2) ? p.h : p.f;
    const int cols = (tl.which == 2) ? p.f : p.h;
    float *base = (tl.which == 0) ? p.fout0 : (tl.which == 1) ? p.fout1 : p.fout2;
    float *dst = base + (size_t)tl.e * rows * cols + (size_t)(tl.m * BM + r) * cols;
    const int n0 = tl.n * BN;
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= cols) break;
      float fv[16];
      if (tl.kit > 0) {
        uint32_t v[16];
        tmem_ld16(tb + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) fv[i] = __uint_as_float(v[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) fv[i] = 0.0f;  // expert without rows: exact zeros
      }
      store16_f32(dst + n0 + c, fv);
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_grouped_gemm(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_u32 = smem_u32(smem_raw);
  uint8_t *tiles = smem_raw + ((1024u - (base_u32 & 1023u)) & 1023u);
  uint64_t *bars = reinterpret_cast<uint64_t *>(tiles + STAGES * STAGE_BYTES);
  uint64_t *full = bars;                     // [STAGES] TMA landed
  uint64_t *empty = bars + STAGES;           // [STAGES] MMAs done reading
  uint64_t *tfull = bars + 2 * STAGES;       // [2] accumulator ready
  uint64_t *tempty = bars + 2 * STAGES + 2;  // [2] accumulator drained
  uint64_t *drain = bars + 2 * STAGES + 4;   // teardown: all MMAs finished
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], EPI_THREADS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
#pragma unroll
    for (int i = 0; i < 5; ++i) prefetch_tmap(&p.tm[i]);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int nb = (MODE == MODE_WGRAD) ? 0 : *p.num_blocks;
  const int total = total_tiles<MODE>(p, nb);

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tl = decode<MODE>(p, t, nb);
      if (MODE != MODE_WGRAD && tl.e < 0) {  // cannot happen with a map from dmoe_sparse_map
        set_status(p.status, DMOE_STATUS_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      bool ok = true;
      for (int kb = 0; kb < tl.kit; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t *sa = tiles + stage * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
        load_stage<MODE>(p, tl, kb, sa, sa + A_BYTES, &full[stage]);
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    // Teardown: every issued copy must have landed before the CTA may exit.
    for (long long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
      mbar_wait_plain(&full[i % STAGES], (uint32_t)((i / STAGES) & 1));
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc =
        idesc_bf16_f32(BM, BN, ModeTraits<MODE>::a_mn, ModeTraits<MODE>::b_mn);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tl = decode<MODE>(p, t, nb);
      if (tl.kit == 0) continue;  // weight gradient of an expert without rows: no MMA
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
      bool ok = true;
      for (int kb = 0; kb < tl.kit; ++kb) {
        if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + stage * STAGE_BYTES);
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = ModeTraits<MODE>::a_mn
                                  ? sdesc_mnmajor_sw128(a_addr + kk * 2048, CHUNK_BYTES)
                                  : sdesc_kmajor_sw128(a_addr + kk * 32);
          const uint64_t bd = ModeTraits<MODE>::b_mn
                                  ? sdesc_mnmajor_sw128(b_addr + kk * 2048, CHUNK_BYTES)
                                  : sdesc_kmajor_sw128(b_addr + kk * 32);
          tc_mma(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      tc_commit(&tfull[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // Teardown: wait until every MMA issued by this thread has completed.
    tc_commit(drain);
    mbar_wait_plain(drain, 0);
  } else if (warp >= 2) {
    // ---------------- epilogue ----------------
    const int sub = warp & 3;  // TMEM sub-partition this warp may read
    const int r = sub * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tl = decode<MODE>(p, t, nb);
      if (tl.kit == 0) {  // no accumulator involved
        epilogue_tile<MODE>(p, tl, 0u, r);
        continue;
      }
      if (!mbar_wait(&tfull[acc], acc_phase, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      epilogue_tile<MODE>(p, tl, tb, r);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---- host side -------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Row-major bf16 matrix [rows, cols] as a 2D tensor; box = box_rows x 64 columns, 128-byte
// swizzle (64 bf16 per box row = exactly one swizzle row).
static bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols,
                      uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64u, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  static int cached = 0;
  if (cached > 0) return cached;
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  cached = n > 0 ? n : 148;
  return cached;
}

template <int MODE>
static cudaError_t launch_gemm(const GemmParams &p, long long max_tiles, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(k_grouped_gemm<MODE>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMM_SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  long long grid = device_sm_count();
  if (max_tiles < grid) grid = max_tiles;
  if (grid < 1) grid = 1;
  k_grouped_gemm<MODE><<<(int)grid, GEMM_THREADS, GEMM_SMEM, st>>>(p);
  return cudaGetLastError();
}

static GemmParams base_params(int h, int f, int E, const int32_t *num_blocks,
                              const int32_t *block_expert, const int32_t *padded_bins,
                              int32_t *status) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.num_blocks = num_blocks;
  p.block_expert = block_expert;
  p.padded_bins = padded_bins;
  p.E = E;
  p.h = h;
  p.f = f;
  p.status = status;
  return p;
}

static inline __nv_bfloat16 *bf(void *q) { return static_cast<__nv_bfloat16 *>(q); }
static inline const __nv_bfloat16 *cbf(const void *q) {
  return static_cast<const __nv_bfloat16 *>(q);
}

cudaError_t launch_glu_gemm(const GemmProblem &g, const void *x_pad, const void *w1,
                            const void *w3, void *h_out, void *a_out, void *b_out,
                            cudaStream_t st) {
  GemmParams p = base_params(g.h, g.f, g.E, g.num_blocks, g.block_expert, g.padded_bins, g.status);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  if (!make_tmap(&p.tm[0], x_pad, P, g.h, BM) || !make_tmap(&p.tm[1], w1, (uint64_t)g.E * g.f, g.h, BN / 2) ||
      !make_tmap(&p.tm[2], w3, (uint64_t)g.E * g.f, g.h, BN / 2))
    return cudaErrorInvalidValue;
  p.tm[3] = p.tm[0];
  p.tm[4] = p.tm[0];
  p.n_tiles = g.f / (BN / 2);
  p.k_iters = g.h / BK;
  p.out0 = bf(h_out);
  p.out1 = bf(a_out);
  p.out2 = bf(b_out);
  return launch_gemm<MODE_GLU>(p, (long long)g.nblk_cap * p.n_tiles, st);
}

cudaError_t launch_down_gemm(const GemmProblem &g, const void *h_in, const void *w2, void *y_pad,
                             cudaStream_t st) {
  GemmParams p = base_params(g.h, g.f, g.E, g.num_blocks, g.block_expert, g.padded_bins, g.status);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  if (!make_tmap(&p.tm[0], h_in, P, g.f, BM) || !make_tmap(&p.tm[1], w2, (uint64_t)g.E * g.h, g.f, BN))
    return cudaErrorInvalidValue;
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.n_tiles = (g.h + BN - 1) / BN;
  p.k_iters = g.f / BK;
  p.out0 = bf(y_pad);
  return launch_gemm<MODE_DOWN>(p, (long long)g.nblk_cap * p.n_tiles, st);
}

cudaError_t launch_dglu_gemm(const GemmProblem &g, const void *dy_pad, const void *w2,
                             const void *a_in, const void *b_in, void *da_out, void *db_out,
                             cudaStream_t st) {
  GemmParams p = base_params(g.h, g.f, g.E, g.num_blocks, g.block_expert, g.padded_bins, g.status);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  if (!make_tmap(&p.tm[0], dy_pad, P, g.h, BM) || !make_tmap(&p.tm[1], w2, (uint64_t)g.E * g.h, g.f, 64))
    return cudaErrorInvalidValue;
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.n_tiles = (g.f + BN - 1) / BN;
  p.k_iters = g.h / BK;
  p.out0 = bf(da_out);
  p.out1 = bf(db_out);
  p.in0 = cbf(a_in);
  p.in1 = cbf(b_in);
  return launch_gemm<MODE_DGLU>(p, (long long)g.nblk_cap * p.n_tiles, st);
}

cudaError_t launch_dx_gemm(const GemmProblem &g, const void *da, const void *db, const void *w1,
                           const void *w3, void *dx_pad, cudaStream_t st) {
  GemmParams p = base_params(g.h, g.f, g.E, g.num_blocks, g.block_expert, g.padded_bins, g.status);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  if (!make_tmap(&p.tm[0], da, P, g.f, BM) || !make_tmap(&p.tm[1], db, P, g.f, BM) ||
      !make_tmap(&p.tm[2], w1, (uint64_t)g.E * g.f, g.h, 64) ||
      !make_tmap(&p.tm[3], w3, (uint64_t)g.E * g.f, g.h, 64))
    return cudaErrorInvalidValue;
  p.tm[4] = p.tm[0];
  p.n_tiles = (g.h + BN - 1) / BN;
  p.k_iters = 2 * (g.f / BK);
  p.out0 = bf(dx_pad);
  return launch_gemm<MODE_DX>(p, (long long)g.nblk_cap * p.n_tiles, st);
}

cudaError_t launch_wgrad_gemm(const GemmProblem &g, const void *x_pad, const void *h_in,
                              const void *dy_pad, const void *da, const void *db, float *dw1,
                              float *dw3, float *dw2, cudaStream_t st) {
  GemmParams p = base_params(g.h, g.f, g.E, g.num_blocks, g.block_expert, g.padded_bins, g.status);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  if (!make_tmap(&p.tm[0], da, P, g.f, 64) || !make_tmap(&p.tm[1], db, P, g.f, 64) ||
      !make_tmap(&p.tm[2], dy_pad, P, g.h, 64) || !make_tmap(&p.tm[3], x_pad, P, g.h, 64) ||
      !make_tmap(&p.tm[4], h_in, P, g.f, 64))
    return cudaErrorInvalidValue;
  p.fout0 = dw1;
  p.fout1 = dw3;
  p.fout2 = dw2;
  const long long t13 = (long long)(g.f / BM) * ((g.h + BN - 1) / BN);
  const long long t2 = (long long)(g.h / BM) * ((g.f + BN - 1) / BN);
  return launch_gemm<MODE_WGRAD>(p, (long long)g.E * (2 * t13 + t2), st);
}

}  // namespace dmoe
