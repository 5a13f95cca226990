// gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The walkthrough ("02 · dropless MoE 与 block-sparse 重构", sections 2-3) views the expert
// FFN as a block-sparse product in which 128-row block i of the padded activations only
// meets the ffn/128 column blocks of its own expert.  Here that non-zero set is enumerated
// directly: a tile is (row block b, output column tile n); its B operand is the weight slab
// of expert block_expert[b].  The tile list is read on the device from num_blocks, so no
// host synchronisation is needed and no tile past the real padded size is ever issued.
//
// Kernel structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile (128 x 64 bf16) and B tile (256 x 64 bf16) per stage,
//               4-stage ring, 128-byte swizzle, completion on an mbarrier (expect-tx).
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma (M=128, N=256,
//               K=16; bf16 in, fp32 accumulate) and tcgen05.commit to release smem stages
//               and to hand a finished accumulator to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp its 32-lane TMEM
//               sub-partition), fused activation, bf16 stores.
// Two accumulators (2 x 256 columns) let the epilogue of tile i overlap the MMAs of i+1.
//
// Modes
//   GLU:  B = [W1_e rows n*128 .. +128 ; W3_e rows n*128 .. +128] stacked, so one N=256 MMA
//         yields the gate (columns 0-127) and the up projection (128-255) of the same f
//         columns; epilogue H = bf16(silu(gate) * up), optionally bf16(gate), bf16(up).
//   DOWN: B = W2_e rows n*256 .. +256; epilogue Y = bf16(acc), columns >= hidden skipped.
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
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;
constexpr int GEMM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr int RASTER_GROUP = 16;  // row blocks per raster group
constexpr size_t GEMM_SMEM = (size_t)STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

enum GemmMode { MODE_GLU = 0, MODE_DOWN = 1 };

struct GemmArgs {
  const int32_t *num_blocks;
  const int32_t *block_expert;
  int n_tiles;  // column tiles per row block
  int k_iters;  // K / 64
  int b_rows;   // rows per expert in the B matrix view (ffn for GLU, hidden for DOWN)
  int ld_out;   // output row stride in elements
  int n_valid;  // valid output columns
  __nv_bfloat16 *out;
  __nv_bfloat16 *out_a;
  __nv_bfloat16 *out_b;
  int32_t *status;
};

// Tile t -> (row block b, column tile n).  Groups of RASTER_GROUP row blocks; inside a group
// the row block varies fastest, so CTAs running at the same time share B tiles and the
// group's A tiles stay in L2.
__device__ __forceinline__ void tile_coords(int t, int nb, int n_tiles, int &b, int &n) {
  const int per_group = RASTER_GROUP * n_tiles;
  const int g = t / per_group;
  const int local = t - g * per_group;
  const int gb0 = g * RASTER_GROUP;
  const int gsz = min(RASTER_GROUP, nb - gb0);
  n = local / gsz;
  b = gb0 + (local - n * gsz);
}

template <int MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_u32 = smem_u32(smem_raw);
  uint8_t *tiles = smem_raw + ((1024u - (base_u32 & 1023u)) & 1023u);
  uint64_t *bars = reinterpret_cast<uint64_t *>(tiles + STAGES * STAGE_BYTES);
  uint64_t *full = bars;                 // [STAGES] TMA landed
  uint64_t *empty = bars + STAGES;       // [STAGES] MMAs done reading
  uint64_t *tfull = bars + 2 * STAGES;   // [2] accumulator ready
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
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    if (MODE == MODE_GLU) prefetch_tmap(&tmB1);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int nb = *args.num_blocks;
  const int total = nb * args.n_tiles;
  const int k_iters = args.k_iters;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      int b, n;
      tile_coords(t, nb, args.n_tiles, b, n);
      const int e = args.block_expert[b];
      if (e < 0) {
        set_status(args.status, DMOE_STATUS_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      const int brow = e * args.b_rows + n * (MODE == MODE_GLU ? BN / 2 : BN);
      bool ok = true;
      for (int kb = 0; kb < k_iters; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, args.status, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t *sa = tiles + stage * STAGE_BYTES;
        uint8_t *sb = sa + A_BYTES;
        mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
        tma_load_2d(sa, &tmA, &full[stage], kb * BK, b * BM);
        if (MODE == MODE_GLU) {
          tma_load_2d(sb, &tmB0, &full[stage], kb * BK, brow);
          tma_load_2d(sb + B_BYTES / 2, &tmB1, &full[stage], kb * BK, brow);
        } else {
          tma_load_2d(sb, &tmB0, &full[stage], kb * BK, brow);
        }
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
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, args.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
      bool ok = true;
      for (int kb = 0; kb < k_iters; ++kb) {
        if (!mbar_wait(&full[stage], phase, args.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + stage * STAGE_BYTES);
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          tc_mma(d_tmem, sdesc_kmajor_sw128(a_addr + kk * 32), sdesc_kmajor_sw128(b_addr + kk * 32),
                 idesc, (kb | kk) != 0 ? 1u : 0u);
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
    const int row_in_tile = sub * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      int b, n;
      tile_coords(t, nb, args.n_tiles, b, n);
      if (!mbar_wait(&tfull[acc], acc_phase, args.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      const size_t grow = (size_t)b * BM + row_in_tile;
      if (MODE == MODE_GLU) {
        const int n0 = n * (BN / 2);
        __nv_bfloat16 *hrow = args.out + grow * args.ld_out + n0;
        for (int c = 0; c < BN / 2; c += 16) {
          uint32_t g[16], u[16];
          tmem_ld16(tb + c, g);
          tmem_ld16(tb + BN / 2 + c, u);
          tmem_ld_wait();
          uint32_t hp[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            hp[i] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
          }
          st_global_v4(hrow + c, hp[0], hp[1], hp[2], hp[3]);
          st_global_v4(hrow + c + 8, hp[4], hp[5], hp[6], hp[7]);
          if (args.out_a) {
            __nv_bfloat16 *arow = args.out_a + grow * args.ld_out + n0 + c;
            uint32_t p[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              p[i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
            st_global_v4(arow, p[0], p[1], p[2], p[3]);
            st_global_v4(arow + 8, p[4], p[5], p[6], p[7]);
          }
          if (args.out_b) {
            __nv_bfloat16 *brw = args.out_b + grow * args.ld_out + n0 + c;
            uint32_t p[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              p[i] = pack_bf16x2(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
            st_global_v4(brw, p[0], p[1], p[2], p[3]);
            st_global_v4(brw + 8, p[4], p[5], p[6], p[7]);
          }
        }
      } else {
        const int n0 = n * BN;
        __nv_bfloat16 *yrow = args.out + grow * args.ld_out + n0;
        for (int c = 0; c < BN; c += 16) {
          if (n0 + c >= args.n_valid) break;  // uniform across the warp
          uint32_t v[16];
          tmem_ld16(tb + c, v);
          tmem_ld_wait();
          uint32_t p[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            p[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          st_global_v4(yrow + c, p[0], p[1], p[2], p[3]);
          st_global_v4(yrow + c + 8, p[4], p[5], p[6], p[7]);
        }
      }
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
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major bf16 matrix [rows, cols] viewed as a 2D tensor; box = box_rows x 64 columns,
// 128-byte swizzle (64 bf16 per row = exactly one swizzle row).
static bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols,
                      uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int MODE>
static cudaError_t launch_gemm(const CUtensorMap &a, const CUtensorMap &b0, const CUtensorMap &b1,
                               const GemmArgs &args, int max_tiles, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(k_grouped_gemm<MODE>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMM_SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  int grid = device_sm_count();
  if (max_tiles < grid) grid = max_tiles;
  if (grid < 1) grid = 1;
  k_grouped_gemm<MODE><<<grid, GEMM_THREADS, GEMM_SMEM, st>>>(a, b0, b1, args);
  return cudaGetLastError();
}

cudaError_t launch_glu_gemm(int h, int f, int E, int nblk_cap, const void *x_pad,
                            const void *w1, const void *w3, const int32_t *num_blocks,
                            const int32_t *block_expert, void *h_out, void *a_out, void *b_out,
                            int32_t *status, cudaStream_t st) {
  CUtensorMap ta, tb0, tb1;
  if (!make_tmap(&ta, x_pad, (uint64_t)nblk_cap * BM, h, BM) ||
      !make_tmap(&tb0, w1, (uint64_t)E * f, h, BN / 2) ||
      !make_tmap(&tb1, w3, (uint64_t)E * f, h, BN / 2))
    return cudaErrorInvalidValue;
  GemmArgs args;
  args.num_blocks = num_blocks;
  args.block_expert = block_expert;
  args.n_tiles = f / (BN / 2);
  args.k_iters = h / BK;
  args.b_rows = f;
  args.ld_out = f;
  args.n_valid = f;
  args.out = static_cast<__nv_bfloat16 *>(h_out);
  args.out_a = static_cast<__nv_bfloat16 *>(a_out);
  args.out_b = static_cast<__nv_bfloat16 *>(b_out);
  args.status = status;
  return launch_gemm<MODE_GLU>(ta, tb0, tb1, args, nblk_cap * args.n_tiles, st);
}

cudaError_t launch_down_gemm(int h, int f, int E, int nblk_cap, const void *h_in,
                             const void *w2, const int32_t *num_blocks,
                             const int32_t *block_expert, void *y_pad, int32_t *status,
                             cudaStream_t st) {
  CUtensorMap ta, tb0;
  if (!make_tmap(&ta, h_in, (uint64_t)nblk_cap * BM, f, BM) ||
      !make_tmap(&tb0, w2, (uint64_t)E * h, f, BN))
    return cudaErrorInvalidValue;
  GemmArgs args;
  args.num_blocks = num_blocks;
  args.block_expert = block_expert;
  args.n_tiles = (h + BN - 1) / BN;
  args.k_iters = f / BK;
  args.b_rows = h;
  args.ld_out = h;
  args.n_valid = h;
  args.out = static_cast<__nv_bfloat16 *>(y_pad);
  args.out_a = nullptr;
  args.out_b = nullptr;
  args.status = status;
  return launch_gemm<MODE_DOWN>(ta, tb0, tb0, args, nblk_cap * args.n_tiles, st);
}

}  // namespace dmoe
