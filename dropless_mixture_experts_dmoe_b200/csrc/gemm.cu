// gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// one SM pair per tile (tcgen05.mma.cta_group::2, M = 256, N = 256).
//
// The walkthrough ("02 · dropless MoE 与 block-sparse 重构", sections 2-3) views the expert
// FFN as a block-sparse product in which 128-row block i of the padded activations only
// meets the ffn/128 column blocks of its own expert.  Here that non-zero set is enumerated
// directly: the unit of work is a pair of consecutive row blocks of one expert (they share the
// expert's weight slab as the B operand) times an output column tile.  The unit list is built
// on the device from padded_bins, so no host synchronisation is needed and no tile past the
// real padded size is ever issued.  The backward's weight gradients (section 4.2's role swap;
// section 4.3's transposed topology) are a tile per (expert, pair of output row tiles, column
// tile) whose K loop walks that expert's padded rows.
//
// Kernel structure (clusters of 2 CTAs on an SM pair, 192 or 320 threads each, persistent,
// tiles taken in snake order: round r of the loop covers tiles [r*n, r*n + n), increasing on
// even rounds and decreasing on odd ones):
//   warp 0      TMA producer (both CTAs): this CTA's 128 rows of A and its half (128 rows)
//               of B per stage, 128-byte swizzle; every load completes on the pair leader's
//               mbarrier (expect-tx of both halves).  GLU, DOWN (ffn > 256) and DX stages hold
//               two 64-deep K slabs (64 KB, three stages), each operand brought by one box of a
//               3D view of its tensor; the other modes use 32 KB one-slab stages (five, four
//               with 8 epilogue warps), MN-major operands again as one 3D box of two 64-column
//               chunks.
//   warp 1      allocates 512 TMEM columns in both CTAs; one thread of the leader issues
//               tcgen05.mma.cta_group::2 (bf16 in, fp32 accumulate), which reads both CTAs'
//               shared memory and writes each CTA's 128 accumulator rows into its own TMEM,
//               and tcgen05.commit (multicast to both CTAs) to free stages and hand over
//               accumulators.  In the weight-gradient mode the peer CTA's warp 1 stores the zero
//               tiles of experts without rows.
//   warps 2..   epilogue (both CTAs; 4 warps, or 8 for a DOWN GEMM with ffn <= 256 and the
//               router's dx GEMM): tcgen05.ld of the accumulator (each warp its 32-lane TMEM
//               sub-partition and, with 8 warps, half of the columns), fused element-wise work,
//               results staged in 128-byte-swizzled shared memory (32 rows x 128 B per box)
//               and written with TMA bulk-tensor stores; one arrival per warp releases the
//               accumulator.
// Two accumulators (2 x 256 columns) let the epilogue of tile i overlap the MMAs of i+1.
// An expert with an odd number of row blocks ends with a unit whose second CTA reads zero
// rows (TMA fill past the last padded row) and stores nothing.
//
// Modes (operand majors: K = K-major, MN = M/N-major; weights are (out, in) = [E, f, h] for
// W1/W3 and [E, h, f] for W2):
//   GLU   A = X_pad (K)      B = W1_e rows (leader) / W3_e rows (peer), 128 f-columns each (K)
//         out H = bf16(silu(gate) * up); optionally bf16(gate), bf16(up) for the backward
//   GLU_GATHER  the same, with A's 128 rows gathered straight from x by the map (TMA
//         tile::gather4, four rows per lane per stage; padding rows read zeros), so the
//         padded copy X_pad is never written or read (the gather of walkthrough section 4.2
//         fused into the GEMM's operand load).  32 gather instructions per 16 KB stage are
//         more than the TMA unit issues in one stage's MMA time: about 3x slower than
//         gather kernel + GLU on B200, so it is not the default path.
//   DOWN  A = H (K)          B = W2_e (K)                 out Y_pad (block floating point:
//         fp16 values and a power-of-two scale per row and 128 columns)
//   DGLU  A = dY_pad (K)     B = W2_e^T (MN)              G = dy W2_e (dY_pad holds the
//         token rows of dy, unweighted); the epilogue recomputes the activation from the saved
//         A, Bm (s = sigmoid(A), h = A*s*Bm) and, with w the routing weight of the row, writes
//         dA = w*G*Bm*s*(1+A(1-s)), dBm = w*G*A*s, Hw = w*h (the dW2 operand) and the partial
//         routing-weight gradient sum_cols G*h of the row over the tile's columns
//   DX    A = dA then dBm (K), B = W1_e then W3_e (MN), one accumulator over both K passes;
//         out dX_pad, block floating point as Y_pad (the k rows of a token are summed
//         afterwards; rounding each of them to bf16 first would put k bf16 roundings into every
//         output element)
//   WGRAD dW1_e = dA^T X_pad, dW3_e = dBm^T X_pad, dW2_e = dY_pad^T Hw over the expert's
//         padded rows (both operands MN-major); fp32 outputs; experts without rows get exact
//         zeros.
// and the dense GEMMs of the linear router (its output is the (scores, top_experts) pair of
// the issue's error log; "router(x)" of walkthrough section 4.5), over T unpadded token rows:
//   ROUTER  A = x (K)        B = W_r (K)                  out logits [T, E]
//   RDX     A = dlogits (K)  B = W_r (MN)                 dx += dlogits W_r (read-add-store)
//   RWGRAD  A = dlogits (MN) B = x (MN), K = tokens       fp32 partial dW_r per K split
//
// Every mbarrier wait is bounded; on expiry the kernel sets DMOE_STATUS_TIMEOUT, raises an
// abort flag for the other roles of its CTA, drains what it issued and returns.
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dmoe {

constexpr int BM = 128;  // rows of A per CTA (= one padded row block)
constexpr int BN = 256;  // output columns per tile
constexpr int BK = 64;   // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int A_BYTES = BM * BK * 2;        // 16 KB: this CTA's 128 rows of A
constexpr int B_BYTES = (BN / 2) * BK * 2;  // 16 KB: this CTA's half of B
constexpr int CHUNK_BYTES = 64 * BK * 2;    // one 64 x 64 MN-major box: 8 KB
constexpr int TMEM_COLS = 512;
constexpr int BOX_BYTES = 32 * 128;  // one result box: 32 rows x 128 B

enum GemmMode {
  MODE_GLU = 0,
  MODE_DOWN = 1,
  MODE_DGLU = 2,
  MODE_DX = 3,
  MODE_WGRAD = 4,
  MODE_GLU_GATHER = 5,  // GLU whose A rows are gathered from the token rows of x
  MODE_ROUTER = 6,      // router logits
  MODE_RDX = 7,         // router input gradient, accumulated into dx
  MODE_RWGRAD = 8,      // router weight gradient, split over the token dimension
  MODE_DOWN_RED = 9     // down GEMM with the weighted combine in its epilogue
};

__host__ __device__ constexpr bool is_glu(int mode) {
  return mode == MODE_GLU || mode == MODE_GLU_GATHER;
}

// 64-deep K slabs per pipeline stage: two (operands as 3D TMA boxes, one instruction per
// operand and stage, a 3-deep ring of 64 KB stages and one staging buffer per epilogue warp)
// for the GEMMs with 4 epilogue warps and few result boxes per tile; one for the others.
// Measured: two slabs speed up GLU, DOWN and DX, and slow DGLU (12 result boxes per tile
// through one staging buffer) and the weight gradients.
__host__ __device__ constexpr int mode_kslabs(int mode, int epi) {
  return (epi == 4 && (mode == MODE_GLU || mode == MODE_DOWN || mode == MODE_DOWN_RED ||
                       mode == MODE_DX))
             ? 2
             : 1;
}

// Modes whose tiles are (pair of an expert's row blocks, column tile), enumerated from
// padded_bins; the others are the weight gradients and the dense router GEMMs.
__host__ __device__ constexpr bool uses_units(int mode) {
  return mode == MODE_GLU || mode == MODE_GLU_GATHER || mode == MODE_DOWN ||
         mode == MODE_DOWN_RED || mode == MODE_DGLU || mode == MODE_DX;
}

// Unit modes whose last unit of an expert with an odd block count runs as one block on the
// pair (M = 128 paired MMA, 64 rows from each CTA) instead of a block and an empty half.
__host__ __device__ constexpr bool half_units(int mode) {
  return mode == MODE_GLU || mode == MODE_DOWN || mode == MODE_DX || mode == MODE_DGLU;
}

// Dense row modes: tiles are (pair of 128-row blocks of the T token rows, column tile).
__host__ __device__ constexpr bool is_dense_rows(int mode) {
  return mode == MODE_ROUTER || mode == MODE_RDX;
}

// Per-launch configuration.  4 epilogue warps (one per TMEM sub-partition) by default, or 8
// (two per sub-partition, each taking half of the tile's columns) for GEMMs whose K is so short
// (a few K steps per tile) that the epilogue, not the MMA, bounds a tile.  The ring of 32 KB
// stages is as deep as shared memory allows next to the result staging: for the forward GEMMs
// (few result boxes per tile) 3 stages of two K slabs (64 KB) and one 4 KB staging buffer per
// warp; for the weight gradients, whose operand loads are the bound, 6 stages of one slab and
// one staging buffer (measured 2-6 % faster than 5 and two); else 5 stages (4 with 8 warps)
// and two staging buffers.
template <int MODE, int EPI>
struct Cfg {
  static constexpr int a_mn = (MODE == MODE_WGRAD || MODE == MODE_RWGRAD) ? 1 : 0;
  static constexpr int b_mn = (MODE == MODE_DGLU || MODE == MODE_DX || MODE == MODE_WGRAD ||
                               MODE == MODE_RDX || MODE == MODE_RWGRAD)
                                  ? 1
                                  : 0;
  static constexpr int epi_warps = EPI;
  static constexpr int col_split = epi_warps / 4;  // warps per TMEM sub-partition
  static constexpr int threads = 64 + 32 * epi_warps;
  // K slabs (64 deep) per stage: the forward GEMMs with K-major operands load two slabs of
  // each operand with one 3D box, halving the TMA instructions per byte.
  static constexpr int kslabs = mode_kslabs(MODE, EPI);
  static constexpr int bk = BK * kslabs;  // K per stage
  static constexpr int a_bytes = A_BYTES * kslabs;
  // WGRAD stages hold three operand slabs: two products per K step share the third
  static constexpr int stage_bytes = (MODE == MODE_WGRAD) ? 3 * A_BYTES : (A_BYTES + B_BYTES) * kslabs;
  // (the eight-warp DOWN takes the fifth stage and one staging buffer per warp: measured 8 %
  // faster at ffn 512 than four stages with two buffers)
  static constexpr int stages =
      (kslabs == 2) ? 3 : ((EPI == 8 && MODE != MODE_DOWN) ? 4 : (MODE == MODE_WGRAD ? 4 : 5));
  // accumulator buffers in tensor memory: two of 256 columns (tile i's epilogue overlaps tile
  // i+1's MMAs), or for WGRAD one of 512 columns holding its two products
  static constexpr int nacc = (MODE == MODE_WGRAD) ? 1 : 2;
  static constexpr int acc_stride = TMEM_COLS / nacc;
  static constexpr int out_bufs =
      (kslabs == 2 || MODE == MODE_WGRAD || (MODE == MODE_DOWN && EPI == 8)) ? 1 : 2;
  static constexpr int out_bytes = epi_warps * out_bufs * BOX_BYTES;
  // WGRAD: one zeroed result box, the source of the zero tiles' stores
  static constexpr int zero_bytes = (MODE == MODE_WGRAD) ? BOX_BYTES : 0;
  static constexpr size_t smem = 1024 /*align*/ + (size_t)stages * stage_bytes + out_bytes +
                                 zero_bytes + 256 /*barriers*/ +
                                 sizeof(int) * (DMOE_MAX_EXPERTS + 1);
};

struct GemmParams {
  CUtensorMap tm[5];   // operand tensor maps (loads)
  CUtensorMap tmo[3];  // result tensor maps (stores)
  const int32_t *padded_bins;
  const int32_t *bins;     // GLU_GATHER: real expert boundaries
  const int32_t *indices;  // GLU_GATHER: sorted entry -> flattened (token, slot)
  int T, k;                // GLU_GATHER: tokens, top_k
  int E, h, f;
  int n_tiles;   // row-block modes: column tiles per unit
  int k_iters;   // row-block modes: 64-wide K steps per tile
  int nblk_cap;  // P_max / 128: rows at or past nblk_cap * 128 read as zeros
  int group;     // row-block modes: units per raster chunk
  int outs;      // GLU: bit 0 H, bit 1 A and Bm
  int inject;    // test-only: pair leaders withhold their first stage (waits then expire)
  long long wait_cycles;  // budget of every bounded wait of this launch
  const __nv_bfloat16 *in0, *in1;  // DGLU: saved A, Bm
  const float *weights;            // DGLU: routing weight of each flattened entry
  float *part;                     // DGLU: [P_max, ceil(f/128)] partial routing-weight gradients;
                                   // DOWN, DX: [P_max, dmoe_scale_stride(h)] scales of the rows
  int total;                       // router modes: number of pair tiles
  int half_ok;                     // half_units modes: run single-block units with M = 128
  int split_k;                     // RWGRAD: 64-wide K steps per split
  int Ep;                          // RWGRAD: rows of one split's slab (E rounded up to 128)
  int32_t *status;
};

struct Tile {
  int e, n, m, which, row0, kit;
  bool dummy;  // this CTA's half of the unit has no rows: load zeros, store nothing
  bool half;   // a unit of one block (half_units modes): M = 128, this CTA's 64 rows at row0
};

// Pair tile t -> expert, column tile, this CTA's rows.
template <int MODE>
__device__ __forceinline__ Tile decode(const GemmParams &p, int t, const int *ustart,
                                       uint32_t rank) {
  Tile tl;
  tl.which = 0;
  tl.m = 0;
  tl.half = false;
  if (is_dense_rows(MODE)) {
    const int u = t / p.n_tiles;
    tl.n = t - u * p.n_tiles;
    tl.e = 0;
    tl.row0 = (2 * u + (int)rank) * BM;
    tl.dummy = tl.row0 >= p.T;  // past the last token row: loads read zeros, nothing stored
    tl.kit = p.k_iters;
    return tl;
  }
  if (MODE == MODE_RWGRAD) {  // t -> (K split, pair of 128-row tiles of E, column tile)
    const int mt = (p.E + BM - 1) / BM, mpairs = (mt + 1) / 2;
    const int per_split = mpairs * p.n_tiles;
    const int sp = t / per_split;
    const int r = t - sp * per_split;
    const int mp = r / p.n_tiles;
    tl.n = r - mp * p.n_tiles;
    tl.m = 2 * mp + (int)rank;
    tl.dummy = tl.m >= mt;
    tl.e = sp;
    tl.row0 = sp * p.split_k * BK;
    tl.kit = min(p.split_k, p.k_iters - sp * p.split_k);
    return tl;
  }
  if (MODE == MODE_WGRAD) {
    // which 0: the (dW1, dW3) blocks of one (m, n) tile, sharing the X_pad operand;
    // which 2: two 256-column halves of one dW2 row-tile pair, sharing the dY_pad operand
    const int mt13 = p.f / BM, mt2 = p.h / BM;
    const int mp13 = (mt13 + 1) / 2, mp2 = (mt2 + 1) / 2;
    const int nt13 = (p.h + BN - 1) / BN, nt2 = (p.f + 2 * BN - 1) / (2 * BN);
    const int tpe = mp13 * nt13 + mp2 * nt2;
    tl.e = t / tpe;
    int r = t - tl.e * tpe;
    int ncols, mtiles;
    if (r < mp13 * nt13) {
      tl.which = 0;
      ncols = nt13;
      mtiles = mt13;
    } else {
      tl.which = 2;
      r -= mp13 * nt13;
      ncols = nt2;
      mtiles = mt2;
    }
    const int mp = r / ncols;
    tl.n = r - mp * ncols;
    tl.m = 2 * mp + (int)rank;
    tl.dummy = tl.m >= mtiles;  // its A boxes start past the matrix: zeros
    const int start = (tl.e > 0) ? p.padded_bins[tl.e - 1] : 0;
    tl.row0 = start;
    tl.kit = (p.padded_bins[tl.e] - start) / (BK * mode_kslabs(MODE_WGRAD, 4));
    return tl;
  }
  const int vu = t / p.n_tiles;  // units partition the tile list in order
  int lo = 0, hi = p.E - 1;      // the expert whose unit range holds vu
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ustart[mid] <= vu)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int e = lo;
  const int units = ustart[e + 1] - ustart[e];
  const int c0 = ((vu - ustart[e]) / p.group) * p.group;  // raster chunk inside the expert
  const int cs = min(p.group, units - c0);
  const int lt = t - (ustart[e] + c0) * p.n_tiles;
  tl.n = lt / cs;  // the unit varies fastest: concurrent pairs share B
  const int unit = c0 + (lt - tl.n * cs);
  const int first = ((e > 0) ? p.padded_bins[e - 1] : 0) / BM;
  const int end = p.padded_bins[e] / BM;
  const int b0 = first + 2 * unit;  // the unit's first block
  tl.e = e;
  tl.kit = p.k_iters;
  if (half_units(MODE) && p.half_ok && b0 + 1 >= end) {  // one block: 64 rows from each CTA
    tl.half = true;
    tl.dummy = false;
    tl.row0 = b0 * BM + (int)rank * (BM / 2);
    return tl;
  }
  const int b = b0 + (int)rank;
  tl.dummy = b >= end;
  tl.row0 = tl.dummy ? p.nblk_cap * BM : b * BM;  // a dummy half reads rows past P_max: zeros
  return tl;
}

// GLU_GATHER: the token rows (rows of x) behind padded rows row0 + 4*lane .. +3 of this
// CTA's block; padding rows and a dummy half get T, past the last row of x: TMA reads zeros.
__device__ __forceinline__ void gather_rows(const GemmParams &p, const Tile &tl, int lane,
                                            int (&rows)[4]) {
  const int e = tl.e;
  const int pstart = (e > 0) ? p.padded_bins[e - 1] : 0;
  const int bstart = (e > 0) ? p.bins[e - 1] : 0;
  const int count = p.bins[e] - bstart;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int local = tl.row0 + 4 * lane + i - pstart;  // position inside the expert's rows
    rows[i] = (!tl.dummy && local < count) ? p.indices[bstart + local] / p.k : p.T;
  }
}

// DOWN, DGLU: routing weight of padded row `row` of expert e (0 for a padding row).
__device__ __forceinline__ float row_weight(const GemmParams &p, int e, int row) {
  const int pstart = (e > 0) ? p.padded_bins[e - 1] : 0;
  const int bstart = (e > 0) ? p.bins[e - 1] : 0;
  const int local = row - pstart;
  return (local < p.bins[e] - bstart) ? __ldg(p.weights + __ldg(p.indices + bstart + local))
                                      : 0.0f;
}

// The operand boxes of stage kb (KSLABS slabs of 64 K) of tile tl, this CTA's half of the pair.
template <int MODE, int KSLABS>
__device__ __forceinline__ void load_stage(const GemmParams &p, const Tile &tl, int kb,
                                           uint32_t rank, uint8_t *sa, uint8_t *sb,
                                           uint32_t bar) {
  if (MODE == MODE_GLU) {  // two K slabs per stage: 3D maps {64, rows, K/64}
    static_assert(MODE != MODE_GLU || KSLABS == 2, "GLU stages hold two K slabs");
    tma_load_3d_pair(sa, &p.tm[0], bar, 0, tl.row0, 2 * kb);
    if (tl.half) {
      // a single-block unit (M = 128): this CTA's B half holds 64 f-rows of W1 then the same
      // 64 of W3 in each K slab, so a thread's accumulator row has gate and up side by side;
      // maps 3 and 4 have 64-row boxes of one slab
      const int fr = tl.e * p.f + tl.n * (BN / 2) + (int)rank * (BN / 4);
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        uint8_t *d = sb + s2 * (BN / 2) * 128;
        tma_load_3d_pair(d, &p.tm[3], bar, 0, fr, 2 * kb + s2);
        tma_load_3d_pair(d + (BN / 4) * 128, &p.tm[4], bar, 0, fr, 2 * kb + s2);
      }
    } else {
      tma_load_3d_pair(sb, &p.tm[rank == 0 ? 1 : 2], bar, 0, tl.e * p.f + tl.n * (BN / 2),
                       2 * kb);
    }
  } else if ((MODE == MODE_DOWN || MODE == MODE_DOWN_RED) && KSLABS == 2) {
    tma_load_3d_pair(sa, &p.tm[0], bar, 0, tl.row0, 2 * kb);
    tma_load_3d_pair(sb, &p.tm[1], bar, 0, tl.e * p.h + tl.n * BN + (int)rank * (BN / 2), 2 * kb);
  } else if (MODE == MODE_DOWN || MODE == MODE_DOWN_RED) {
    tma_load_2d_pair(sa, &p.tm[0], bar, kb * BK, tl.row0);
    tma_load_2d_pair(sb, &p.tm[1], bar, kb * BK, tl.e * p.h + tl.n * BN + (int)rank * (BN / 2));
  } else if (MODE == MODE_DGLU) {
    tma_load_2d_pair(sa, &p.tm[0], bar, kb * BK, tl.row0);
    // MN-major B: both 64-column chunks of this CTA's half in one box of the chunked map
    tma_load_3d_pair(sb, &p.tm[1], bar, 0, tl.e * p.h + kb * BK, (tl.n * BN) / 64 + 2 * (int)rank);
  } else if (MODE == MODE_DX) {  // two K slabs per stage
    const int kf = p.f / (2 * BK);
    const int pass = (kb < kf) ? 0 : 1;
    const int kk = kb - pass * kf;
    tma_load_3d_pair(sa, &p.tm[pass], bar, 0, tl.row0, 2 * kk);
    tma_load_3d_pair(sb, &p.tm[2 + pass], bar, 0, tl.e * p.f + kk * 2 * BK,
                     (tl.n * BN) / 64 + 2 * (int)rank);
  } else if (MODE == MODE_ROUTER) {
    tma_load_2d_pair(sa, &p.tm[0], bar, kb * BK, tl.row0);
    tma_load_2d_pair(sb, &p.tm[1], bar, kb * BK, tl.n * BN + (int)rank * (BN / 2));
  } else if (MODE == MODE_RDX) {
    tma_load_2d_pair(sa, &p.tm[0], bar, kb * BK, tl.row0);
#pragma unroll
    for (int c = 0; c < 2; ++c)
      tma_load_2d_pair(sb + c * CHUNK_BYTES, &p.tm[1], bar, tl.n * BN + (2 * (int)rank + c) * 64,
                       kb * BK);
  } else if (MODE == MODE_RWGRAD) {
    const int y = tl.row0 + kb * BK;
#pragma unroll
    for (int c = 0; c < 2; ++c) tma_load_2d_pair(sa + c * CHUNK_BYTES, &p.tm[0], bar, tl.m * BM + c * 64, y);
#pragma unroll
    for (int c = 0; c < 2; ++c)
      tma_load_2d_pair(sb + c * CHUNK_BYTES, &p.tm[1], bar, tl.n * BN + (2 * (int)rank + c) * 64, y);
  } else {  // MODE_WGRAD: three MN-major slabs, each one box of two 64-column chunks
    const int y = tl.row0 + kb * BK;
    if (tl.which == 0) {  // dA, dBm (128 f-rows each), X_pad (this CTA's 128 h-columns)
      tma_load_3d_pair(sa, &p.tm[0], bar, 0, y, (tl.m * BM) / 64);
      tma_load_3d_pair(sa + A_BYTES, &p.tm[1], bar, 0, y, (tl.m * BM) / 64);
      tma_load_3d_pair(sa + 2 * A_BYTES, &p.tm[3], bar, 0, y, (tl.n * BN) / 64 + 2 * (int)rank);
    } else {  // dY_pad (128 h-rows), Hw of the two 256-column halves (this CTA's 128 of each)
      const int c0 = (tl.n * 2 * BN) / 64 + 2 * (int)rank;
      tma_load_3d_pair(sa, &p.tm[2], bar, 0, y, (tl.m * BM) / 64);
      tma_load_3d_pair(sa + A_BYTES, &p.tm[4], bar, 0, y, c0);
      tma_load_3d_pair(sa + 2 * A_BYTES, &p.tm[4], bar, 0, y, c0 + BN / 64);
    }
  }
}

// ---- epilogue ---------------------------------------------------------------------------------

// Per-warp result staging: two 4 KB buffers, each one box of 32 rows x 128 B in the 128-byte
// swizzled layout that a SWIZZLE_128B tensor map expects (16-byte chunk c of row r sits at
// chunk position c ^ (r & 7)).  Lane l writes row l; lane 0 issues the TMA store.
template <int OUT_BUFS>
struct Stager {
  uint32_t bufs;  // shared address of buffer 0 (the others follow)
  int cur;
  int lane;

  __device__ __forceinline__ void emit(const CUtensorMap *map, const uint32_t (&w)[32], int x,
                                       int y) {
    const uint32_t buf = bufs + (uint32_t)(cur * BOX_BYTES);
    if (lane == 0) bulk_wait_read<OUT_BUFS - 1>();  // the store that last used it has read it
    __syncwarp();
    const uint32_t row = buf + (uint32_t)(lane * 128);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      st_shared_v4(row + (uint32_t)((c ^ (lane & 7)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                   w[4 * c + 3]);
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d_u32(map, buf, x, y);
      bulk_commit();
    }
    cur = (cur + 1) % OUT_BUFS;
  }

  // Batched form: write box i of a batch into buffer i (put), then publish the whole batch
  // with one proxy fence and one store per box (flush).  reclaim() first waits until the
  // previous batch's stores have read their buffers.
  __device__ __forceinline__ void reclaim() {
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
  }
  __device__ __forceinline__ void put(int i, const uint32_t (&w)[32]) {
    const uint32_t row = bufs + (uint32_t)(i * BOX_BYTES) + (uint32_t)(lane * 128);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      st_shared_v4(row + (uint32_t)((c ^ (lane & 7)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                   w[4 * c + 3]);
  }
  __device__ __forceinline__ void flush(const CUtensorMap *map, int n, int x0, int dx, int y) {
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      for (int i = 0; i < n; ++i) tma_store_2d_u32(map, bufs + (uint32_t)(i * BOX_BYTES), x0 + i * dx, y);
      bulk_commit();
    }
  }
};

__device__ __forceinline__ void pack_bf16_row(const uint32_t (&lo)[32], const uint32_t (&hi)[32],
                                              uint32_t (&w)[32]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    w[i] = pack_bf16x2(__uint_as_float(lo[2 * i]), __uint_as_float(lo[2 * i + 1]));
    w[16 + i] = pack_bf16x2(__uint_as_float(hi[2 * i]), __uint_as_float(hi[2 * i + 1]));
  }
}

// This warp's share of a tile of DOWN, DX or DGLU: output rows y0 .. y0+31 (one per lane),
// columns n0 .. n0+kw-1, at TMEM column tcol of the accumulator.  A unit of one block
// (M = 128 paired MMA) holds each CTA's 64 rows in lanes 0-63 for columns 0-127 and again in
// lanes 64-127 for columns 128-255, all at TMEM columns 0-127: the warp of sub-partition sub
// owns rows (sub & 1) * 32 and columns (sub >> 1) * 128; with 8 epilogue warps the second
// column half of warps (half = 1) has nothing to do.
struct Share {
  int y0, n0, kw, tcol;
  bool on;
};
template <int MODE, int EPI>
__device__ __forceinline__ Share share_of(const Tile &tl, int sub, int half) {
  constexpr int kw = BN / Cfg<MODE, EPI>::col_split;
  Share s;
  if (half_units(MODE) && tl.half) {
    s.y0 = tl.row0 + (sub & 1) * 32;
    s.n0 = tl.n * BN + (sub >> 1) * (BN / 2);
    s.kw = BN / 2;
    s.tcol = 0;
    s.on = half == 0;
  } else {
    s.y0 = tl.row0 + sub * 32;
    s.n0 = tl.n * BN + half * kw;
    s.kw = kw;
    s.tcol = half * kw;
    s.on = true;
  }
  return s;
}

// Epilogue of one tile for the warp owning TMEM sub-partition `sub` (rows sub*32 .. +31 of
// this CTA's 128 rows); tb = TMEM address of the warp's lanes at accumulator column 0.
// Work of a tile's epilogue that does not depend on the accumulator, done before waiting for
// it: DOWN and DGLU look up the routing weight of this thread's row (a chain of dependent
// loads), and DGLU starts pulling the row's saved A and Bm columns of the tile into L2.
template <int MODE, int EPI>
__device__ __forceinline__ float epilogue_prologue(const GemmParams &p, const Tile &tl, int sub,
                                                   int half, int lane) {
  if (MODE == MODE_RDX && !tl.dummy) {  // the dx values this thread will add to
    constexpr int kw = BN / Cfg<MODE, EPI>::col_split;
    const int grow = tl.row0 + sub * 32 + lane;
    const int n0 = tl.n * BN + half * kw;
    const int ncols = min(kw, p.h - n0);
    if (grow < p.T)
      for (int c = 0; c < ncols; c += 64) prefetch_l2(p.in0 + (size_t)grow * p.h + n0 + c);
    return 0.0f;
  }
  if (MODE == MODE_DOWN && !tl.dummy)  // the row's routing weight, ahead of the accumulator
    return row_weight(p, tl.e, share_of<MODE, EPI>(tl, sub, half).y0 + lane);
  if (MODE != MODE_DGLU || tl.dummy) return 0.0f;
  const Share sh = share_of<MODE, EPI>(tl, sub, half);
  const int grow = sh.y0 + lane;
  const int n0 = sh.n0;
  const int ncols = min(sh.kw, p.f - n0);
  const __nv_bfloat16 *ra = p.in0 + (size_t)grow * p.f + n0;
  const __nv_bfloat16 *rb = p.in1 + (size_t)grow * p.f + n0;
  for (int c = 0; c < ncols; c += 64) {  // one 128-byte line per 64 columns
    prefetch_l2(ra + c);
    prefetch_l2(rb + c);
  }
  return row_weight(p, tl.e, grow);
}

template <int MODE, int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmParams &p, const Tile &tl, uint32_t tb,
                                              int sub, int half, int lane, float wr,
                                              Stager<Cfg<MODE, EPI>::out_bufs> &st) {
  const int y0 = tl.row0 + sub * 32;  // first row of this warp's boxes
  constexpr int kw = BN / Cfg<MODE, EPI>::col_split;  // accumulator columns per warp (non-GLU)
  if (is_glu(MODE)) {
    // gate columns at TMEM 0 .. gw-1, up at gw .. 2gw-1.  A single-block unit (M = 128) holds
    // 64 f-columns per warp: rows (sub & 1) * 32 of this CTA's 64, f-columns (sub >> 1) * 64
    const bool hu = half_units(MODE) && tl.half;
    const int gw = hu ? BN / 4 : BN / 2;
    const int n0 = tl.n * (BN / 2) + (hu ? (sub >> 1) * (BN / 4) : 0);
    const int yg = hu ? tl.row0 + (sub & 1) * 32 : y0;
#pragma unroll 1
    for (int c = 0; c < gw; c += 64) {  // one 64-column box of H (and of A, Bm)
      uint32_t g0[32], g1[32], u0[32], u1[32], w[32];
      tmem_ld32(tb + c, g0);
      tmem_ld32(tb + c + 32, g1);
      tmem_ld32(tb + gw + c, u0);
      tmem_ld32(tb + gw + c + 32, u1);
      tmem_ld_wait();
      if (p.outs & 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          w[i] = pack_bf16x2(silu_f(__uint_as_float(g0[2 * i])) * __uint_as_float(u0[2 * i]),
                             silu_f(__uint_as_float(g0[2 * i + 1])) * __uint_as_float(u0[2 * i + 1]));
          w[16 + i] = pack_bf16x2(silu_f(__uint_as_float(g1[2 * i])) * __uint_as_float(u1[2 * i]),
                                  silu_f(__uint_as_float(g1[2 * i + 1])) * __uint_as_float(u1[2 * i + 1]));
        }
        st.emit(&p.tmo[0], w, n0 + c, yg);
      }
      if (p.outs & 2) {
        pack_bf16_row(g0, g1, w);
        st.emit(&p.tmo[1], w, n0 + c, yg);
        pack_bf16_row(u0, u1, w);
        st.emit(&p.tmo[2], w, n0 + c, yg);
      }
    }
  } else if (MODE == MODE_DOWN || MODE == MODE_DX) {
    // Y_pad / dX_pad in block floating point.  DOWN first weights the row by its routing
    // weight (0 for a padding row), so the combine sums unweighted rows.  Per DMOE_SCALE_COLS
    // columns of this thread's row, the largest magnitude m picks a power-of-two scale that
    // puts it into [2^13, 2^14) -- for m < 2^-11 the scale stops at 2^24 (fp16's range of
    // powers of two), which still leaves the group's largest value a normal fp16 down to
    // m = 2^-38.  The values go out as fp16 (11 significant bits) and 1/scale to
    // p.part[row * nsc + chunk], its sign set when fp16 cannot hold 1/scale (m < 2^-38 or
    // m >= 2^29) or when the group holds an inf or NaN (values unscaled, 1/scale = -1).
    const Share sh = share_of<MODE, EPI>(tl, sub, half);
    if (!sh.on) return;
    const int n0 = sh.n0;                     // this warp's first column
    const int ncols = min(sh.kw, p.h - n0);   // multiple of 64 (may be <= 0)
    if (ncols <= 0) return;
    tb += (uint32_t)sh.tcol;
    const int nsc = dmoe_scale_stride(p.h);
    const int y0 = sh.y0;
    const int grow = y0 + lane;
    const float wrow = (MODE == MODE_DOWN) ? wr : 1.0f;  // DOWN: from epilogue_prologue
    float *srow = p.part + (size_t)grow * nsc;
    // one pass per group: its 128 accumulator columns in registers (the last group of a
    // 64-column remainder reads 64 columns past it, inside this CTA's TMEM allocation, and
    // leaves them out), one wait, then the maximum, the scale and the conversion
    static_assert(DMOE_SCALE_COLS == 128, "four 32-column loads per group");
#pragma unroll 1
    for (int c0 = 0; c0 < ncols; c0 += DMOE_SCALE_COLS) {
      const bool full = ncols - c0 >= DMOE_SCALE_COLS;
      uint32_t v[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(tb + c0 + 32 * j, v[j]);
      tmem_ld_wait();
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (j < 2 || full) m = fmaxf(m, fabsf(__uint_as_float(v[j][i])));
      m *= fabsf(wrow);  // the largest weighted magnitude (rounding is monotone)
      int es = 13 - ((int)((__float_as_uint(m) >> 23) & 0xFFu) - 127);  // m * 2^es < 2^14
      const bool finite = m <= 3.402823466e38f;
      if (m == 0.0f || !finite) es = 0;  // zero, inf or NaN: unscaled
      if (es > 24 && es <= 51) es = 24;  // see above
      es = min(max(es, -126), 126);
      const bool fits = finite && es >= -15 && es <= 24;
      const float sc = __uint_as_float((uint32_t)(127 + es) << 23);
      const float k = wrow * sc;  // weight and scale in one exact product
      srow[(n0 + c0) / DMOE_SCALE_COLS] =
          __uint_as_float(((uint32_t)(127 - es) << 23) | (fits ? 0u : 0x80000000u));
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        if (h2 == 1 && !full) break;
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          w[i] = pack_f16x2(__uint_as_float(v[2 * h2][2 * i]) * k,
                            __uint_as_float(v[2 * h2][2 * i + 1]) * k);
          w[16 + i] = pack_f16x2(__uint_as_float(v[2 * h2 + 1][2 * i]) * k,
                                 __uint_as_float(v[2 * h2 + 1][2 * i + 1]) * k);
        }
        st.emit(&p.tmo[0], w, n0 + c0 + 64 * h2, y0);
      }
    }
  } else if (MODE == MODE_DOWN_RED) {
    // the weighted combine fused in: the row's routing weight times its fp32 accumulator row,
    // added into y_acc [T, h] fp32 at the row's token with vector reductions (no Y_pad)
    const int n0 = tl.n * BN + half * kw;
    const int ncols = min(kw, p.h - n0);  // multiple of 64 (may be <= 0)
    if (ncols <= 0) return;
    const int grow = y0 + lane;
    const int pstart = (tl.e > 0) ? p.padded_bins[tl.e - 1] : 0;
    const int bstart = (tl.e > 0) ? p.bins[tl.e - 1] : 0;
    const int local = grow - pstart;
    int tok = -1;
    float wr = 0.0f;
    if (local < p.bins[tl.e] - bstart) {  // a real row, not padding
      const int j = __ldg(p.indices + bstart + local);
      tok = j / p.k;
      wr = __ldg(p.weights + j);
    }
    tb += (uint32_t)(half * kw);
    float *dst = p.part + (size_t)(tok < 0 ? 0 : tok) * p.h + n0;
#pragma unroll 1
    for (int c = 0; c < ncols; c += 32) {
      uint32_t v[32];
      tmem_ld32(tb + c, v);
      tmem_ld_wait();
      if (tok >= 0) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          red_add_v4(dst + c + 4 * q, wr * __uint_as_float(v[4 * q]),
                     wr * __uint_as_float(v[4 * q + 1]), wr * __uint_as_float(v[4 * q + 2]),
                     wr * __uint_as_float(v[4 * q + 3]));
      }
    }
  } else if (MODE == MODE_DGLU) {
    static_assert(MODE != MODE_DGLU || EPI == 4, "one warp per row holds a row's partial sum");
    const Share sh = share_of<MODE, EPI>(tl, sub, half);
    const int n0 = sh.n0;
    const int yw = sh.y0;         // first row of this warp's boxes
    const int grow = yw + lane;   // this thread's padded row; wr = its routing weight
    tb += (uint32_t)sh.tcol;
    float dot0 = 0.0f, dot1 = 0.0f;  // per 128 columns: the sum of G * h, in column order
#pragma unroll 1
    for (int c = 0; c < sh.kw; c += 64) {
      if (n0 + c >= p.f) break;
      float dot = (c < DMOE_DGLU_TILE_COLS) ? dot0 : dot1;
      uint32_t v0[32], v1[32], wa[32], wb[32], wh[32];
      uint4 qa[8], qb[8];
      tmem_ld32(tb + c, v0);
      tmem_ld32(tb + c + 32, v1);
      const uint4 *sa = reinterpret_cast<const uint4 *>(p.in0 + (size_t)grow * p.f + n0 + c);
      const uint4 *sb = reinterpret_cast<const uint4 *>(p.in1 + (size_t)grow * p.f + n0 + c);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        qa[i] = __ldg(sa + i);
        qb[i] = __ldg(sb + i);
      }
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {  // bf16 pairs 2i, 2i+1 of this 64-column chunk
        const uint32_t aw = reinterpret_cast<const uint32_t *>(qa)[i];
        const uint32_t bw = reinterpret_cast<const uint32_t *>(qb)[i];
        const float g0 = __uint_as_float(i < 16 ? v0[2 * i] : v1[2 * i - 32]);
        const float g1 = __uint_as_float(i < 16 ? v0[2 * i + 1] : v1[2 * i - 31]);
        const float a0 = bf16_lo(aw), a1 = bf16_hi(aw), b0 = bf16_lo(bw), b1 = bf16_hi(bw);
        const float s0 = sigmoid_f(a0), s1 = sigmoid_f(a1);
        const float h0 = a0 * s0 * b0, h1 = a1 * s1 * b1;
        dot = fmaf(g0, h0, dot);
        dot = fmaf(g1, h1, dot);
        const float dh0 = wr * g0, dh1 = wr * g1;
        wa[i] = pack_bf16x2(dh0 * b0 * s0 * (1.0f + a0 * (1.0f - s0)),
                            dh1 * b1 * s1 * (1.0f + a1 * (1.0f - s1)));
        wb[i] = pack_bf16x2(dh0 * a0 * s0, dh1 * a1 * s1);
        wh[i] = pack_bf16x2(wr * h0, wr * h1);
      }
      if (c < DMOE_DGLU_TILE_COLS)
        dot0 = dot;
      else
        dot1 = dot;
      st.emit(&p.tmo[0], wa, n0 + c, yw);
      st.emit(&p.tmo[1], wb, n0 + c, yw);
      st.emit(&p.tmo[2], wh, n0 + c, yw);
    }
    const int pt = (p.f + DMOE_DGLU_TILE_COLS - 1) / DMOE_DGLU_TILE_COLS;  // partials per row
    float *prow = p.part + (size_t)grow * pt + n0 / DMOE_DGLU_TILE_COLS;
    prow[0] = dot0;
    if (DMOE_DGLU_TILE_COLS < sh.kw && n0 + DMOE_DGLU_TILE_COLS < p.f) prow[1] = dot1;
  } else if (MODE == MODE_ROUTER) {  // logits [T, E]: bf16 boxes, rows past T not stored
    if (y0 >= p.T) return;
    const int n0 = tl.n * BN;
    const int ncols = min(BN, p.E - n0);
    uint32_t v0[32], v1[32], w[32];
#pragma unroll 1
    for (int c = 0; c < ncols; c += 64) {
      tmem_ld32(tb + c, v0);
      tmem_ld32(tb + c + 32, v1);
      tmem_ld_wait();
      pack_bf16_row(v0, v1, w);
      st.emit(&p.tmo[0], w, n0 + c, y0);
    }
  } else if (MODE == MODE_RDX) {  // dx [T, h] += accumulator, in fp32, rounded once
    if (y0 >= p.T) return;
    const int n0 = tl.n * BN + half * kw;  // this warp's columns
    const int ncols = min(kw, p.h - n0);   // multiple of 64 (may be <= 0)
    if (ncols <= 0) return;
    tb += (uint32_t)(half * kw);
    const int grow = y0 + lane;
    const bool live = grow < p.T;
#pragma unroll 1
    for (int c = 0; c < ncols; c += 64) {
      uint32_t v0[32], v1[32], w[32];
      uint4 q[8];
      tmem_ld32(tb + c, v0);
      tmem_ld32(tb + c + 32, v1);
      const uint4 *src = reinterpret_cast<const uint4 *>(p.in0 + (size_t)grow * p.h + n0 + c);
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = live ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t ow = reinterpret_cast<const uint32_t *>(q)[i];
        const float a0 = __uint_as_float(i < 16 ? v0[2 * i] : v1[2 * i - 32]);
        const float a1 = __uint_as_float(i < 16 ? v0[2 * i + 1] : v1[2 * i - 31]);
        w[i] = pack_bf16x2(bf16_lo(ow) + a0, bf16_hi(ow) + a1);
      }
      st.emit(&p.tmo[0], w, n0 + c, y0);
    }
  } else if (MODE == MODE_RWGRAD) {  // fp32 partial of split tl.e, slab rows [tl.e * Ep, +Ep)
    const int r0 = tl.m * BM + sub * 32;
    if (r0 >= p.E) return;
    const int yw = tl.e * p.Ep + r0;
    const int n0 = tl.n * BN;
    const int ncols = min(BN, p.h - n0);
    uint32_t v[32], w[32];
    tmem_ld32(tb, v);
    tmem_ld_wait();
#pragma unroll 1
    for (int c = 0; c < ncols; c += 32) {
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = v[i];
      if (c + 32 < ncols) tmem_ld32(tb + c + 32, v);
      st.emit(&p.tmo[0], w, n0 + c, yw);
      tmem_ld_wait();
    }
  } else {  // MODE_WGRAD: two products, fp32 results, boxes of 32 columns
    const int rows = (tl.which == 2) ? p.h : p.f;
    const int cols = (tl.which == 2) ? p.f : p.h;
    const int yw = tl.e * rows + tl.m * BM + sub * 32;
#pragma unroll 1
    for (int q = 0; q < 2; ++q) {  // product q: dW1 / dW3 (which 0), or dW2's half q
      const CUtensorMap *map = &p.tmo[tl.which == 0 ? q : 2];
      const int n0 = (tl.which == 0 ? tl.n * BN : tl.n * 2 * BN + q * BN) + half * kw;
      const int ncols = min(kw, cols - n0);  // multiple of 32 (may be <= 0)
      if (ncols <= 0) continue;
      const uint32_t tq = tb + (uint32_t)(q * BN + half * kw);
      uint32_t v[32], w[32];
      tmem_ld32(tq, v);
      tmem_ld_wait();
#pragma unroll 1
      for (int c = 0; c < ncols; c += 32) {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = v[i];
        if (c + 32 < ncols) tmem_ld32(tq + c + 32, v);  // overlaps the store
        st.emit(map, w, n0 + c, yw);
        tmem_ld_wait();
      }
    }
  }
}

// ---- the kernel -------------------------------------------------------------------------------

// The r-th tile of a cluster in the persistent loop.  Round r covers tiles [r*n, r*n + n); the
// clusters take them in increasing order on even rounds and in decreasing order on odd ones
// (a snake), which evens out the per-cluster sums when tile costs fall along the list (the
// weight-gradient tiles of large experts first, then ever smaller ones).  Every role of both
// CTAs uses the same sequence.
__device__ __forceinline__ int snake_tile(int r, int cluster, int nclusters) {
  return r * nclusters + ((r & 1) ? nclusters - 1 - cluster : cluster);
}

template <int MODE, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<MODE, EPI>::threads, 1)
    k_grouped_gemm(const __grid_constant__ GemmParams p) {
  using C = Cfg<MODE, EPI>;
  constexpr int STAGES = C::stages;
  constexpr int EPI_THREADS = 32 * C::epi_warps;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_u32 = smem_u32(smem_raw);
  uint8_t *tiles = smem_raw + ((1024u - (base_u32 & 1023u)) & 1023u);
  uint8_t *outbuf = tiles + STAGES * C::stage_bytes;  // 1024-aligned
  uint8_t *zbuf = outbuf + C::out_bytes;           // 1024-aligned (WGRAD only)
  uint64_t *bars = reinterpret_cast<uint64_t *>(zbuf + C::zero_bytes);
  uint64_t *full = bars;                       // [STAGES] leader: both halves landed
  uint64_t *empty = bars + STAGES;             // [STAGES] MMAs done reading the stage
  uint64_t *tfull = bars + 2 * STAGES;         // [2] accumulator ready
  uint64_t *tempty = bars + 2 * STAGES + 2;    // [2] leader: accumulator drained (one arrival
                                               //     per epilogue warp of both CTAs)
  uint64_t *drain = bars + 2 * STAGES + 4;     // leader: all MMAs finished
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *ustart = reinterpret_cast<int *>(zbuf + C::zero_bytes + 256);  // [E + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * C::epi_warps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
#pragma unroll
    for (int i = 0; i < 5; ++i) prefetch_tmap(&p.tm[i]);
  }
  // First global access below (the tile schedule).  No explicit pdl_trigger(): the next
  // kernel is released as this grid's CTAs exit, so that it does not sit resident for the
  // whole GEMM (measured: an early trigger cost 1-2 % per step, the exit trigger gains 2-3 %
  // on the short forward steps against no programmatic launch).
  pdl_wait();
  if (uses_units(MODE)) {
    // units (pairs of row blocks) per expert -> exclusive prefix ustart[0..E]
    for (int e = threadIdx.x; e < p.E; e += C::threads) {
      const int blocks = (p.padded_bins[e] - ((e > 0) ? p.padded_bins[e - 1] : 0)) / BM;
      ustart[e + 1] = (blocks + 1) / 2;
    }
    __syncthreads();
    if (warp == 0) {
      int carry = 0;
      for (int base = 0; base < p.E; base += 32) {
        const int e = base + lane;
        int v = (e < p.E) ? ustart[e + 1] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int nv = __shfl_up_sync(0xFFFFFFFFu, v, off);
          if (lane >= off) v += nv;
        }
        if (e < p.E) ustart[e + 1] = carry + v;
        carry += __shfl_sync(0xFFFFFFFFu, v, 31);
      }
      if (lane == 0) ustart[0] = 0;
    }
  }
  if (MODE == MODE_WGRAD) {  // zero box for the stores of experts without rows
    for (int i = threadIdx.x; i < C::zero_bytes / 16; i += C::threads)
      st_shared_v4(smem_u32(zbuf) + (uint32_t)(i * 16), 0u, 0u, 0u, 0u);
    fence_async_smem();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  int total;
  if (!uses_units(MODE) && MODE != MODE_WGRAD) {
    total = p.total;
  } else if (MODE == MODE_WGRAD) {
    const int mp13 = (p.f / BM + 1) / 2, mp2 = (p.h / BM + 1) / 2;
    total = p.E * (mp13 * ((p.h + BN - 1) / BN) + mp2 * ((p.f + 2 * BN - 1) / (2 * BN)));
  } else {
    total = ustart[p.E] * p.n_tiles;
  }
  const uint32_t leader_full0 = mapa_shared(smem_u32(&full[0]), 0);
  const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    // Lane 0 waits for free stages and issues the tile loads; in GLU_GATHER mode every lane
    // also issues one 4-row gather of the A tile (32 x 4 = 128 rows).
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    int rows[4] = {0, 0, 0, 0};
    for (int r = 0, t = snake_tile(0, cluster, nclusters); t < total;
         t = snake_tile(++r, cluster, nclusters)) {
      const Tile tl = decode<MODE>(p, t, ustart, rank);
      if (MODE == MODE_WGRAD && tl.kit == 0) continue;  // zero tile: see the peer's warp 1
      if (MODE == MODE_GLU_GATHER) gather_rows(p, tl, lane, rows);
      bool ok = true;
      for (int kb = 0; kb < tl.kit; ++kb) {
        int good = 1;
        if (lane == 0)
          good = mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag, p.wait_cycles) ? 1 : 0;
        if (!__shfl_sync(0xFFFFFFFFu, good, 0)) {
          ok = false;
          break;
        }
        uint8_t *sa = tiles + stage * C::stage_bytes;
        const uint32_t bar = leader_full0 + (uint32_t)(stage * sizeof(uint64_t));
        if (p.inject && leader && issued == 0 && kb == 0) {
          // test-only stall: this stage is never armed, so the MMA's wait on it expires
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          ++issued;
          continue;
        }
        if (lane == 0 && leader) mbar_arrive_expect_tx(&full[stage], 2 * C::stage_bytes);
        if (MODE == MODE_GLU_GATHER) {
          tma_gather4_pair(sa + lane * 4 * 128, &p.tm[3], bar, kb * BK, rows[0], rows[1], rows[2],
                           rows[3]);
          if (lane == 0)
            tma_load_2d_pair(sa + C::a_bytes, &p.tm[rank == 0 ? 1 : 2], bar, kb * BK,
                             tl.e * p.f + tl.n * (BN / 2));
        } else if (lane == 0) {
          load_stage<MODE, C::kslabs>(p, tl, kb, rank, sa, sa + C::a_bytes, bar);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    if (lane == 0 && leader)  // every issued copy (of both CTAs) has landed before exit
      for (long long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
        mbar_wait_plain(&full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.wait_cycles);
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------- MMA issuer (leader only) ----------------
    constexpr uint32_t idesc =
        idesc_bf16_f32(2 * BM, BN, C::a_mn, C::b_mn);
    constexpr uint32_t idesc_half = idesc_bf16_f32(BM, BN, C::a_mn, C::b_mn);  // M = 128
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int r = 0, t = snake_tile(0, cluster, nclusters); t < total;
         t = snake_tile(++r, cluster, nclusters)) {
      const Tile tl = decode<MODE>(p, t, ustart, rank);
      if (tl.kit == 0) continue;  // weight gradient of an expert without rows: no MMA
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status, abort_flag, p.wait_cycles)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * C::acc_stride);
      bool ok = true;
      for (int kb = 0; kb < tl.kit; ++kb) {
        if (!mbar_wait(&full[stage], phase, p.status, abort_flag, p.wait_cycles)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + stage * C::stage_bytes);
        const uint32_t b_addr = a_addr + C::a_bytes;
        if (MODE == MODE_WGRAD) {  // two products per K step; slabs s0, s1, s2 of the stage
          const bool shared_b = tl.which == 0;  // (dA, dBm) x X_pad, else dY_pad x (Hw, Hw')
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t s0 = sdesc_mnmajor_sw128(a_addr + kk * 2048, CHUNK_BYTES);
            const uint64_t s1 = sdesc_mnmajor_sw128(a_addr + A_BYTES + kk * 2048, CHUNK_BYTES);
            const uint64_t s2 = sdesc_mnmajor_sw128(a_addr + 2 * A_BYTES + kk * 2048, CHUNK_BYTES);
            const uint32_t acc_flag = (kb | kk) != 0 ? 1u : 0u;
            tc_mma_pair(d_tmem, s0, shared_b ? s2 : s1, idesc, acc_flag);
            tc_mma_pair(d_tmem + BN, shared_b ? s1 : s0, s2, idesc, acc_flag);
          }
        } else {
#pragma unroll
        for (int kk = 0; kk < C::bk / 16; ++kk) {
          // K-major: slab kk / 4 (one 128 B swizzle row of 64 K per slab), 32 B per 16 K inside
          const uint64_t ad = C::a_mn
                                  ? sdesc_mnmajor_sw128(a_addr + kk * 2048, CHUNK_BYTES * C::kslabs)
                                  : sdesc_kmajor_sw128(a_addr + (kk >> 2) * A_BYTES + (kk & 3) * 32);
          const uint64_t bd = C::b_mn
                                  ? sdesc_mnmajor_sw128(b_addr + kk * 2048, CHUNK_BYTES * C::kslabs)
                                  : sdesc_kmajor_sw128(b_addr + (kk >> 2) * B_BYTES + (kk & 3) * 32);
          tc_mma_pair(d_tmem, ad, bd, (half_units(MODE) && tl.half) ? idesc_half : idesc,
                      (kb | kk) != 0 ? 1u : 0u);
        }
        }
        tc_commit_pair_mc(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      tc_commit_pair_mc(&tfull[acc]);
      if (++acc == C::nacc) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    tc_commit_pair(drain);
    mbar_wait_plain(drain, 0, p.wait_cycles);
  } else if (MODE == MODE_WGRAD && warp == 1 && lane == 0 && !leader) {
    // ---------------- zero tiles (peer CTA; its warp 1 has no MMA to issue) ----------------
    // Experts without rows have zero weight gradients.  Both halves of such a pair tile are
    // stored here from the zero box, as a background stream of TMA stores that overlaps the
    // other tiles' MMAs and never touches the accumulator hand-off.
    for (int r = 0, t = snake_tile(0, cluster, nclusters); t < total;
         t = snake_tile(++r, cluster, nclusters)) {
#pragma unroll 1
      for (uint32_t half = 0; half < 2; ++half) {
        const Tile tl = decode<MODE>(p, t, ustart, half);
        if (tl.kit != 0 || tl.dummy) break;
        const int rows_ = (tl.which == 2) ? p.h : p.f;
        const int cols = (tl.which == 2) ? p.f : p.h;
        const int y = tl.e * rows_ + tl.m * BM;
        for (int q = 0; q < 2; ++q) {  // both products of the tile
          const CUtensorMap *map = &p.tmo[tl.which == 0 ? q : 2];
          const int n0 = (tl.which == 0) ? tl.n * BN : tl.n * 2 * BN + q * BN;
          const int ncols = min(BN, cols - n0);
          for (int r = 0; r < BM; r += 32)
            for (int c = 0; c < ncols; c += 32) tma_store_2d_u32(map, smem_u32(zbuf), n0 + c, y + r);
          bulk_commit();
          bulk_wait_read<8>();  // bounded number of groups in flight
        }
      }
    }
    bulk_wait_all();  // every zero store has completed before the CTA exits
  } else if (warp >= 2) {
    // ---------------- epilogue (both CTAs) ----------------
    const int sub = warp & 3;           // TMEM sub-partition this warp may read
    const int half = (warp - 2) >> 2;   // which part of the tile's columns (8-warp modes)
    Stager<C::out_bufs> st;
    st.bufs = smem_u32(outbuf) + (uint32_t)((warp - 2) * C::out_bufs * BOX_BYTES);
    st.cur = 0;
    st.lane = lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int r = 0, t = snake_tile(0, cluster, nclusters); t < total;
         t = snake_tile(++r, cluster, nclusters)) {
      const Tile tl = decode<MODE>(p, t, ustart, rank);
      if (tl.kit == 0) continue;  // WGRAD zero tile: stored by the producer warp
      const float wr = epilogue_prologue<MODE, EPI>(p, tl, sub, half, lane);
      int good = 1;  // lane 0 waits for the accumulator; the warp follows its verdict
      if (lane == 0) good = mbar_wait(&tfull[acc], acc_phase, p.status, abort_flag, p.wait_cycles) ? 1 : 0;
      if (!__shfl_sync(0xFFFFFFFFu, good, 0)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * C::acc_stride);
      if (!tl.dummy) epilogue_tile<MODE, EPI>(p, tl, tb, sub, half, lane, wr, st);
      // every lane's accumulator reads are complete (tcgen05.wait::ld inside the tile), ordered
      // before the warp barrier by the fence; one arrival per warp releases the accumulator
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty0 + (uint32_t)(acc * sizeof(uint64_t)));
      if (++acc == C::nacc) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_all();  // results written before the CTA exits
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs into this CTA's TMEM are done; no more remote traffic
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
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

// Row-major matrix [rows, cols] of bf16 (esize 2) or fp32 (esize 4) as a 2D tensor; box =
// box_rows x (128 / esize) columns, 128-byte swizzle (one box row = one swizzle row).
static bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols,
                      uint32_t box_rows, int esize = 2) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)esize};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esize), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   2, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// MN-major operand [rows, cols] bf16 (cols % 64 == 0) viewed as 3D: dim0 = 64 columns of a
// chunk (contiguous), dim1 = rows (stride = row pitch), dim2 = 64-column chunks (stride 128 B).
// A box of {64, box_rows, 2} lands as two consecutive [box_rows x 128 B] swizzled chunks,
// exactly the layout of two 2D boxes of 64 columns, in one TMA instruction.
static bool make_tmap_chunked(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols,
                              uint32_t box_rows, uint32_t box_chunks = 2) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc || cols % 64 != 0) return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
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

// Raster chunk: as many units (2 row blocks) as keep their A tiles (2 x 128 x K bf16 per
// unit) within about 40 MB of L2, 1..64.
static int raster_units(int K) {
  const long long per_unit = 2LL * BM * K * 2;
  long long g = (40LL << 20) / per_unit;
  if (g < 1) g = 1;
  if (g > 64) g = 64;
  return (int)g;
}

// Test-only stall injection (dmoe_debug_inject_stall): consumed by the next GEMM launch.
static std::atomic<int> g_inject_stall{0};

void set_inject_stall(int on) { g_inject_stall.store(on ? 1 : 0); }

template <int MODE, int EPI>
static cudaError_t launch_gemm(const GemmParams &p_in, long long max_tiles, cudaStream_t st) {
  using C = Cfg<MODE, EPI>;
  GemmParams p = p_in;
  p.inject = g_inject_stall.exchange(0);
  p.wait_cycles = p.inject ? kInjectedWaitCycles : kWaitCycles;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(k_grouped_gemm<MODE, EPI>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
    cfg.blockDim = dim3(C::threads, 1, 1);
    cfg.dynamicSmemBytes = C::smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_grouped_gemm<MODE, EPI>, &cfg) != cudaSuccess ||
        n < 1)
      n = device_sm_count() / 2;
    max_clusters = n;
  });
  if (attr_err != cudaSuccess) return attr_err;
  long long clusters = max_clusters;
  if (max_tiles < clusters) clusters = max_tiles;
  if (clusters < 1) clusters = 1;
  return launch_pdl(k_grouped_gemm<MODE, EPI>, (int)(2 * clusters), C::threads, C::smem, st, p);
}

static GemmParams base_params(const GemmProblem &g) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.padded_bins = g.padded_bins;
  p.bins = g.bins;
  p.indices = g.indices;
  p.T = g.T;
  p.k = g.k;
  p.E = g.E;
  p.h = g.h;
  p.f = g.f;
  p.nblk_cap = g.nblk_cap;
  p.group = 1;
  p.outs = 1;
  p.status = g.status;
  return p;
}

static inline long long max_units(const GemmProblem &g) { return (long long)g.nblk_cap / 2 + g.E; }

cudaError_t launch_glu_gemm(const GemmProblem &g, const void *x_pad, const void *w1,
                            const void *w3, void *h_out, void *a_out, void *b_out,
                            cudaStream_t st) {
  GemmParams p = base_params(g);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  const uint64_t EF = (uint64_t)g.E * g.f;
  // K-major operands viewed as {64, rows, K/64}: one box brings two 64-deep K slabs
  if (!make_tmap_chunked(&p.tm[0], x_pad, P, g.h, BM) ||
      !make_tmap_chunked(&p.tm[1], w1, EF, g.h, BN / 2) ||
      !make_tmap_chunked(&p.tm[2], w3, EF, g.h, BN / 2))
    return cudaErrorInvalidValue;
  p.outs = 0;
  if (h_out) {
    if (!make_tmap(&p.tmo[0], h_out, P, g.f, 32)) return cudaErrorInvalidValue;
    p.outs |= 1;
  }
  if (a_out && b_out) {
    if (!make_tmap(&p.tmo[1], a_out, P, g.f, 32) || !make_tmap(&p.tmo[2], b_out, P, g.f, 32))
      return cudaErrorInvalidValue;
    p.outs |= 2;
  }
  if (p.outs == 0) return cudaErrorInvalidValue;
  // single-block units: 64-row, one-slab boxes of W1 and W3 (see load_stage)
  if (!make_tmap_chunked(&p.tm[3], w1, EF, g.h, BN / 4, 1) ||
      !make_tmap_chunked(&p.tm[4], w3, EF, g.h, BN / 4, 1))
    return cudaErrorInvalidValue;
  p.half_ok = 1;
  p.n_tiles = g.f / (BN / 2);
  p.k_iters = g.h / Cfg<MODE_GLU, 4>::bk;
  p.group = raster_units(g.h);
  return launch_gemm<MODE_GLU, 4>(p, max_units(g) * p.n_tiles, st);
}

cudaError_t launch_glu_gather_gemm(const GemmProblem &g, const void *x, const void *w1,
                                   const void *w3, void *h_out, void *a_out, void *b_out,
                                   cudaStream_t st) {
  GemmParams p = base_params(g);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  const uint64_t EF = (uint64_t)g.E * g.f;
  if (!make_tmap(&p.tm[3], x, (uint64_t)g.T, g.h, 1) ||
      !make_tmap(&p.tm[1], w1, EF, g.h, BN / 2) || !make_tmap(&p.tm[2], w3, EF, g.h, BN / 2) ||
      !make_tmap(&p.tmo[0], h_out, P, g.f, 32))
    return cudaErrorInvalidValue;
  if (a_out && b_out) {
    if (!make_tmap(&p.tmo[1], a_out, P, g.f, 32) || !make_tmap(&p.tmo[2], b_out, P, g.f, 32))
      return cudaErrorInvalidValue;
    p.outs = 3;
  }
  p.tm[0] = p.tm[4] = p.tm[3];
  p.n_tiles = g.f / (BN / 2);
  p.k_iters = g.h / BK;
  p.group = raster_units(g.h);
  return launch_gemm<MODE_GLU_GATHER, 4>(p, max_units(g) * p.n_tiles, st);
}

cudaError_t launch_down_gemm(const GemmProblem &g, const void *h_in, const void *w2, void *y_pad,
                             float *y_scale, cudaStream_t st) {
  GemmParams p = base_params(g);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  // ffn <= 512: the epilogue bounds a tile, so 8 epilogue warps (measured: -9 % at ffn 512)
  const bool short_k = g.f / BK <= 8;
  const bool ok = short_k ? (make_tmap(&p.tm[0], h_in, P, g.f, BM) &&
                             make_tmap(&p.tm[1], w2, (uint64_t)g.E * g.h, g.f, BN / 2))
                          : (make_tmap_chunked(&p.tm[0], h_in, P, g.f, BM) &&
                             make_tmap_chunked(&p.tm[1], w2, (uint64_t)g.E * g.h, g.f, BN / 2));
  if (!ok || !make_tmap(&p.tmo[0], y_pad, P, g.h, 32)) return cudaErrorInvalidValue;  // fp16
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.weights = g.weights;  // the rows go out weighted
  p.part = y_scale;
  p.n_tiles = (g.h + BN - 1) / BN;
  p.group = raster_units(g.f);
  if (short_k) {
    p.k_iters = g.f / Cfg<MODE_DOWN, 8>::bk;
    return launch_gemm<MODE_DOWN, 8>(p, max_units(g) * p.n_tiles, st);
  }
  // single-block units as M = 128 MMAs only with 4 epilogue warps: with 8 the epilogue bounds
  // the tile and half of its warps would idle (measured slower)
  p.half_ok = 1;
  p.k_iters = g.f / Cfg<MODE_DOWN, 4>::bk;
  return launch_gemm<MODE_DOWN, 4>(p, max_units(g) * p.n_tiles, st);
}

cudaError_t launch_down_red_gemm(const GemmProblem &g, const void *h_in, const void *w2,
                                 float *y_acc, cudaStream_t st) {
  GemmParams p = base_params(g);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  const bool short_k = g.f / BK <= 4;  // ffn <= 256: the epilogue bounds a tile (8 warps)
  const bool ok = short_k ? (make_tmap(&p.tm[0], h_in, P, g.f, BM) &&
                             make_tmap(&p.tm[1], w2, (uint64_t)g.E * g.h, g.f, BN / 2))
                          : (make_tmap_chunked(&p.tm[0], h_in, P, g.f, BM) &&
                             make_tmap_chunked(&p.tm[1], w2, (uint64_t)g.E * g.h, g.f, BN / 2));
  if (!ok) return cudaErrorInvalidValue;
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.tmo[0] = p.tm[0];  // no result stores: the epilogue reduces into y_acc
  p.weights = g.weights;
  p.part = y_acc;
  p.n_tiles = (g.h + BN - 1) / BN;
  p.group = raster_units(g.f);
  if (short_k) {
    p.k_iters = g.f / Cfg<MODE_DOWN_RED, 8>::bk;
    return launch_gemm<MODE_DOWN_RED, 8>(p, max_units(g) * p.n_tiles, st);
  }
  p.k_iters = g.f / Cfg<MODE_DOWN_RED, 4>::bk;
  return launch_gemm<MODE_DOWN_RED, 4>(p, max_units(g) * p.n_tiles, st);
}

cudaError_t launch_dglu_gemm(const GemmProblem &g, const void *dy_pad, const void *w2,
                             const void *a_in, const void *b_in, void *da_out, void *db_out,
                             void *hw_out, float *part, cudaStream_t st) {
  GemmParams p = base_params(g);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  if (!make_tmap(&p.tm[0], dy_pad, P, g.h, BM) ||
      !make_tmap_chunked(&p.tm[1], w2, (uint64_t)g.E * g.h, g.f, BK) ||
      !make_tmap(&p.tmo[0], da_out, P, g.f, 32) || !make_tmap(&p.tmo[1], db_out, P, g.f, 32) ||
      !make_tmap(&p.tmo[2], hw_out, P, g.f, 32))
    return cudaErrorInvalidValue;
  p.weights = g.weights;
  p.part = part;
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.n_tiles = (g.f + BN - 1) / BN;
  p.k_iters = g.h / Cfg<MODE_DGLU, 4>::bk;
  p.group = raster_units(g.h);
  p.in0 = static_cast<const __nv_bfloat16 *>(a_in);
  p.in1 = static_cast<const __nv_bfloat16 *>(b_in);
  p.half_ok = 1;
  return launch_gemm<MODE_DGLU, 4>(p, max_units(g) * p.n_tiles, st);
}

cudaError_t launch_dx_gemm(const GemmProblem &g, const void *da, const void *db, const void *w1,
                           const void *w3, void *dx_pad, float *dx_scale, cudaStream_t st) {
  GemmParams p = base_params(g);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  const uint64_t EF = (uint64_t)g.E * g.f;
  if (!make_tmap_chunked(&p.tm[0], da, P, g.f, BM) ||
      !make_tmap_chunked(&p.tm[1], db, P, g.f, BM) ||
      !make_tmap_chunked(&p.tm[2], w1, EF, g.h, 2 * BK) ||
      !make_tmap_chunked(&p.tm[3], w3, EF, g.h, 2 * BK) ||
      !make_tmap(&p.tmo[0], dx_pad, P, g.h, 32))  // fp16 boxes (2-byte copies)
    return cudaErrorInvalidValue;
  p.tm[4] = p.tm[0];
  p.part = dx_scale;
  p.n_tiles = (g.h + BN - 1) / BN;
  p.k_iters = 2 * (g.f / Cfg<MODE_DX, 4>::bk);
  p.group = raster_units(2 * g.f);
  p.half_ok = 1;
  return launch_gemm<MODE_DX, 4>(p, max_units(g) * p.n_tiles, st);
}

cudaError_t launch_wgrad_gemm(const GemmProblem &g, const void *x_pad, const void *h_in,
                              const void *dy_pad, const void *da, const void *db, float *dw1,
                              float *dw3, float *dw2, cudaStream_t st) {
  GemmParams p = base_params(g);
  const uint64_t P = (uint64_t)g.nblk_cap * BM;
  const uint64_t EF = (uint64_t)g.E * g.f, EH = (uint64_t)g.E * g.h;
  if (!make_tmap_chunked(&p.tm[0], da, P, g.f, BK) ||
      !make_tmap_chunked(&p.tm[1], db, P, g.f, BK) ||
      !make_tmap_chunked(&p.tm[2], dy_pad, P, g.h, BK) ||
      !make_tmap_chunked(&p.tm[3], x_pad, P, g.h, BK) ||
      !make_tmap_chunked(&p.tm[4], h_in, P, g.f, BK) || !make_tmap(&p.tmo[0], dw1, EF, g.h, 32, 4) ||
      !make_tmap(&p.tmo[1], dw3, EF, g.h, 32, 4) || !make_tmap(&p.tmo[2], dw2, EH, g.f, 32, 4))
    return cudaErrorInvalidValue;
  const long long t13 = (long long)((g.f / BM + 1) / 2) * ((g.h + BN - 1) / BN);
  const long long t2 = (long long)((g.h / BM + 1) / 2) * ((g.f + 2 * BN - 1) / (2 * BN));
  return launch_gemm<MODE_WGRAD, 4>(p, (long long)g.E * (t13 + t2), st);
}

// ---- the linear router's GEMMs (dense token rows) ----------------------------------------------

static GemmParams dense_params(int T, int h, int E, int32_t *status) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.T = T;
  p.h = h;
  p.E = E;
  p.group = 1;
  p.outs = 1;
  p.status = status;
  return p;
}

static inline int row_units(int T) { return (T + 2 * BM - 1) / (2 * BM); }

cudaError_t launch_router_gemm(int T, int h, int E, const void *x, const void *wr, void *logits,
                               int32_t *status, cudaStream_t st) {
  GemmParams p = dense_params(T, h, E, status);
  if (!make_tmap(&p.tm[0], x, (uint64_t)T, h, BM) || !make_tmap(&p.tm[1], wr, (uint64_t)E, h, BN / 2) ||
      !make_tmap(&p.tmo[0], logits, (uint64_t)T, E, 32))
    return cudaErrorInvalidValue;
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.n_tiles = (E + BN - 1) / BN;
  p.k_iters = h / BK;
  p.total = row_units(T) * p.n_tiles;
  return launch_gemm<MODE_ROUTER, 4>(p, p.total, st);
}

cudaError_t launch_router_dx_gemm(int T, int h, int E, const void *dlogits, const void *wr, void *dx,
                                  int32_t *status, cudaStream_t st) {
  GemmParams p = dense_params(T, h, E, status);
  if (!make_tmap(&p.tm[0], dlogits, (uint64_t)T, E, BM) ||
      !make_tmap(&p.tm[1], wr, (uint64_t)E, h, 64) || !make_tmap(&p.tmo[0], dx, (uint64_t)T, h, 32))
    return cudaErrorInvalidValue;
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.in0 = static_cast<const __nv_bfloat16 *>(dx);
  p.n_tiles = (h + BN - 1) / BN;
  p.k_iters = (E + BK - 1) / BK;
  p.total = row_units(T) * p.n_tiles;
  // K = E is short (a few K steps per tile): the read-add-store epilogue bounds a tile, so it
  // gets 8 warps (two per TMEM sub-partition, each half of the columns)
  return launch_gemm<MODE_RDX, 8>(p, p.total, st);
}

int router_wgrad_splits(int T, int h, int E) {
  const int mpairs = ((E + BM - 1) / BM + 1) / 2;
  const int tiles = mpairs * ((h + BN - 1) / BN);
  const int k_iters = (T + BK - 1) / BK;
  int s = (device_sm_count() / 2) / tiles;  // at most one tile per SM pair: a single wave
  s = min(s, kRouterMaxSplits);
  s = min(s, k_iters);
  if (s < 1) s = 1;
  const int per = (k_iters + s - 1) / s;
  return (k_iters + per - 1) / per;  // no empty split
}

cudaError_t launch_router_wgrad_gemm(int T, int h, int E, const void *dlogits, const void *x,
                                     float *partials, int splits, int32_t *status,
                                     cudaStream_t st) {
  GemmParams p = dense_params(T, h, E, status);
  p.Ep = (E + BM - 1) / BM * BM;
  if (!make_tmap(&p.tm[0], dlogits, (uint64_t)T, E, 64) || !make_tmap(&p.tm[1], x, (uint64_t)T, h, 64) ||
      !make_tmap(&p.tmo[0], partials, (uint64_t)splits * p.Ep, h, 32, 4))
    return cudaErrorInvalidValue;
  p.tm[2] = p.tm[3] = p.tm[4] = p.tm[0];
  p.n_tiles = (h + BN - 1) / BN;
  p.k_iters = (T + BK - 1) / BK;
  p.split_k = (p.k_iters + splits - 1) / splits;
  if (splits < 1 || splits > kRouterMaxSplits || (splits - 1) * p.split_k >= p.k_iters)
    return cudaErrorInvalidValue;  // every split must own K steps: its slab is read back
  const int mpairs = ((E + BM - 1) / BM + 1) / 2;
  p.total = splits * mpairs * p.n_tiles;
  return launch_gemm<MODE_RWGRAD, 4>(p, p.total, st);
}

}  // namespace dmoe
