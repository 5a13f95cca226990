// map.cu -- routing and sparse-map construction (MegaBlocks walkthrough "02 · dropless MoE 与
// block-sparse 重构", sections 4.1-4.3; Fast-LLM issue #56 get_sparse_map).
//
// Three kernels, no spin-waits, deterministic results (the only global atomic is the scan's
// completion ticket):
//   k_route_hist   16 warps per 64-token tile, 4 tokens per warp with all their logits loaded
//                  at once: top-k by integer max over order-preserving keys (ties -> lower
//                  expert index; each lane keeps its three best candidates, the picks checked
//                  afterwards), fp32 softmax weights, per-tile histogram in shared memory
//                  (O(E) bytes, independent of T) and a per-tile status word.
//   k_map_scan     one CTA per 32 experts: per-expert exclusive offsets of every tile; the
//                  last CTA to finish (a ticket counter, no waiting) computes bins,
//                  padded_bins (round_up to 128), num_blocks and stores the status word.
//   k_map_scatter  one CTA per up to 2048 entries (up to 4 tiles at top-8): stable rank of
//                  every entry inside its expert (warp histograms + __match_any_sync ranks in
//                  entry order), then indices, bin_ids (staged per expert in shared memory)
//                  and dest_row from the index math of section 4.2; every CTA also fills a
//                  slice of the block -> expert table.
#include "common.cuh"
#include "kernels.h"

namespace dmoe {

constexpr int kMapThreads = 256;
constexpr int kMapWarps = kMapThreads / 32;


// 2^x with the hardware approximation (a few ulp; subnormal results kept).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Selection key of a logit given as its fp32 image u (a bf16 value in the high half): the high
// half is the order-preserving image (negative -> bits inverted, else sign bit set; -0 taken as
// +0), the low half is `low` = 0xFFFF - expert, so among equal logits the lower expert has the
// larger key.  Exact for every value but NaN; route_key_nan also maps NaN to 0 (below -inf).
__device__ __forceinline__ uint32_t route_key(uint32_t u, uint32_t low) {
  const float f = __fadd_rn(__uint_as_float(u), 0.0f);  // -0 + 0 = +0
  const uint32_t z = __float_as_uint(f);
  const uint32_t neg = (uint32_t)((int32_t)z >> 31);
  return (z ^ (neg & 0x7FFF0000u)) ^ (0x80000000u | low);
}
__device__ __forceinline__ uint32_t route_key_nan(uint32_t u, uint32_t low) {
  return ((u & 0x7FFFFFFFu) > 0x7F800000u) ? low : route_key(u, low);
}

// The bf16 value whose order-preserving image (the high half of a route key) is `ord`, for
// any image but that of NaN.
__device__ __forceinline__ float bf16_from_order(uint32_t ord) {
  const uint32_t bits = (ord & 0x8000u) ? (ord & 0x7FFFu) : (~ord & 0xFFFFu);
  return __uint_as_float(bits << 16);
}

// ---- routing + histogram ---------------------------------------------------------------------

// The routing kernel runs 16 warps per 64-token tile, 4 tokens per warp, so that each warp has
// all of its tokens' logits in flight at once: ranking a token is a chain of k dependent
// warp reductions, and with one token loaded ahead the load latency was not hidden.
constexpr int kRouteThreads = 512;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kRouteTPW = kMapTokTile / kRouteWarps;  // tokens per warp
static_assert(kRouteTPW * kRouteWarps == kMapTokTile, "routing tile");

// One lane's share of a token's logits.  KPL = logits per lane (E <= 32*KPL).  PACKED (E even,
// KPL >= 2): word c of lane l holds experts 64c + 2l and 64c + 2l + 1, two per word, so that
// each word is one coalesced 128-byte load across the warp and a run of strong experts (the
// low indices of a Zipf-skewed router) spreads over many lanes; otherwise lane l owns experts
// l, l + 32, ..., one per word.
template <int KPL, bool PACKED>
struct RouteRow {
  static_assert(!PACKED || KPL >= 2, "two logits per word");
  static constexpr int kWords = PACKED ? KPL / 2 : KPL;
  uint32_t w[kWords];

  __device__ __forceinline__ static int expert(int lane, int i) {
    return PACKED ? 64 * (i >> 1) + 2 * lane + (i & 1) : lane + 32 * i;
  }
  // fp32 image of logit i (the bf16 bits in the high half)
  __device__ __forceinline__ uint32_t image(int i) const {
    if constexpr (PACKED) return (i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16);
    return w[i] << 16;
  }
  __device__ __forceinline__ void load(const uint16_t *__restrict__ row, int E, int lane) {
#pragma unroll
    for (int c = 0; c < kWords; ++c) {
      if constexpr (PACKED) {
        const int e = 64 * c + 2 * lane;  // E even: both experts of the pair exist or neither
        w[c] = (e < E) ? __ldg(reinterpret_cast<const unsigned int *>(row + e)) : 0u;
      } else {
        const int e = lane + 32 * c;
        w[c] = (e < E) ? (uint32_t)__ldg(row + e) : 0u;
      }
    }
  }
};

// Order-preserving 16-bit images of the two bf16 values packed in w, in the same halves:
// -0 is first turned into +0 (-0 + +0 = +0) so that the two zeros tie; then a negative half
// has every bit inverted and any other half its sign bit set.  For non-NaN a, b: a < b iff
// image(a) < image(b).  NaN is not ordered here (the caller takes a separate path for it).
__device__ __forceinline__ uint32_t order2(uint32_t w) {
  uint32_t z, sgn, o;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(z) : "r"(w), "r"(0u));
  // per half: its sign bit replicated (prmt with the selector's sign-extension bit set, which
  // __byte_perm does not pass on)
  asm("prmt.b32 %0, %1, %2, 0xBB99;" : "=r"(sgn) : "r"(z), "r"(0u));
  // per half: bits 0-14 z ^ sgn, bit 15 ~z  (lookup table of c ? a ^ b : ~a)
  asm("lop3.b32 %0, %1, %2, %3, 0x2D;" : "=r"(o) : "r"(z), "r"(sgn), "r"(0x7FFF7FFFu));
  return o;
}

// Non-finite detector over packed bf16 pairs: acc = w * 0 + acc stays +0 in both halves while
// every value seen is finite (x * 0 = +-0 and +0 + -0 = +0) and is NaN from the first Inf or
// NaN on.
__device__ __forceinline__ uint32_t nonfinite_acc(uint32_t acc, uint32_t w) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0u), "r"(acc));
  return r;
}

// 2^x without subnormal results (flushed to +0): the terms of a softmax sum, which is >= 1.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The two bf16 values packed in w minus m, in fp32 (one rounding each: x * 1 + (-m) on the
// mixed-precision fused multiply-add, with no unpacking of the pair).
__device__ __forceinline__ void sub_bf16x2_f32(uint32_t w, float m, float &d0, float &d1) {
  asm("{.reg .b16 lo, hi, one;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "mov.b16 one, 0x3F80;\n\t"
      "fma.rn.f32.bf16 %0, lo, one, %3;\n\t"
      "fma.rn.f32.bf16 %1, hi, one, %3;}"
      : "=f"(d0), "=f"(d1)
      : "r"(w), "f"(-m));
}

// (a, b) * s on the paired fp32 pipe, and the sum of two pairs.
__device__ __forceinline__ void mul_f32x2(float &a, float &b, float s) {
  asm("{.reg .b64 x, y, m;\n\t"
      "mov.b64 x, {%0, %1};\n\t"
      "mov.b64 m, {%2, %2};\n\t"
      "mul.rn.f32x2 y, x, m;\n\t"
      "mov.b64 {%0, %1}, y;}"
      : "+f"(a), "+f"(b)
      : "f"(s));
}
__device__ __forceinline__ void add_f32x2(float &a, float &b, float c, float d) {
  asm("{.reg .b64 x, y, z;\n\t"
      "mov.b64 x, {%0, %1};\n\t"
      "mov.b64 y, {%2, %3};\n\t"
      "add.rn.f32x2 z, x, y;\n\t"
      "mov.b64 {%0, %1}, z;}"
      : "+f"(a), "+f"(b)
      : "f"(c), "f"(d));
}

// The C largest keys seen so far, largest first (0 = empty slot): one insertion costs C
// max/min pairs, with no branches.
template <int C>
struct TopC {
  uint32_t c[C];
  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int i = 0; i < C; ++i) c[i] = 0u;
  }
  __device__ __forceinline__ void insert(uint32_t x) {
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const uint32_t hi = max(c[i], x);
      x = min(c[i], x);
      c[i] = hi;
    }
  }
};

struct Picks {
  uint32_t mine;   // lane s < k: the key of pick s
  uint32_t first;  // every lane: pick 0 (the largest key)
  uint32_t last;   // every lane: pick k - 1
  bool dry;        // this lane has no candidate left
};

// The k rounds of a warp-wide integer max over the lanes' best candidates: keys are unique,
// so exactly one lane holds each winner and drops it.  KC > 0 fixes k at compile time.  Every
// lane keeps its C largest keys; with REFILL, a lane that has given up all C while rounds
// remain refills them from its keys below the last pick (warp-uniform test).  Without it the
// picks are the top-k of the candidates, and the caller checks that they are the top-k of all.
template <int C, int KPL, int KC, bool REFILL>
__device__ __forceinline__ Picks select_rounds(const uint32_t (&key)[KPL], int k, int lane) {
  TopC<C> cand;
  cand.clear();
#pragma unroll
  for (int i = 0; i < KPL; ++i) cand.insert(key[i]);
  Picks r;
  r.mine = 0u;
  r.first = 0u;
  uint32_t wb = 0u;
  auto round = [&](int s) {
    wb = __reduce_max_sync(0xFFFFFFFFu, cand.c[0]);
    if (s == 0) r.first = wb;
    r.mine = (lane == s) ? wb : r.mine;
    const bool win = cand.c[0] == wb;
#pragma unroll
    for (int i = 0; i + 1 < C; ++i) cand.c[i] = win ? cand.c[i + 1] : cand.c[i];
    cand.c[C - 1] = win ? 0u : cand.c[C - 1];
    if constexpr (REFILL && KPL > C) {
      const bool dry = win && cand.c[0] == 0u && s + 1 < k;
      if (__any_sync(0xFFFFFFFFu, dry)) {
        if (dry) {
#pragma unroll
          for (int i = 0; i < KPL; ++i)
            if (key[i] < wb) cand.insert(key[i]);
        }
      }
    }
  };
  if constexpr (KC > 0) {
#pragma unroll
    for (int s = 0; s < KC; ++s) round(s);
  } else {
#pragma unroll 1
    for (int s = 0; s < k; ++s) round(s);
  }
  r.last = wb;
  r.dry = cand.c[0] == 0u;
  return r;
}

// Grid: one CTA per 64-token tile.  Per token: every lane turns its logits into unique integer
// keys (order-preserving image of the bf16 value in the high half, 0xFFFF - expert in the low
// half, so the larger key is the larger logit and, on equal logits, the lower expert) and
// keeps its three largest; k rounds of a warp-wide integer max then pick the top-k in rank
// order.  Those are the top-k of all keys unless some lane holds more than three keys at or
// above the last pick (if a key of the true top-k were missing from the candidates, its lane
// would hold three larger ones and it, all above the last pick): then, rarely, the rounds run
// again with refills.  Weights: fp32 softmax over all E logits (or, renormalised, over the k
// picks) with the first pick as the maximum.  The tile's expert histogram is built in shared
// memory and written to tile_hist; the tile's status bits go to tile_flags (a plain store, so
// the workspace needs no initialisation).  Up to 8 logits per lane two CTAs share an SM
// (at most 64 registers a thread).
template <int KPL, bool PACKED, int KC>
__global__ void __launch_bounds__(kRouteThreads, KPL <= 8 ? 2 : 1)
    k_route_hist(const uint16_t *__restrict__ logits, int T, int E, int k, int renorm,
                 int32_t *__restrict__ top, float *__restrict__ weights,
                 int32_t *__restrict__ tile_hist, int32_t *__restrict__ tile_flags,
                 unsigned int *__restrict__ done) {
  using Row = RouteRow<KPL, PACKED>;
  constexpr int C = (KPL < 3) ? KPL : 3;                  // candidates kept per lane
  constexpr int kInFlight = (KPL <= 8) ? kRouteTPW : 1;  // token rows loaded ahead per warp
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ int hist[];  // [E]
  __shared__ int s_flags;
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) *done = 0u;  // ticket counter of k_map_scan
  if (threadIdx.x == 0) s_flags = 0;
  for (int e = threadIdx.x; e < E; e += kRouteThreads) hist[e] = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kMapTokTile + warp;
  const bool full_rows = (E == 32 * KPL);  // every slot of every lane holds an expert
  // low halves of this lane's keys, per word (PACKED: key 2c in bits 0-15, key 2c + 1 in bits
  // 16-31); 0 marks a word past the last expert
  uint32_t lowp[Row::kWords];
#pragma unroll
  for (int c = 0; c < Row::kWords; ++c) {
    const int e = Row::expert(lane, PACKED ? 2 * c : c);
    lowp[c] = (e >= E) ? 0u
              : PACKED ? (((0xFFFEu - (uint32_t)e) << 16) | (0xFFFFu - (uint32_t)e))
                       : 0xFFFFu - (uint32_t)e;
  }
  auto low_of = [&](int i) -> uint32_t {
    if constexpr (PACKED) return (i & 1) ? (lowp[i >> 1] >> 16) : (lowp[i >> 1] & 0xFFFFu);
    return lowp[i];
  };
  Row rows[kInFlight];
#pragma unroll
  for (int j = 0; j < kInFlight; ++j) {
    const int t = t0 + kRouteWarps * j;
    if (t < T) rows[j].load(logits + (size_t)t * E, E, lane);
  }
  __syncthreads();
  bool bad = false;
#pragma unroll
  for (int j = 0; j < kRouteTPW; ++j) {
    const int t = t0 + kRouteWarps * j;
    if (t >= T) break;
    Row cur;
    if constexpr (kInFlight == kRouteTPW) {
      cur = rows[j];
    } else {
      cur.load(logits + (size_t)t * E, E, lane);
    }
    uint32_t key[KPL];
    uint32_t nfa = 0u;  // slots past E hold +0: finite
#pragma unroll
    for (int i = 0; i < Row::kWords; ++i) {
      const uint32_t wv = cur.w[i];
      nfa = nonfinite_acc(nfa, wv);
      const uint32_t o = order2(wv);
      if constexpr (PACKED) {
        key[2 * i] = __byte_perm(o, lowp[i], 0x1054);      // (image lo << 16) | low lo
        key[2 * i + 1] = __byte_perm(o, lowp[i], 0x3276);  // (image hi << 16) | low hi
      } else {
        key[i] = __byte_perm(o, lowp[i], 0x1054);
      }
    }
    if (!full_rows) {  // warp-uniform: slots past the last expert hold no candidate
#pragma unroll
      for (int i = 0; i < KPL; ++i) key[i] = low_of(i) ? key[i] : 0u;
    }
    if (__any_sync(0xFFFFFFFFu, nfa != 0u)) {  // rare: NaN ranked lowest
      bad = true;
#pragma unroll
      for (int i = 0; i < KPL; ++i) {
        const uint32_t lo = low_of(i);
        key[i] = lo ? route_key_nan(cur.image(i), lo) : 0u;
      }
    }
    // a valid key is never 0 (its low half is >= 0xFFFF - 1023)
    Picks pk = select_rounds<C, KPL, KC, false>(key, k, lane);
    if constexpr (KPL > C) {
      if (__any_sync(0xFFFFFFFFu, pk.dry)) {
        int cnt = 0;
#pragma unroll
        for (int i = 0; i < KPL; ++i) cnt += (key[i] >= pk.last) ? 1 : 0;
        if (__any_sync(0xFFFFFFFFu, cnt > C)) pk = select_rounds<C, KPL, KC, true>(key, k, lane);
      }
    }
    const uint32_t my_key = pk.mine;
    const int my_e = 0xFFFF - (int)(my_key & 0xFFFFu);
    // softmax over all E logits (or, renormalised, over the k picks), max m = the first pick
    // (lane 0's); e^(x - m) = 2^((x - m) log2(e)), x - m rounded once
    const float v = (lane < k) ? (((my_key >> 16) == 0u) ? __uint_as_float(0x7FC00000u)
                                                         : bf16_from_order(my_key >> 16))
                               : 0.0f;
    const float m = __shfl_sync(0xFFFFFFFFu, v, 0);
    const float ev = ex2_approx((v - m) * kLog2e);
    float sum = 0.0f;
    if (renorm) {
      if (lane < k) sum = ev;
    } else if (PACKED && full_rows) {  // two logits per word, on the paired fp32 pipe
      float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
      for (int i = 0; i < Row::kWords; ++i) {
        float a, b;
        sub_bf16x2_f32(cur.w[i], m, a, b);
        mul_f32x2(a, b, kLog2e);
        add_f32x2(s0, s1, ex2_ftz(a), ex2_ftz(b));
      }
      sum = s0 + s1;
    } else if (full_rows) {
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        sum += ex2_ftz((__uint_as_float(cur.image(i)) - m) * kLog2e);
    } else {
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        if (low_of(i)) sum += ex2_ftz((__uint_as_float(cur.image(i)) - m) * kLog2e);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    if (lane < k) {
      top[(size_t)t * k + lane] = my_e;
      weights[(size_t)t * k + lane] = __fdividef(ev, sum);  // 1 <= sum <= E
      atomicAdd(&hist[my_e], 1);
    }
  }
  if (bad && lane == 0) atomicOr(&s_flags, DMOE_STATUS_NONFINITE_LOGITS);  // warp-uniform
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kRouteThreads)
    tile_hist[(size_t)blockIdx.x * E + e] = hist[e];
  if (threadIdx.x == 0) tile_flags[blockIdx.x] = s_flags;
}

// Histogram of caller-given top_experts; invalid ids are reported (in tile_flags) and left
// out of the map.
__global__ void __launch_bounds__(kMapThreads) k_given_hist(const int32_t *__restrict__ top,
                                                            int T, int E, int k, int absent_ok,
                                                            int32_t *__restrict__ tile_hist,
                                                            int32_t *__restrict__ tile_flags,
                                                            unsigned int *__restrict__ done) {
  extern __shared__ int hist[];
  __shared__ int s_flags;
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) *done = 0u;  // ticket counter of k_map_scan
  if (threadIdx.x == 0) s_flags = 0;
  for (int e = threadIdx.x; e < E; e += kMapThreads) hist[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kMapTokTile;
  int flags = 0;
  if (k == 1) {  // one entry per token (the rounded routing's entry list): 32 tokens a warp
    for (int tt = warp * 32; tt < kMapTokTile; tt += kMapWarps * 32) {
      const int t = t0 + tt + lane;
      int e = -1;
      if (t < T) {
        e = top[t];
        if (e < -1 || e >= E || (e == -1 && !absent_ok)) {
          flags |= DMOE_STATUS_EXPERT_OUT_OF_RANGE;
          e = -1;
        }
      }
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[e], __popc(peers));
    }
  }
  for (int tt = warp; k > 1 && tt < kMapTokTile; tt += kMapWarps) {
    const int t = t0 + tt;
    if (t >= T) break;
    int e = -1 - lane;  // distinct sentinels for lanes >= k
    if (lane < k) {
      e = top[(size_t)t * k + lane];
      if (e < 0 || e >= E) {
        if (!(absent_ok && e == -1)) flags |= DMOE_STATUS_EXPERT_OUT_OF_RANGE;
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
  if (flags && lane == 0) atomicOr(&s_flags, flags);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kMapThreads)
    tile_hist[(size_t)blockIdx.x * E + e] = hist[e];
  if (threadIdx.x == 0) tile_flags[blockIdx.x] = s_flags;
}

// ---- scan ------------------------------------------------------------------------------------

constexpr int kScanThreads = 1024;
static_assert(kScanSeg == 32 * kScanCache, "a scan CTA holds its segment in registers");

// Inclusive block-wide scan of one int per thread (whole warps, at most 1024 threads);
// warp_tot holds 32 ints of shared memory.
__device__ __forceinline__ int block_incl_scan(int v, int *warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (int)(blockDim.x >> 5);
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xFFFFFFFFu, v, off);
    if (lane >= off) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < nwarps) ? warp_tot[lane] : 0;
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

// Two-level scan of the per-tile histograms.  Grid (ceil(E/32), S): CTA (x, y) covers experts
// 32x .. 32x+31 over the y-th segment of kScanSeg tiles; warp c of it owns kScanCache
// consecutive tiles of the segment, lane l owns expert 32x + l, so every load of a tile's
// histogram row is one coalesced access and all of a thread's loads are in flight at once.
// It rewrites each count as the tile's exclusive offset inside its expert and segment and
// writes the segment's total per expert to seg_sum[y][e].  The CTA that takes the last ticket
// of `done` (zeroed by the routing kernel; no CTA waits for another) turns seg_sum into
// exclusive prefixes over segments and computes tokens_per_expert, bins, padded_bins,
// num_blocks and the call's status word.
__global__ void __launch_bounds__(kScanThreads, 1) k_map_scan(int n_tiles, int E,
                                                           int32_t *__restrict__ tile_hist,
                                                           const int32_t *__restrict__ tile_flags,
                                                           int32_t *__restrict__ seg_sum,
                                                           int32_t *__restrict__ tokens_per_expert,
                                                           int32_t *__restrict__ bins,
                                                           int32_t *__restrict__ padded_bins,
                                                           int32_t *__restrict__ num_blocks,
                                                           int32_t *__restrict__ status,
                                                           unsigned int *__restrict__ done,
                                                           int or_status) {
  __shared__ int chunk[32][33];
  __shared__ int warp_tot[32];
  __shared__ int s_flags;
  __shared__ bool is_last;
  pdl_wait();
  pdl_trigger();
  const int c = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + lane;
  const int seg = blockIdx.y;
  const int tb = seg * kScanSeg + c * kScanCache;
  const int te = min(n_tiles, tb + kScanCache);
  int cache[kScanCache];
  int sum = 0;
  if (e < E) {
#pragma unroll
    for (int i = 0; i < kScanCache; ++i) {
      cache[i] = (tb + i < te) ? tile_hist[(size_t)(tb + i) * E + e] : 0;
      sum += cache[i];
    }
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
    if (e < E) seg_sum[(size_t)seg * E + e] = run;
  }
  __syncthreads();
  if (e < E) {  // counts -> exclusive offsets inside the expert and segment
    int run = chunk[c][lane];
#pragma unroll
    for (int i = 0; i < kScanCache; ++i) {
      if (tb + i < te) tile_hist[(size_t)(tb + i) * E + e] = run;
      run += cache[i];
    }
  }
  // ---- last CTA: segment prefixes, bins, padded_bins, num_blocks, status ----
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1u) == gridDim.x * gridDim.y - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int tid = threadIdx.x;
  if (tid == 0) s_flags = 0;
  int flags = 0;
  for (int t = tid; t < n_tiles; t += kScanThreads) flags |= tile_flags[t];
  int cnt = 0;
  if (tid < E) {
    volatile int32_t *ss = seg_sum;
    for (int y = 0; y < (int)gridDim.y; ++y) {
      const int v = ss[(size_t)y * E + tid];
      ss[(size_t)y * E + tid] = cnt;
      cnt += v;
    }
    tokens_per_expert[tid] = cnt;
  }
  const int pad = ((cnt + kBlock - 1) / kBlock) * kBlock;
  const int incl = block_incl_scan(cnt, warp_tot);  // (its barriers also order s_flags = 0)
  const int pincl = block_incl_scan(pad, warp_tot);
  if (tid < E) {
    bins[tid] = incl;
    padded_bins[tid] = pincl;
  }
  if (tid == E - 1) *num_blocks = pincl / kBlock;
  flags = __reduce_or_sync(0xFFFFFFFFu, flags);
  if (flags && lane == 0) atomicOr(&s_flags, flags);
  __syncthreads();
  if (tid == 0) {
    // the map call's own bits (later calls OR theirs in); a second map of the same call ORs
    if (or_status) {
      if (s_flags) atomicOr(status, s_flags);
    } else {
      *status = s_flags;
    }
    *done = 0u;  // ready for the next call
  }
}

// ---- stable scatter --------------------------------------------------------------------------

// Entries a lane keeps in registers between the scatter's two passes: a tile has at most
// 64 * DMOE_MAX_TOP_K entries, split over 8 warps in whole 32-entry rounds.
constexpr int kScatRounds = 8;
static_assert(kMapTokTile * DMOE_MAX_TOP_K <= kMapWarps * 32 * kScatRounds, "scatter rounds");

// Entries of one scatter CTA: its staging buffers in shared memory hold that many.
constexpr int kScatEntries = kMapWarps * 32 * kScatRounds;

// Grid: one CTA per S consecutive tiles (S a power of two dividing kScanSeg, at most
// kScatEntries entries: up to 4 for top-8, fewer where the grid would drop below two CTAs per
// SM), so that the per-expert work of a CTA (offsets, warp histograms) is shared by S tiles.  The rank r of an entry inside its expert among the CTA's
// entries (warp histograms and __match_any_sync ranks, in entry order) gives its sorted
// position s_base[e] + r by the index math of section 4.2: dest_row is stored from there in
// entry order, while indices and bin_ids are first staged in shared memory, expert by
// expert, and then stored by consecutive threads, so that each expert's run of the CTA (one
// contiguous range of both arrays) takes a few wide stores instead of one per entry.  Every
// CTA also writes a grid-strided slice of the block -> expert table (entry b = the expert
// whose padded range holds row 128*b, -1 past num_blocks).
__global__ void __launch_bounds__(kMapThreads) k_map_scatter(int T, int E, int k, int S,
                                                             int nblk_cap,
                                                             const int32_t *__restrict__ top,
                                                             const int32_t *__restrict__ tile_off,
                                                             const int32_t *__restrict__ seg_off,
                                                             const int32_t *__restrict__ bins,
                                                             const int32_t *__restrict__ padded_bins,
                                                             int32_t *__restrict__ indices,
                                                             int32_t *__restrict__ bin_ids,
                                                             int32_t *__restrict__ dest_row,
                                                             int32_t *__restrict__ block_expert) {
  extern __shared__ int sm[];
  int *wh = sm;                      // [kMapWarps][E] counts, then offsets inside (CTA, expert)
  int *s_base = wh + kMapWarps * E;  // [E] bins[e-1] + offset of this CTA's tiles inside e
  int *s_shift = s_base + E;         // [E] padded_bins[e-1] - bins[e-1]
  int *s_pb = s_shift + E;           // [E] padded_bins
  int *s_loff = s_pb + E;            // [E] staging slot of the CTA's first entry of e
  int *st_j = s_loff + E;            // [kScatEntries] staged entry index, by slot
  int *st_e = st_j + kScatEntries;   // [kScatEntries] staged expert, by slot
  __shared__ int warp_tot[32];
  __shared__ int s_nv;
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long N = (long long)T * k;
  const int tile0 = blockIdx.x * S;  // the CTA's first tile
  const long long j0 = (long long)tile0 * kMapTokTile * k;
  const long long j1 = min(N, j0 + (long long)S * kMapTokTile * k);
  const int n = (int)(j1 - j0);
  const int per_warp = (((n + kMapWarps - 1) / kMapWarps) + 31) & ~31;
  const long long wb = j0 + (long long)warp * per_warp;
  const long long we = min(j1, wb + per_warp);
  // this warp's entries, loaded once (all rounds in flight) and kept for both passes
  int ev[kScatRounds];
#pragma unroll
  for (int r = 0; r < kScatRounds; ++r) {
    const long long j = wb + 32 * r + lane;
    int e = -1 - lane;
    if (j < we) {
      const int v = top[j];
      if (v >= 0 && v < E) e = v;
    }
    ev[r] = e;
  }
  for (int i = threadIdx.x; i < kMapWarps * E; i += kMapThreads) wh[i] = 0;
  for (int e = threadIdx.x; e < E; e += kMapThreads) {
    const int bp = (e > 0) ? bins[e - 1] : 0;
    const int pp = (e > 0) ? padded_bins[e - 1] : 0;
    s_base[e] = bp + seg_off[(size_t)(tile0 / kScanSeg) * E + e] +
                tile_off[(size_t)tile0 * E + e];
    s_shift[e] = pp - bp;
    s_pb[e] = padded_bins[e];
  }
  __syncthreads();
  int *my = wh + warp * E;
  const unsigned lt_mask = (1u << lane) - 1u;
  // pass 1: per-warp histogram of its contiguous entry range; the lanes sharing each lane's
  // expert in a round are kept for pass 2
  unsigned peers_of[kScatRounds];
#pragma unroll
  for (int r = 0; r < kScatRounds; ++r) peers_of[r] = 0u;
#pragma unroll
  for (int r = 0; r < kScatRounds; ++r) {
    if (wb + 32 * r >= we) break;
    const int e = ev[r];
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    peers_of[r] = peers;
    if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per expert: warp counts -> offsets inside (CTA, expert); the CTA's count of each expert,
  // scanned over the experts in order, gives its staging slots (a thread takes a run of up
  // to ceil(E / kMapThreads) consecutive experts)
  const int ept = (E + kMapThreads - 1) / kMapThreads;
  const int e_lo = min(E, threadIdx.x * ept), e_hi = min(E, e_lo + ept);
  int tsum = 0;
  for (int e = e_lo; e < e_hi; ++e) {
    int run = 0;
    for (int w = 0; w < kMapWarps; ++w) {
      const int v = wh[w * E + e];
      wh[w * E + e] = run;
      run += v;
    }
    s_loff[e] = run;  // the count, for now
    tsum += run;
  }
  const int incl = block_incl_scan(tsum, warp_tot);
  if (threadIdx.x == kMapThreads - 1) s_nv = incl;
  {
    int pre = incl - tsum;
    for (int e = e_lo; e < e_hi; ++e) {
      const int c = s_loff[e];
      s_loff[e] = pre;
      pre += c;
    }
  }
  __syncthreads();
  // pass 2: rank of every entry inside (CTA, expert), in entry order: dest_row, and the
  // entry's staging slot
#pragma unroll
  for (int r = 0; r < kScatRounds; ++r) {
    if (wb + 32 * r >= we) break;
    const long long j = wb + 32 * r + lane;
    const int e = ev[r];
    const unsigned peers = peers_of[r];
    if (e >= 0) {
      const int rr = my[e] + __popc(peers & lt_mask);
      dest_row[j] = s_base[e] + rr + s_shift[e];  // offset_in_bin + padded_bins[e-1]
      const int slot = s_loff[e] + rr;
      st_j[slot] = (int)j;  // T * k <= 2^25
      st_e[slot] = e;
    } else if (j < we) {
      dest_row[j] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // pass 3: indices and bin_ids, slot by slot (slot - s_loff[e] = the rank inside the expert)
  for (int t = threadIdx.x; t < s_nv; t += kMapThreads) {
    const int e = st_e[t];
    const int i = s_base[e] + (t - s_loff[e]);
    indices[i] = st_j[t];
    bin_ids[i] = e;
  }
  // block -> expert table slice
  const int nb = s_pb[E - 1] / kBlock;
  for (int b = blockIdx.x * kMapThreads + threadIdx.x; b < nblk_cap;
       b += gridDim.x * kMapThreads) {
    int owner = -1;
    if (b < nb) {  // smallest e with padded_bins[e] > 128*b
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

// ---- launchers -------------------------------------------------------------------------------

cudaError_t launch_route_hist(const uint16_t *logits, int T, int E, int k, bool renorm, int32_t *top,
                              float *weights, int32_t *tile_hist, cudaStream_t st,
                              bool absent_ok) {
  const int tiles = map_tiles(T);
  const size_t smem = sizeof(int) * (size_t)E;
  unsigned int *done = map_ticket(tile_hist, T, E);
  int32_t *flags = map_flags(tile_hist, T, E);
  if (!logits)
    return launch_pdl(k_given_hist, tiles, kMapThreads, smem, st, top, T, E, k,
                      absent_ok ? 1 : 0, tile_hist, flags, done);
  // logits per lane: the smallest power of two with E <= 32 * KPL; two per word when E is
  // even; the round count fixed at compile time for top-2 and top-8 on those layouts
  using Kernel = void (*)(const uint16_t *, int, int, int, int, int32_t *, float *, int32_t *,
                          int32_t *, unsigned int *);
  Kernel kernel;
#define DMOE_ROUTE_K(KPL, PK) \
  kernel = (k == 8) ? k_route_hist<KPL, PK, 8> : (k == 2) ? k_route_hist<KPL, PK, 2> : k_route_hist<KPL, PK, 0>
#define DMOE_ROUTE(KPL)           \
  if (E % 2 == 0)                 \
    DMOE_ROUTE_K(KPL, true);      \
  else                            \
    kernel = k_route_hist<KPL, false, 0>
  if (E <= 32)
    kernel = (k == 2) ? k_route_hist<1, false, 2> : k_route_hist<1, false, 0>;
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
#undef DMOE_ROUTE_K
  return launch_pdl(kernel, tiles, kRouteThreads, smem, st, logits, T, E, k, renorm ? 1 : 0, top,
                    weights, tile_hist, flags, done);
}

cudaError_t launch_map_scan(int T, int E, int32_t *tile_hist, int32_t *tokens_per_expert,
                            int32_t *bins, int32_t *padded_bins, int32_t *num_blocks,
                            int32_t *status, cudaStream_t st, bool or_status) {
  return launch_pdl(k_map_scan, dim3((E + 31) / 32, map_segments(T)), kScanThreads, 0, st,
                    map_tiles(T), E, tile_hist, map_flags(tile_hist, T, E),
                    map_segs(tile_hist, T, E), tokens_per_expert, bins, padded_bins, num_blocks,
                    status, map_ticket(tile_hist, T, E), or_status ? 1 : 0);
}

cudaError_t launch_map_scatter(int T, int E, int k, int nblk_cap, const int32_t *top,
                               const int32_t *tile_off, const int32_t *bins,
                               const int32_t *padded_bins, int32_t *indices, int32_t *bin_ids,
                               int32_t *dest_row, int32_t *block_expert, cudaStream_t st) {
  const size_t smem = sizeof(int) * ((size_t)(kMapWarps + 4) * E + 2 * kScatEntries);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        k_map_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  // tiles per CTA: as many as the staging buffers hold while the grid keeps at least two
  // CTAs per SM (a small map keeps one tile per CTA)
  const int tiles = map_tiles(T), min_ctas = 2 * device_sm_count();
  int S = 1;
  while (2 * S * kMapTokTile * k <= kScatEntries && 2 * S <= kScanSeg &&
         tiles / (2 * S) >= min_ctas)
    S *= 2;
  return launch_pdl(k_map_scatter, (map_tiles(T) + S - 1) / S, kMapThreads, smem, st, T, E, k, S,
                    nblk_cap, top,
                    tile_off, map_segs(const_cast<int32_t *>(tile_off), T, E), bins, padded_bins,
                    indices, bin_ids, dest_row, block_expert);
}

}  // namespace dmoe
