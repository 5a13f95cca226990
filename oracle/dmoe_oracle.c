/*
 * dmoe_oracle.c -- plain, slow CPU oracle for the dropless-MoE (dMoE) expert layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU-baseline
 * leg may load this library.  It shares no code, header, table or helper with the CUDA
 * path, and the CUDA path never calls it.
 *
 * Conventions
 *   - Floating-point inputs arrive as fp32 arrays.  The layer's inputs are bf16, and widening
 *     bf16 to fp32 is exact, so the caller widens them before the call.  All arithmetic is
 *     double precision; all floating outputs are double.
 *   - Entries are flattened j = t*k + s (token t, slot s).  This is the flattening that the
 *     gather rule "source row = index_a // TOP_K" implies (MegaBlocks walkthrough,
 *     "dropless MoE and block-sparse", section 4.2).  In the forward and backward, an entry
 *     whose expert is -1 is absent (the rounded routing's unused positions).
 *   - Weights use the (out, in) layout: W1, W3 are [E, f, h]; W2 is [E, h, f].
 *   - Gated SiLU: W1 is the gate projection (passed through silu), W3 the up projection.
 *     silu(z) = z / (1 + exp(-z)).
 *
 * Every function is a direct restatement of the definition it cites; there is no blocking,
 * fusion or reordering beyond the per-token loop that the definition states.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define BLOCKING 128 /* rows per block; "self.blocking = 128" (walkthrough, section 2) */

/* ------------------------------------------------------------------------------------ */
/* Routing: top-k of softmax over all E logits.                                          */
/* ------------------------------------------------------------------------------------ */

/* Order used to pick experts: larger value first; NaN below everything (including -inf);
 * equal values (+0 and -0 included) are not "greater", so the earlier (lower) expert index
 * keeps its place.  Returns 1 when a is strictly preferred over b. */
static int preferred(double a, double b) {
  if (isnan(a)) return 0;
  if (isnan(b)) return 1;
  return a > b;
}

/* Router output (scores, top_experts) of the Fast-LLM dropless forward (issue #56 error log)
 * and the "router(x)" step of the walkthrough's schematic forward (section 4.5).
 * For each token: pick k experts by repeatedly taking the preferred remaining logit; slot s
 * holds the s-th pick.  The weight of slot s is the softmax over all E logits read at the
 * chosen expert: w = exp(l_e - m) / sum_j exp(l_j - m), m = max logit.  No renormalisation
 * over the k chosen experts -- unless renorm != 0, the routing variant in which the weights are
 * the softmax over the k chosen logits only: w = exp(l_e - m) / sum_{chosen j} exp(l_j - m),
 * so that they sum to 1.
 * logits: [T, E] (fp32 widened from bf16); top: [T, k] int32 out; w: [T, k] double out. */
int oracle_route(int T, int E, int k, int renorm, const float *logits, int32_t *top,
                 double *w) {
  if (T < 0 || E < 1 || k < 1 || k > E) return -1;
  unsigned char *chosen = (unsigned char *)malloc((size_t)E);
  if (!chosen) return -2;
  for (int t = 0; t < T; ++t) {
    const float *l = logits + (size_t)t * E;
    memset(chosen, 0, (size_t)E);
    for (int s = 0; s < k; ++s) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (chosen[e]) continue;
        if (best < 0 || preferred(l[e], l[best])) best = e;
      }
      chosen[best] = 1;
      top[(size_t)t * k + s] = best;
    }
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
      if (!isnan(l[e]) && (double)l[e] > m) m = l[e];
    double denom = 0.0;
    if (renorm)
      for (int s = 0; s < k; ++s) denom += exp((double)l[top[(size_t)t * k + s]] - m);
    else
      for (int e = 0; e < E; ++e) denom += exp((double)l[e] - m);
    for (int s = 0; s < k; ++s) {
      int e = top[(size_t)t * k + s];
      w[(size_t)t * k + s] = exp((double)l[e] - m) / denom;
    }
  }
  free(chosen);
  return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Tile-aware token rounding (SonicMoE abstract: the routing is rounded so that each       */
/* expert's token count is a multiple of the GEMM tile, removing the padding the grouped   */
/* GEMM would otherwise compute; reported 1.16x kernel time).                              */
/* ------------------------------------------------------------------------------------ */

/* One (token, logit) candidate of an expert. */
typedef struct {
  float v;
  int32_t t;
} rank_item;

/* Rank order of the rounding: the larger logit first; equal logits (+0 and -0 included)
 * -> the lower token index first; NaN last.  qsort comparator: negative when a ranks first. */
static int rank_cmp(const void *pa, const void *pb) {
  const rank_item *a = (const rank_item *)pa, *b = (const rank_item *)pb;
  if (preferred(a->v, b->v)) return -1;
  if (preferred(b->v, a->v)) return 1;
  return (a->t < b->t) ? -1 : (a->t > b->t);
}

/* The abstract gives the method in one sentence; the reading taken here:
 *   - start from the top-k routing `top` [T, k] and its counts c_e;
 *   - for every expert with r = c_e mod B != 0: round up -- add the B - r best-ranked tokens
 *     not routed to e -- when r >= B/2 and at least B - r such tokens exist; otherwise round
 *     down -- drop e's r worst-ranked entries.  So each count becomes the multiple of B
 *     nearest to it (ties upward), or the one below when too few tokens are left to add;
 *   - rank of a token for expert e: its logit l[t][e] (rank_cmp), the quantity both the
 *     softmax weight and the top-k choice are monotone in for a token;
 *   - a token keeps its surviving slots in slot order, then its added experts in increasing
 *     expert index; every entry's weight is the softmax over all E logits at its expert
 *     (as for a routed entry, no renormalisation).
 * out_top / out_w: [T, kmax] entries per token; unused positions hold expert -1, weight 0.
 * Returns the largest number of entries of a token (<= kmax), -4 if kmax is too small. */
int oracle_round_tokens(int T, int E, int k, int B, const float *logits, const int32_t *top,
                        int kmax, int32_t *out_top, double *out_w) {
  if (T < 0 || E < 1 || k < 1 || k > E || B < 1 || kmax < 1) return -1;
  const long N = (long)T * k;
  long *count = (long *)calloc((size_t)E, sizeof(long));
  unsigned char *drop = (unsigned char *)calloc((size_t)(N > 0 ? N : 1), 1);
  unsigned char *add = (unsigned char *)calloc((size_t)T * E > 0 ? (size_t)T * E : 1, 1);
  unsigned char *routed = (unsigned char *)calloc((size_t)T * E > 0 ? (size_t)T * E : 1, 1);
  rank_item *items = (rank_item *)malloc(sizeof(rank_item) * (size_t)(T > 0 ? T : 1));
  long *where = (long *)malloc(sizeof(long) * (size_t)(T > 0 ? T : 1));
  if (!count || !drop || !add || !routed || !items || !where) {
    free(count); free(drop); free(add); free(routed); free(items); free(where);
    return -2;
  }
  for (long j = 0; j < N; ++j) {
    count[top[j]] += 1;
    routed[(size_t)(j / k) * E + top[j]] = 1;
  }
  for (int e = 0; e < E; ++e) {
    const long r = count[e] % B;
    if (r == 0) continue;
    const long need = B - r;
    if (2 * r >= B && (long)T - count[e] >= need) {  /* round up */
      int n = 0;
      for (int t = 0; t < T; ++t)
        if (!routed[(size_t)t * E + e]) {
          items[n].v = logits[(size_t)t * E + e];
          items[n].t = t;
          ++n;
        }
      qsort(items, (size_t)n, sizeof(rank_item), rank_cmp);
      for (long q = 0; q < need; ++q) add[(size_t)items[q].t * E + e] = 1;
    } else {  /* round down: the r worst-ranked entries of e */
      int n = 0;
      for (long j = 0; j < N; ++j)
        if (top[j] == e) {
          items[n].v = logits[(size_t)(j / k) * E + e];
          items[n].t = (int32_t)(j / k);
          where[n] = j;
          ++n;
        }
      /* sort the positions along with the items: order indices by rank */
      for (int a = 1; a < n; ++a) { /* insertion sort keeps it plain; n is one expert's count */
        rank_item it = items[a];
        long wj = where[a];
        int b = a - 1;
        while (b >= 0 && rank_cmp(&items[b], &it) > 0) {
          items[b + 1] = items[b];
          where[b + 1] = where[b];
          --b;
        }
        items[b + 1] = it;
        where[b + 1] = wj;
      }
      for (long q = n - r; q < n; ++q) drop[where[q]] = 1;
    }
  }
  int most = 0, err = 0;
  for (int t = 0; t < T && !err; ++t) {
    const float *l = logits + (size_t)t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
      if (!isnan(l[e]) && (double)l[e] > m) m = l[e];
    double denom = 0.0;
    for (int e = 0; e < E; ++e) denom += exp((double)l[e] - m);
    int n = 0;
    for (int s = 0; s < k; ++s) {
      const long j = (long)t * k + s;
      if (drop[j]) continue;
      if (n >= kmax) { err = 1; break; }
      out_top[(size_t)t * kmax + n] = top[j];
      out_w[(size_t)t * kmax + n] = exp((double)l[top[j]] - m) / denom;
      ++n;
    }
    for (int e = 0; e < E && !err; ++e) {
      if (!add[(size_t)t * E + e]) continue;
      if (n >= kmax) { err = 1; break; }
      out_top[(size_t)t * kmax + n] = e;
      out_w[(size_t)t * kmax + n] = exp((double)l[e] - m) / denom;
      ++n;
    }
    for (int q = n; q < kmax; ++q) {
      out_top[(size_t)t * kmax + q] = -1;
      out_w[(size_t)t * kmax + q] = 0.0;
    }
    if (n > most) most = n;
  }
  free(count); free(drop); free(add); free(routed); free(items); free(where);
  return err ? -4 : most;
}

/* ------------------------------------------------------------------------------------ */
/* Sparse map (walkthrough, sections 4.1-4.3).                                           */
/* ------------------------------------------------------------------------------------ */

/* Builds, from top_experts [T*k]:
 *   counts[e]       = number of entries routed to e (histogram, tokens_per_expert)
 *   bins[e]         = inclusive cumulative sum of counts (real expert boundaries)
 *   padded_bins[e]  = inclusive cumulative sum of round_up(counts, 128) (padded boundaries)
 *   indices[i], bin_ids[i]: entries stably sorted by expert (i-th sorted entry's flattened
 *                     position and its expert)
 *   dest_row[j]     = padded row of entry j, from the three-line index math of section 4.2:
 *                     offset_in_bin = i - bins[e-1]; index_b = offset_in_bin + padded_bins[e-1]
 *                     with bins[-1] = padded_bins[-1] = 0 for e = 0
 *   block_expert[b] = expert owning 128-row block b (section 2: every 128-row block belongs
 *                     to exactly one expert), -1 for b >= num_blocks, b < nblk_cap
 *   num_blocks      = padded_bins[E-1] / 128
 * Returns -3 if an expert id is out of range. */
int oracle_sparse_map(int T, int E, int k, const int32_t *top, int32_t *counts, int32_t *bins,
                      int32_t *padded_bins, int32_t *indices, int32_t *bin_ids, int32_t *dest_row,
                      int32_t *block_expert, int nblk_cap, int32_t *num_blocks) {
  if (T < 0 || E < 1 || k < 1) return -1;
  const long N = (long)T * k;
  for (long j = 0; j < N; ++j)
    if (top[j] < 0 || top[j] >= E) return -3;

  /* histogram */
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (long j = 0; j < N; ++j) counts[top[j]] += 1;

  /* bins = inclusive cumsum(counts); padded = round_up(counts, 128);
   * padded_bins = inclusive cumsum(padded) */
  long run = 0, prun = 0;
  for (int e = 0; e < E; ++e) {
    long padded = ((counts[e] + BLOCKING - 1) / BLOCKING) * BLOCKING;
    run += counts[e];
    prun += padded;
    bins[e] = (int32_t)run;
    padded_bins[e] = (int32_t)prun;
  }

  /* stable sort of entries by expert: walk j in increasing order and append j to its
   * expert's list; the lists, concatenated in expert order, are the sorted sequence */
  long *fill = (long *)calloc((size_t)E, sizeof(long));
  if (!fill) return -2;
  for (long j = 0; j < N; ++j) {
    int e = top[j];
    long start = (e > 0) ? bins[e - 1] : 0;
    long i = start + fill[e];
    indices[i] = (int32_t)j;
    bin_ids[i] = e;
    fill[e] += 1;
  }
  free(fill);

  /* padded-row index math, one sorted entry at a time */
  for (long i = 0; i < N; ++i) {
    long index_a = indices[i];
    int bin_idx = bin_ids[i];
    long offset_in_bin = i - ((bin_idx > 0) ? bins[bin_idx - 1] : 0);
    long index_b = offset_in_bin + ((bin_idx > 0) ? padded_bins[bin_idx - 1] : 0);
    dest_row[index_a] = (int32_t)index_b;
  }

  /* block -> expert table */
  *num_blocks = padded_bins[E - 1] / BLOCKING;
  for (int b = 0; b < nblk_cap; ++b) block_expert[b] = -1;
  for (int e = 0; e < E; ++e) {
    int b0 = ((e > 0) ? padded_bins[e - 1] : 0) / BLOCKING;
    int b1 = padded_bins[e] / BLOCKING;
    for (int b = b0; b < b1 && b < nblk_cap; ++b) block_expert[b] = e;
  }
  return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Expert FFN and the forward (schematic forward, walkthrough section 4.5, with the gated   */
/* SiLU expert of the Fast-LLM config "gated: true, activation_type: silu").             */
/* ------------------------------------------------------------------------------------ */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One expert applied to one token row x (length h):
 *   a = W1_e x, b = W3_e x (length f); hh = silu(a) * b; yts = W2_e hh (length h). */
static void expert_ffn(int h, int f, const float *x, const float *W1e, const float *W3e,
                       const float *W2e, double *a, double *b, double *hh, double *yts) {
  for (int i = 0; i < f; ++i) {
    double sa = 0.0, sb = 0.0;
    const float *r1 = W1e + (size_t)i * h, *r3 = W3e + (size_t)i * h;
    for (int j = 0; j < h; ++j) {
      sa += (double)r1[j] * (double)x[j];
      sb += (double)r3[j] * (double)x[j];
    }
    a[i] = sa;
    b[i] = sb;
    hh[i] = silu(sa) * sb;
  }
  for (int o = 0; o < h; ++o) {
    double s = 0.0;
    const float *r2 = W2e + (size_t)o * f;
    for (int i = 0; i < f; ++i) s += (double)r2[i] * hh[i];
    yts[o] = s;
  }
}

/* Per-token forward: y_t = sum_s w_ts * W2_e(silu(W1_e x_t) * W3_e x_t), e = top[t*k+s].
 * Computes the tokens listed in toks[0..ntok) (toks == NULL: tokens 0..ntok-1).
 * y: [ntok, h] double out.  yts (optional, may be NULL): [ntok, k, h] per-slot expert output.
 * nthreads > 1 splits the token list over OpenMP threads (each token's arithmetic is
 * unchanged). */
int oracle_forward(int T, int h, int f, int E, int k, const float *x, const float *W1,
                   const float *W3, const float *W2, const int32_t *top, const double *w,
                   int ntok, const int32_t *toks, double *y, double *yts, int nthreads) {
  (void)T;
  int err = 0;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads) reduction(| : err)
#endif
  {
    double *a = (double *)malloc(sizeof(double) * f), *b = (double *)malloc(sizeof(double) * f);
    double *hh = (double *)malloc(sizeof(double) * f), *yo = (double *)malloc(sizeof(double) * h);
    if (!a || !b || !hh || !yo) {
      err |= 1;
    } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int n = 0; n < ntok; ++n) {
        int t = toks ? toks[n] : n;
        const float *xt = x + (size_t)t * h;
        double *yt = y + (size_t)n * h;
        for (int o = 0; o < h; ++o) yt[o] = 0.0;
        for (int s = 0; s < k; ++s) {
          int e = top[(size_t)t * k + s];
          if (e < 0) { /* no entry in this position (rounded routing) */
            if (yts)
              for (int o = 0; o < h; ++o) yts[((size_t)n * k + s) * h + o] = 0.0;
            continue;
          }
          expert_ffn(h, f, xt, W1 + (size_t)e * f * h, W3 + (size_t)e * f * h,
                     W2 + (size_t)e * h * f, a, b, hh, yo);
          double wts = w[(size_t)t * k + s];
          for (int o = 0; o < h; ++o) yt[o] += wts * yo[o];
          if (yts)
            for (int o = 0; o < h; ++o) yts[((size_t)n * k + s) * h + o] = yo[o];
        }
      }
    }
    free(a);
    free(b);
    free(hh);
    free(yo);
  }
  return err ? -2 : 0;
}

/* ------------------------------------------------------------------------------------ */
/* Backward.  The walkthrough (section 4.2) fixes the structure: the gradient of the       */
/* weighted scatter is a gather of dy plus a routing-weight gradient; the gradient of the  */
/* gather sums the k copies back into dx; section 4.4 recomputes the activation instead   */
/* of storing it.  Written per (token, slot) from the chain rule:                          */
/*   dw_ts = <dy_t, yts>;  g = w_ts dy_t;  dhh = W2_e^T g;                                  */
/*   sig = 1/(1+exp(-a));  da = dhh * b * sig * (1 + a (1 - sig));  db = dhh * silu(a);     */
/*   dx_t += W1_e^T da + W3_e^T db;                                                         */
/*   dW2_e += g hh^T;  dW1_e += da x_t^T;  dW3_e += db x_t^T.                               */
/* ------------------------------------------------------------------------------------ */

/* One (token, slot) entry's backward.  Accumulates into dx_t (length h) and, if dW1e is not
 * NULL, into dW1e/dW3e [f,h] and dW2e [h,f]; returns dw_ts. */
static double entry_backward(int h, int f, const float *xt, const float *dyt, double wts,
                             const float *W1e, const float *W3e, const float *W2e, double *a,
                             double *b, double *hh, double *yo, double *g, double *dhh,
                             double *dx_t, double *dW1e, double *dW3e, double *dW2e) {
  expert_ffn(h, f, xt, W1e, W3e, W2e, a, b, hh, yo);
  double dw = 0.0;
  for (int o = 0; o < h; ++o) dw += (double)dyt[o] * yo[o];
  for (int o = 0; o < h; ++o) g[o] = wts * (double)dyt[o];
  for (int i = 0; i < f; ++i) {
    double s = 0.0;
    for (int o = 0; o < h; ++o) s += (double)W2e[(size_t)o * f + i] * g[o];
    dhh[i] = s;
  }
  for (int i = 0; i < f; ++i) {
    double sig = 1.0 / (1.0 + exp(-a[i]));
    double da = dhh[i] * b[i] * sig * (1.0 + a[i] * (1.0 - sig));
    double db = dhh[i] * (a[i] * sig);
    const float *r1 = W1e + (size_t)i * h, *r3 = W3e + (size_t)i * h;
    for (int j = 0; j < h; ++j) dx_t[j] += da * (double)r1[j] + db * (double)r3[j];
    if (dW1e) {
      for (int j = 0; j < h; ++j) {
        dW1e[(size_t)i * h + j] += da * (double)xt[j];
        dW3e[(size_t)i * h + j] += db * (double)xt[j];
      }
    }
  }
  if (dW2e)
    for (int o = 0; o < h; ++o)
      for (int i = 0; i < f; ++i) dW2e[(size_t)o * f + i] += g[o] * hh[i];
  return dw;
}

/* Full backward over all T tokens, single-threaded (meant for small shapes).
 * dy: [T,h]; outputs dx [T,h], dW1, dW3 [E,f,h], dW2 [E,h,f], dw [T,k], all double,
 * overwritten. */
int oracle_backward(int T, int h, int f, int E, int k, const float *x, const float *dy,
                    const float *W1, const float *W3, const float *W2, const int32_t *top,
                    const double *w, double *dx, double *dW1, double *dW3, double *dW2,
                    double *dw) {
  size_t nW = (size_t)E * f * h;
  memset(dx, 0, sizeof(double) * (size_t)T * h);
  memset(dW1, 0, sizeof(double) * nW);
  memset(dW3, 0, sizeof(double) * nW);
  memset(dW2, 0, sizeof(double) * nW);
  double *buf = (double *)malloc(sizeof(double) * (size_t)(4 * f + 2 * h));
  if (!buf) return -2;
  double *a = buf, *b = a + f, *hh = b + f, *dhh = hh + f, *yo = dhh + f, *g = yo + h;
  for (int t = 0; t < T; ++t) {
    for (int s = 0; s < k; ++s) {
      int e = top[(size_t)t * k + s];
      if (e < 0) { /* no entry in this position (rounded routing) */
        dw[(size_t)t * k + s] = 0.0;
        continue;
      }
      dw[(size_t)t * k + s] = entry_backward(
          h, f, x + (size_t)t * h, dy + (size_t)t * h, w[(size_t)t * k + s],
          W1 + (size_t)e * f * h, W3 + (size_t)e * f * h, W2 + (size_t)e * h * f, a, b, hh, yo,
          g, dhh, dx + (size_t)t * h, dW1 + (size_t)e * f * h, dW3 + (size_t)e * f * h,
          dW2 + (size_t)e * h * f);
    }
  }
  free(buf);
  return 0;
}

/* Token-sampled backward: dx_t [ntok,h] and dw [ntok,k] for the listed tokens only (the
 * weight gradients are not touched).  Parallel over the token list. */
int oracle_backward_tokens(int T, int h, int f, int E, int k, const float *x, const float *dy,
                           const float *W1, const float *W3, const float *W2,
                           const int32_t *top, const double *w, int ntok, const int32_t *toks,
                           double *dx, double *dw, int nthreads) {
  (void)T;
  (void)E;
  int err = 0;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads) reduction(| : err)
#endif
  {
    double *buf = (double *)malloc(sizeof(double) * (size_t)(4 * f + 2 * h));
    if (!buf) {
      err |= 1;
    } else {
      double *a = buf, *b = a + f, *hh = b + f, *dhh = hh + f, *yo = dhh + f, *g = yo + h;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int n = 0; n < ntok; ++n) {
        int t = toks[n];
        double *dxt = dx + (size_t)n * h;
        for (int j = 0; j < h; ++j) dxt[j] = 0.0;
        for (int s = 0; s < k; ++s) {
          int e = top[(size_t)t * k + s];
          if (e < 0) { /* no entry in this position (rounded routing) */
            dw[(size_t)n * k + s] = 0.0;
            continue;
          }
          dw[(size_t)n * k + s] = entry_backward(
              h, f, x + (size_t)t * h, dy + (size_t)t * h, w[(size_t)t * k + s],
              W1 + (size_t)e * f * h, W3 + (size_t)e * f * h, W2 + (size_t)e * h * f, a, b,
              hh, yo, g, dhh, dxt, NULL, NULL, NULL);
        }
      }
      free(buf);
    }
  }
  return err ? -2 : 0;
}

/* Single elements of the weight gradients, each summed over every entry routed to its
 * expert (entries visited in increasing j):
 *   which 1: dW1[e][r][c] = sum da_ts[r] x_t[c]
 *   which 3: dW3[e][r][c] = sum db_ts[r] x_t[c]
 *   which 2: dW2[e][r][c] = sum g_ts[r] hh_ts[c]   (r in [0,h), c in [0,f))
 * q: [nq, 4] int32 rows (which, e, r, c); out: [nq] double.  Parallel over the queries. */
int oracle_wgrad_elements(int T, int h, int f, int E, int k, const float *x, const float *dy,
                          const float *W1, const float *W3, const float *W2,
                          const int32_t *top, const double *w, int nq, const int32_t *q,
                          double *out, int nthreads) {
  (void)E;
  long N = (long)T * k;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
#endif
  for (int n = 0; n < nq; ++n) {
    int which = q[4 * n], e = q[4 * n + 1], r = q[4 * n + 2], c = q[4 * n + 3];
    const float *W1e = W1 + (size_t)e * f * h, *W3e = W3 + (size_t)e * f * h;
    const float *W2e = W2 + (size_t)e * h * f;
    double acc = 0.0;
    for (long j = 0; j < N; ++j) {
      if (top[j] != e) continue;
      long t = j / k;
      const float *xt = x + (size_t)t * h, *dyt = dy + (size_t)t * h;
      double wts = w[j];
      if (which == 2) {
        /* hh_ts[c] = silu(a[c]) * b[c] */
        double sa = 0.0, sb = 0.0;
        for (int jj = 0; jj < h; ++jj) {
          sa += (double)W1e[(size_t)c * h + jj] * (double)xt[jj];
          sb += (double)W3e[(size_t)c * h + jj] * (double)xt[jj];
        }
        acc += wts * (double)dyt[r] * (silu(sa) * sb);
      } else {
        /* a[r], b[r], dhh[r] = sum_o W2e[o][r] g[o] */
        double sa = 0.0, sb = 0.0, d = 0.0;
        for (int jj = 0; jj < h; ++jj) {
          sa += (double)W1e[(size_t)r * h + jj] * (double)xt[jj];
          sb += (double)W3e[(size_t)r * h + jj] * (double)xt[jj];
        }
        for (int o = 0; o < h; ++o) d += (double)W2e[(size_t)o * f + r] * (wts * (double)dyt[o]);
        double sig = 1.0 / (1.0 + exp(-sa));
        double grad = (which == 1) ? d * sb * sig * (1.0 + sa * (1.0 - sig)) : d * (sa * sig);
        acc += grad * (double)xt[c];
      }
    }
    out[n] = acc;
  }
  return 0;
}

/* The three weight-gradient slabs of one expert e, summed over every entry routed to it
 * (entries visited in increasing j, the chain rule of entry_backward):
 *   dW1e[r][c] = sum da_ts[r] x_t[c],  dW3e[r][c] = sum db_ts[r] x_t[c]   ([f, h])
 *   dW2e[r][c] = sum g_ts[r] hh_ts[c]                                      ([h, f])
 * The per-entry vectors (da, db, hh, g) of a chunk of entries are formed first (parallel over
 * the entries), then added to the slabs (parallel over slab rows, entries in order), so every
 * slab element is the same ordered sum whatever the thread count.  Outputs double,
 * overwritten. */
int oracle_wgrad_expert(int T, int h, int f, int E, int k, const float *x, const float *dy,
                        const float *W1, const float *W3, const float *W2, const int32_t *top,
                        const double *w, int e, double *dW1e, double *dW3e, double *dW2e,
                        int nthreads) {
  if (e < 0 || e >= E) return -1;
  const long N = (long)T * k;
  const int CH = 512; /* entries per chunk */
  const float *W1e = W1 + (size_t)e * f * h, *W3e = W3 + (size_t)e * f * h;
  const float *W2e = W2 + (size_t)e * h * f;
  long *ent = (long *)malloc(sizeof(long) * (size_t)(N > 0 ? N : 1));
  double *da = (double *)malloc(sizeof(double) * (size_t)CH * f);
  double *db = (double *)malloc(sizeof(double) * (size_t)CH * f);
  double *hh = (double *)malloc(sizeof(double) * (size_t)CH * f);
  double *g = (double *)malloc(sizeof(double) * (size_t)CH * h);
  if (!ent || !da || !db || !hh || !g) {
    free(ent); free(da); free(db); free(hh); free(g);
    return -2;
  }
  long n = 0;
  for (long j = 0; j < N; ++j)
    if (top[j] == e) ent[n++] = j;
  memset(dW1e, 0, sizeof(double) * (size_t)f * h);
  memset(dW3e, 0, sizeof(double) * (size_t)f * h);
  memset(dW2e, 0, sizeof(double) * (size_t)h * f);
  if (nthreads < 1) nthreads = 1;
  for (long c0 = 0; c0 < n; c0 += CH) {
    const int m = (int)((n - c0 < CH) ? n - c0 : CH);
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
#endif
    for (int q = 0; q < m; ++q) {
      const long j = ent[c0 + q];
      const long t = j / k;
      const float *xt = x + (size_t)t * h, *dyt = dy + (size_t)t * h;
      double *gq = g + (size_t)q * h;
      for (int o = 0; o < h; ++o) gq[o] = w[j] * (double)dyt[o];
      for (int i = 0; i < f; ++i) {
        double sa = 0.0, sb = 0.0, d = 0.0;
        const float *r1 = W1e + (size_t)i * h, *r3 = W3e + (size_t)i * h;
        for (int jj = 0; jj < h; ++jj) {
          sa += (double)r1[jj] * (double)xt[jj];
          sb += (double)r3[jj] * (double)xt[jj];
        }
        for (int o = 0; o < h; ++o) d += (double)W2e[(size_t)o * f + i] * gq[o];
        const double sig = 1.0 / (1.0 + exp(-sa));
        da[(size_t)q * f + i] = d * sb * sig * (1.0 + sa * (1.0 - sig));
        db[(size_t)q * f + i] = d * (sa * sig);
        hh[(size_t)q * f + i] = silu(sa) * sb;
      }
    }
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads) schedule(static)
#endif
    for (int r = 0; r < f + h; ++r) {
      for (int q = 0; q < m; ++q) {
        const long t = ent[c0 + q] / k;
        if (r < f) { /* row r of dW1e and dW3e */
          const float *xt = x + (size_t)t * h;
          const double a1 = da[(size_t)q * f + r], a3 = db[(size_t)q * f + r];
          double *o1 = dW1e + (size_t)r * h, *o3 = dW3e + (size_t)r * h;
          for (int c = 0; c < h; ++c) {
            o1[c] += a1 * (double)xt[c];
            o3[c] += a3 * (double)xt[c];
          }
        } else { /* row r - f of dW2e */
          const int o = r - f;
          const double go = g[(size_t)q * h + o];
          double *o2 = dW2e + (size_t)o * f;
          const double *hq = hh + (size_t)q * f;
          for (int c = 0; c < f; ++c) o2[c] += go * hq[c];
        }
      }
    }
  }
  free(ent); free(da); free(db); free(hh); free(g);
  return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Router GEMM and the gradient through the routing weights.                             */
/* ------------------------------------------------------------------------------------ */

/* Router scores: the "router(x)" step of the walkthrough's schematic forward (section 4.5)
 * whose output the issue's error log shows as (scores, top_experts).  The pages fix only that
 * output; the plainest reading is a linear router without bias:
 *   logits[t][e] = sum_i x[t][i] * Wr[e][i],   Wr [E, h] in the (out, in) layout.
 * tokens: n token ids, or NULL for all T tokens (then n = T).  out: [n, E] double. */
int oracle_router_logits(int T, int h, int E, const float *x, const float *Wr, int n,
                         const int32_t *tokens, double *out, int threads) {
  if (T < 0 || h < 1 || E < 1 || n < 0) return -1;
  if (!tokens && n != T) return -1;
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic, 4) if (threads > 1)
#endif
  for (int q = 0; q < n; ++q) {
    const int t = tokens ? tokens[q] : q;
    const float *xt = x + (size_t)t * h;
    for (int e = 0; e < E; ++e) {
      const float *we = Wr + (size_t)e * h;
      double acc = 0.0;
      for (int i = 0; i < h; ++i) acc += (double)xt[i] * (double)we[i];
      out[(size_t)q * E + e] = acc;
    }
  }
  (void)threads;
  return 0;
}

/* Gradient through the routing weights of oracle_route; the choice of experts is piecewise
 * constant, so it carries no gradient.  With j_s = top[t][s] and p_t the softmax of logits_t
 * over all E experts (renorm == 0), or over the k chosen experts only, zero elsewhere
 * (renorm != 0):
 *   w_ts = p_t[j_s],   d w_ts / d l_ti = p_t[j_s] * ([i == j_s] - p_t[i]),
 *   dlogits[t][i] = sum_s dw[t][s] * d w_ts / d l_ti                       (chain rule),
 * and, through logits = x Wr^T,
 *   dx_r[t][c] = sum_e dlogits[t][e] * Wr[e][c],   dWr[e][c] = sum_t dlogits[t][e] * x[t][c].
 * logits [T, E] are the routed scores (fp32 widened from bf16), dw [T, k] double.
 * dlogits: [T, E] double out (always computed).
 * dx_r: [n_tok, h] for tokens (NULL = all T, n_tok = T); skipped when dx_r is NULL.
 * dWr: one value per (e, c) pair of `elems` ([n_el, 2] int32), or the full [E, h] when elems
 *      is NULL; skipped when dWr is NULL. */
int oracle_router_backward(int T, int h, int E, int k, int renorm, const float *x,
                           const float *Wr, const float *logits, const int32_t *top,
                           const double *dw,
                           double *dlogits, int n_tok, const int32_t *tokens, double *dx_r,
                           int n_el, const int32_t *elems, double *dWr, int threads) {
  if (T < 0 || h < 1 || E < 1 || k < 1 || k > E) return -1;
  if (!tokens && dx_r && n_tok != T) return -1;
  double *prob = (double *)malloc(sizeof(double) * (size_t)E);
  if (!prob) return -2;
  for (int t = 0; t < T; ++t) {
    const float *l = logits + (size_t)t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
      if ((double)l[e] > m) m = (double)l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) prob[e] = renorm ? 0.0 : exp((double)l[e] - m);
    if (renorm)
      for (int s = 0; s < k; ++s) {
        const int j = top[(size_t)t * k + s];
        if (j >= 0 && j < E) prob[j] = exp((double)l[j] - m);
      }
    for (int e = 0; e < E; ++e) z += prob[e];
    for (int e = 0; e < E; ++e) prob[e] /= z;
    for (int i = 0; i < E; ++i) {
      double g = 0.0;
      for (int s = 0; s < k; ++s) {
        const int j = top[(size_t)t * k + s];
        if (j < 0 || j >= E) continue;
        g += dw[(size_t)t * k + s] * prob[j] * ((i == j ? 1.0 : 0.0) - prob[i]);
      }
      dlogits[(size_t)t * E + i] = g;
    }
  }
  free(prob);
  if (dx_r) {
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic, 4) if (threads > 1)
#endif
    for (int q = 0; q < n_tok; ++q) {
      const int t = tokens ? tokens[q] : q;
      for (int c = 0; c < h; ++c) {
        double acc = 0.0;
        for (int e = 0; e < E; ++e) acc += dlogits[(size_t)t * E + e] * (double)Wr[(size_t)e * h + c];
        dx_r[(size_t)q * h + c] = acc;
      }
    }
  }
  if (dWr) {
    const int n = elems ? n_el : E * h;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic, 16) if (threads > 1)
#endif
    for (int q = 0; q < n; ++q) {
      const int e = elems ? elems[2 * q] : q / h;
      const int c = elems ? elems[2 * q + 1] : q % h;
      double acc = 0.0;
      for (int t = 0; t < T; ++t) acc += dlogits[(size_t)t * E + e] * (double)x[(size_t)t * h + c];
      dWr[q] = acc;
    }
  }
  (void)threads;
  return 0;
}

/* Number of OpenMP threads this build can use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
