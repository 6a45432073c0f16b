/*
 * oracle_moe.c -- plain, slow, fp64 CPU reference for one routed MoE FFN layer
 * whose experts are stored as 2-bit (Q2) blocks.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity oracle: only the test
 * suite, the package smoke check and the bench's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (per token t, independently):
 *   1. W[r][c] = d(r, c/32) * (q(r,c) - 1)                 Q2 "affine, bias = -1" codebook
 *      (devlabs page, section 4 "验证方法", second layer: the Q2_0 -> S2
 *       round-trip reports codebook=affine bias=-1, bit-exact)
 *   2. logit[e] = sum_h x[h] * Wr[e][h] + bias[e]          router
 *   3. S = the top_k experts by logit, ties to the lower expert index
 *      (each token goes to 10 of 512 routed experts: devlabs page, section 1;
 *       Strata tuning page, section 2 model table)
 *   4. w[e] = exp(logit[e] - max) / sum_{e' in S} exp(logit[e'] - max)
 *   5. E_e(x) = Wd_e (silu(Wg_e x) * (Wu_e x)),  silu(z) = z / (1 + exp(-z))
 *   6. y = E_shared(x) + sum_{e in S} w[e] E_e(x)          (plus 1 shared expert,
 *      Strata tuning page, section 2 model table)
 *   7. (a stack of layers, orc_stack) r <- r + layer(bf16(RMSNorm(r))), r in binary64
 * Everything is computed in binary64 with no intermediate rounding (the one
 * exception: a stacked layer's input is rounded to bf16, the layer's input type).  Steps the
 * pages leave open (block bit layout, softmax placement, tie rule, shared-expert
 * weight, SwiGLU form) follow the readings listed in the design notes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "oracle_moe.h"

/* ---------- scalar decoding ---------------------------------------------- */

/* IEEE 754 binary16 -> binary64, written from the format's definition. */
double orc_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 0x1f;
  int mant = h & 0x3ff;
  double v;
  if (expo == 0) {
    v = ldexp((double)mant, -24);             /* subnormal: mant * 2^-24 */
  } else if (expo == 31) {
    v = mant ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + mant), expo - 25); /* (1 + mant/2^10) * 2^(expo-15) */
  }
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double orc_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* binary64 -> bfloat16, round to nearest even, written from the format:
 * keep 8 significant bits.  Finite, normal-range inputs only (what the stack
 * produces); returns the bit pattern. */
uint16_t orc_double_to_bf16(double v) {
  if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
  int sign = v < 0;
  double a = fabs(v);
  int e;
  double m = frexp(a, &e);                    /* a = m * 2^e, m in [0.5, 1) */
  double scaled = ldexp(m, 8);                /* 8 significant bits -> [128, 256) */
  double fl = floor(scaled);
  double rem = scaled - fl;
  if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
  double r = ldexp(fl, e - 8);
  float f = (float)r;                         /* exact: r has 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint16_t bits = (uint16_t)(u >> 16);
  return sign ? (uint16_t)(bits | 0x8000) : bits;
}

void orc_double_to_bf16_array(size_t n, const double *v, uint16_t *out) {
  for (size_t i = 0; i < n; ++i) out[i] = orc_double_to_bf16(v[i]);
}

/* ---------- Q2 blocks ------------------------------------------------------ */

/* One canonical 10-byte block -> 32 weights.  Element j sits in byte j>>2 of
 * the code bytes at bit offset 2*(j&3); the weight is d * (q - 1). */
void orc_dequant_block(const uint8_t *blk, double *w) {
  uint16_t dbits = (uint16_t)(blk[0] | ((uint16_t)blk[1] << 8));
  double d = orc_half_to_double(dbits);
  for (int j = 0; j < ORC_QBLOCK; ++j) {
    int q = (blk[2 + (j >> 2)] >> (2 * (j & 3))) & 3;
    w[j] = d * (double)(q - 1);
  }
}

/* Dense dequantisation of a [rows x cols] Q2 matrix (blocks along cols). */
void orc_dequant_matrix(const uint8_t *blocks, int rows, int cols, double *W) {
  int nb = cols / ORC_QBLOCK;
  for (int r = 0; r < rows; ++r)
    for (int b = 0; b < nb; ++b)
      orc_dequant_block(blocks + ((size_t)r * nb + b) * ORC_QBLOCK_BYTES, W + (size_t)r * cols + (size_t)b * ORC_QBLOCK);
}

/* y[r] = sum_c W[r][c] v[c] for one Q2 matrix, decoding each block on the fly. */
static void q2_matvec(const uint8_t *blocks, int rows, int cols, const double *v, double *y) {
  int nb = cols / ORC_QBLOCK;
  double w[ORC_QBLOCK];
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int b = 0; b < nb; ++b) {
      orc_dequant_block(blocks + ((size_t)r * nb + b) * ORC_QBLOCK_BYTES, w);
      for (int j = 0; j < ORC_QBLOCK; ++j) acc += w[j] * v[(size_t)b * ORC_QBLOCK + j];
    }
    y[r] = acc;
  }
}

size_t orc_expert_bytes(int hidden, int inter) {
  return (size_t)3 * hidden * inter / ORC_QBLOCK * ORC_QBLOCK_BYTES;
}

double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* SwiGLU expert: gate [I x H], up [I x H], down [H x I], stored back to back. */
void orc_expert_forward(int hidden, int inter, const uint8_t *expert, const double *x, double *y) {
  size_t mat_gu = (size_t)inter * hidden / ORC_QBLOCK * ORC_QBLOCK_BYTES;
  const uint8_t *gate = expert;
  const uint8_t *up = expert + mat_gu;
  const uint8_t *down = expert + 2 * mat_gu;
  double *g = (double *)malloc(sizeof(double) * inter);
  double *u = (double *)malloc(sizeof(double) * inter);
  double *h = (double *)malloc(sizeof(double) * inter);
  q2_matvec(gate, inter, hidden, x, g);
  q2_matvec(up, inter, hidden, x, u);
  for (int i = 0; i < inter; ++i) h[i] = orc_silu(g[i]) * u[i];
  q2_matvec(down, hidden, inter, h, y);
  free(g);
  free(u);
  free(h);
}

/* ---------- routing -------------------------------------------------------- */

typedef struct {
  double v;
  int e;
} keyed;

/* Order: larger logit first; equal logits -> lower expert index first. */
static int by_logit_desc(const void *a, const void *b) {
  const keyed *x = (const keyed *)a, *y = (const keyed *)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->e > y->e) - (x->e < y->e);
}

/* Top-k of one token's logits by a full sort, then the softmax over the
 * selected set (equal to the full softmax renormalised over the set). */
void orc_topk_one(const double *logits, int n_experts, int top_k, int32_t *idx, double *w, double *gap) {
  keyed *all = (keyed *)malloc(sizeof(keyed) * n_experts);
  for (int e = 0; e < n_experts; ++e) {
    all[e].v = logits[e];
    all[e].e = e;
  }
  qsort(all, n_experts, sizeof(keyed), by_logit_desc);
  double mx = all[0].v, sum = 0.0;
  for (int j = 0; j < top_k; ++j) {
    idx[j] = all[j].e;
    w[j] = exp(all[j].v - mx);
    sum += w[j];
  }
  for (int j = 0; j < top_k; ++j) w[j] /= sum;
  if (gap) *gap = (top_k < n_experts) ? all[top_k - 1].v - all[top_k].v : INFINITY;
  free(all);
}

/* Softmax over an externally chosen set (used when the caller fixes the set). */
static void weights_for_set(const double *logits, int top_k, const int32_t *sel, double *w) {
  double mx = -INFINITY, sum = 0.0;
  for (int j = 0; j < top_k; ++j) mx = logits[sel[j]] > mx ? logits[sel[j]] : mx;
  for (int j = 0; j < top_k; ++j) {
    w[j] = exp(logits[sel[j]] - mx);
    sum += w[j];
  }
  for (int j = 0; j < top_k; ++j) w[j] /= sum;
}

void orc_logits_one(int hidden, int n_experts, const double *x, const float *router_w, const float *router_b,
                    double *logits) {
  for (int e = 0; e < n_experts; ++e) {
    double acc = 0.0;
    const float *row = router_w + (size_t)e * hidden;
    for (int h = 0; h < hidden; ++h) acc += x[h] * (double)row[h];
    logits[e] = acc + (router_b ? (double)router_b[e] : 0.0);
  }
}

int orc_route(int hidden, int n_experts, int top_k, int tokens, const uint16_t *x_bf16, const float *router_w,
              const float *router_b, int32_t *idx, double *w, double *gap, double *logits_out) {
  if (top_k < 1 || top_k > n_experts || hidden % ORC_QBLOCK) return 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < tokens; ++t) {
    double *x = (double *)malloc(sizeof(double) * hidden);
    double *lg = (double *)malloc(sizeof(double) * n_experts);
    for (int h = 0; h < hidden; ++h) x[h] = orc_bf16_to_double(x_bf16[(size_t)t * hidden + h]);
    orc_logits_one(hidden, n_experts, x, router_w, router_b, lg);
    orc_topk_one(lg, n_experts, top_k, idx + (size_t)t * top_k, w + (size_t)t * top_k, gap ? gap + t : NULL);
    if (logits_out) memcpy(logits_out + (size_t)t * n_experts, lg, sizeof(double) * n_experts);
    free(x);
    free(lg);
  }
  return 0;
}

/* ---------- the layer ------------------------------------------------------ */

int orc_layer(int hidden, int inter, int n_experts, int top_k, int tokens, const uint16_t *x_bf16,
              const float *router_w, const float *router_b, const uint8_t *experts, const uint8_t *shared,
              const int32_t *forced_idx, double *y, int32_t *idx_out, double *w_out, double *gap_out) {
  if (top_k < 1 || top_k > n_experts || hidden % ORC_QBLOCK || inter % ORC_QBLOCK) return 1;
  size_t ebytes = orc_expert_bytes(hidden, inter);
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < tokens; ++t) {
    double *x = (double *)malloc(sizeof(double) * hidden);
    double *lg = (double *)malloc(sizeof(double) * n_experts);
    double *ye = (double *)malloc(sizeof(double) * hidden);
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * top_k);
    double *wt = (double *)malloc(sizeof(double) * top_k);
    double g = INFINITY;
    for (int h = 0; h < hidden; ++h) x[h] = orc_bf16_to_double(x_bf16[(size_t)t * hidden + h]);
    orc_logits_one(hidden, n_experts, x, router_w, router_b, lg);
    orc_topk_one(lg, n_experts, top_k, sel, wt, &g);
    if (forced_idx) {
      memcpy(sel, forced_idx + (size_t)t * top_k, sizeof(int32_t) * top_k);
      weights_for_set(lg, top_k, sel, wt);
    }
    double *yt = y + (size_t)t * hidden;
    orc_expert_forward(hidden, inter, shared, x, yt); /* shared expert, weight 1 */
    for (int j = 0; j < top_k; ++j) {
      orc_expert_forward(hidden, inter, experts + (size_t)sel[j] * ebytes, x, ye);
      for (int h = 0; h < hidden; ++h) yt[h] += wt[j] * ye[h];
    }
    if (idx_out) memcpy(idx_out + (size_t)t * top_k, sel, sizeof(int32_t) * top_k);
    if (w_out) memcpy(w_out + (size_t)t * top_k, wt, sizeof(double) * top_k);
    if (gap_out) gap_out[t] = g;
    free(x);
    free(lg);
    free(ye);
    free(sel);
    free(wt);
  }
  return 0;
}

/* RMSNorm with unit gain: v / sqrt(mean(v^2) + eps), one row of length n. */
void orc_rmsnorm(int n, const double *v, double eps, double *out) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += v[i] * v[i];
  double r = 1.0 / sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) out[i] = v[i] * r;
}

/* ---------- a stack of layers ------------------------------------------------
 * The pages' model runs 48 such layers one after another (Strata tuning page,
 * section 2 model table); between layers the stack keeps a residual stream and
 * normalises the layer input (unit-gain RMSNorm, eps given):
 *   r_0 = x
 *   for l = 0 .. L-1:  u_l = bf16(RMSNorm(r_l));  r_{l+1} = r_l + layer_l(u_l)
 * The residual r stays in binary64 here; the layer input u_l is rounded to
 * bfloat16 (nearest even) because the layer consumes bf16 activations.  Each
 * layer routes u_l exactly as orc_layer does.
 * follow_idx (nullable, [L][tokens][top_k]): a routing made elsewhere.  Where
 * its set for (layer, token) differs from this oracle's own and the oracle's
 * k-th/(k+1)-th logit gap is below tie_gap, the stack takes that set (weights
 * = softmax over its logits) so that both sides stay on one trajectory; such
 * (layer, token) pairs are counted in *n_followed.  Where the sets differ with
 * a larger gap the oracle keeps its own set and counts the pair in
 * *n_mismatch.  idx_out [L][tokens][top_k] and gap_out [L][tokens] (nullable)
 * receive the routing actually used and the oracle's own gap.
 * resid_in (nullable, [tokens][hidden]): start from this residual instead of
 * x (so that a long stack can be run a few layers at a time; the layers of
 * one token run in order either way, so the result is the same). */
int orc_stack(int hidden, int inter, int n_experts, int top_k, int n_layers, int tokens, const uint16_t *x_bf16,
              const double *resid_in,
              const float *const *router_w, const float *const *router_b, const uint8_t *const *experts,
              const uint8_t *const *shared, double eps, const int32_t *follow_idx, double tie_gap, double *resid,
              int32_t *idx_out, double *gap_out, int *n_followed, int *n_mismatch) {
  if (top_k < 1 || top_k > n_experts || hidden % ORC_QBLOCK || inter % ORC_QBLOCK || n_layers < 0) return 1;
  size_t ebytes = orc_expert_bytes(hidden, inter);
  int followed = 0, mismatch = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : followed, mismatch)
  for (int t = 0; t < tokens; ++t) {
    double *r = resid + (size_t)t * hidden;
    double *v = (double *)malloc(sizeof(double) * hidden);
    double *u = (double *)malloc(sizeof(double) * hidden);
    double *lg = (double *)malloc(sizeof(double) * n_experts);
    double *y = (double *)malloc(sizeof(double) * hidden);
    double *ye = (double *)malloc(sizeof(double) * hidden);
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * top_k);
    double *wt = (double *)malloc(sizeof(double) * top_k);
    for (int h = 0; h < hidden; ++h)
      r[h] = resid_in ? resid_in[(size_t)t * hidden + h] : orc_bf16_to_double(x_bf16[(size_t)t * hidden + h]);
    for (int l = 0; l < n_layers; ++l) {
      orc_rmsnorm(hidden, r, eps, v);
      for (int h = 0; h < hidden; ++h) u[h] = orc_bf16_to_double(orc_double_to_bf16(v[h]));
      double g = INFINITY;
      orc_logits_one(hidden, n_experts, u, router_w[l], router_b ? router_b[l] : NULL, lg);
      orc_topk_one(lg, n_experts, top_k, sel, wt, &g);
      if (follow_idx) {
        const int32_t *f = follow_idx + ((size_t)l * tokens + t) * top_k;
        int same = 1;
        for (int j = 0; j < top_k && same; ++j) {
          int found = 0;
          for (int i = 0; i < top_k; ++i) found |= f[i] == sel[j];
          same = found;
        }
        if (!same) {
          if (g < tie_gap) {
            memcpy(sel, f, sizeof(int32_t) * top_k);
            weights_for_set(lg, top_k, sel, wt);
            ++followed;
          } else {
            ++mismatch;
          }
        }
      }
      orc_expert_forward(hidden, inter, shared[l], u, y); /* shared expert, weight 1 */
      for (int j = 0; j < top_k; ++j) {
        orc_expert_forward(hidden, inter, experts[l] + (size_t)sel[j] * ebytes, u, ye);
        for (int h = 0; h < hidden; ++h) y[h] += wt[j] * ye[h];
      }
      for (int h = 0; h < hidden; ++h) r[h] += y[h];
      if (idx_out) memcpy(idx_out + ((size_t)l * tokens + t) * top_k, sel, sizeof(int32_t) * top_k);
      if (gap_out) gap_out[(size_t)l * tokens + t] = g;
    }
    free(v);
    free(u);
    free(lg);
    free(y);
    free(ye);
    free(sel);
    free(wt);
  }
  if (n_followed) *n_followed = followed;
  if (n_mismatch) *n_mismatch = mismatch;
  return 0;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads the oracle's token loops use from now on (n < 1: all host threads). */
void orc_set_num_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n >= 1 ? n : omp_get_num_procs());
#else
  (void)n;
#endif
}
