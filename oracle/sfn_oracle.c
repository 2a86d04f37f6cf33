/*
 * sfn_oracle.c -- plain fp64 CPU oracle for the predictor-gated bank-wise
 * top-k sparse SwiGLU FFN forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library and its Python binding) never calls it and shares no code with
 * it.
 *
 * Source: "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity
 * Training Recipe for Dense-to-Sparse LLMs" (arXiv 2606.10722), as summarised
 * on gist.science, section "Methodologie / 1. Architectuur: Predictor-Gated
 * Sparse SwiGLU" (predictor R^d -> R^448 -> R^{d_i}; banks of 64 with a hard
 * top-16; hard binary mask, inactive channels exactly zero) and section
 * "3. Hardware Implicaties" (gate, up and down all skip inactive channels).
 *
 * Everything here is the plain definition written out with double-precision
 * loops in the order the method states it; no blocking, fusion or
 * reordering.  Inputs are widened exactly to double from their stored type
 * (f64, f32 or bf16), so the oracle sees the same numbers the GPU sees.
 *
 * Readings of points the pages leave open (each is also listed in the design
 * notes of the repository):
 *   - predictor is a plain linear factorisation p = B (A x), no bias, no
 *     inner activation;
 *   - the predictor's logits take the place of the dense SwiGLU gate's
 *     sigma: silu(g) = g*sigma(g) becomes g*sigma(p), so a_j = sigma(p_j) * g_j * u_j with
 *     g_j = Wg[j].x and u_j = Wu[j].x;
 *   - banks are contiguous index ranges [b*bank, (b+1)*bank);
 *   - ranking is on p (not sigma(p)); equal logits go to the lower index;
 *     +0 and -0 are equal; NaN ranks below every number (including -inf),
 *     and NaNs among themselves go to the lower index;
 *   - y = sum_j a_j * W_down[:, j]; the column j of W_down is stored as the
 *     contiguous row j of Wd ([d_i][d], channel-major).
 *
 * OpenMP parallelises over tokens only (tokens are independent); every
 * token's arithmetic is sequential and deterministic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SFN_ORACLE_F64 0
#define SFN_ORACLE_F32 1
#define SFN_ORACLE_BF16 2

/* Exact widening of one stored element to double. */
static double ld(const void *p, int dtype, int64_t i) {
  if (dtype == SFN_ORACLE_F64) return ((const double *)p)[i];
  if (dtype == SFN_ORACLE_F32) return (double)((const float *)p)[i];
  /* bf16: the upper 16 bits of an IEEE binary32 value */
  uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Logistic sigma(z) = 1 / (1 + e^{-z}), evaluated on the side that does not
 * overflow. */
double sfn_oracle_sigmoid(double z) {
  if (z >= 0.0) return 1.0 / (1.0 + exp(-z));
  double e = exp(z);
  return e / (1.0 + e);
}

/* Predictor, a two-layer map R^d -> R^448 -> R^{d_i}:  h = A x  (A is [r][d]),  p = B h
 * (B is [d_i][r]).  logits is [T][d_i] double. */
void sfn_oracle_predict(const void *x, int x_dt, const void *A, int A_dt,
                        const void *B, int B_dt, int64_t T, int d, int d_i,
                        int r, double *logits) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    double *h = (double *)malloc(sizeof(double) * (size_t)r);
    for (int m = 0; m < r; ++m) {
      double s = 0.0;
      for (int n = 0; n < d; ++n)
        s += ld(A, A_dt, (int64_t)m * d + n) * ld(x, x_dt, t * d + n);
      h[m] = s;
    }
    for (int j = 0; j < d_i; ++j) {
      double s = 0.0;
      for (int m = 0; m < r; ++m) s += ld(B, B_dt, (int64_t)j * r + m) * h[m];
      logits[t * d_i + j] = s;
    }
    free(h);
  }
}

/* "a beats b" in the bank ranking: larger value first; NaN below all. */
static int beats(double a, double b) {
  if (isnan(a)) return 0;
  if (isnan(b)) return 1;
  return a > b;
}
static int same(double a, double b) {
  if (isnan(a) && isnan(b)) return 1;
  return a == b; /* +0 == -0 */
}

/* Bank-wise hard top-k: in every bank of `bank` consecutive channels keep the
 * k channels of highest logit.  rank_j = #{i in bank : p_i beats p_j, or
 * p_i equals p_j and i < j};  channel j is kept iff rank_j < k.
 * mask is [T][d_i/bank] uint64; bit i of word b is channel b*bank + i. */
void sfn_oracle_bank_topk(const double *logits, int64_t T, int d_i, int bank,
                          int k, uint64_t *mask) {
  int nb = d_i / bank;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int b = 0; b < nb; ++b) {
      const double *p = logits + t * d_i + (int64_t)b * bank;
      uint64_t word = 0;
      for (int j = 0; j < bank; ++j) {
        int rank = 0;
        for (int i = 0; i < bank; ++i)
          if (beats(p[i], p[j]) || (same(p[i], p[j]) && i < j)) ++rank;
        if (rank < k) word |= (uint64_t)1 << j;
      }
      mask[t * nb + b] = word;
    }
  }
}

/* Sparse gate/up/down given the mask: for every kept channel j,
 *   g_j = Wg[j] . x,  u_j = Wu[j] . x,  a_j = sigma(p_j) g_j u_j,
 * and y = sum_{kept j} a_j Wd[j, :].  Unkept channels contribute exactly
 * nothing (they are never touched).  y is [T][d] double. */
void sfn_oracle_forward_given_mask(const void *x, int x_dt,
                                   const double *logits, const uint64_t *mask,
                                   const void *Wg, int Wg_dt, const void *Wu,
                                   int Wu_dt, const void *Wd, int Wd_dt,
                                   int64_t T, int d, int d_i, int bank,
                                   double *y) {
  int nb = d_i / bank;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    double *yt = y + t * d;
    for (int n = 0; n < d; ++n) yt[n] = 0.0;
    for (int j = 0; j < d_i; ++j) {
      uint64_t word = mask[t * nb + j / bank];
      if (!((word >> (j % bank)) & 1)) continue;
      double g = 0.0, u = 0.0;
      for (int n = 0; n < d; ++n) {
        double xn = ld(x, x_dt, t * d + n);
        g += ld(Wg, Wg_dt, (int64_t)j * d + n) * xn;
        u += ld(Wu, Wu_dt, (int64_t)j * d + n) * xn;
      }
      double a = sfn_oracle_sigmoid(logits[t * d_i + j]) * g * u;
      for (int n = 0; n < d; ++n) yt[n] += a * ld(Wd, Wd_dt, (int64_t)j * d + n);
    }
  }
}

/* The whole forward: predictor, bank top-k, sparse gate/up/down.
 * logits_out ([T][d_i]) and mask_out ([T][d_i/bank]) receive the
 * intermediates; y is [T][d]. */
void sfn_oracle_forward(const void *x, int x_dt, const void *A, int A_dt,
                        const void *B, int B_dt, const void *Wg, int Wg_dt,
                        const void *Wu, int Wu_dt, const void *Wd, int Wd_dt,
                        int64_t T, int d, int d_i, int r, int bank, int k,
                        double *logits_out, uint64_t *mask_out, double *y) {
  sfn_oracle_predict(x, x_dt, A, A_dt, B, B_dt, T, d, d_i, r, logits_out);
  sfn_oracle_bank_topk(logits_out, T, d_i, bank, k, mask_out);
  sfn_oracle_forward_given_mask(x, x_dt, logits_out, mask_out, Wg, Wg_dt, Wu,
                                Wu_dt, Wd, Wd_dt, T, d, d_i, bank, y);
}

/* The form of the pages' own GPU code, which simulates the sparsity: materialise the dense gate
 * and up projections for every channel, form the predictor-gated product,
 * multiply by the 0/1 mask, then run the dense down projection.  A separate
 * loop nest from sfn_oracle_forward_given_mask, used to check that skipping
 * channels and masking after the fact give the same y. */
void sfn_oracle_dense_then_mask(const void *x, int x_dt, const double *logits,
                                const uint64_t *mask, const void *Wg,
                                int Wg_dt, const void *Wu, int Wu_dt,
                                const void *Wd, int Wd_dt, int64_t T, int d,
                                int d_i, int bank, double *y) {
  int nb = d_i / bank;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    double *act = (double *)malloc(sizeof(double) * (size_t)d_i);
    /* dense gate and up for all channels */
    for (int j = 0; j < d_i; ++j) {
      double g = 0.0, u = 0.0;
      for (int n = 0; n < d; ++n) {
        double xn = ld(x, x_dt, t * d + n);
        g += ld(Wg, Wg_dt, (int64_t)j * d + n) * xn;
        u += ld(Wu, Wu_dt, (int64_t)j * d + n) * xn;
      }
      act[j] = sfn_oracle_sigmoid(logits[t * d_i + j]) * g * u;
    }
    /* hard binary mask */
    for (int j = 0; j < d_i; ++j) {
      double m = (double)((mask[t * nb + j / bank] >> (j % bank)) & 1);
      act[j] = act[j] * m;
    }
    /* dense down: y_n = sum_j W_down[n][j] act_j with W_down[n][j] = Wd[j][n] */
    for (int n = 0; n < d; ++n) {
      double s = 0.0;
      for (int j = 0; j < d_i; ++j) s += ld(Wd, Wd_dt, (int64_t)j * d + n) * act[j];
      y[t * d + n] = s;
    }
    free(act);
  }
}

/* The pages' "Dense-4x" comparison (gist.science summary, "Resultaten": a
 * dense model with a naive 4x sparsity applied post hoc from the activation
 * amplitude).  Reading: the standard SwiGLU FFN, act_j = silu(g_j) u_j with
 * silu(z) = z sigma(z), g_j = Wg[j].x, u_j = Wu[j].x; in every bank keep the
 * k channels of largest |act_j| (ties to the lower index, the same rule as
 * sfn_oracle_bank_topk); y = sum_{kept j} act_j Wd[j, :].  No predictor.
 * mask_io is [T][d_i/bank]: written, or (use_given_mask) read as the mask to
 * apply; act_out, if not NULL, receives act [T][d_i]; y is [T][d]. */
void sfn_oracle_dense4x(const void *x, int x_dt, const void *Wg, int Wg_dt, const void *Wu,
                        int Wu_dt, const void *Wd, int Wd_dt, int64_t T, int d, int d_i,
                        int bank, int k, int use_given_mask, uint64_t *mask_io, double *act_out,
                        double *y) {
  int nb = d_i / bank;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    double *act = (double *)malloc(sizeof(double) * (size_t)d_i);
    double *amp = (double *)malloc(sizeof(double) * (size_t)d_i);
    for (int j = 0; j < d_i; ++j) {
      double g = 0.0, u = 0.0;
      for (int n = 0; n < d; ++n) {
        double xn = ld(x, x_dt, t * d + n);
        g += ld(Wg, Wg_dt, (int64_t)j * d + n) * xn;
        u += ld(Wu, Wu_dt, (int64_t)j * d + n) * xn;
      }
      act[j] = g * sfn_oracle_sigmoid(g) * u;
      amp[j] = fabs(act[j]);
    }
    if (act_out)
      for (int j = 0; j < d_i; ++j) act_out[t * d_i + j] = act[j];
    if (!use_given_mask) sfn_oracle_bank_topk(amp, 1, d_i, bank, k, mask_io + t * nb);
    double *yt = y + t * d;
    for (int n = 0; n < d; ++n) yt[n] = 0.0;
    for (int j = 0; j < d_i; ++j) {
      if (!((mask_io[t * nb + j / bank] >> (j % bank)) & 1)) continue;
      for (int n = 0; n < d; ++n) yt[n] += act[j] * ld(Wd, Wd_dt, (int64_t)j * d + n);
    }
    free(act);
    free(amp);
  }
}

/* Threads the OpenMP runtime will use (reported beside CPU timings). */
/* Backward of the whole layer, for predictor training ("Executie / Backward
 * Pass" in the architecture section of the same summary: the hard top-k is
 * not differentiable, so a soft, sigmoid-like surrogate gradient around the
 * selection threshold lets the loss reach the predictor).
 *
 * The forward is the one above: h = A x, p = B h, m_j = hard bank top-k,
 * s_j = sigma(p_j), g_j = Wg[j].x, u_j = Wu[j].x, a_j = m_j s_j g_j u_j,
 * y = sum_j a_j Wd[j].  Given dy = dL/dy this returns dL/dx, dL/dA, dL/dB,
 * dL/dWg, dL/dWu, dL/dWd, with one reading for the surrogate (the pages
 * give neither formula nor temperature):
 *   - bank b's threshold is tau_b = (p_(k) + p_(k+1)) / 2, the midpoint of
 *     its k-th and (k+1)-th logits in the ranking order; it is held constant
 *     (no gradient flows through it).  With k = bank there is no threshold
 *     and no surrogate term;
 *   - dm_j/dp_j is replaced by sigma'(z_j) / temp with z_j = (p_j - tau_b) /
 *     temp and sigma'(z) = sigma(z) (1 - sigma(z)): the derivative of a
 *     sigmoid step of width temp centred on the threshold.  m_j itself stays
 *     hard (0 or 1) everywhere else.
 * The chain rule then gives, per token and channel j (da_j = Wd[j].dy):
 *   dg_j = da_j m_j s_j u_j,   du_j = da_j m_j s_j g_j,
 *   dp_j = da_j g_j u_j (m_j s_j (1 - s_j) + s_j sigma'(z_j) / temp),
 *   dWd[j] += a_j dy,  dWg[j] += dg_j x,  dWu[j] += du_j x,  dB[j] += dp_j h,
 *   dh = sum_j dp_j B[j],  dA += dh x^T,
 *   dx = sum_j (dg_j Wg[j] + du_j Wu[j]) + A^T dh.
 * The surrogate term needs g_j u_j of every channel, kept or not.
 *
 * mask_in (may be NULL): use this mask instead of the own top-k (the
 * threshold still comes from the own logits).  mask_out (may be NULL)
 * receives the mask used.  Every gradient output is overwritten. */
void sfn_oracle_backward(const void *x, int x_dt, const void *A, int A_dt,
                         const void *B, int B_dt, const void *Wg, int Wg_dt,
                         const void *Wu, int Wu_dt, const void *Wd, int Wd_dt,
                         const void *dy, int dy_dt, int64_t T, int d, int d_i,
                         int r, int bank, int k, double temp,
                         const uint64_t *mask_in, double *dx, double *dA,
                         double *dB, double *dWg, double *dWu, double *dWd,
                         uint64_t *mask_out) {
  const int nb = d_i / bank;
  memset(dA, 0, sizeof(double) * (size_t)r * d);
  memset(dB, 0, sizeof(double) * (size_t)d_i * r);
  memset(dWg, 0, sizeof(double) * (size_t)d_i * d);
  memset(dWu, 0, sizeof(double) * (size_t)d_i * d);
  memset(dWd, 0, sizeof(double) * (size_t)d_i * d);
  double *h = (double *)malloc(sizeof(double) * (size_t)r);
  double *dh = (double *)malloc(sizeof(double) * (size_t)r);
  double *p = (double *)malloc(sizeof(double) * (size_t)d_i);
  double *tau = (double *)malloc(sizeof(double) * (size_t)nb);
  double *dg = (double *)malloc(sizeof(double) * (size_t)d_i);
  double *du = (double *)malloc(sizeof(double) * (size_t)d_i);
  uint64_t *mw = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)nb);
  for (int64_t t = 0; t < T; ++t) {
    /* forward of this token: h, p, mask, thresholds */
    for (int m = 0; m < r; ++m) {
      double acc = 0.0;
      for (int n = 0; n < d; ++n) acc += ld(x, x_dt, t * d + n) * ld(A, A_dt, (int64_t)m * d + n);
      h[m] = acc;
    }
    for (int j = 0; j < d_i; ++j) {
      double acc = 0.0;
      for (int m = 0; m < r; ++m) acc += h[m] * ld(B, B_dt, m + (int64_t)j * r);
      p[j] = acc;
    }
    for (int b = 0; b < nb; ++b) {
      const double *pb = p + (int64_t)b * bank;
      uint64_t word = 0;
      double pk = 0.0, pk1 = 0.0;
      for (int j = 0; j < bank; ++j) {
        int rk = 0;
        for (int i = 0; i < bank; ++i)
          if (beats(pb[i], pb[j]) || (same(pb[i], pb[j]) && i < j)) ++rk;
        if (rk < k) word |= ((uint64_t)1) << j;
        if (rk == k - 1) pk = pb[j];
        if (rk == k) pk1 = pb[j];
      }
      tau[b] = (k < bank) ? 0.5 * (pk + pk1) : NAN;
      mw[b] = mask_in ? mask_in[t * nb + b] : word;
      if (mask_out) mask_out[t * nb + b] = mw[b];
    }
    /* every channel: g, u, da; the chain rule; weight gradients of row j */
#pragma omp parallel for schedule(static)
    for (int j = 0; j < d_i; ++j) {
      double g = 0.0, u = 0.0, da = 0.0;
      for (int n = 0; n < d; ++n) {
        const double xn = ld(x, x_dt, t * d + n);
        g += ld(Wg, Wg_dt, (int64_t)j * d + n) * xn;
        u += ld(Wu, Wu_dt, (int64_t)j * d + n) * xn;
        da += ld(Wd, Wd_dt, (int64_t)j * d + n) * ld(dy, dy_dt, t * d + n);
      }
      const double mj = (double)((mw[j / bank] >> (j % bank)) & 1);
      const double s = sfn_oracle_sigmoid(p[j]);
      const double tb = tau[j / bank];
      double sur = 0.0;
      if (!isnan(tb)) {
        const double sz = sfn_oracle_sigmoid((p[j] - tb) / temp);
        sur = sz * (1.0 - sz) / temp;
      }
      const double a = mj * s * g * u;
      dg[j] = da * mj * s * u;
      du[j] = da * mj * s * g;
      const double dp = da * g * u * (mj * s * (1.0 - s) + s * sur);
      for (int n = 0; n < d; ++n) {
        const double xn = ld(x, x_dt, t * d + n);
        dWd[(int64_t)j * d + n] += a * ld(dy, dy_dt, t * d + n);
        dWg[(int64_t)j * d + n] += dg[j] * xn;
        dWu[(int64_t)j * d + n] += du[j] * xn;
      }
      for (int m = 0; m < r; ++m) dB[(int64_t)j * r + m] += dp * h[m];
      p[j] = dp; /* p[j] is not read again for this token: keep dp there */
    }
    /* dh = B^T dp (p now holds dp), dA += dh x^T */
#pragma omp parallel for schedule(static)
    for (int m = 0; m < r; ++m) {
      double acc = 0.0;
      for (int j = 0; j < d_i; ++j) acc += p[j] * ld(B, B_dt, m + (int64_t)j * r);
      dh[m] = acc;
      for (int n = 0; n < d; ++n) dA[(int64_t)m * d + n] += acc * ld(x, x_dt, t * d + n);
    }
    /* dx = Wg^T dg + Wu^T du + A^T dh */
#pragma omp parallel for schedule(static)
    for (int n = 0; n < d; ++n) {
      double acc = 0.0;
      for (int j = 0; j < d_i; ++j)
        acc += dg[j] * ld(Wg, Wg_dt, (int64_t)j * d + n) + du[j] * ld(Wu, Wu_dt, (int64_t)j * d + n);
      for (int m = 0; m < r; ++m) acc += dh[m] * ld(A, A_dt, (int64_t)m * d + n);
      dx[t * d + n] = acc;
    }
  }
  free(h);
  free(dh);
  free(p);
  free(tau);
  free(dg);
  free(du);
  free(mw);
}

int sfn_oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
