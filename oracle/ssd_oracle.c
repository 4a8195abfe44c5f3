/*
 * ssd_oracle.c -- plain, slow, sequential fp64 CPU oracle for the Mamba-2 mixer
 * scan (causal depthwise conv1d + SiLU, softplus dt, scalar-decay-per-head SSM
 * recurrence, z-gated RMSNorm, single-token decode step).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: it exists so that the tests, the smoke check and the benchmark's
 * CPU-baseline leg can check the CUDA library against an independent,
 * obviously-correct definition.  It shares no code, header or constant with
 * the CUDA sources.
 *
 * What it follows (page titles and sections of the source pages):
 *  - "NVIDIA Nemotron Nano 2" summary (hyper.ai), section "Method": the Mamba-2
 *    layers use 8 groups, state dimension 128, head dimension 64, expansion 2
 *    and a convolution window of 4; the model normalises with RMSNorm and has
 *    no linear-layer bias.  The neurohive.io article, section "Model
 *    architecture", states the same numbers.
 *  - neurohive.io article, section "Deployment and usage": the SSM cache is
 *    kept in float32 (here every intermediate is fp64, wider still).
 *  - The recurrence itself is the Mamba-2 scalar-decay selective SSM:
 *        h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T   (P x N per head)
 *        y_t = h_t C_t + D_h * x_t                            (uses h_t after
 *                                                              the update)
 *    with x = conv+SiLU output of the head's channels, B/C the conv+SiLU
 *    output of the head's group channels, dt = softplus(dt_raw + dt_bias)
 *    optionally clamped to [dt_min, dt_max].
 *  - z-gated RMSNorm: g = y * silu(z); out = g / sqrt(mean_group(g^2) + eps) * w,
 *    groups of d_inner / norm_groups consecutive channels (gate first, then
 *    normalise).
 *
 * Every element is read in its stored precision (fp64, fp32 or bf16 bit
 * pattern) and widened to double exactly; nothing is rounded afterwards.
 * Work is split over independent (batch, head) pairs with OpenMP when asked;
 * the arithmetic inside one pair is the plain sequential recurrence.
 *
 * Parity status: every function here is pinned by the CPU tests against
 * brute force, closed forms or textbook routines (quadratic form, prefix sums,
 * geometric series, chunked form, split/carry and decode equivalence, conv
 * impulse response, norm invariants, linearity).
 *
 * ORACLE_MUTANT: the CPU tests rebuild this file with -DORACLE_MUTANT=k to
 * plant one deliberate mistake and check that some pin fails.  The default
 * build (ORACLE_MUTANT undefined or 0) is the oracle.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

enum { OR_F64 = 0, OR_F32 = 1, OR_BF16 = 2 };

/* Read element i of a buffer stored as fp64, fp32 or bf16 bits; exact widening. */
static double ld(const void *p, int dtype, long long i) {
  if (dtype == OR_F64) return ((const double *)p)[i];
  if (dtype == OR_F32) return (double)((const float *)p)[i];
  uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round to the nearest bf16 value (8 significant bits), ties to even, computed directly from
 * the double (no intermediate float rounding).  Used only where the layer materialises a
 * bf16 activation tensor. */
double oracle_round_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  const double m = frexp(x, &e); /* x = m * 2^e, 0.5 <= |m| < 1 */
  return ldexp(nearbyint(ldexp(m, 8)), e - 8);
}

/* SiLU(x) = x * sigmoid(x) = x / (1 + e^{-x}). */
double oracle_silu(double x) { return x / (1.0 + exp(-x)); }

/* softplus(x) = log(1 + e^x), written so that large x does not overflow
 * (x + log1p(e^{-x}) is the same quantity). */
double oracle_softplus(double x) {
#if ORACLE_MUTANT == 6
  return x; /* mutant: softplus skipped */
#else
  return x > 30.0 ? x + log1p(exp(-x)) : log1p(exp(x));
#endif
}

/* Effective time step: softplus(dt_raw + bias) when softplus != 0, else
 * dt_raw + bias; then clamped to [dt_min, dt_max] (pass 0 and +inf for none). */
double oracle_dt(double dt_raw, double bias, int softplus, double dt_min, double dt_max) {
  double v = dt_raw + bias;
  if (softplus) v = oracle_softplus(v);
  if (v < dt_min) v = dt_min;
  if (v > dt_max) v = dt_max;
  return v;
}

/* Causal depthwise conv1d of window W, plus bias, then SiLU, for channel c of
 * batch row b at time t.  Inputs before t = 0 come from the conv cache
 * conv_state [B, W, C] (row W-1 is the most recent raw input, i.e. time -1);
 * a NULL cache means zeros.  W == 0 means "no conv": the raw input is
 * returned unchanged (no activation either).  Weights w are [C, W] with
 * w[c, W-1] multiplying the current input. */
static double conv_at(int L, int C, int W, const void *xin, int xdt, long long row_stride,
                      const void *state_in, int sdt, const void *w, int wdt, const void *bias,
                      int bdt, int b, int t, int c) {
  if (W == 0) return ld(xin, xdt, ((long long)b * L + t) * row_stride + c);
  double acc = bias ? ld(bias, bdt, c) : 0.0;
  for (int k = 0; k < W; ++k) {
#if ORACLE_MUTANT == 5
    int tau = t - k; /* mutant: taps applied in reversed order */
#else
    int tau = t - (W - 1) + k; /* the input time that tap k multiplies */
#endif
    double xv;
    if (tau >= 0)
      xv = ld(xin, xdt, ((long long)b * L + tau) * row_stride + c);
    else
      xv = state_in ? ld(state_in, sdt, ((long long)b * W + (W + tau)) * C + c) : 0.0;
    acc += ld(w, wdt, (long long)c * W + k) * xv;
  }
  return oracle_silu(acc);
}

/* Materialise the conv front end: u[b, t, c] for all channels (small cases). */
void oracle_conv1d_silu(int B, int L, int C, int W, const void *xin, int xdt, long long row_stride,
                        const void *state_in, int sdt, const void *w, int wdt, const void *bias,
                        int bdt, double *u) {
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < L; ++t)
      for (int c = 0; c < C; ++c)
        u[((long long)b * L + t) * C + c] =
            conv_at(L, C, W, xin, xdt, row_stride, state_in, sdt, w, wdt, bias, bdt, b, t, c);
}

/* Shapes and optional parts shared by the prefill and decode oracles. */
typedef struct {
  int batch, seqlen, nheads, headdim, dstate, ngroups, conv_width;
  int dt_softplus;
  double dt_min, dt_max;
} oracle_shape_t;

/*
 * Prefill: runs the plain recurrence for heads [h_lo, h_hi) of every batch row.
 *  xBC   [B, L, conv_dim] raw (pre-conv) channels x | B | C, row stride in elements
 *        conv_dim = H*P + 2*G*N; head h owns x channels h*P .. h*P+P-1, its group
 *        g = h / (H/G) owns B channels H*P + g*N .. and C channels H*P + G*N + g*N ..
 *  dt    [B, L, H] raw time steps (row stride in elements)
 *  A, D, dt_bias [H]; conv_w [conv_dim, W]; conv_b [conv_dim] or NULL
 *  h0    [B, H, P, N] or NULL (zeros); conv_state_in [B, W, conv_dim] or NULL
 * Outputs (fp64): y [B, L, h_hi-h_lo, P] (no gating), h_final [B, h_hi-h_lo, P, N].
 */
void oracle_ssd_prefill(const oracle_shape_t *s, const void *xBC, int xdt, long long xBC_stride,
                        const void *dtr, int ddt, long long dt_stride, const void *A, const void *D,
                        const void *dt_bias, int pdt, const void *conv_w, const void *conv_b,
                        int cdt, const void *h0, int h0dt, const void *conv_state_in, int sdt,
                        int h_lo, int h_hi, double *y, double *h_final, int threads) {
  const int Bn = s->batch, L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate;
  const int G = s->ngroups, W = s->conv_width;
  const int hpg = H / G, d_inner = H * P, conv_dim = d_inner + 2 * G * N, nh = h_hi - h_lo;
  const long long pairs = (long long)Bn * nh;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1)
  for (long long pr = 0; pr < pairs; ++pr) {
    const int b = (int)(pr / nh), hi = (int)(pr % nh), h = h_lo + hi;
#if ORACLE_MUTANT == 4
    const int g = h % G; /* mutant: heads assigned to groups round-robin */
#else
    const int g = h / hpg;
#endif
    double *st = (double *)malloc(sizeof(double) * P * N);
    double *ux = (double *)malloc(sizeof(double) * P);
    double *uB = (double *)malloc(sizeof(double) * N);
    double *uC = (double *)malloc(sizeof(double) * N);
    for (int i = 0; i < P * N; ++i)
      st[i] = h0 ? ld(h0, h0dt, ((long long)b * H + h) * P * N + i) : 0.0;
    const double Ah = ld(A, pdt, h), Dh = ld(D, pdt, h), bias = ld(dt_bias, pdt, h);
    for (int t = 0; t < L; ++t) {
      for (int p = 0; p < P; ++p)
        ux[p] = conv_at(L, conv_dim, W, xBC, xdt, xBC_stride, conv_state_in, sdt, conv_w, cdt,
                        conv_b, cdt, b, t, h * P + p);
      for (int n = 0; n < N; ++n) {
        uB[n] = conv_at(L, conv_dim, W, xBC, xdt, xBC_stride, conv_state_in, sdt, conv_w, cdt,
                        conv_b, cdt, b, t, d_inner + g * N + n);
        uC[n] = conv_at(L, conv_dim, W, xBC, xdt, xBC_stride, conv_state_in, sdt, conv_w, cdt,
                        conv_b, cdt, b, t, d_inner + G * N + g * N + n);
      }
      const double dt = oracle_dt(ld(dtr, ddt, ((long long)b * L + t) * dt_stride + h), bias,
                                  s->dt_softplus, s->dt_min, s->dt_max);
#if ORACLE_MUTANT == 2
      const double a = exp(-dt * Ah); /* mutant: sign of A flipped */
#else
      const double a = exp(dt * Ah);
#endif
      double *yt = y + (((long long)b * L + t) * nh + hi) * P;
#if ORACLE_MUTANT == 3
      for (int p = 0; p < P; ++p) { /* mutant: output read before the update */
        double acc = 0.0;
        for (int n = 0; n < N; ++n) acc += st[p * N + n] * uC[n];
        yt[p] = acc + Dh * ux[p];
      }
#endif
      for (int p = 0; p < P; ++p)
        for (int n = 0; n < N; ++n) st[p * N + n] = a * st[p * N + n] + dt * ux[p] * uB[n];
#if ORACLE_MUTANT != 3
      for (int p = 0; p < P; ++p) {
        double acc = 0.0;
#if ORACLE_MUTANT == 7
        for (int n = 0; n < N; ++n) acc += st[p * N + n] * uB[n]; /* mutant: B read for C */
#else
        for (int n = 0; n < N; ++n) acc += st[p * N + n] * uC[n];
#endif
#if ORACLE_MUTANT == 1
        yt[p] = acc; /* mutant: skip term D*x dropped */
#else
        yt[p] = acc + Dh * ux[p];
#endif
      }
#endif
    }
    if (h_final)
      memcpy(h_final + ((long long)b * nh + hi) * P * N, st, sizeof(double) * P * N);
    free(st);
    free(ux);
    free(uB);
    free(uC);
  }
}

/*
 * z-gated RMSNorm over rows of width Dn split into ngroups groups of Dn/ngroups
 * consecutive channels.  Gate first (norm_before_gate = 0):
 *   g = y * silu(z);  out = g / sqrt(mean(g^2) + eps) * w.
 * Normalise first (norm_before_gate = 1):
 *   out = y / sqrt(mean(y^2) + eps) * w * silu(z).
 * y, out: fp64 [T, Dn]; z [T, Dn] with row stride z_stride (NULL = no gate); w [Dn]
 * (NULL = ones).
 */
void oracle_gated_rmsnorm(long long T, int Dn, int ngroups, const double *y, const void *z, int zdt,
                          long long z_stride, const void *w, int wdt, double eps, int norm_before_gate,
                          double *out) {
  const int gs = Dn / ngroups;
  double *g = (double *)malloc(sizeof(double) * gs);
  for (long long t = 0; t < T; ++t)
    for (int k = 0; k < ngroups; ++k) {
      double ss = 0.0;
      for (int i = 0; i < gs; ++i) {
        const int c = k * gs + i;
        const double gate = z ? oracle_silu(ld(z, zdt, t * z_stride + c)) : 1.0;
        g[i] = norm_before_gate ? y[t * Dn + c] : y[t * Dn + c] * gate;
        ss += g[i] * g[i];
      }
      const double r = 1.0 / sqrt(ss / gs + eps);
      for (int i = 0; i < gs; ++i) {
        const int c = k * gs + i;
        const double gate = (norm_before_gate && z) ? oracle_silu(ld(z, zdt, t * z_stride + c)) : 1.0;
        out[t * Dn + c] = g[i] * r * (w ? ld(w, wdt, c) : 1.0) * gate;
      }
    }
  free(g);
}

/* Plain RMSNorm of rows of width Dn: out = x / sqrt(mean(x^2) + eps) * w. */
void oracle_rmsnorm(long long T, int Dn, const void *x, int xdt, const void *w, int wdt, double eps,
                    double *out) {
  for (long long t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int c = 0; c < Dn; ++c) {
      const double v = ld(x, xdt, t * Dn + c);
      ss += v * v;
    }
    const double r = 1.0 / sqrt(ss / Dn + eps);
    for (int c = 0; c < Dn; ++c) out[t * Dn + c] = ld(x, xdt, t * Dn + c) * r * (w ? ld(w, wdt, c) : 1.0);
  }
}

/*
 * One decode step (a single new token per batch row) for heads [h_lo, h_hi).
 *  xBC_t [B, conv_dim] raw channels of the new token; dt_t [B, H] raw.
 *  conv_state_in [B, W, conv_dim]: the last W raw inputs, oldest first.
 *  conv_state_out [B, W, conv_dim] (fp64): the cache shifted by one with the new
 *    token appended as row W-1 (written for every channel when h_lo == 0).
 *  state [B, h_hi-h_lo, P, N] fp64, updated in place.
 *  y [B, h_hi-h_lo, P] fp64 (no gating).
 * The conv output for channel c is silu(bias_c + sum_k w[c,k] * cache_out[k, c]),
 * which is the prefill conv of a one-token sequence whose history is the cache.
 */
void oracle_decode_step(const oracle_shape_t *s, const void *xBC_t, int xdt, const void *dt_t,
                        int ddt, const void *A, const void *D, const void *dt_bias, int pdt,
                        const void *conv_w, const void *conv_b, int cdt, const void *conv_state_in,
                        int sdt, double *conv_state_out, double *state, int h_lo, int h_hi,
                        double *y, int threads) {
  const int Bn = s->batch, H = s->nheads, P = s->headdim, N = s->dstate, G = s->ngroups;
  const int W = s->conv_width, hpg = H / G, d_inner = H * P, conv_dim = d_inner + 2 * G * N;
  const int nh = h_hi - h_lo;
  const int Wr = W > 0 ? W : 1;
  double *cache = (double *)malloc(sizeof(double) * (size_t)Bn * Wr * conv_dim);
  double *u = (double *)malloc(sizeof(double) * (size_t)Bn * conv_dim);
  for (int b = 0; b < Bn; ++b) {
    double *cb = cache + (size_t)b * Wr * conv_dim, *ub = u + (size_t)b * conv_dim;
    /* shift the cache and append the new raw input */
    for (int c = 0; c < conv_dim; ++c) {
      for (int k = 0; k + 1 < W; ++k)
        cb[k * conv_dim + c] = ld(conv_state_in, sdt, ((long long)b * W + k + 1) * conv_dim + c);
      if (W > 0) cb[(W - 1) * conv_dim + c] = ld(xBC_t, xdt, (long long)b * conv_dim + c);
    }
    for (int c = 0; c < conv_dim; ++c) {
      if (W == 0) {
        ub[c] = ld(xBC_t, xdt, (long long)b * conv_dim + c);
        continue;
      }
      double acc = conv_b ? ld(conv_b, cdt, c) : 0.0;
      for (int k = 0; k < W; ++k) acc += ld(conv_w, cdt, (long long)c * W + k) * cb[k * conv_dim + c];
      ub[c] = oracle_silu(acc);
    }
    if (conv_state_out && W > 0)
      memcpy(conv_state_out + (long long)b * W * conv_dim, cb, sizeof(double) * W * conv_dim);
  }
  const long long pairs = (long long)Bn * nh;
#pragma omp parallel for schedule(static) num_threads(threads > 0 ? threads : 1)
  for (long long pr = 0; pr < pairs; ++pr) {
    const int b = (int)(pr / nh), hi = (int)(pr % nh);
    const int h = h_lo + hi, g = h / hpg;
    const double *ub = u + (size_t)b * conv_dim;
    const double dt = oracle_dt(ld(dt_t, ddt, (long long)b * H + h), ld(dt_bias, pdt, h),
                                s->dt_softplus, s->dt_min, s->dt_max);
    const double a = exp(dt * ld(A, pdt, h)), Dh = ld(D, pdt, h);
    double *st = state + ((long long)b * nh + hi) * P * N;
    const double *ux = ub + h * P, *uB = ub + d_inner + g * N, *uC = ub + d_inner + G * N + g * N;
    for (int p = 0; p < P; ++p) {
      double acc = 0.0;
      for (int n = 0; n < N; ++n) {
        st[p * N + n] = a * st[p * N + n] + dt * ux[p] * uB[n];
        acc += st[p * N + n] * uC[n];
      }
      y[((long long)b * nh + hi) * P + p] = acc + Dh * ux[p];
    }
  }
  free(cache);
  free(u);
}
