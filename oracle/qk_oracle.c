/*
 * qk_oracle.c -- plain CPU oracle for the block-quantized expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY (see qk_oracle.h).  C99 + libm, optional OpenMP
 * over output rows; each output element is summed sequentially in index order,
 * so results are bit-identical for any thread count.
 */
#include "qk_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- codes --
 * e2m1 (OCP Microscaling Formats v1.0, FP4 E2M1; the pages name the format but
 * do not print its table): bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa.  Exponent field 0 is subnormal: value = m * 0.5.  Otherwise
 * value = 2^(e-1) * (1 + m/2).  Magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6. */
double qko_e2m1_value(uint8_t code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

/* e8m0 / UE8M0: unsigned power of two 2^(c-127); 255 is NaN. */
double qko_e8m0_value(uint8_t code) {
  if (code == 255) return NAN;
  return ldexp(1.0, (int)code - 127);
}

/* E4M3FN: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa; no
 * infinities; S.1111.111 is NaN; exponent 0 is subnormal (m/8)*2^-6. */
double qko_e4m3_value(uint8_t code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m, -9);
  else mag = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

static double round_half_even(double q) { /* q >= 0 with few significant bits */
  double f = floor(q), r = q - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Cast to E4M3FN, round to nearest even, saturating finite values to +-448. */
uint8_t qko_e4m3_encode(double v) {
  uint8_t sign;
  double a;
  int ex, m;
  if (isnan(v)) return 0x7F;
  sign = signbit(v) ? 0x80 : 0x00;
  a = fabs(v);
  if (a == 0.0) return sign;
  if (a >= 448.0) return sign | 0x7E;
  if (a < ldexp(1.0, -6)) {                    /* subnormal range: steps of 2^-9 */
    m = (int)round_half_even(a * 512.0);
    return sign | (uint8_t)m;                  /* m == 8 is the min normal 0x08 */
  }
  frexp(a, &ex);
  ex -= 1;                                     /* a = f * 2^ex, f in [1,2) */
  m = (int)round_half_even((ldexp(a, -ex) - 1.0) * 8.0);
  if (m == 8) { m = 0; ex += 1; }
  if (ex > 8 || (ex == 8 && m == 7)) return sign | 0x7E;
  return sign | (uint8_t)(((ex + 7) << 3) | m);
}

/* Cast to e2m1: round to nearest, ties to the even code (mantissa bit 0),
 * saturating to +-6 (FP4 has no infinity or NaN; OCP Microscaling v1.0
 * conversions clamp).  Returns the 4-bit code. */
uint8_t qko_e2m1_encode(double v) {
  uint8_t sign = signbit(v) ? 8 : 0;
  double a = fabs(v);
  int ex, n;
  if (a >= 6.0) return sign | 7;
  if (a < 1.0) return sign | (uint8_t)round_half_even(a * 2.0); /* 0, 0.5, 1: codes 0, 1, 2 */
  frexp(a, &ex);
  ex -= 1;                                 /* a = f * 2^ex, f in [1,2), ex in {0, 1, 2} */
  n = (int)round_half_even(ldexp(a, 1 - ex)); /* a / 2^(ex-1) in [2, 4) -> 2, 3 or 4 */
  if (n == 4) return sign | (uint8_t)((ex + 2) << 1);
  return sign | (uint8_t)(((ex + 1) << 1) | (n - 2));
}

double qko_bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ------------------------------------------------------------ dequant --
 * Nibble order (pages silent; reading adopted): element 2i of a row is the low
 * nibble of byte i, element 2i+1 the high nibble.  Rows are contiguous along
 * the input dimension; quantization blocks run along it. */
static int nibble(const uint8_t* row_q, int32_t k) {
  uint8_t b = row_q[k >> 1];
  return (k & 1) ? (b >> 4) : (b & 15);
}

/* The dequantized value is held in fp64, where it is exact for every code of
 * every format: e2m1 (2 significant bits) x e8m0 (a power of two, 2^-127 ..
 * 2^127) for MXFP4; e2m1 x e4m3 (4 bits) x an fp32 scale_2 (24 bits) for
 * NVFP4, at most 30 significant bits and within fp64's exponent range.
 * Rounding it to fp32 would change general NVFP4 weights (scale_2 not a power
 * of two) and overflow MXFP4 codes >= 253. */
int qko_dequant_row(const qko_weight* w, int32_t e, int32_t row, double* out) {
  int64_t r = (int64_t)e * w->rows + row;
  const uint8_t* rq = w->q + r * (w->cols / 2);
  int32_t k;
  if (w->fmt == QKO_FMT_MXFP4) {
    const uint8_t* rs = w->scales + r * (w->cols / 32);
    for (k = 0; k < w->cols; ++k) {
      uint8_t c = rs[k / 32];
      if (c == 255) return QKO_ERR_NAN_SCALE;
      out[k] = qko_e2m1_value((uint8_t)nibble(rq, k)) * qko_e8m0_value(c);
    }
    return QKO_OK;
  }
  if (w->fmt == QKO_FMT_NVFP4) {
    const uint8_t* rs = w->scales + r * (w->cols / 16);
    double s2 = (double)w->scale_2[e];
    for (k = 0; k < w->cols; ++k) {
      uint8_t c = rs[k / 16];
      if ((c & 0x7F) == 0x7F) return QKO_ERR_NAN_SCALE;
      out[k] = qko_e2m1_value((uint8_t)nibble(rq, k)) * qko_e4m3_value(c) * s2;
    }
    return QKO_OK;
  }
  return QKO_ERR_INVALID_ARG;
}

/* --------------------------------------------------------- conversion --
 * MXFP4 -> NVFP4, scales only (REAP-K180-NVFP4 page: the nibbles are kept and
 * e8m0/32 becomes e4m3/16 + per-expert fp32 scale_2).  Lossless needs
 * 2^(c-127) == e4m3(s) * scale_2, so scale_2 is a power of two.  Rule adopted
 * (the page gives none): anchor at the expert's largest code c_max,
 *   scale_2 = 2^(c_max - 127 - 8),
 * and each 32-block with code c gets, in both of its 16-halves, the e4m3
 * cast (round to nearest even) of 2^(c - c_max + 8).  Exponents down to -9
 * are exact; a block whose cast is not exact counts once in n_inexact. */
int qko_convert_mx_to_nv(const uint8_t* e8m0, int32_t E, int32_t N, int32_t K,
                         uint8_t* e4m3, float* scale_2, uint64_t* n_inexact) {
  int32_t e;
  int64_t per, i;
  uint64_t bad = 0;
  if (!e8m0 || !e4m3 || !scale_2 || E < 0 || N < 0 || K <= 0 || K % 32) return QKO_ERR_INVALID_ARG;
  per = (int64_t)N * (K / 32);
  for (e = 0; e < E; ++e) {
    const uint8_t* s = e8m0 + (int64_t)e * per;
    int cmax = 0;
    for (i = 0; i < per; ++i) {
      if (s[i] == 255) return QKO_ERR_NAN_SCALE;
      if (s[i] > cmax) cmax = s[i];
    }
    scale_2[e] = (float)ldexp(1.0, cmax - 127 - 8);
    for (i = 0; i < per; ++i) {
      double target = ldexp(1.0, (int)s[i] - cmax + 8);
      uint8_t c = qko_e4m3_encode(target);
      e4m3[(int64_t)e * per * 2 + 2 * i] = c;
      e4m3[(int64_t)e * per * 2 + 2 * i + 1] = c;
      if (qko_e4m3_value(c) != target) ++bad;
    }
  }
  if (n_inexact) *n_inexact = bad;
  return QKO_OK;
}

/* NVFP4 -> MXFP4, scales only (the reverse of the conversion above; the pages
 * define only the forward direction, so the rule is the reading adopted).  A
 * 32-block's two half scales e4m3(s0) * scale_2 and e4m3(s1) * scale_2 (exact
 * in fp64) convert exactly when they are equal and a power of two 2^p with
 * -127 <= p <= 127: code p + 127.  Any other block is counted once in
 * n_inexact and gets the code whose power of two is nearest in log2 to the
 * larger magnitude of the two (2^p for a mantissa below sqrt 2, else 2^(p+1);
 * clamped to codes 0 .. 254; code 0 for two zero scales: e8m0 has no zero, so
 * such a block's nonzero nibbles turn into values of 2^-127 scale and the block
 * counts as inexact).  A NaN code or a non-finite product is
 * QKO_ERR_NAN_SCALE. */
int qko_convert_nv_to_mx(const uint8_t* e4m3, const float* scale_2, int32_t E, int32_t N, int32_t K,
                         uint8_t* e8m0, uint64_t* n_inexact) {
  int64_t e, i, per;
  uint64_t bad = 0;
  if (!e4m3 || !scale_2 || !e8m0 || E < 0 || N < 0 || K <= 0 || K % 32) return QKO_ERR_INVALID_ARG;
  per = (int64_t)N * (K / 32);
  for (e = 0; e < E; ++e) {
    double s2 = (double)scale_2[e];
    for (i = 0; i < per; ++i) {
      uint8_t c0 = e4m3[(e * per + i) * 2], c1 = e4m3[(e * per + i) * 2 + 1];
      double a = qko_e4m3_value(c0) * s2, b = qko_e4m3_value(c1) * s2, v, f;
      int ex, p;
      if (isnan(a) || isnan(b) || isinf(a) || isinf(b)) return QKO_ERR_NAN_SCALE;
      if (a == b && a > 0.0) {
        f = frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1) */
        if (f == 0.5 && ex - 1 >= -127 && ex - 1 <= 127) {
          e8m0[e * per + i] = (uint8_t)(ex - 1 + 127);
          continue;
        }
      }
      ++bad;
      v = fabs(a) > fabs(b) ? fabs(a) : fabs(b);
      if (v == 0.0) {
        e8m0[e * per + i] = 0;
        continue;
      }
      f = frexp(v, &ex);                   /* v = (2f) * 2^(ex-1), 2f in [1, 2) */
      p = (2.0 * f < sqrt(2.0)) ? ex - 1 : ex;
      if (p < -127) p = -127;
      if (p > 127) p = 127;
      e8m0[e * per + i] = (uint8_t)(p + 127);
    }
  }
  if (n_inexact) *n_inexact = bad;
  return QKO_OK;
}

/* -------------------------------------------------------------- router --
 * Softmax over the E logits in fp64, the k largest probabilities (equal
 * probabilities: lower expert id first), renormalised to sum to 1, slots in
 * that order.  (The pages name 256 experts and top-6 but not the function.) */
int qko_route_topk(const float* logits, int32_t T, int32_t E, int32_t k,
                   int32_t* ids, double* w) {
  int32_t t, i, s;
  double* p;
  char* taken;
  if (!logits || !ids || !w || T < 0 || E <= 0 || k <= 0 || k > E) return QKO_ERR_INVALID_ARG;
  p = (double*)malloc(sizeof(double) * E);
  taken = (char*)malloc(E);
  for (t = 0; t < T; ++t) {
    const float* l = logits + (int64_t)t * E;
    double mx = -INFINITY, z = 0.0, tot = 0.0;
    for (i = 0; i < E; ++i) if ((double)l[i] > mx) mx = l[i];
    if (!isfinite(mx)) { free(p); free(taken); return QKO_ERR_INVALID_ARG; }
    for (i = 0; i < E; ++i) { p[i] = exp((double)l[i] - mx); z += p[i]; }
    for (i = 0; i < E; ++i) p[i] /= z;
    memset(taken, 0, E);
    for (s = 0; s < k; ++s) {
      int32_t best = -1;
      for (i = 0; i < E; ++i)
        if (!taken[i] && (best < 0 || p[i] > p[best])) best = i;
      taken[best] = 1;
      ids[(int64_t)t * k + s] = best;
    }
    for (s = 0; s < k; ++s) tot += p[ids[(int64_t)t * k + s]];
    for (s = 0; s < k; ++s) w[(int64_t)t * k + s] = p[ids[(int64_t)t * k + s]] / tot;
  }
  free(p);
  free(taken);
  return QKO_OK;
}

/* ------------------------------------------------- activation quantization --
 * The activation-quantized modes: fp4 weights times MXFP4 or E4M3
 * activations on block-scaled tensor cores, the latter being the expert
 * numerics DeepSeek-V4-Flash's own config names ("DeepSeekv4 Flash for 1x
 * Spark [REAP25]", the v0.2.3 update: fp4 weights x dynamic E4M3
 * activations on the f8f6f4 tensor cores).  The block-scaled MMA takes one
 * e8m0 scale per 32 activations; the scale rule is the OCP Microscaling v1.0
 * one (reading adopted; the pages give none): per block of 32,
 *   X = floor(log2 max|v|) - emax,  emax = 2 (e2m1) or 8 (e4m3),
 * clamped to the e8m0 range [-127, 127] (X = -127 for an all-zero block), and
 * each element is cast from v / 2^X with round-to-nearest-even, saturating.
 * codes: one element code per value (e2m1 in the low nibble, or e4m3);
 * scales: one e8m0 code per block; out: the dequantized values.  Any of the
 * three outputs may be NULL.  A non-finite value is an argument error. */
int qko_act_quant(const double* v, int32_t n, int32_t aq, uint8_t* codes, uint8_t* scales,
                  double* out) {
  int32_t b, i;
  int emax;
  if (!v || n < 0 || n % 32) return QKO_ERR_INVALID_ARG;
  if (aq == QKO_ACT_MXFP4) emax = 2;
  else if (aq == QKO_ACT_E4M3) emax = 8;
  else return QKO_ERR_INVALID_ARG;
  for (b = 0; b < n / 32; ++b) {
    const double* vb = v + (int64_t)b * 32;
    double amax = 0.0;
    int X = -127, ex;
    for (i = 0; i < 32; ++i) {
      if (isnan(vb[i]) || isinf(vb[i])) return QKO_ERR_INVALID_ARG;
      if (fabs(vb[i]) > amax) amax = fabs(vb[i]);
    }
    if (amax > 0.0) {
      frexp(amax, &ex);
      X = (ex - 1) - emax;
      if (X < -127) X = -127;
      if (X > 127) X = 127;
    }
    if (scales) scales[b] = (uint8_t)(X + 127);
    for (i = 0; i < 32; ++i) {
      double q = ldexp(vb[i], -X), val;
      uint8_t c;
      if (aq == QKO_ACT_MXFP4) {
        c = qko_e2m1_encode(q);
        val = qko_e2m1_value(c);
      } else {
        c = qko_e4m3_encode(q);
        val = qko_e4m3_value(c);
      }
      if (codes) codes[(int64_t)b * 32 + i] = c;
      if (out) out[(int64_t)b * 32 + i] = ldexp(val, X);
    }
  }
  return QKO_OK;
}

/* ----------------------------------------------------------------- FFN --
 * Routed expert (pages: gate/up/down projections; SwiGLU form not printed,
 * reading adopted: h = silu(gate) * up, silu(g) = g / (1 + exp(-g)), no clamp,
 * no routed scaling factor). */
static int matvec_rows(const qko_weight* w, int32_t e, const double* x, double* out) {
  int err = QKO_OK;
  int32_t n;
#pragma omp parallel
  {
    double* row = (double*)malloc(sizeof(double) * w->cols);
#pragma omp for schedule(static)
    for (n = 0; n < w->rows; ++n) {
      int32_t k;
      double acc = 0.0;
      if (qko_dequant_row(w, e, n, row) != QKO_OK) {
#pragma omp atomic write
        err = QKO_ERR_NAN_SCALE;
        continue;
      }
      for (k = 0; k < w->cols; ++k) acc += row[k] * x[k];
      out[n] = acc;
    }
    free(row);
  }
  return err;
}

static int check_layer(const qko_layer* L) {
  if (!L) return 0;
  if (L->gate.rows != L->inter || L->gate.cols != L->hidden) return 0;
  if (L->up.rows != L->inter || L->up.cols != L->hidden) return 0;
  if (L->down.rows != L->hidden || L->down.cols != L->inter) return 0;
  if (L->hidden % 32 || L->inter % 32) return 0;
  return 1;
}

/* One expert on one token.  With an activation-quantized mode, x is
 * quantized before gate/up, and h is rounded to fp32 (the precision in which
 * the GPU takes the same decision) and quantized before down; h then returns
 * the quantized values down consumes. */
int qko_expert_ffn_aq(const qko_layer* L, int32_t e, const uint16_t* x_bf16, int32_t aq,
                      double* g, double* u, double* h, double* d) {
  int32_t I, H, i, err = QKO_OK, aq_err = QKO_OK;
  double *xg, *gg, *uu, *hh, *dd;
  if (!check_layer(L) || !x_bf16 || e < 0 || e >= L->gate.n_experts) return QKO_ERR_INVALID_ARG;
  if (aq != QKO_ACT_NONE && aq != QKO_ACT_MXFP4 && aq != QKO_ACT_E4M3) return QKO_ERR_INVALID_ARG;
  I = L->inter;
  H = L->hidden;
  xg = (double*)malloc(sizeof(double) * H);
  gg = (double*)malloc(sizeof(double) * I);
  uu = (double*)malloc(sizeof(double) * I);
  hh = (double*)malloc(sizeof(double) * I);
  dd = (double*)malloc(sizeof(double) * H);
  for (i = 0; i < H; ++i) xg[i] = qko_bf16_value(x_bf16[i]);
  if (aq != QKO_ACT_NONE) aq_err |= qko_act_quant(xg, H, aq, NULL, NULL, xg);
  err |= matvec_rows(&L->gate, e, xg, gg);
  err |= matvec_rows(&L->up, e, xg, uu);
  for (i = 0; i < I; ++i) hh[i] = gg[i] / (1.0 + exp(-gg[i])) * uu[i];
  if (aq != QKO_ACT_NONE && !err) {
    for (i = 0; i < I; ++i) hh[i] = (double)(float)hh[i];
    aq_err |= qko_act_quant(hh, I, aq, NULL, NULL, hh);
  }
  err |= matvec_rows(&L->down, e, hh, dd);
  if (g) memcpy(g, gg, sizeof(double) * I);
  if (u) memcpy(u, uu, sizeof(double) * I);
  if (h) memcpy(h, hh, sizeof(double) * I);
  if (d) memcpy(d, dd, sizeof(double) * H);
  free(xg); free(gg); free(uu); free(hh); free(dd);
  if (err) return QKO_ERR_NAN_SCALE;
  return aq_err ? QKO_ERR_INVALID_ARG : QKO_OK;  /* a non-finite activation */
}

int qko_expert_ffn(const qko_layer* L, int32_t e, const uint16_t* x_bf16,
                   double* g, double* u, double* h, double* d) {
  return qko_expert_ffn_aq(L, e, x_bf16, QKO_ACT_NONE, g, u, h, d);
}

/* Weighted combine: y[t] = sum over slots s = 0..k-1, in that order, of
 * w[t][s] * d_{t,s}. */
int qko_moe_forward_aq(const qko_layer* L, const uint16_t* x_bf16, int32_t T,
                       const int32_t* ids, const double* w, int32_t k, int32_t aq, double* y) {
  int32_t t, s, m, H;
  double* d;
  if (!check_layer(L) || T < 0 || k <= 0 || (T > 0 && (!x_bf16 || !ids || !w || !y)))
    return QKO_ERR_INVALID_ARG;
  H = L->hidden;
  for (t = 0; t < T; ++t)
    for (s = 0; s < k; ++s) {
      int32_t e = ids[(int64_t)t * k + s];
      if (e < 0 || e >= L->gate.n_experts || e >= L->up.n_experts || e >= L->down.n_experts)
        return QKO_ERR_INVALID_ARG;
    }
  d = (double*)malloc(sizeof(double) * H);
  for (t = 0; t < T; ++t) {
    double* yt = y + (int64_t)t * H;
    for (m = 0; m < H; ++m) yt[m] = 0.0;
    for (s = 0; s < k; ++s) {
      int err = qko_expert_ffn_aq(L, ids[(int64_t)t * k + s], x_bf16 + (int64_t)t * H, aq, NULL,
                                  NULL, NULL, d);
      if (err) { free(d); return err; }
      for (m = 0; m < H; ++m) yt[m] += w[(int64_t)t * k + s] * d[m];
    }
  }
  free(d);
  return QKO_OK;
}

int qko_moe_forward(const qko_layer* L, const uint16_t* x_bf16, int32_t T,
                    const int32_t* ids, const double* w, int32_t k, double* y) {
  return qko_moe_forward_aq(L, x_bf16, T, ids, w, k, QKO_ACT_NONE, y);
}

/* ------------------------------------------------------ FP8 block-128 --
 * Dense FP8 linear (IQ2XXS-Q2K-FP8 page: "FP8 E4M3, block-128, UE8M0
 * scales"): weight [N][K] e4m3 with one power-of-two scale per b x b tile,
 * scales [ceil(N/b)][ceil(K/b)].  dq = e4m3 * 2^(s-127), exact in fp64. */
static int fp8_linear_d(const double* x, int32_t M, int32_t K, const uint8_t* w,
                        const uint8_t* ws, int32_t N, int32_t b, double* y) {
  int32_t kb = (K + b - 1) / b, n, err = QKO_OK;
#pragma omp parallel
  {
    double* row = (double*)malloc(sizeof(double) * K);
#pragma omp for schedule(static)
    for (n = 0; n < N; ++n) {
      int32_t k, mm, bad = 0;
      for (k = 0; k < K; ++k) {
        uint8_t sc = ws[(int64_t)(n / b) * kb + k / b];
        if (sc == 255) bad = 1;
        row[k] = qko_e4m3_value(w[(int64_t)n * K + k]) * qko_e8m0_value(sc);
      }
      if (bad) {
#pragma omp atomic write
        err = QKO_ERR_NAN_SCALE;
      }
      for (mm = 0; mm < M; ++mm) {
        double acc = 0.0;
        const double* xr = x + (int64_t)mm * K;
        for (k = 0; k < K; ++k) acc += row[k] * xr[k];
        y[(int64_t)mm * N + n] = acc;
      }
    }
    free(row);
  }
  return err;
}

int qko_fp8_block_linear(const uint16_t* x_bf16, int32_t M, int32_t K,
                         const uint8_t* w, const uint8_t* w_scale, int32_t N,
                         int32_t block, double* y) {
  int64_t i;
  double* x;
  int err;
  if (!x_bf16 || !w || !w_scale || !y || M < 0 || K <= 0 || N <= 0 || block <= 0)
    return QKO_ERR_INVALID_ARG;
  x = (double*)malloc(sizeof(double) * (size_t)M * K);
  for (i = 0; i < (int64_t)M * K; ++i) x[i] = qko_bf16_value(x_bf16[i]);
  err = fp8_linear_d(x, M, K, w, w_scale, N, block, y);
  free(x);
  return err;
}

int qko_fp8_swiglu_ffn(const uint16_t* x_bf16, int32_t M, int32_t H, int32_t I,
                       const uint8_t* wg, const uint8_t* sg,
                       const uint8_t* wu, const uint8_t* su,
                       const uint8_t* wd, const uint8_t* sd,
                       int32_t block, double* y) {
  int64_t i;
  int err = QKO_OK;
  double *x, *g, *u;
  if (!x_bf16 || !wg || !sg || !wu || !su || !wd || !sd || !y || M < 0 || H <= 0 || I <= 0 ||
      block <= 0)
    return QKO_ERR_INVALID_ARG;
  x = (double*)malloc(sizeof(double) * (size_t)M * H);
  g = (double*)malloc(sizeof(double) * (size_t)M * I);
  u = (double*)malloc(sizeof(double) * (size_t)M * I);
  for (i = 0; i < (int64_t)M * H; ++i) x[i] = qko_bf16_value(x_bf16[i]);
  err |= fp8_linear_d(x, M, H, wg, sg, I, block, g);
  err |= fp8_linear_d(x, M, H, wu, su, I, block, u);
  for (i = 0; i < (int64_t)M * I; ++i) g[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
  err |= fp8_linear_d(g, M, I, wd, sd, H, block, y);
  free(x); free(g); free(u);
  return err ? QKO_ERR_NAN_SCALE : QKO_OK;
}

void qko_set_threads(int32_t n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int32_t qko_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
