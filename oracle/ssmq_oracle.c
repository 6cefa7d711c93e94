/*
 * ssmq_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * The plain, slow, double-precision CPU oracle for the W8A8 selective
 * state-space hot path.  Every function states the passage it follows:
 *
 *   [Q2]  "Quamba2: A Robust and Scalable Post-training Quantization
 *         Framework for Selective State Space Models" (shd-paper.top card):
 *         abstract (8-bit inputs of a linear recurrence; sort-and-cluster of
 *         x; per-state-group quantization of B and C; offline weight
 *         rearrangement for compute invariance) and the technical-framework
 *         steps 1-4 of the method section.
 *   [SD]  "SSDi8" (arxivdaily card): English abstract (SSD integrates the
 *         recurrent and attention modes; a persistent INT8 path).
 *   [SE]  Quamba-SE soft-edge quantization write-up (wmrh.cn): section 1
 *         (one scale maps floats to INT8), 2.1 (three modes: scale/4 for
 *         |v| < L, scale, scale*4 for |v| > H), 2.2 (range classifier and the
 *         0xxxxxxx / 10xxxxxx / 11xxxxxx byte codes with 6 data bits),
 *         4.1 (L = 5th, H = 99.9th percentile; shift-only ratio 2).
 *
 * The recurrence itself is the Mamba selective state-space model that [Q2]
 * and [SD] quantize (Mamba-1 and Mamba-2 backbones):
 *     h_t = exp(delta_t * A) (.) h_{t-1} + delta_t * B_t * x_t
 *     y_t = C_t . h_t + D * x_t,   optionally y_t *= silu(z_t)
 * with delta_t = softplus(dt_t + dt_bias) when requested.  The oracle runs
 * that definition sequentially in time, in double precision.  Where the pages
 * are silent (operand layouts, the soft-edge payload width, the comparison
 * operators lost from the RTL snippet) the readings are the ones listed in
 * the design notes; each is restated at the function that uses it.
 *
 * No blocking, fusion or reordering beyond the definitions: the chunked SSD
 * form below exists only as an independent cross-check of the sequential one.
 */
#include "ssmq_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* conversions                                                               */
/* ------------------------------------------------------------------------ */

/* IEEE binary16 -> double, exact (1 sign, 5 exponent, 10 fraction bits). */
double orc_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 31;
  int m = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* zero or subnormal */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m + 1024), e - 25);
  return sign ? -v : v;
}

static float orc_load_f32(const void* src, int32_t is_f16, int64_t i) {
  if (is_f16) return (float)orc_half_to_double(((const uint16_t*)src)[i]);
  return ((const float*)src)[i];
}

/* ------------------------------------------------------------------------ */
/* symmetric int8 quantization, binary32 semantics                           */
/* ------------------------------------------------------------------------ */

/* q = clamp(round_half_even(fl32(v / step)), -lim, lim).
 * [SE] section 1: one scale factor maps floats onto the 8-bit integer grid.
 * The fp32 quotient is formed first (double division rounded once to float
 * is the correctly rounded binary32 quotient, since 53 >= 2*24 + 2), and only
 * then rounded to an integer, ties to even (nearbyint under the default
 * FE_TONEAREST mode). */
static int32_t orc_q_rne(float v, float step, int32_t lim) {
  float r = (float)((double)v / (double)step);
  double k = nearbyint((double)r);
  if (k > (double)lim) k = (double)lim;
  if (k < -(double)lim) k = -(double)lim;
  return (int32_t)k;
}

/* [Q2] abstract and method steps 2-3: one scale per group (a cluster of
 * x channels, or a block of states of B/C).  STATIC: scales are calibrated
 * offline and given.  ABSMAX: scale_g = fl32(max|v| over the group / 127).
 * A zero (or negative / non-finite) scale quantizes every element to 0.
 * Non-finite inputs are encoded as 0 and counted. */
int64_t orc_quantize_groups(const void* src, int32_t src_is_f16, int64_t outer,
                            int64_t mid, int64_t inner,
                            const int32_t* group_of_mid, int32_t n_groups,
                            int32_t mode, float* scales, int8_t* q) {
  if (outer < 0 || mid < 0 || inner < 0 || n_groups <= 0) return -1;
  for (int64_t m = 0; m < mid; ++m)
    if (group_of_mid[m] < 0 || group_of_mid[m] >= n_groups) return -1;
  if (mode == ORC_SCALE_ABSMAX) {
    double* amax = (double*)calloc((size_t)n_groups, sizeof(double));
    for (int64_t o = 0; o < outer; ++o)
      for (int64_t m = 0; m < mid; ++m)
        for (int64_t i = 0; i < inner; ++i) {
          float v = orc_load_f32(src, src_is_f16, (o * mid + m) * inner + i);
          if (!isfinite(v)) continue;
          double a = fabs((double)v);
          if (a > amax[group_of_mid[m]]) amax[group_of_mid[m]] = a;
        }
    for (int32_t g = 0; g < n_groups; ++g)
      scales[g] = (float)(amax[g] / 127.0); /* fl32 of the exact quotient */
    free(amax);
  } else if (mode != ORC_SCALE_STATIC) {
    return -1;
  }
  int64_t nonfinite = 0;
  for (int64_t o = 0; o < outer; ++o)
    for (int64_t m = 0; m < mid; ++m) {
      float s = scales[group_of_mid[m]];
      int ok = isfinite(s) && s > 0.0f;
      for (int64_t i = 0; i < inner; ++i) {
        int64_t e = (o * mid + m) * inner + i;
        float v = orc_load_f32(src, src_is_f16, e);
        if (!isfinite(v)) {
          q[e] = 0;
          ++nonfinite;
          continue;
        }
        q[e] = ok ? (int8_t)orc_q_rne(v, s, 127) : (int8_t)0;
      }
    }
  return nonfinite;
}

/* ------------------------------------------------------------------------ */
/* three-mode soft-edge codec                                                */
/* ------------------------------------------------------------------------ */

enum { ORC_MODE_STD = 0, ORC_MODE_SMALL = 1, ORC_MODE_LARGE = 2 };

/* Step size of a mode, [SE] 2.1: scale / 2^r for the high-precision (small)
 * mode, scale for the standard mode, scale * 2^r for the outlier (large)
 * mode; r = 2 gives the page's /4 and x4, r = 1 the shift-only /2 and x2 of
 * 4.1.  The product is exact in double and rounded once to binary32. */
static float orc_mode_step(float s, int mode, int32_t r) {
  double f = 1.0;
  if (mode == ORC_MODE_SMALL) f = ldexp(1.0, -r);
  if (mode == ORC_MODE_LARGE) f = ldexp(1.0, r);
  return (float)((double)s * f);
}

/* [SE] 2.1 / 2.2.  Classification compares |v| with the thresholds (2.1
 * speaks of absolute value): |v| < L -> small, |v| > H -> large, otherwise
 * standard (the RTL's default branch).  Byte layout (2.2): standard mode is
 * 0xxxxxxx with a 7-bit two's-complement payload (clamped to +-63); small is
 * 10xxxxxx and large is 11xxxxxx, each with a 6-bit two's-complement payload
 * (clamped to +-31).  The mode is chosen by the thresholds alone; the payload
 * then saturates inside that mode.  L > H is rejected.  Non-finite inputs
 * become code 0x00 and are counted. */
int64_t orc_softedge_encode(const void* src, int32_t src_is_f16, int64_t n,
                            float scale, float thr_lo, float thr_hi,
                            int32_t log2_ratio, uint8_t* codes) {
  if (n < 0 || !(thr_lo <= thr_hi) || log2_ratio < 0 || log2_ratio > 8)
    return -1;
  int64_t nonfinite = 0;
  for (int64_t i = 0; i < n; ++i) {
    float v = orc_load_f32(src, src_is_f16, i);
    if (!isfinite(v)) {
      codes[i] = 0;
      ++nonfinite;
      continue;
    }
    float a = fabsf(v);
    int mode = ORC_MODE_STD;
    if (a < thr_lo)
      mode = ORC_MODE_SMALL;
    else if (a > thr_hi)
      mode = ORC_MODE_LARGE;
    float step = orc_mode_step(scale, mode, log2_ratio);
    int32_t lim = (mode == ORC_MODE_STD) ? 63 : 31;
    int32_t qv = (isfinite(step) && step > 0.0f) ? orc_q_rne(v, step, lim) : 0;
    uint8_t c;
    if (mode == ORC_MODE_STD)
      c = (uint8_t)(qv & 0x7F);
    else if (mode == ORC_MODE_SMALL)
      c = (uint8_t)(0x80 | (qv & 0x3F));
    else
      c = (uint8_t)(0xC0 | (qv & 0x3F));
    codes[i] = c;
  }
  return nonfinite;
}

/* Splits a code into (mode, signed payload), [SE] 2.2. */
static void orc_se_split(uint8_t c, int* mode, int32_t* qv) {
  if ((c & 0x80) == 0) {
    int32_t v = c & 0x7F;
    *qv = v >= 64 ? v - 128 : v;
    *mode = ORC_MODE_STD;
  } else {
    int32_t v = c & 0x3F;
    *qv = v >= 32 ? v - 64 : v;
    *mode = (c & 0x40) ? ORC_MODE_LARGE : ORC_MODE_SMALL;
  }
}

/* value = payload * step(mode), rounded once to binary32. */
void orc_softedge_decode(const uint8_t* codes, int64_t n, float scale,
                         int32_t log2_ratio, float* out) {
  for (int64_t i = 0; i < n; ++i) {
    int mode;
    int32_t qv;
    orc_se_split(codes[i], &mode, &qv);
    out[i] = (float)((double)qv * (double)orc_mode_step(scale, mode, log2_ratio));
  }
}

/* ------------------------------------------------------------------------ */
/* scan helpers                                                              */
/* ------------------------------------------------------------------------ */

/* Dequantized x in double: code * scale of the channel's cluster ([Q2]), or a
 * soft-edge code times its mode's step ([SE] 2.2).  Exact in double. */
static double orc_x_value(int32_t fmt, const void* x, int64_t idx,
                          int64_t channel, const int32_t* x_group,
                          const float* x_scale, float se_scale, int32_t r) {
  if (fmt == ORC_X_SOFTEDGE) {
    int mode;
    int32_t qv;
    orc_se_split(((const uint8_t*)x)[idx], &mode, &qv);
    return (double)qv * (double)orc_mode_step(se_scale, mode, r);
  }
  return (double)((const int8_t*)x)[idx] * (double)x_scale[x_group[channel]];
}

/* softplus(v) = log(1 + e^v), evaluated without overflow. */
static double orc_softplus(double v) {
  return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v));
}

/* silu(z) = z * sigmoid(z) */
static double orc_silu(double z) { return z / (1.0 + exp(-z)); }

static double orc_delta(double dtv, double bias, int32_t softplus) {
  double v = dtv + bias;
  return softplus ? orc_softplus(v) : v;
}

/* ---- thread fan-out over independent recurrences ------------------------ */
typedef void (*orc_unit_fn)(const void* prob, int64_t k, int64_t u, void* ctx);
typedef struct {
  orc_unit_fn fn;
  const void* prob;
  const int64_t* units;
  int64_t lo, hi;
  void* ctx;
} orc_job;

static void* orc_job_run(void* arg) {
  orc_job* j = (orc_job*)arg;
  for (int64_t k = j->lo; k < j->hi; ++k)
    j->fn(j->prob, k, j->units ? j->units[k] : k, j->ctx);
  return NULL;
}

static void orc_parallel(orc_unit_fn fn, const void* prob, int64_t n_units,
                         const int64_t* units, void* ctx, int32_t n_threads) {
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  if ((int64_t)n_threads > n_units) n_threads = (int32_t)(n_units > 0 ? n_units : 1);
  orc_job jobs[256];
  pthread_t tid[256];
  for (int32_t t = 0; t < n_threads; ++t) {
    jobs[t].fn = fn;
    jobs[t].prob = prob;
    jobs[t].units = units;
    jobs[t].lo = n_units * t / n_threads;
    jobs[t].hi = n_units * (t + 1) / n_threads;
    jobs[t].ctx = ctx;
  }
  if (n_threads == 1) {
    orc_job_run(&jobs[0]);
    return;
  }
  for (int32_t t = 0; t < n_threads; ++t)
    pthread_create(&tid[t], NULL, orc_job_run, &jobs[t]);
  for (int32_t t = 0; t < n_threads; ++t) pthread_join(tid[t], NULL);
}

typedef struct {
  double* y;
  double* h_final;
  int64_t chunk;
} orc_out;

/* ------------------------------------------------------------------------ */
/* Mamba-1 diagonal selective scan                                           */
/* ------------------------------------------------------------------------ */

/* One (batch, channel) recurrence, sequential over t, N states in double.
 * A is diagonal per (channel, state); B and C are shared by the channels of
 * group g = floor(c * G / d) and carry one fp32 scale per block of
 * state_group_size states ([Q2] per-state-group quantization). */
static void orc_m1_unit(const void* vp, int64_t k, int64_t u, void* vctx) {
  const orc_m1_problem* p = (const orc_m1_problem*)vp;
  orc_out* o = (orc_out*)vctx;
  const int64_t d = p->dim, L = p->seqlen, N = p->dstate, G = p->ngroups;
  const int64_t b = u / d, c = u % d, g = c * G / d;
  const int64_t spg = N / p->state_group_size;
  double* h = (double*)malloc((size_t)N * sizeof(double));
  for (int64_t n = 0; n < N; ++n) h[n] = p->h0 ? (double)p->h0[(b * d + c) * N + n] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const int64_t idx = (b * d + c) * L + t;
    const double x = orc_x_value(p->x_format, p->x, idx, c, p->x_group, p->x_scale,
                                 p->se_scale, p->se_log2_ratio);
    const double delta = orc_delta(orc_half_to_double(p->dt[idx]),
                                   p->dt_bias ? (double)p->dt_bias[c] : 0.0, p->dt_softplus);
    double acc = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const int64_t bi = ((b * G + g) * N + n) * L + t;
      const int64_t si = g * spg + n / p->state_group_size;
      const double Bv = (double)p->B[bi] * (double)p->B_scale[si];
      const double Cv = (double)p->C[bi] * (double)p->C_scale[si];
      h[n] = exp(delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;
      acc += Cv * h[n];
    }
    if (p->D) acc += (double)p->D[c] * x;
    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));
    if (o->y) o->y[k * L + t] = acc;
  }
  if (o->h_final)
    for (int64_t n = 0; n < N; ++n) o->h_final[k * N + n] = h[n];
  free(h);
}

static int orc_m1_valid(const orc_m1_problem* p) {
  if (p->batch < 0 || p->seqlen < 0 || p->dim <= 0 || p->dstate <= 0 || p->ngroups <= 0)
    return 0;
  if (p->dim % p->ngroups) return 0;
  if (p->state_group_size <= 0 || p->dstate % p->state_group_size) return 0;
  return 1;
}

int32_t orc_m1_scan(const orc_m1_problem* p, int64_t n_units,
                    const int64_t* units, double* y, double* h_final,
                    int32_t n_threads) {
  if (!orc_m1_valid(p)) return -1;
  if (!units) n_units = p->batch * p->dim;
  orc_out o = {y, h_final, 0};
  orc_parallel(orc_m1_unit, p, n_units, units, &o, n_threads);
  return 0;
}

/* Mamba-1 single-token step: the same update for one t; x, dt, z: (b, d);
 * B, C: (b, G, N). */
typedef struct {
  double* state;
  double* y;
} orc_dec_out;

static void orc_m1_decode_unit(const void* vp, int64_t k, int64_t u, void* vctx) {
  const orc_m1_problem* p = (const orc_m1_problem*)vp;
  orc_dec_out* o = (orc_dec_out*)vctx;
  const int64_t d = p->dim, N = p->dstate, G = p->ngroups;
  const int64_t b = u / d, c = u % d, g = c * G / d;
  const int64_t spg = N / p->state_group_size;
  const int64_t idx = b * d + c;
  const double x = orc_x_value(p->x_format, p->x, idx, c, p->x_group, p->x_scale,
                               p->se_scale, p->se_log2_ratio);
  const double delta = orc_delta(orc_half_to_double(p->dt[idx]),
                                 p->dt_bias ? (double)p->dt_bias[c] : 0.0, p->dt_softplus);
  double acc = 0.0;
  double* h = o->state + k * N;
  for (int64_t n = 0; n < N; ++n) {
    const int64_t bi = (b * G + g) * N + n;
    const int64_t si = g * spg + n / p->state_group_size;
    const double Bv = (double)p->B[bi] * (double)p->B_scale[si];
    const double Cv = (double)p->C[bi] * (double)p->C_scale[si];
    h[n] = exp(delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;
    acc += Cv * h[n];
  }
  if (p->D) acc += (double)p->D[c] * x;
  if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));
  if (o->y) o->y[k] = acc;
}

int32_t orc_m1_decode_step(const orc_m1_problem* p, int64_t n_units,
                           const int64_t* units, double* state, double* y) {
  if (!orc_m1_valid(p)) return -1;
  if (!units) n_units = p->batch * p->dim;
  orc_dec_out o = {state, y};
  orc_parallel(orc_m1_decode_unit, p, n_units, units, &o, 1);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Mamba-2 SSD: sequential definition                                        */
/* ------------------------------------------------------------------------ */

static int orc_ssd_valid(const orc_ssd_problem* p) {
  if (p->batch < 0 || p->seqlen < 0 || p->nheads <= 0 || p->headdim <= 0 ||
      p->dstate <= 0 || p->ngroups <= 0)
    return 0;
  if (p->nheads % p->ngroups) return 0;
  if (p->state_group_size <= 0 || p->dstate % p->state_group_size) return 0;
  return 1;
}

/* [SD]: Mamba-2's SSD layer is the same recurrence with a scalar A per head
 * and a P x N state per head; head h reads B/C group floor(h * G / H). */
static void orc_ssd_unit(const void* vp, int64_t k, int64_t u, void* vctx) {
  const orc_ssd_problem* p = (const orc_ssd_problem*)vp;
  orc_out* o = (orc_out*)vctx;
  const int64_t H = p->nheads, P = p->headdim, N = p->dstate, G = p->ngroups, L = p->seqlen;
  const int64_t b = u / H, hd = u % H, g = hd * G / H;
  const int64_t spg = N / p->state_group_size;
  double* h = (double*)malloc((size_t)(P * N) * sizeof(double));
  double* Bv = (double*)malloc((size_t)N * sizeof(double));
  double* Cv = (double*)malloc((size_t)N * sizeof(double));
  for (int64_t i = 0; i < P * N; ++i)
    h[i] = p->h0 ? (double)p->h0[(b * H + hd) * P * N + i] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const double delta = orc_delta(orc_half_to_double(p->dt[(b * L + t) * H + hd]),
                                   p->dt_bias ? (double)p->dt_bias[hd] : 0.0, p->dt_softplus);
    const double dA = exp(delta * (double)p->A[hd]);
    for (int64_t n = 0; n < N; ++n) {
      const int64_t bi = ((b * L + t) * G + g) * N + n;
      const int64_t si = g * spg + n / p->state_group_size;
      Bv[n] = (double)p->B[bi] * (double)p->B_scale[si];
      Cv[n] = (double)p->C[bi] * (double)p->C_scale[si];
    }
    for (int64_t pp = 0; pp < P; ++pp) {
      const int64_t xi = ((b * L + t) * H + hd) * P + pp;
      const double x = orc_x_value(p->x_format, p->x, xi, hd * P + pp, p->x_group,
                                   p->x_scale, p->se_scale, p->se_log2_ratio);
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        h[pp * N + n] = dA * h[pp * N + n] + delta * Bv[n] * x;
        acc += Cv[n] * h[pp * N + n];
      }
      if (p->D) acc += (double)p->D[hd] * x;
      if (p->z) acc *= orc_silu(orc_half_to_double(p->z[xi]));
      if (o->y) o->y[(k * L + t) * P + pp] = acc;
    }
  }
  if (o->h_final)
    for (int64_t i = 0; i < P * N; ++i) o->h_final[k * P * N + i] = h[i];
  free(h);
  free(Bv);
  free(Cv);
}

int32_t orc_ssd_scan(const orc_ssd_problem* p, int64_t n_units,
                     const int64_t* units, double* y, double* h_final,
                     int32_t n_threads) {
  if (!orc_ssd_valid(p)) return -1;
  if (!units) n_units = p->batch * p->nheads;
  orc_out o = {y, h_final, 0};
  orc_parallel(orc_ssd_unit, p, n_units, units, &o, n_threads);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Mamba-2 SSD: chunked (state-space-duality) form, self-check only          */
/* ------------------------------------------------------------------------ */

/* [SD] abstract: SSD combines a recurrent mode and an attention mode.  Split
 * the sequence into chunks of Q steps; inside a chunk, with the inclusive
 * cumulative sum S_t = sum_{r <= t} delta_r * A:
 *   y_t = sum_{s <= t} (C_t . B_s) exp(S_t - S_s) delta_s x_s     (attention)
 *       + exp(S_t) C_t . h_prev                                    (carry in)
 *       + D x_t
 *   h_next = exp(S_last) h_prev + sum_s exp(S_last - S_s) delta_s x_s B_s^T
 * This is algebraically the recurrence unrolled over one chunk. */
static void orc_ssd_chunk_unit(const void* vp, int64_t k, int64_t u, void* vctx) {
  const orc_ssd_problem* p = (const orc_ssd_problem*)vp;
  orc_out* o = (orc_out*)vctx;
  const int64_t H = p->nheads, P = p->headdim, N = p->dstate, G = p->ngroups, L = p->seqlen;
  const int64_t Q = o->chunk;
  const int64_t b = u / H, hd = u % H, g = hd * G / H;
  const int64_t spg = N / p->state_group_size;
  double* h = (double*)malloc((size_t)(P * N) * sizeof(double));
  double* hn = (double*)malloc((size_t)(P * N) * sizeof(double));
  double* S = (double*)malloc((size_t)Q * sizeof(double));
  double* dl = (double*)malloc((size_t)Q * sizeof(double));
  double* xs = (double*)malloc((size_t)(Q * P) * sizeof(double));
  double* Bs = (double*)malloc((size_t)(Q * N) * sizeof(double));
  double* Cs = (double*)malloc((size_t)(Q * N) * sizeof(double));
  double* CB = (double*)malloc((size_t)(Q * Q) * sizeof(double));
  for (int64_t i = 0; i < P * N; ++i)
    h[i] = p->h0 ? (double)p->h0[(b * H + hd) * P * N + i] : 0.0;
  for (int64_t c0 = 0; c0 < L; c0 += Q) {
    const int64_t Qc = (L - c0 < Q) ? (L - c0) : Q;
    double run = 0.0;
    for (int64_t t = 0; t < Qc; ++t) {
      const int64_t tt = c0 + t;
      dl[t] = orc_delta(orc_half_to_double(p->dt[(b * L + tt) * H + hd]),
                        p->dt_bias ? (double)p->dt_bias[hd] : 0.0, p->dt_softplus);
      run += dl[t] * (double)p->A[hd];
      S[t] = run;
      for (int64_t pp = 0; pp < P; ++pp) {
        const int64_t xi = ((b * L + tt) * H + hd) * P + pp;
        xs[t * P + pp] = orc_x_value(p->x_format, p->x, xi, hd * P + pp, p->x_group,
                                     p->x_scale, p->se_scale, p->se_log2_ratio);
      }
      for (int64_t n = 0; n < N; ++n) {
        const int64_t bi = ((b * L + tt) * G + g) * N + n;
        const int64_t si = g * spg + n / p->state_group_size;
        Bs[t * N + n] = (double)p->B[bi] * (double)p->B_scale[si];
        Cs[t * N + n] = (double)p->C[bi] * (double)p->C_scale[si];
      }
    }
    for (int64_t t = 0; t < Qc; ++t)
      for (int64_t s = 0; s <= t; ++s) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) acc += Cs[t * N + n] * Bs[s * N + n];
        CB[t * Q + s] = acc;
      }
    for (int64_t t = 0; t < Qc; ++t) {
      const int64_t tt = c0 + t;
      for (int64_t pp = 0; pp < P; ++pp) {
        double yd = 0.0;
        for (int64_t s = 0; s <= t; ++s)
          yd += CB[t * Q + s] * exp(S[t] - S[s]) * dl[s] * xs[s * P + pp];
        double yo = 0.0;
        for (int64_t n = 0; n < N; ++n) yo += Cs[t * N + n] * h[pp * N + n];
        double acc = yd + exp(S[t]) * yo;
        if (p->D) acc += (double)p->D[hd] * xs[t * P + pp];
        const int64_t xi = ((b * L + tt) * H + hd) * P + pp;
        if (p->z) acc *= orc_silu(orc_half_to_double(p->z[xi]));
        if (o->y) o->y[(k * L + tt) * P + pp] = acc;
      }
    }
    const double Sl = S[Qc - 1];
    for (int64_t pp = 0; pp < P; ++pp)
      for (int64_t n = 0; n < N; ++n) {
        double acc = exp(Sl) * h[pp * N + n];
        for (int64_t s = 0; s < Qc; ++s)
          acc += exp(Sl - S[s]) * dl[s] * Bs[s * N + n] * xs[s * P + pp];
        hn[pp * N + n] = acc;
      }
    memcpy(h, hn, (size_t)(P * N) * sizeof(double));
  }
  if (o->h_final)
    for (int64_t i = 0; i < P * N; ++i) o->h_final[k * P * N + i] = h[i];
  free(h);
  free(hn);
  free(S);
  free(dl);
  free(xs);
  free(Bs);
  free(Cs);
  free(CB);
}

int32_t orc_ssd_scan_chunked(const orc_ssd_problem* p, int64_t chunk,
                             int64_t n_units, const int64_t* units, double* y,
                             double* h_final, int32_t n_threads) {
  if (!orc_ssd_valid(p) || chunk <= 0) return -1;
  if (!units) n_units = p->batch * p->nheads;
  orc_out o = {y, h_final, chunk};
  orc_parallel(orc_ssd_chunk_unit, p, n_units, units, &o, n_threads);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Mamba-2 single-token decode state update                                  */
/* ------------------------------------------------------------------------ */

/* [Q2] abstract / generation stage: one step of the recurrence on the
 * persistent state, in place. */
static void orc_decode_unit(const void* vp, int64_t k, int64_t u, void* vctx) {
  const orc_decode_problem* p = (const orc_decode_problem*)vp;
  orc_dec_out* o = (orc_dec_out*)vctx;
  const int64_t H = p->nheads, P = p->headdim, N = p->dstate, G = p->ngroups;
  const int64_t b = u / H, hd = u % H, g = hd * G / H;
  const int64_t spg = N / p->state_group_size;
  const double delta = orc_delta(orc_half_to_double(p->dt[b * H + hd]),
                                 p->dt_bias ? (double)p->dt_bias[hd] : 0.0, p->dt_softplus);
  const double dA = exp(delta * (double)p->A[hd]);
  double* h = o->state + k * P * N;
  for (int64_t pp = 0; pp < P; ++pp) {
    const int64_t xi = (b * H + hd) * P + pp;
    const double x = orc_x_value(p->x_format, p->x, xi, hd * P + pp, p->x_group,
                                 p->x_scale, p->se_scale, p->se_log2_ratio);
    double acc = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const int64_t bi = (b * G + g) * N + n;
      const int64_t si = g * spg + n / p->state_group_size;
      const double Bv = (double)p->B[bi] * (double)p->B_scale[si];
      const double Cv = (double)p->C[bi] * (double)p->C_scale[si];
      h[pp * N + n] = dA * h[pp * N + n] + delta * Bv * x;
      acc += Cv * h[pp * N + n];
    }
    if (p->D) acc += (double)p->D[hd] * x;
    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[xi]));
    if (o->y) o->y[k * P + pp] = acc;
  }
}

int32_t orc_decode_step(const orc_decode_problem* p, int64_t n_units,
                        const int64_t* units, double* state, double* y) {
  if (p->batch < 0 || p->nheads <= 0 || p->headdim <= 0 || p->dstate <= 0 ||
      p->ngroups <= 0 || p->nheads % p->ngroups || p->state_group_size <= 0 ||
      p->dstate % p->state_group_size)
    return -1;
  if (!units) n_units = p->batch * p->nheads;
  orc_dec_out o = {state, y};
  orc_parallel(orc_decode_unit, p, n_units, units, &o, 1);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* offline calibration                                                       */
/* ------------------------------------------------------------------------ */

/* [Q2] method step 1: activation statistics per channel (max |v|). */
void orc_absmax_per_mid(const void* src, int32_t src_is_f16, int64_t outer,
                        int64_t mid, int64_t inner, double* absmax) {
  for (int64_t m = 0; m < mid; ++m) absmax[m] = 0.0;
  for (int64_t o = 0; o < outer; ++o)
    for (int64_t m = 0; m < mid; ++m)
      for (int64_t i = 0; i < inner; ++i) {
        float v = orc_load_f32(src, src_is_f16, (o * mid + m) * inner + i);
        if (!isfinite(v)) continue;
        double a = fabs((double)v);
        if (a > absmax[m]) absmax[m] = a;
      }
}

typedef struct {
  double v;
  int64_t i;
} orc_vi;

static int orc_vi_cmp(const void* a, const void* b) {
  const orc_vi* x = (const orc_vi*)a;
  const orc_vi* y = (const orc_vi*)b;
  if (x->v < y->v) return -1;
  if (x->v > y->v) return 1;
  return (x->i > y->i) - (x->i < y->i);
}

/* [Q2] method step 2 and key design 1: sort the channels by their
 * calibration magnitude and cut the sorted order into k clusters; each
 * cluster gets one scale, fl32(largest member absmax / 127).  Reading: k
 * contiguous clusters of (near-)equal size, cluster j holding sorted
 * positions [floor(j n / k), floor((j + 1) n / k)). */
int32_t orc_cluster_by_absmax(const double* absmax, int64_t n, int32_t k,
                              int32_t* cluster_of, float* scales) {
  if (n <= 0 || k <= 0 || k > n) return -1;
  orc_vi* a = (orc_vi*)malloc((size_t)n * sizeof(orc_vi));
  for (int64_t i = 0; i < n; ++i) {
    a[i].v = absmax[i];
    a[i].i = i;
  }
  qsort(a, (size_t)n, sizeof(orc_vi), orc_vi_cmp);
  for (int32_t j = 0; j < k; ++j) {
    const int64_t lo = n * j / k, hi = n * (j + 1) / k;
    for (int64_t r = lo; r < hi; ++r) cluster_of[a[r].i] = j;
    scales[j] = (float)(a[hi - 1].v / 127.0);
  }
  free(a);
  return 0;
}

/* k-th smallest (0-based) of v[0..n), rearranging v (Hoare quickselect). */
static double orc_select(double* v, int64_t n, int64_t k) {
  int64_t lo = 0, hi = n - 1;
  while (lo < hi) {
    const double pivot = v[lo + (hi - lo) / 2];
    int64_t i = lo, j = hi;
    while (i <= j) {
      while (v[i] < pivot) ++i;
      while (v[j] > pivot) --j;
      if (i <= j) {
        double t = v[i];
        v[i] = v[j];
        v[j] = t;
        ++i;
        --j;
      }
    }
    if (k <= j)
      hi = j;
    else if (k >= i)
      lo = i;
    else
      return v[k];
  }
  return v[k];
}

/* [SE] 4.1: L and H are percentiles (5th and 99.9th) of the activation
 * distribution.  Reading: percentiles of |v| over the whole tensor, with
 * linear interpolation between order statistics at position (n - 1) q / 100.
 * Non-finite values are excluded. */
double orc_percentile_abs(const void* src, int32_t src_is_f16, int64_t n,
                          double q) {
  double* v = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
  int64_t m = 0;
  for (int64_t i = 0; i < n; ++i) {
    float f = orc_load_f32(src, src_is_f16, i);
    if (isfinite(f)) v[m++] = fabs((double)f);
  }
  if (m == 0) {
    free(v);
    return 0.0;
  }
  const double pos = (double)(m - 1) * (q / 100.0);
  int64_t k = (int64_t)floor(pos);
  if (k < 0) k = 0;
  if (k > m - 1) k = m - 1;
  const double frac = pos - (double)k;
  const double vk = orc_select(v, m, k);
  double vk1 = vk;
  if (k + 1 < m) {
    /* after selection every element right of k is >= v[k]: take their min */
    vk1 = v[k + 1];
    for (int64_t i = k + 2; i < m; ++i)
      if (v[i] < vk1) vk1 = v[i];
  }
  free(v);
  return vk + frac * (vk1 - vk);
}

/* [SE] 4.1: L at the 5th and H at the 99.9th percentile of the activation
 * magnitudes, refreshed from a new batch by alpha * new + (1 - alpha) *
 * running (alpha = 0.1 there); the base scale puts H at the top of the
 * standard mode (reading: s = H / 63). */
void orc_softedge_thresholds(const void* src, int32_t src_is_f16, int64_t n, double q_lo,
                             double q_hi, double alpha, float* thr) {
  float lo = (float)orc_percentile_abs(src, src_is_f16, n, q_lo);
  float hi = (float)orc_percentile_abs(src, src_is_f16, n, q_hi);
  if (alpha != 1.0) {
    lo = (float)(alpha * (double)lo + (1.0 - alpha) * (double)thr[1]);
    hi = (float)(alpha * (double)hi + (1.0 - alpha) * (double)thr[2]);
  }
  thr[1] = lo;
  thr[2] = hi;
  thr[0] = (float)((double)hi / 63.0);
}

/* ------------------------------------------------------------------------ */
/* causal depthwise convolution + SiLU: the producer of the scan input       */
/* ------------------------------------------------------------------------ */
/* In the Mamba-1 block the scan input x is the output of a short causal
 * depthwise convolution along time followed by SiLU; [SE] 4.1 puts the range
 * check (the quantizer or the soft-edge encoder) where that activation is
 * produced.  The quantizer's code is decided in binary32 (the quantizer's
 * own rule), so the value it is given is defined as a binary32 evaluation,
 * step by step, with IEEE operations only (fused multiply-add, add, multiply,
 * correctly rounded reciprocal) -- reproducible to the bit by any IEEE
 * implementation.  The tests pin every step against double-precision
 * mathematics. */

/* 2^k as an exact binary32 number, -126 <= k <= 127. */
static float orc_pow2f(int k) {
  union {
    uint32_t u;
    float f;
  } b;
  b.u = (uint32_t)(k + 127) << 23;
  return b.f;
}

/* e^v in binary32 by Cody and Waite's argument reduction (published method):
 *   k = round-half-even(fl32(v * log2 e))
 *   r = (v - k LN2_HI) - k LN2_LO, two fused multiply-adds, with
 *       LN2_HI = 0.693145751953125 (16 significant bits: k LN2_HI is exact)
 *       and LN2_LO = fl32(ln 2 - LN2_HI), so |r| <= ln2 / 2 + tiny
 *   p = sum_{n<=7} r^n / n!  (Taylor series, Horner form, fused multiply-adds,
 *       coefficients fl32(1 / n!); the truncation is below 5e-9 relative)
 *   e^v = p * 2^k  (one rounding; subnormal results rounded as IEEE does)
 * Range of this definition: v > 88 gives +inf, v < -87 gives 0, NaN stays
 * NaN. */
float orc_exp_f32(float v) {
  if (v != v) return v;
  if (v > 88.0f) return INFINITY;
  if (v < -87.0f) return 0.0f;
  const float log2e = 1.44269504088896340736f;
  const float ln2_hi = 0.693145751953125f;
  const float ln2_lo = (float)(0.69314718055994530942 - 0.693145751953125);
  const float kf = nearbyintf(v * log2e);
  float r = fmaf(-kf, ln2_hi, v);
  r = fmaf(-kf, ln2_lo, r);
  float p = (float)(1.0 / 5040.0);
  p = fmaf(p, r, (float)(1.0 / 720.0));
  p = fmaf(p, r, (float)(1.0 / 120.0));
  p = fmaf(p, r, (float)(1.0 / 24.0));
  p = fmaf(p, r, (float)(1.0 / 6.0));
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  return p * orc_pow2f((int)kf);
}

/* silu(a) = a sigmoid(a) = a / (1 + e^-a), in binary32:
 *   e = orc_exp_f32(-a); den = fl32(1 + e); r = fl32(1 / den); u = fl32(a r). */
float orc_silu_f32(float a) {
  const float e = orc_exp_f32(-a);
  const float den = 1.0f + e;
  const float r = 1.0f / den;
  return a * r;
}

void orc_exp_f32_n(const float* v, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_exp_f32(v[i]);
}

void orc_silu_f32_n(const float* a, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_silu_f32(a[i]);
}

/* The scan input of channel c at step t, for x (b, d, L) binary16:
 *   a = fl32 chain: a = bias_c (0 without bias); for tap k = 0 .. W-1:
 *       a = fma(w[c][k], x[t - (W - 1) + k], a)   (oldest tap first)
 *   u = orc_silu_f32(a)
 * Steps before t = 0 read the conv state x_prev (b, d, W-1: the W-1 inputs
 * before the call, oldest first), or zero without one.  x_prev_out (if not
 * NULL) receives the W-1 most recent inputs, the state of the next call.
 * Returns the number of non-finite u, or -1 on invalid arguments. */
int64_t orc_conv_silu(const uint16_t* x, const uint16_t* x_prev, const float* weight,
                      const float* bias, int64_t batch, int64_t dim, int64_t seqlen,
                      int32_t width, float* u, uint16_t* x_prev_out) {
  if (batch < 0 || dim < 0 || seqlen < 0 || width < 1 || width > 4) return -1;
  const int64_t W = width, S = width - 1;
  int64_t nonfinite = 0;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t c = 0; c < dim; ++c) {
      const uint16_t* xr = x + (b * dim + c) * seqlen;
      const uint16_t* pr = x_prev ? x_prev + (b * dim + c) * S : NULL;
      for (int64_t t = 0; t < seqlen; ++t) {
        float a = bias ? bias[c] : 0.0f;
        for (int64_t k = 0; k < W; ++k) {
          const int64_t s = t - (W - 1) + k;
          float xv = 0.0f;
          if (s >= 0)
            xv = (float)orc_half_to_double(xr[s]);
          else if (pr)
            xv = (float)orc_half_to_double(pr[S + s]);
          a = fmaf(weight[c * W + k], xv, a);
        }
        const float v = orc_silu_f32(a);
        if (!isfinite(v)) ++nonfinite;
        u[(b * dim + c) * seqlen + t] = v;
      }
      if (x_prev_out)
        for (int64_t j = 0; j < S; ++j) {
          const int64_t s = seqlen - S + j; /* time of state slot j */
          uint16_t h = 0;
          if (s >= 0)
            h = xr[s];
          else if (pr)
            h = pr[S + s];
          x_prev_out[(b * dim + c) * S + j] = h;
        }
    }
  return nonfinite;
}
