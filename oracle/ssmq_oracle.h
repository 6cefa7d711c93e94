/*
 * ssmq_oracle.h -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * Plain, sequential, double-precision CPU oracle for the W8A8 selective
 * state-space hot path: the symmetric int8 group quantizer, the three-mode
 * soft-edge codec, the Mamba-1 diagonal selective scan, the Mamba-2 SSD scan
 * (sequential definition plus an independent chunked form used only as a
 * self-check), the single-token decode state update and the offline
 * calibration steps (per-channel absmax, sort-and-cluster, percentile
 * thresholds).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may load
 * this library.  It shares no code, header, table or helper with the CUDA
 * library; neither includes or links the other.
 *
 * Conventions shared with the GPU path only through the *problem statement*:
 *   - binary16 inputs are passed as raw uint16_t bit patterns and converted to
 *     double exactly;
 *   - every floating-point step of the scans runs in double, sequential in
 *     time, so the oracle is the plain definition of the recurrence;
 *   - the quantizers follow binary32 semantics exactly (correctly rounded fp32
 *     quotient, then round-half-to-even to an integer, then clamp), so their
 *     outputs are unique and can be compared bit for bit.
 */
#ifndef SSMQ_ORACLE_H
#define SSMQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* x operand formats */
#define ORC_X_INT8_GROUP 0 /* int8 code, per-channel-cluster fp32 scale */
#define ORC_X_SOFTEDGE 1   /* soft-edge byte code, one base scale */

/* quantizer scale modes */
#define ORC_SCALE_STATIC 0 /* scales are inputs */
#define ORC_SCALE_ABSMAX 1 /* scales are outputs: fl32(absmax / 127) */

/* ---- conversions ------------------------------------------------------- */
double orc_half_to_double(uint16_t h);

/* ---- symmetric int8 group quantizer ------------------------------------
 * Element (o, m, i) of an (outer, mid, inner) array lives at
 * (o * mid + m) * inner + i and belongs to group group_of_mid[m].
 * src_is_f16 = 1: src holds binary16 bits; 0: binary32.
 * Returns the number of non-finite inputs (each encoded as 0), or -1 on
 * invalid arguments. */
int64_t orc_quantize_groups(const void* src, int32_t src_is_f16, int64_t outer,
                            int64_t mid, int64_t inner,
                            const int32_t* group_of_mid, int32_t n_groups,
                            int32_t mode, float* scales, int8_t* q);

/* ---- three-mode soft-edge codec ---------------------------------------- */
int64_t orc_softedge_encode(const void* src, int32_t src_is_f16, int64_t n,
                            float scale, float thr_lo, float thr_hi,
                            int32_t log2_ratio, uint8_t* codes);
void orc_softedge_decode(const uint8_t* codes, int64_t n, float scale,
                         int32_t log2_ratio, float* out);

/* ---- Mamba-1 diagonal selective scan ----------------------------------- */
typedef struct {
  int64_t batch, seqlen, dim, dstate, ngroups; /* b, L, d, N, G */
  int32_t state_group_size;                    /* states per B/C scale */
  int32_t x_format;                            /* ORC_X_* */
  const void* x;                               /* (b, d, L) int8 / uint8 */
  const int32_t* x_group;                      /* [d] cluster id */
  const float* x_scale;                        /* [clusters] */
  float se_scale;                              /* soft-edge base scale */
  int32_t se_log2_ratio;                       /* 2: /4 and x4 */
  const uint16_t* dt;                          /* (b, d, L) binary16 */
  const float* dt_bias;                        /* [d] or NULL */
  int32_t dt_softplus;                         /* 1: delta = softplus */
  const float* A;                              /* (d, N) */
  const float* D;                              /* [d] or NULL */
  const uint16_t* z;                           /* (b, d, L) or NULL */
  const int8_t* B;                             /* (b, G, N, L) */
  const int8_t* C;                             /* (b, G, N, L) */
  const float* B_scale;                        /* [G * N / gs] */
  const float* C_scale;                        /* [G * N / gs] */
  const float* h0;                             /* (b, d, N) or NULL */
} orc_m1_problem;

/* units: NULL for all b*d (batch, channel) recurrences in order, else a list
 * of unit ids u = batch * d + channel.  y: [n_units, L]; h_final:
 * [n_units, N] (either may be NULL).  Returns 0, or -1 on invalid args. */
int32_t orc_m1_scan(const orc_m1_problem* p, int64_t n_units,
                    const int64_t* units, double* y, double* h_final,
                    int32_t n_threads);

/* ---- Mamba-2 SSD scan (scalar A per head) ------------------------------ */
typedef struct {
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups; /* b L H P N G */
  int32_t state_group_size;
  int32_t x_format;
  const void* x;           /* (b, L, H, P) */
  const int32_t* x_group;  /* [H * P] */
  const float* x_scale;
  float se_scale;
  int32_t se_log2_ratio;
  const uint16_t* dt;      /* (b, L, H) */
  const float* dt_bias;    /* [H] or NULL */
  int32_t dt_softplus;
  const float* A;          /* [H] */
  const float* D;          /* [H] or NULL */
  const uint16_t* z;       /* (b, L, H, P) or NULL */
  const int8_t* B;         /* (b, L, G, N) */
  const int8_t* C;         /* (b, L, G, N) */
  const float* B_scale;    /* [G * N / gs] */
  const float* C_scale;
  const float* h0;         /* (b, H, P, N) or NULL */
} orc_ssd_problem;

/* Sequential definition.  units: u = batch * H + head.  y: [n_units, L, P];
 * h_final: [n_units, P, N]. */
int32_t orc_ssd_scan(const orc_ssd_problem* p, int64_t n_units,
                     const int64_t* units, double* y, double* h_final,
                     int32_t n_threads);
/* Chunked (state-space-duality) form of the same map, used only to pin the
 * sequential definition and vice versa. */
int32_t orc_ssd_scan_chunked(const orc_ssd_problem* p, int64_t chunk,
                             int64_t n_units, const int64_t* units, double* y,
                             double* h_final, int32_t n_threads);

/* ---- single-token decode state update ---------------------------------- */
typedef struct {
  int64_t batch, nheads, headdim, dstate, ngroups; /* b H P N G */
  int32_t state_group_size;
  int32_t x_format;
  const void* x;           /* (b, H, P) */
  const int32_t* x_group;  /* [H * P] */
  const float* x_scale;
  float se_scale;
  int32_t se_log2_ratio;
  const uint16_t* dt;      /* (b, H) */
  const float* dt_bias;    /* [H] or NULL */
  int32_t dt_softplus;
  const float* A;          /* [H] */
  const float* D;          /* [H] or NULL */
  const uint16_t* z;       /* (b, H, P) or NULL */
  const int8_t* B;         /* (b, G, N) */
  const int8_t* C;         /* (b, G, N) */
  const float* B_scale;
  const float* C_scale;
} orc_decode_problem;

/* state: [n_units, P, N] in/out (double); y: [n_units, P]. */
int32_t orc_decode_step(const orc_decode_problem* p, int64_t n_units,
                        const int64_t* units, double* state, double* y);

/* Mamba-1 decode (diagonal A per (channel, state)); units u = batch*d + c.
 * x, dt, z: (b, d); B, C: (b, G, N); state [n_units, N]; y [n_units]. */
int32_t orc_m1_decode_step(const orc_m1_problem* p, int64_t n_units,
                           const int64_t* units, double* state, double* y);

/* ---- offline calibration ----------------------------------------------- */
/* absmax over (outer, inner) for every mid index; non-finite values skipped */
void orc_absmax_per_mid(const void* src, int32_t src_is_f16, int64_t outer,
                        int64_t mid, int64_t inner, double* absmax);
/* sort channels by absmax (ascending, ties by index), cut into k contiguous
 * clusters of floor-divided size, scale_j = fl32(max absmax in j / 127). */
int32_t orc_cluster_by_absmax(const double* absmax, int64_t n, int32_t k,
                              int32_t* cluster_of, float* scales);
/* q-th percentile (linear interpolation between order statistics) of |v| */
double orc_percentile_abs(const void* src, int32_t src_is_f16, int64_t n,
                          double q);
/* soft-edge parameters thr = {scale, lo, hi}: lo, hi from the q_lo / q_hi
 * percentiles of |v| (rounded to binary32), blended as alpha new +
 * (1 - alpha) previous when alpha != 1, then scale = fl32(hi / 63). */
void orc_softedge_thresholds(const void* src, int32_t src_is_f16, int64_t n, double q_lo,
                             double q_hi, double alpha, float* thr);


/* ---- causal depthwise convolution + SiLU (producer of the scan input) ---
 * binary32 evaluation defined step by step in ssmq_oracle.c; x (b, d, L)
 * binary16 bits, weight (d, W) fp32, bias fp32[d] or NULL, x_prev (b, d, W-1)
 * binary16 or NULL (zeros), u (b, d, L) fp32 out, x_prev_out (b, d, W-1) or
 * NULL.  Returns the number of non-finite u, -1 on invalid arguments. */
float orc_exp_f32(float v);
float orc_silu_f32(float a);
void orc_exp_f32_n(const float* v, int64_t n, float* out);
void orc_silu_f32_n(const float* a, int64_t n, float* out);
int64_t orc_conv_silu(const uint16_t* x, const uint16_t* x_prev, const float* weight,
                      const float* bias, int64_t batch, int64_t dim, int64_t seqlen,
                      int32_t width, float* u, uint16_t* x_prev_out);

#ifdef __cplusplus
}
#endif
#endif /* SSMQ_ORACLE_H */
