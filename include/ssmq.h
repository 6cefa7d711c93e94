/*
 * ssmq.h -- C ABI of the B200 (sm_100a) W8A8 selective state-space library.
 *
 * The library computes the hot path of quantized selective state-space
 * models: the Mamba selective-SSM linear recurrence
 *
 *     h_t = exp(delta_t * A) (.) h_{t-1} + delta_t * B_t * x_t
 *     y_t = C_t . h_t + D * x_t          (optionally y_t *= silu(z_t))
 *     delta_t = softplus(dt_t + dt_bias)  (or dt_t when softplus is off)
 *
 * with int8 x (one fp32 scale per sorted-and-clustered channel group) and
 * int8 B / C (one fp32 scale per block of states), an fp32 state, binary16
 * dt / z / y.  Sources ("the pages"):
 *   - "Quamba2: A Robust and Scalable Post-training Quantization Framework
 *     for Selective State Space Models" (shd-paper.top card), abstract and
 *     the method section's technical framework (steps 1-4): 8-bit inputs of
 *     a linear recurrence, sort-and-cluster of x, per-state-group
 *     quantization of B and C, offline rearrangement for compute invariance;
 *     Mamba1 and Mamba2 backbones; prefill and generation stages.
 *   - "SSDi8" (arxivdaily card), abstract: Mamba-2's structured state-space
 *     duality (SSD) runs a recurrent and an attention mode; a persistent INT8
 *     path; element-wise products decoupled from the matrix products.
 *   - Quamba-SE soft-edge quantization write-up (wmrh.cn), sections 1, 2.1,
 *     2.2, 4.1: one scale maps floats to INT8; three modes scale/4, scale,
 *     scale*4 chosen by |v| < L, |v| > H; byte codes 0xxxxxxx / 10xxxxxx /
 *     11xxxxxx; a range check inside a CUDA quantize/dequantize kernel.
 *
 * General conventions
 *   - Every pointer argument named "device" is CUDA device memory owned by
 *     the caller; the library never allocates, frees or retains memory and
 *     keeps no state besides a thread-local error message.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  SSMQ_OK means the arguments were valid and every
 *     kernel was launched; results are ready once the stream reaches them.
 *   - Argument errors are returned before anything is launched.  No C++
 *     exception crosses the ABI.  ssmq_last_error() describes the most recent
 *     non-OK status of the calling thread.
 *   - Device-side anomalies (non-finite inputs, out-of-range group ids in
 *     device maps, invalid device scales) are OR-ed into the optional device
 *     word `status` as SSMQ_DEV_* bits; the caller reads it after a
 *     synchronisation.  Kernels never trap or assert.
 *   - binary16 tensors are passed as uint16_t bit patterns.
 *   - Tensors are dense, row-major, with the layouts stated per call.  Base
 *     pointers of int8/uint8/binary16 tensors must be 16-byte aligned, fp32
 *     tensors 16-byte aligned (SSMQ_ERR_ALIGNMENT otherwise).
 */
#ifndef SSMQ_H
#define SSMQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSMQ_OK = 0,
  SSMQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad enum, L > H ... */
  SSMQ_ERR_ALIGNMENT = 2,   /* a base pointer violates the alignment rule */
  SSMQ_ERR_UNSUPPORTED = 3, /* valid, but outside the shapes the kernels implement */
  SSMQ_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
  SSMQ_ERR_TIMEOUT = 5,     /* reserved: a bounded device wait gave up */
  SSMQ_ERR_NONFINITE = 6    /* reserved for host-detected non-finite scalars */
} ssmq_status;

/* bits OR-ed into the optional device status word */
#define SSMQ_DEV_NONFINITE 1u /* a non-finite input element was met (coded 0) */
#define SSMQ_DEV_BAD_GROUP 2u /* a device group id was out of range (coded 0) */
#define SSMQ_DEV_BAD_SCALE 4u /* a device scale was negative / non-finite */
#define SSMQ_DEV_TIMEOUT 8u   /* a bounded device wait (tensor core, bulk copy) gave up;
                                 the call's outputs are then incomplete.  Every such
                                 wait probes at most ~2^20 times (about a second).
                                 For tests of this path, the environment variable
                                 SSMQ_WAIT_LIMIT=<probes> (read at each call) lowers
                                 the limit of ssmq_quantize_groups' pipeline waits;
                                 0 makes them give up at once. */

typedef enum { SSMQ_F32 = 0, SSMQ_F16 = 1 } ssmq_dtype;
typedef enum { SSMQ_SCALE_STATIC = 0, SSMQ_SCALE_ABSMAX = 1 } ssmq_scale_mode;
typedef enum {
  SSMQ_X_INT8_GROUP = 0,   /* int8 codes, one fp32 scale per channel cluster */
  SSMQ_X_SOFTEDGE = 1,     /* soft-edge uint8 codes (se_scale, se_log2_ratio) */
  SSMQ_X_F16_GROUP = 2,    /* binary16 x quantized inside the kernel (Mamba-1 scan only) */
  SSMQ_X_F16_SOFTEDGE = 3  /* binary16 x soft-edge encoded inside the kernel (Mamba-1 scan only) */
} ssmq_x_format;

/* ------------------------------------------------------------------------ */
/* Symmetric int8 group quantizer                                           */
/* ------------------------------------------------------------------------ */
/*
 * Passage: Quamba-SE write-up section 1 (one scale factor maps floats onto the
 * 8-bit grid); Quamba2 abstract and method step 3 (one scale per cluster of x
 * channels, one per block of B/C states).
 *
 *   q = clamp(round_half_even(fl32(v / s_g)), -127, 127)
 *
 * with fl32(v / s_g) the correctly rounded binary32 quotient (formed before
 * the integer rounding).  `src` is viewed as an (outer, mid, inner) array:
 * element (o, m, i) sits at (o * mid + m) * inner + i and belongs to group
 * group_of_mid[m] in [0, n_groups).  This covers every layout of the path:
 *   Mamba-1 x (b, d, L):       outer = b,     mid = d,     inner = L
 *   Mamba-1 B/C (b, G, N, L):  outer = b,     mid = G * N, inner = L
 *   Mamba-2 x (b, L, H, P):    outer = b * L, mid = H * P, inner = 1
 *   Mamba-2 B/C (b, L, G, N):  outer = b * L, mid = G * N, inner = 1
 *
 * src          device, binary16 bits or fp32 (dtype), outer*mid*inner elems
 * group_of_mid device int32[mid]
 * mode         SSMQ_SCALE_STATIC: scales[n_groups] (device) are inputs;
 *              SSMQ_SCALE_ABSMAX: scales[g] = fl32(max |v| in g / 127) are
 *              computed and written first (the buffer is also used as the
 *              reduction accumulator)
 * q_out        device int8, same element count
 * status       device uint32 word or NULL
 * Non-finite elements are coded 0 and excluded from the absmax.  A zero scale
 * codes its group as 0.  Errors: INVALID_ARG for null pointers / negative
 * sizes / n_groups < 1 / bad enums; ALIGNMENT for unaligned bases.
 */
ssmq_status ssmq_quantize_groups(const void* src, ssmq_dtype dtype,
                                 int64_t outer, int64_t mid, int64_t inner,
                                 const int32_t* group_of_mid, int32_t n_groups,
                                 ssmq_scale_mode mode, float* scales,
                                 int8_t* q_out, uint32_t* status,
                                 void* stream);

/*
 * Batched static quantization: ssmq_quantize_groups with SSMQ_SCALE_STATIC
 * for n_jobs (1..8) tensors, in one launch for all jobs of one dtype and
 * layout class (e.g. the Mamba-1 layer's x, B and C), each job's tiles taken
 * by its own share of the CTAs.  Results are byte-identical to one
 * ssmq_quantize_groups call per job.  The pages have no counterpart: this is
 * a launch-count optimisation of this library.
 *
 * jobs    host array of n_jobs descriptors (read during the call); each
 *         field as for ssmq_quantize_groups (scales are inputs); the jobs'
 *         q_out ranges must not overlap each other or any src
 * status  device uint32 word or NULL (flags of all jobs)
 * Errors: INVALID_ARG for n_jobs outside [1, 8] or a job that
 * ssmq_quantize_groups would reject; ALIGNMENT likewise.
 */
typedef struct {
  const void* src;
  ssmq_dtype dtype;
  int64_t outer, mid, inner;
  const int32_t* group_of_mid;
  int32_t n_groups;
  const float* scales;
  int8_t* q_out;
} ssmq_quant_job;

ssmq_status ssmq_quantize_groups_batch(const ssmq_quant_job* jobs, int32_t n_jobs,
                                       uint32_t* status, void* stream);

/* ------------------------------------------------------------------------ */
/* Three-mode soft-edge codec                                                */
/* ------------------------------------------------------------------------ */
/*
 * Passage: Quamba-SE write-up 2.1 (small |v| < L coded at scale / 2^r,
 * standard at scale, large |v| > H at scale * 2^r; r = 2 is the page's /4 and
 * x4, r = 1 the shift-only variant of 4.1) and 2.2 (byte codes 0xxxxxxx
 * standard, 10xxxxxx small, 11xxxxxx large, 6 data bits for small / large).
 *
 * Readings: |v| is compared (strict < L, strict > H, equality is standard);
 * the standard payload is 7-bit two's complement clamped to +-63, the small /
 * large payload 6-bit two's complement clamped to +-31; the quotient by the
 * mode's step follows the quantizer's binary32 rule.  Decoding multiplies the
 * payload by fl32(scale * 2^{-r, 0, +r}).
 *
 * encode: src device (binary16 bits or fp32), n elements -> codes device
 *         uint8[n].  thr_lo <= thr_hi is required (INVALID_ARG otherwise);
 *         0 <= log2_ratio <= 8.  Non-finite inputs -> code 0x00 and
 *         SSMQ_DEV_NONFINITE.
 * decode: codes device uint8[n] -> out device fp32[n].
 */
ssmq_status ssmq_softedge_encode(const void* src, ssmq_dtype dtype, int64_t n,
                                 float scale, float thr_lo, float thr_hi,
                                 int32_t log2_ratio, uint8_t* codes,
                                 uint32_t* status, void* stream);
ssmq_status ssmq_softedge_decode(const uint8_t* codes, int64_t n, float scale,
                                 int32_t log2_ratio, float* out, void* stream);

/* ------------------------------------------------------------------------ */
/* Calibration on the device                                                 */
/* ------------------------------------------------------------------------ */
/*
 * Passages: Quamba2 method steps 1-2 (activation statistics; channels sorted
 * by magnitude and cut into clusters sharing one scale) and the Quamba-SE
 * write-up 4.1 (thresholds L = 5th, H = 99.9th percentile of the activation
 * magnitudes, refreshed as alpha * new + (1 - alpha) * running, alpha 0.1).
 *
 * ssmq_group_absmax: absmax[g] = largest |v| over the finite elements of
 *   group g (same tensor / group-map conventions as ssmq_quantize_groups);
 *   0 for a group without finite elements.  Exact (no rounding).  Status:
 *   NONFINITE / BAD_GROUP as the quantizer.  absmax is device fp32[n_groups].
 *
 * ssmq_cluster_by_absmax: channels sorted by (absmax, index) ascending; the
 *   sorted order is cut into k clusters, cluster j holding sorted positions
 *   [floor(n j / k), floor(n (j + 1) / k)); cluster_of[c] (device int32[n])
 *   gets the cluster of channel c, scales[j] (device fp32[k]) the binary32
 *   quotient fl32(max member absmax / 127).  1 <= k <= n <= 65536
 *   (SSMQ_ERR_UNSUPPORTED above).  Negative or non-finite absmax values set
 *   SSMQ_DEV_NONFINITE and sort last.
 *
 * ssmq_percentile_abs: out[i] (device fp32[nq]) = the q[i]-th percentile
 *   (host doubles in [0, 100], 1 <= nq <= 4) of |v| over the m finite
 *   elements of src: with pos = (m - 1) q / 100, k = floor(pos) (clamped to
 *   [0, m - 1]), the k-th and (k+1)-th smallest (0-based) values a, b give
 *   fl32(a + (pos - k) (b - a)) evaluated in double; 0 when m == 0.  Exact
 *   order statistics (radix selection on the magnitude bits).
 *
 * ssmq_softedge_calibrate: thresholds (device fp32[3] = {scale, lo, hi},
 *   in/out): lo' = fl32(P(q_lo)), hi' = fl32(P(q_hi)) as above; then, for
 *   alpha < 1, lo = fl32(alpha lo' + (1 - alpha) lo), hi likewise (in double),
 *   else lo = lo', hi = hi'; finally scale = fl32(hi / 63) -- the parameters of
 *   ssmq_softedge_encode.  0 <= q_lo <= q_hi <= 100, 0 < alpha <= 1.
 *
 * The two percentile calls need a caller-owned device workspace of
 * ssmq_percentile_workspace_size() bytes, 256-byte aligned (contents need
 * not be initialised; one call at a time per workspace).
 */
ssmq_status ssmq_group_absmax(const void* src, ssmq_dtype dtype, int64_t outer, int64_t mid,
                              int64_t inner, const int32_t* group_of_mid, int32_t n_groups,
                              float* absmax, uint32_t* status, void* stream);
ssmq_status ssmq_cluster_by_absmax(const float* absmax, int64_t n, int32_t k,
                                   int32_t* cluster_of, float* scales, uint32_t* status,
                                   void* stream);
size_t ssmq_percentile_workspace_size(void);
ssmq_status ssmq_percentile_abs(const void* src, ssmq_dtype dtype, int64_t n, const double* q,
                                int32_t nq, float* out, void* workspace, size_t ws_bytes,
                                void* stream);
ssmq_status ssmq_softedge_calibrate(const void* src, ssmq_dtype dtype, int64_t n, double q_lo,
                                    double q_hi, float alpha, float* thresholds,
                                    void* workspace, size_t ws_bytes, void* stream);

/*
 * Allocation-free variants of the two percentile calls, for callers that may
 * not allocate device memory: code running while a CUDA graph is captured,
 * or a serving loop whose memory is fixed at start-up, cannot call cudaMalloc
 * or an allocator for the workspace.  Same computation and results as the
 * workspace forms; the scratch is the library's own file-scope device array
 * of about 136 KB (ssmq_percentile_workspace_size() bytes), which every GPU
 * that loads the library holds until the process exits.  Nothing is
 * allocated or freed.
 *   - The calls run on the current device (like every entry point): src,
 *     out / thresholds and stream must belong to it.
 *   - The first call on a device, with that device current, looks up the
 *     device address of that device's copy of the array (cudaGetSymbolAddress)
 *     and keeps it; make that first call before any stream capture.
 *   - All calls on one device share the array and it keeps the last call's
 *     contents (each call clears what it needs).  Calls that overlap on the
 *     GPU race: issue them on one stream, or synchronise between them.
 *   - SSMQ_ERR_UNSUPPORTED if a call needs more scratch than the array holds;
 *     SSMQ_ERR_CUDA if the address lookup fails.
 * The pages have no counterpart: this is a deployment convenience of this
 * library, not part of the method.
 */
ssmq_status ssmq_percentile_abs_noalloc(const void* src, ssmq_dtype dtype, int64_t n,
                                        const double* q, int32_t nq, float* out, void* stream);
ssmq_status ssmq_softedge_calibrate_noalloc(const void* src, ssmq_dtype dtype, int64_t n,
                                            double q_lo, double q_hi, float alpha,
                                            float* thresholds, void* stream);

/* ------------------------------------------------------------------------ */
/* Producer of the scan input: causal conv + SiLU + quantize, fused           */
/* ------------------------------------------------------------------------ */
/*
 * Passage: Quamba-SE write-up 4.1 (the range check is inserted into the
 * quantization where the activation is produced, inside a custom CUDA
 * kernel) and Quamba2 abstract / method step 3 (x quantized per
 * sorted-and-clustered channel group).  In the Mamba-1 block the scan input x
 * is the output of a short causal depthwise convolution along time followed
 * by SiLU; this call computes it and writes its 8-bit codes directly (no
 * binary16 x through HBM).
 *
 * The value coded is a binary32 evaluation, step by step (reproducible to the
 * bit by any IEEE implementation):
 *   a = bias[c] (0 without bias); a = fma(weight[c][k], x[t - (W-1) + k], a)
 *       for k = 0 .. W-1 (oldest tap first; steps before 0 read x_prev)
 *   e = exp32(-a): k = round-half-even(fl32(v * log2 e));
 *       r = fma(-k, LN2_LO, fma(-k, LN2_HI, v)) with LN2_HI = 0.693145751953125,
 *       LN2_LO = fl32(ln 2 - LN2_HI); p = sum_{n<=7} r^n / n! in Horner form
 *       (fused multiply-adds, coefficients fl32(fl64(1 / n!))); e = fl32(p 2^k);
 *       v > 88 gives +inf, v < -87 gives 0
 *   u = fl32(a * fl32(1 / fl32(1 + e)))
 * then u is coded as ssmq_quantize_groups (SCALE_STATIC, binary32 source,
 * group x_group[c]) or ssmq_softedge_encode would code it.
 *
 * Layouts (b, d, L, W):
 *   x        (b, d, L) binary16: the convolution's input (the in_proj output)
 *   weight   fp32 (d, W), W in 1..4;  bias fp32[d] or NULL
 *   x_prev   (b, d, W-1) binary16: the W-1 inputs before step 0, oldest first
 *            (the conv state of a previous call), or NULL for zeros
 *   codes    (b, d, L) int8 (out_format INT8_GROUP: x_group int32[d], x_scale
 *            fp32[n_x_groups]) or uint8 soft-edge codes (SOFTEDGE: se_scale,
 *            se_lo, se_hi, se_log2_ratio as ssmq_softedge_encode)
 *   u        (b, d, L) fp32 out (the values coded) or NULL
 *   x_prev_out (b, d, W-1) binary16 out or NULL: the W-1 most recent inputs,
 *            the x_prev of the next call (a call on steps [0, L1) followed by
 *            one on [L1, L) with that state gives the unsplit call's bytes);
 *            must not overlap x_prev
 * status: NONFINITE (non-finite u, coded 0), BAD_GROUP, BAD_SCALE as the
 * quantizer.  Errors: INVALID_ARG (NULL tensors, W outside 1..4, bad
 * out_format, se_lo > se_hi, overlapping states), ALIGNMENT (x, codes, u not
 * 16-byte aligned).  Rows of L % 16 == 0 steps take the vectorised kernel.
 */
typedef struct {
  int64_t batch, seqlen, dim;
  int32_t width;
  const uint16_t* x;
  const float* weight;
  const float* bias;
  const uint16_t* x_prev;
  int32_t out_format;       /* SSMQ_X_INT8_GROUP or SSMQ_X_SOFTEDGE */
  const int32_t* x_group;
  const float* x_scale;
  int32_t n_x_groups;
  float se_scale, se_lo, se_hi;
  int32_t se_log2_ratio;
  void* codes;
  float* u;
  uint16_t* x_prev_out;
  uint32_t* status;
} ssmq_conv_args;

ssmq_status ssmq_conv_silu_quantize(const ssmq_conv_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* Mamba-1 diagonal selective scan                                           */
/* ------------------------------------------------------------------------ */
/*
 * Passage: Quamba2 abstract (W8A8 for the Mamba1 backbone: 8-bit inputs of
 * the linear recurrence, clustered x, per-state-group B / C) and the
 * recurrence above with A diagonal per (channel, state).
 *
 * Layouts (b = batch, L = seqlen, d = dim, N = dstate, G = ngroups):
 *   x        (b, d, L)  int8 codes (x_format INT8_GROUP) or soft-edge uint8
 *                       codes (x_format SOFTEDGE: se_scale, se_log2_ratio);
 *                       or binary16 activations encoded on the fly ("encode
 *                       then scan"):
 *                       F16_GROUP: each element becomes the int8 code that
 *                         ssmq_quantize_groups (SCALE_STATIC, group x_group[c],
 *                         scale x_scale) gives it, and the recurrence reads
 *                         code * scale;
 *                       F16_SOFTEDGE: each element becomes the code that
 *                         ssmq_softedge_encode(se_scale, se_lo, se_hi,
 *                         se_log2_ratio) gives it, read back as the decoded value;
 *                       either way y and h_final equal, byte for byte, the
 *                       separate encode followed by INT8_GROUP / SOFTEDGE, and
 *                       the status word gets the encoder's bits (NONFINITE,
 *                       BAD_SCALE)
 *   x_group  int32[d]   cluster of each channel; x_scale fp32[n_x_groups]
 *   dt, z    (b, d, L)  binary16; z may be NULL (no gate)
 *   dt_bias  fp32[d] or NULL;  dt_softplus 0/1
 *   A        fp32 (d, N);  D fp32[d] or NULL
 *   B, C     (b, G, N, L) int8; channel c reads group floor(c * G / d)
 *   B_scale, C_scale fp32[G * N / state_group_size]: state n of group g uses
 *            index g * (N / state_group_size) + n / state_group_size
 *   h0       fp32 (b, d, N) or NULL (zero initial state)
 *   y        (b, d, L) binary16 output, or NULL when y_q is given
 *   h_final  fp32 (b, d, N) output or NULL
 *   y_q      (b, d, L) int8 output or NULL: the persistent-INT8 epilogue
 *            (SSDi8 abstract: an INT8 path through the block).  Each y is
 *            rounded to binary16 and quantized with its channel's static
 *            scale, y_group int32[d] -> y_scale fp32[n_y_groups]: the bytes
 *            equal ssmq_quantize_groups (SCALE_STATIC) of the binary16 y.
 * Supported: N in {4, 8, 16, 32, 64}; d % G == 0; any L >= 0.
 * status: device word or NULL (SSMQ_DEV_BAD_GROUP for x_group / y_group ids
 * out of range, which then read scale 0; the quantizer's bits for y_q).
 * time_segments: 0 or 1 scans each (batch, channel) row in one pass.  k > 1
 *   cuts L into k segments of whole 32-step chunks that run in parallel
 *   (segment 0 from h0, the others from a zero state), then a carry-in kernel
 *   adds to each later step the term of the state carried into its segment,
 *   (sum_n C_tn exp(A_n S_t) h_in,n) silu(z_t), S_t the sum of delta over the
 *   segment up to t, and forms h_final: the recurrence is linear in the
 *   state, so the result is the one-pass result up to rounding (y of the
 *   later segments is rounded to binary16 twice).  It multiplies the rows in
 *   flight by k, for shapes with too few (batch, channel) rows to fill the
 *   GPU.  The effective count is ssmq_scan_time_segments(args): 1 when y is
 *   NULL, y_q is given, L < 64 or batch * k > 65535.
 * workspace / workspace_bytes: with an effective count k > 1, caller-owned
 *   device memory of at least ssmq_scan_workspace_size(args) bytes (16-byte
 *   aligned, contents need not be initialised; it receives every segment's
 *   local final state, k * b * d * N fp32); unused otherwise.  Errors:
 *   INVALID_ARG when it is NULL or too small, ALIGNMENT when misaligned.
 * dec_final: fp32 (b, d, N) output or NULL: the log2 decay of the call's
 *   steps, A_cn log2(e) sum_t delta_t per (batch, channel, state), which
 *   chains the slices of a sequence cut over several calls or ranks
 *   (ssmq_state_chain with units b * d * N, elems 1).  A call with dec_final
 *   keeps one pass (no time segments).
 */
typedef struct {
  int64_t batch, seqlen, dim, dstate, ngroups;
  int32_t state_group_size;
  int32_t x_format; /* ssmq_x_format */
  const void* x;
  const int32_t* x_group;
  const float* x_scale;
  int32_t n_x_groups;
  float se_scale;
  int32_t se_log2_ratio;
  const uint16_t* dt;
  const float* dt_bias;
  int32_t dt_softplus;
  const float* A;
  const float* D;
  const uint16_t* z;
  const int8_t* B;
  const int8_t* C;
  const float* B_scale;
  const float* C_scale;
  const float* h0;
  uint16_t* y;
  float* h_final;
  uint32_t* status;
  float se_lo, se_hi; /* soft-edge thresholds of x_format F16_SOFTEDGE (|v| < se_lo small,
                         |v| > se_hi large); ignored otherwise */
  int8_t* y_q;              /* int8 y (see above) or NULL */
  const int32_t* y_group;   /* [d] output cluster of each channel (with y_q) */
  const float* y_scale;     /* [n_y_groups] static output scales (with y_q) */
  int32_t n_y_groups;
  int32_t time_segments;    /* see above; 0 or 1: one pass */
  void* workspace;          /* with time segments (see above) */
  size_t workspace_bytes;
  float* dec_final;         /* (b, d, N) log2 decays of the call, or NULL */
} ssmq_scan_args;

ssmq_status ssmq_selective_scan_w8(const ssmq_scan_args* args, void* stream);

/* Effective number of time segments of a scan call (>= 1; 0 for NULL args). */
int32_t ssmq_scan_time_segments(const ssmq_scan_args* args);

/* Workspace bytes a scan call needs (0 without time segments or for NULL args). */
size_t ssmq_scan_workspace_size(const ssmq_scan_args* args);

/*
 * ssmq_selective_scan_carry_in: a slice of a sequence (the steps of args)
 * was scanned from a zero state while the true state entering it is h_carry
 * (fp32 (b, d, N), device): adds the carried term to every step,
 * y_t += (sum_n C_tn sC_n exp(A_cn S_ct) h_carry,cn) silu(z_t), S_ct the sum
 * of delta over the slice up to t (y rounded to binary16 once more), and,
 * when args->h_final is given, turns the slice's final state into the true
 * one: h_final = exp(A S_c,L) h_carry + h_final.  args are those of the
 * slice's ssmq_selective_scan_w8 call (y required; y_q, h0, dec_final,
 * time_segments and workspace are ignored; x is not read).  With the slices'
 * h_final and dec_final chained by ssmq_state_chain this gives the unsplit
 * scan up to rounding (Mamba-1 sequence sharding).  Errors: INVALID_ARG for
 * NULL args / y / h_carry / dt / A / C / C_scale, UNSUPPORTED dstate,
 * ALIGNMENT for misaligned tensors.
 */
ssmq_status ssmq_selective_scan_carry_in(const ssmq_scan_args* args, const float* h_carry,
                                         void* stream);

/* ------------------------------------------------------------------------ */
/* Mamba-2 SSD chunked scan                                                  */
/* ------------------------------------------------------------------------ */
/*
 * Passage: SSDi8 abstract (SSD combines a recurrent and an attention mode;
 * element-wise products are kept apart from the matrix products) and Quamba2
 * abstract (W8A8 for the Mamba2 backbone).  Scalar A per head; the sequence
 * is processed in chunks of `chunk` steps: inside a chunk the output is the
 * masked, decay-weighted C B^T "attention" applied to delta * x, plus the
 * contribution of the state carried in; between chunks the state is passed
 * on.  The result equals the sequential recurrence up to rounding.
 *
 * Layouts (b, L, H = nheads, P = headdim, N = dstate, G = ngroups):
 *   x        (b, L, H, P) int8 (INT8_GROUP) or soft-edge uint8 (SOFTEDGE)
 *   x_group  int32[H * P]; x_scale fp32[n_x_groups]
 *   dt       (b, L, H) binary16;  dt_bias fp32[H] or NULL
 *   A        fp32[H];  D fp32[H] or NULL
 *   z        (b, L, H, P) binary16 or NULL
 *   B, C     (b, L, G, N) int8; head h reads group floor(h * G / H)
 *   B_scale, C_scale fp32[G * N / state_group_size]
 *   h0       fp32 (b, H, P, N) or NULL
 *   y        (b, L, H, P) binary16 output, or NULL when y_q is given
 *   h_final  fp32 (b, H, P, N) output or NULL
 *   y_q      (b, L, H, P) int8 output or NULL: the persistent-INT8 epilogue,
 *            channel h * P + p quantized with y_scale[y_group[h * P + p]]
 *            after rounding to binary16 (the bytes of ssmq_quantize_groups
 *            of the binary16 y)
 * workspace: device memory of at least ssmq_ssd_workspace_size(args) bytes,
 *   256-byte aligned, caller-owned, contents need not be initialised; it
 *   receives the head-independent binary16 MMA operands (C scaled per state
 *   group, B), 64 KB per (batch, group, 128-step tile), written once for all
 *   heads of a group.
 * Supported: P == 64, N == 128, chunk in {64, 128, 256}, H % G == 0.  The
 * result is the recurrence's for every chunk length (the decomposition is
 * exact up to rounding); the kernel processes 128-step tiles.
 * Segments: when the (batch, head) sequences do not fill the last round of
 * SMs evenly, the remaining sequences are cut into segments run in parallel
 * from a zero state, and a second kernel adds each later segment's carried
 * state term (exp(S_t) C_t h_start, gated like y) and forms h_final; y of
 * those sequences is then rounded to binary16 twice.  max_segments = 1 turns
 * this off (one pass per sequence: a call on steps [0, L) equals, byte for
 * byte, a call on [0, L1) followed by one on [L1, L) with h0 = its h_final,
 * L1 a multiple of 128); so do y_q and a NULL y.
 * seqlen = 0: h_final = h0 (or zeros) and dec_final = 0; the step tensors
 * may then be NULL.
 * status: SSMQ_DEV_BAD_GROUP as above; SSMQ_DEV_TIMEOUT if a bounded wait for
 * the tensor core gave up (the call's outputs are then incomplete).
 * The environment variable SSMQ_SSD_KERNEL=pipelined (read at each call)
 * selects, for binary16 y, an alternative kernel whose warp roles work on
 * different tiles at once; it gives the same bytes.
 */
typedef struct {
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups;
  int64_t chunk;
  int32_t state_group_size;
  int32_t x_format;
  const void* x;
  const int32_t* x_group;
  const float* x_scale;
  int32_t n_x_groups;
  float se_scale;
  int32_t se_log2_ratio;
  const uint16_t* dt;
  const float* dt_bias;
  int32_t dt_softplus;
  const float* A;
  const float* D;
  const uint16_t* z;
  const int8_t* B;
  const int8_t* C;
  const float* B_scale;
  const float* C_scale;
  const float* h0;
  uint16_t* y;
  float* h_final;
  uint32_t* status;
  int8_t* y_q;              /* int8 y (see above) or NULL */
  const int32_t* y_group;   /* [H * P] output cluster of each channel (with y_q) */
  const float* y_scale;     /* [n_y_groups] static output scales (with y_q) */
  int32_t n_y_groups;
  int32_t max_segments;     /* 0: the library may cut some sequences into up
                               to 32 segments (see above); n > 1: up to n;
                               1: one pass per sequence.  The workspace size
                               depends on it, on y and on y_q. */
  float* dec_final;         /* (b, H) fp32 output or NULL: the sequence's total
                               log2 decay, sum_t delta_t A_h log2(e) (binary32,
                               summed per 128-step tile in step order, the
                               tiles in order) -- exp2 of it multiplies the
                               state carried across the call */
} ssmq_ssd_args;

size_t ssmq_ssd_workspace_size(const ssmq_ssd_args* args);
ssmq_status ssmq_ssd_chunk_scan_w8(const ssmq_ssd_args* args, void* workspace,
                                   size_t ws_bytes, void* stream);

/*
 * Sequence sharding: a long sequence cut into consecutive slices (one per
 * device, say).  The pages describe no such split; it follows from the
 * recurrence (Quamba2 abstract, the selective SSM) being linear in the state:
 * a slice scanned from a zero state (h0 = NULL) gives y and h_final of its
 * own inputs; the state h_carry it should have started from adds
 * exp(S_t) C_t h_carry to y_t (S_t the decay from the slice's start through
 * step t; gated like y) and exp(S_L) h_carry to h_final.
 *
 * ssmq_state_chain: h_out[u] = fold over parts q = 0 .. n_parts - 1 of
 *   h <- exp2(dec[q][u]) h + h_end[q][u], from h = 0.  h_end: device fp32
 *   [n_parts][units][elems], dec: device fp32 [n_parts][units] (the slices'
 *   h_final and dec_final, in sequence order), h_out: device fp32
 *   [units][elems].  A slice's carry-in is the chain over the slices before
 *   it (the first slice runs with the true h0 and needs none).
 * ssmq_ssd_carry_in: adds h_carry's contribution (above) to args->y and, when
 *   given, args->h_final, for the inputs of args (the same arguments as the
 *   ssmq_ssd_chunk_scan_w8 call that produced them; y must not be NULL, y_q
 *   must be NULL; h0, dec_final and max_segments are ignored).  y is rounded
 *   to binary16 once more.  h_carry: device fp32 (b, H, P, N).  workspace:
 *   at least ssmq_ssd_workspace_size(args) bytes (the operand blocks are
 *   rebuilt).
 */
ssmq_status ssmq_state_chain(const float* h_end, const float* dec, int32_t n_parts,
                             int64_t units, int64_t elems, float* h_out, void* stream);
ssmq_status ssmq_ssd_carry_in(const ssmq_ssd_args* args, const float* h_carry,
                              void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Single-token decode state update (Mamba-2 form)                           */
/* ------------------------------------------------------------------------ */
/*
 * Passage: Quamba2 abstract (generation stage; W8A8 Mamba2 backbone): one step
 * of the recurrence on the persistent fp32 state, in place.
 *
 * Layouts (b, H, P, N, G):
 *   state    fp32 (b, H, P, N), read and overwritten
 *   x        (b, H, P) int8 (INT8_GROUP) or soft-edge uint8 (SOFTEDGE)
 *   x_group  int32[H * P]; x_scale fp32[n_x_groups]
 *   dt       (b, H) binary16; dt_bias fp32[H] or NULL
 *   A fp32[H]; D fp32[H] or NULL; z (b, H, P) binary16 or NULL
 *   B, C     (b, G, N) int8; head h reads group floor(h * G / H)
 *   B_scale, C_scale fp32[G * N / state_group_size]
 *   y        (b, H, P) binary16 output
 * Supported: N in {16, 32, 64, 128}; H % G == 0.
 */
typedef struct {
  int64_t batch, nheads, headdim, dstate, ngroups;
  int32_t state_group_size;
  int32_t x_format;
  const void* x;
  const int32_t* x_group;
  const float* x_scale;
  int32_t n_x_groups;
  float se_scale;
  int32_t se_log2_ratio;
  const uint16_t* dt;
  const float* dt_bias;
  int32_t dt_softplus;
  const float* A;
  const float* D;
  const uint16_t* z;
  const int8_t* B;
  const int8_t* C;
  const float* B_scale;
  const float* C_scale;
  float* state;
  uint16_t* y;
  uint32_t* status;
} ssmq_decode_args;

ssmq_status ssmq_state_update_w8(const ssmq_decode_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* Single-token decode state update (Mamba-1 form)                           */
/* ------------------------------------------------------------------------ */
/*
 * Passage: Quamba2 abstract (generation stage; W8A8 Mamba1 backbone): one
 * step of the diagonal recurrence on the persistent fp32 state, in place,
 * with A per (channel, state).
 *
 * Layouts (b, d, N, G):
 *   state    fp32 (b, d, N), read and overwritten
 *   x        (b, d) int8 (INT8_GROUP) or soft-edge uint8 (SOFTEDGE)
 *   x_group  int32[d]; x_scale fp32[n_x_groups]
 *   dt       (b, d) binary16; dt_bias fp32[d] or NULL
 *   A fp32 (d, N); D fp32[d] or NULL; z (b, d) binary16 or NULL
 *   B, C     (b, G, N) int8; channel c reads group floor(c * G / d)
 *   B_scale, C_scale fp32[G * N / state_group_size]
 *   y        (b, d) binary16 output
 * Supported: N in {4, 8, 16, 32, 64, 128}; d % G == 0.
 */
typedef struct {
  int64_t batch, dim, dstate, ngroups;
  int32_t state_group_size;
  int32_t x_format;
  const void* x;
  const int32_t* x_group;
  const float* x_scale;
  int32_t n_x_groups;
  float se_scale;
  int32_t se_log2_ratio;
  const uint16_t* dt;
  const float* dt_bias;
  int32_t dt_softplus;
  const float* A;
  const float* D;
  const uint16_t* z;
  const int8_t* B;
  const int8_t* C;
  const float* B_scale;
  const float* C_scale;
  float* state;
  uint16_t* y;
  uint32_t* status;
} ssmq_m1_decode_args;

ssmq_status ssmq_selective_state_update_w8(const ssmq_m1_decode_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics                                                               */
/* ------------------------------------------------------------------------ */
/* Thread-local, NUL-terminated description of the last non-OK status. */
const char* ssmq_last_error(void);
/* Library ABI version (major * 10000 + minor * 100 + patch). */
int32_t ssmq_version(void);

/*
 * Throughput probe of the special-function unit's base-2 exponential, the
 * compute roof of the Mamba-1 scan (one exp(delta A) per state update; the
 * Quamba2 abstract's Mamba1 recurrence, whose decay the pages leave to the
 * hardware).  Launches sms * 8 CTAs of 256 threads; every thread evaluates
 * iters * 8 independent ex2.approx.ftz.f32 and nothing else that the unit
 * executes.  *n_ex2 (host) receives the number of exponentials; the caller
 * times the launch on `stream` (rate = *n_ex2 / time).  sink: device fp32[1],
 * not written.  Not part of the method.
 * Errors: INVALID_ARG for iters < 1 or NULL sink / n_ex2.
 */
ssmq_status ssmq_probe_ex2(int32_t iters, float* sink, int64_t* n_ex2, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SSMQ_H */
