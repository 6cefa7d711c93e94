// extern "C" entry points: argument validation, then the launchers.
// Validation never touches the device, so every error path here can be
// exercised without a GPU.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/ssmq.h"
#include "internal.h"

namespace {

thread_local char g_err[512] = "";

ssmq_status fail(ssmq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

// One NVTX range per entry-point call (named after the entry point), seen by
// profilers as the host-side span of the call; a no-op without a tool.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host-side fault injection for tests of the error path: when the
// environment variable SSMQ_FAULT_INJECT names an entry point (or "all"),
// that entry point reports a launch failure instead of launching.
bool injected(const char* name) {
  const char* v = getenv("SSMQ_FAULT_INJECT");
  if (!v || !*v) return false;
  return strcmp(v, "all") == 0 || strcmp(v, name) == 0;
}

ssmq_status finish(cudaError_t e, const char* name) {
  if (e != cudaSuccess) return fail(SSMQ_ERR_CUDA, "%s: CUDA error %d (%s)", name, (int)e,
                                    cudaGetErrorString(e));
  return SSMQ_OK;
}

#define REQUIRE(cond, code, ...)        \
  do {                                  \
    if (!(cond)) return fail(code, __VA_ARGS__); \
  } while (0)

ssmq_status check_x(int32_t fmt, const void* x, const int32_t* x_group, const float* x_scale,
                    int32_t n_x_groups, int32_t log2_ratio, const char* fn,
                    bool allow_f16 = false) {
  REQUIRE(fmt >= SSMQ_X_INT8_GROUP && fmt <= SSMQ_X_F16_SOFTEDGE, SSMQ_ERR_INVALID_ARG,
          "%s: x_format %d is not an ssmq_x_format", fn, fmt);
  REQUIRE(allow_f16 || fmt == SSMQ_X_INT8_GROUP || fmt == SSMQ_X_SOFTEDGE, SSMQ_ERR_UNSUPPORTED,
          "%s: binary16 x (x_format %d) is accepted by the Mamba-1 scan only", fn, fmt);
  REQUIRE(x != nullptr, SSMQ_ERR_INVALID_ARG, "%s: x is NULL", fn);
  if (fmt == SSMQ_X_INT8_GROUP || fmt == SSMQ_X_F16_GROUP) {
    REQUIRE(x_group && x_scale, SSMQ_ERR_INVALID_ARG, "%s: x_group / x_scale is NULL", fn);
    REQUIRE(n_x_groups >= 1, SSMQ_ERR_INVALID_ARG, "%s: n_x_groups must be >= 1", fn);
  } else {
    REQUIRE(log2_ratio >= 0 && log2_ratio <= 8, SSMQ_ERR_INVALID_ARG,
            "%s: se_log2_ratio must be in [0, 8]", fn);
  }
  return SSMQ_OK;
}

// optional int8 output: the cluster map and scales come with it
ssmq_status check_yq(const int8_t* y_q, const int32_t* y_group, const float* y_scale,
                     int32_t n_y_groups, const char* fn) {
  if (!y_q) return SSMQ_OK;
  REQUIRE(aligned16(y_q), SSMQ_ERR_ALIGNMENT, "%s: y_q must be 16-byte aligned", fn);
  REQUIRE(y_group && y_scale && n_y_groups >= 1, SSMQ_ERR_INVALID_ARG,
          "%s: y_q needs y_group, y_scale and n_y_groups >= 1", fn);
  return SSMQ_OK;
}

ssmq_status check_src(const void* src, ssmq_dtype dtype, int64_t n, const char* fn) {
  REQUIRE(dtype == SSMQ_F32 || dtype == SSMQ_F16, SSMQ_ERR_INVALID_ARG, "%s: bad dtype", fn);
  REQUIRE(n >= 0, SSMQ_ERR_INVALID_ARG, "%s: negative size", fn);
  if (n > 0) REQUIRE(src != nullptr, SSMQ_ERR_INVALID_ARG, "%s: src is NULL", fn);
  return SSMQ_OK;
}

ssmq_status check_ws(void* workspace, size_t ws_bytes, const char* fn) {
  REQUIRE(workspace && ws_bytes >= ssmq::percentile_workspace_bytes(), SSMQ_ERR_INVALID_ARG,
          "%s: workspace of %zu bytes required (got %zu)", fn,
          ssmq::percentile_workspace_bytes(), ws_bytes);
  REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, SSMQ_ERR_ALIGNMENT,
          "%s: workspace must be 256-byte aligned", fn);
  return SSMQ_OK;
}

ssmq_status check_pct_q(const double* q, int32_t nq, const float* out, const char* fn) {
  REQUIRE(q && out && nq >= 1 && nq <= ssmq::percentile_max_q(), SSMQ_ERR_INVALID_ARG,
          "%s: need 1 <= nq <= %d percentiles and out", fn, ssmq::percentile_max_q());
  for (int i = 0; i < nq; ++i)
    REQUIRE(q[i] >= 0.0 && q[i] <= 100.0, SSMQ_ERR_INVALID_ARG,
            "%s: percentile %d outside [0, 100]", fn, i);
  return SSMQ_OK;
}

ssmq_status check_se_cal(double q_lo, double q_hi, float alpha, const float* thresholds,
                         const char* fn) {
  REQUIRE(thresholds != nullptr, SSMQ_ERR_INVALID_ARG, "%s: thresholds is NULL", fn);
  REQUIRE(q_lo >= 0.0 && q_lo <= q_hi && q_hi <= 100.0, SSMQ_ERR_INVALID_ARG,
          "%s: need 0 <= q_lo <= q_hi <= 100", fn);
  REQUIRE(alpha > 0.0f && alpha <= 1.0f, SSMQ_ERR_INVALID_ARG, "%s: alpha must be in (0, 1]", fn);
  return SSMQ_OK;
}

#define CHECK(call)                     \
  do {                                  \
    const ssmq_status s_ = (call);      \
    if (s_ != SSMQ_OK) return s_;       \
  } while (0)

}  // namespace

extern "C" {

const char* ssmq_last_error(void) { return g_err; }

int32_t ssmq_version(void) { return 100; }

ssmq_status ssmq_quantize_groups(const void* src, ssmq_dtype dtype, int64_t outer, int64_t mid,
                                 int64_t inner, const int32_t* group_of_mid, int32_t n_groups,
                                 ssmq_scale_mode mode, float* scales, int8_t* q_out,
                                 uint32_t* status, void* stream) {
  const char* fn = "ssmq_quantize_groups";
  Range nvtx_range(fn);
  REQUIRE(dtype == SSMQ_F32 || dtype == SSMQ_F16, SSMQ_ERR_INVALID_ARG, "%s: bad dtype %d", fn,
          (int)dtype);
  REQUIRE(mode == SSMQ_SCALE_STATIC || mode == SSMQ_SCALE_ABSMAX, SSMQ_ERR_INVALID_ARG,
          "%s: bad scale mode %d", fn, (int)mode);
  REQUIRE(outer >= 0 && mid >= 0 && inner >= 0, SSMQ_ERR_INVALID_ARG, "%s: negative size", fn);
  REQUIRE(n_groups >= 1, SSMQ_ERR_INVALID_ARG, "%s: n_groups must be >= 1", fn);
  REQUIRE(scales != nullptr, SSMQ_ERR_INVALID_ARG, "%s: scales is NULL", fn);
  const bool empty = outer == 0 || mid == 0 || inner == 0;
  if (!empty) {
    REQUIRE(src && q_out && group_of_mid, SSMQ_ERR_INVALID_ARG, "%s: NULL tensor", fn);
    REQUIRE(outer <= (INT64_MAX / mid) / inner, SSMQ_ERR_INVALID_ARG, "%s: size overflow", fn);
  }
  REQUIRE(aligned16(src) && aligned16(q_out), SSMQ_ERR_ALIGNMENT,
          "%s: src and q_out must be 16-byte aligned", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  if (empty && mode == SSMQ_SCALE_STATIC) return SSMQ_OK;
  return finish(ssmq::launch_quantize(src, dtype == SSMQ_F16, empty ? 0 : outer, mid, inner,
                                      group_of_mid, n_groups, mode == SSMQ_SCALE_ABSMAX, scales,
                                      q_out, status, (cudaStream_t)stream),
                fn);
}

ssmq_status ssmq_quantize_groups_batch(const ssmq_quant_job* jobs, int32_t n_jobs,
                                       uint32_t* status, void* stream) {
  const char* fn = "ssmq_quantize_groups_batch";
  Range nvtx_range(fn);
  REQUIRE(jobs != nullptr, SSMQ_ERR_INVALID_ARG, "%s: jobs is NULL", fn);
  REQUIRE(n_jobs >= 1 && n_jobs <= ssmq::kMaxQuantJobs, SSMQ_ERR_INVALID_ARG,
          "%s: n_jobs must be in [1, %d] (got %d)", fn, ssmq::kMaxQuantJobs, (int)n_jobs);
  ssmq::QuantJob hj[ssmq::kMaxQuantJobs];
  for (int k = 0; k < n_jobs; ++k) {
    const ssmq_quant_job& j = jobs[k];
    REQUIRE(j.dtype == SSMQ_F32 || j.dtype == SSMQ_F16, SSMQ_ERR_INVALID_ARG,
            "%s: job %d: bad dtype %d", fn, k, (int)j.dtype);
    REQUIRE(j.outer >= 0 && j.mid >= 0 && j.inner >= 0, SSMQ_ERR_INVALID_ARG,
            "%s: job %d: negative size", fn, k);
    REQUIRE(j.n_groups >= 1, SSMQ_ERR_INVALID_ARG, "%s: job %d: n_groups must be >= 1", fn, k);
    REQUIRE(j.scales != nullptr, SSMQ_ERR_INVALID_ARG, "%s: job %d: scales is NULL", fn, k);
    const bool empty = j.outer == 0 || j.mid == 0 || j.inner == 0;
    if (!empty) {
      REQUIRE(j.src && j.q_out && j.group_of_mid, SSMQ_ERR_INVALID_ARG, "%s: job %d: NULL tensor",
              fn, k);
      REQUIRE(j.outer <= (INT64_MAX / j.mid) / j.inner, SSMQ_ERR_INVALID_ARG,
              "%s: job %d: size overflow", fn, k);
    }
    REQUIRE(aligned16(j.src) && aligned16(j.q_out), SSMQ_ERR_ALIGNMENT,
            "%s: job %d: src and q_out must be 16-byte aligned", fn, k);
    hj[k] = ssmq::QuantJob{j.src, j.dtype == SSMQ_F16, empty ? 0 : j.outer, j.mid, j.inner,
                           j.group_of_mid, j.n_groups, j.scales, j.q_out};
  }
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_quantize_batch(hj, n_jobs, status, (cudaStream_t)stream), fn);
}

ssmq_status ssmq_softedge_encode(const void* src, ssmq_dtype dtype, int64_t n, float scale,
                                 float thr_lo, float thr_hi, int32_t log2_ratio, uint8_t* codes,
                                 uint32_t* status, void* stream) {
  const char* fn = "ssmq_softedge_encode";
  Range nvtx_range(fn);
  REQUIRE(dtype == SSMQ_F32 || dtype == SSMQ_F16, SSMQ_ERR_INVALID_ARG, "%s: bad dtype", fn);
  REQUIRE(n >= 0, SSMQ_ERR_INVALID_ARG, "%s: negative size", fn);
  REQUIRE(thr_lo <= thr_hi, SSMQ_ERR_INVALID_ARG,
          "%s: thr_lo must not exceed thr_hi (got %g > %g)", fn, (double)thr_lo, (double)thr_hi);
  REQUIRE(log2_ratio >= 0 && log2_ratio <= 8, SSMQ_ERR_INVALID_ARG,
          "%s: log2_ratio must be in [0, 8]", fn);
  if (n > 0) REQUIRE(src && codes, SSMQ_ERR_INVALID_ARG, "%s: NULL tensor", fn);
  REQUIRE(aligned16(src) && aligned16(codes), SSMQ_ERR_ALIGNMENT, "%s: 16-byte alignment", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_softedge_encode(src, dtype == SSMQ_F16, n, scale, thr_lo, thr_hi,
                                             log2_ratio, codes, status, (cudaStream_t)stream),
                fn);
}

ssmq_status ssmq_group_absmax(const void* src, ssmq_dtype dtype, int64_t outer, int64_t mid,
                              int64_t inner, const int32_t* group_of_mid, int32_t n_groups,
                              float* absmax, uint32_t* status, void* stream) {
  const char* fn = "ssmq_group_absmax";
  Range nvtx_range(fn);
  REQUIRE(dtype == SSMQ_F32 || dtype == SSMQ_F16, SSMQ_ERR_INVALID_ARG, "%s: bad dtype %d", fn,
          (int)dtype);
  REQUIRE(outer >= 0 && mid >= 0 && inner >= 0, SSMQ_ERR_INVALID_ARG, "%s: negative size", fn);
  REQUIRE(n_groups >= 1 && absmax, SSMQ_ERR_INVALID_ARG, "%s: need n_groups >= 1 and absmax", fn);
  const int64_t n = outer * mid * inner;
  if (n > 0) REQUIRE(src && group_of_mid, SSMQ_ERR_INVALID_ARG, "%s: NULL tensor", fn);
  REQUIRE(aligned16(src), SSMQ_ERR_ALIGNMENT, "%s: src must be 16-byte aligned", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_group_absmax(src, dtype == SSMQ_F16, outer, mid, inner,
                                          group_of_mid, n_groups, absmax, status,
                                          (cudaStream_t)stream),
                fn);
}

ssmq_status ssmq_cluster_by_absmax(const float* absmax, int64_t n, int32_t k, int32_t* cluster_of,
                                   float* scales, uint32_t* status, void* stream) {
  const char* fn = "ssmq_cluster_by_absmax";
  Range nvtx_range(fn);
  REQUIRE(n >= 1 && k >= 1 && k <= n, SSMQ_ERR_INVALID_ARG, "%s: need 1 <= k <= n", fn);
  REQUIRE(n <= 65536, SSMQ_ERR_UNSUPPORTED, "%s: n > 65536 channels", fn);
  REQUIRE(absmax && cluster_of && scales, SSMQ_ERR_INVALID_ARG, "%s: NULL tensor", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_cluster_by_absmax(absmax, (int)n, k, cluster_of, scales, status,
                                               (cudaStream_t)stream),
                fn);
}

ssmq_status ssmq_probe_ex2(int32_t iters, float* sink, int64_t* n_ex2, void* stream) {
  const char* fn = "ssmq_probe_ex2";
  Range nvtx_range(fn);
  REQUIRE(iters >= 1 && sink && n_ex2, SSMQ_ERR_INVALID_ARG,
          "%s: iters >= 1, sink and n_ex2 required", fn);
  REQUIRE(aligned16(sink), SSMQ_ERR_ALIGNMENT, "%s: sink must be 16-byte aligned", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_probe_ex2(iters, sink, n_ex2, (cudaStream_t)stream), fn);
}

size_t ssmq_percentile_workspace_size(void) { return ssmq::percentile_workspace_bytes(); }


ssmq_status ssmq_percentile_abs(const void* src, ssmq_dtype dtype, int64_t n, const double* q,
                                int32_t nq, float* out, void* workspace, size_t ws_bytes,
                                void* stream) {
  const char* fn = "ssmq_percentile_abs";
  Range nvtx_range(fn);
  CHECK(check_src(src, dtype, n, fn));
  CHECK(check_pct_q(q, nq, out, fn));
  CHECK(check_ws(workspace, ws_bytes, fn));
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_percentile_abs(src, dtype == SSMQ_F16, n, q, nq, out, nullptr, 1.0f,
                                            workspace, (cudaStream_t)stream),
                fn);
}

ssmq_status ssmq_softedge_calibrate(const void* src, ssmq_dtype dtype, int64_t n, double q_lo,
                                    double q_hi, float alpha, float* thresholds, void* workspace,
                                    size_t ws_bytes, void* stream) {
  const char* fn = "ssmq_softedge_calibrate";
  Range nvtx_range(fn);
  CHECK(check_src(src, dtype, n, fn));
  CHECK(check_se_cal(q_lo, q_hi, alpha, thresholds, fn));
  CHECK(check_ws(workspace, ws_bytes, fn));
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  const double q[2] = {q_lo, q_hi};
  return finish(ssmq::launch_percentile_abs(src, dtype == SSMQ_F16, n, q, 2,
                                            ssmq::percentile_scratch_out(workspace), thresholds,
                                            alpha, workspace, (cudaStream_t)stream),
                fn);
}

namespace {
// the library's static scratch of the current device, or an error status
ssmq_status static_scratch(void** ws, const char* fn) {
  cudaError_t e;
  const size_t need = ssmq::percentile_workspace_bytes();
  *ws = ssmq::percentile_static_scratch(need, &e);
  REQUIRE(e == cudaSuccess, SSMQ_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  REQUIRE(*ws != nullptr, SSMQ_ERR_UNSUPPORTED, "%s: %zu bytes of scratch exceed the static array",
          fn, need);
  return SSMQ_OK;
}
}  // namespace

ssmq_status ssmq_percentile_abs_noalloc(const void* src, ssmq_dtype dtype, int64_t n,
                                        const double* q, int32_t nq, float* out, void* stream) {
  const char* fn = "ssmq_percentile_abs_noalloc";
  Range nvtx_range(fn);
  CHECK(check_src(src, dtype, n, fn));  // argument errors before any device call
  CHECK(check_pct_q(q, nq, out, fn));
  void* ws = nullptr;
  CHECK(static_scratch(&ws, fn));
  return ssmq_percentile_abs(src, dtype, n, q, nq, out, ws, ssmq::percentile_workspace_bytes(),
                             stream);
}

ssmq_status ssmq_softedge_calibrate_noalloc(const void* src, ssmq_dtype dtype, int64_t n,
                                            double q_lo, double q_hi, float alpha,
                                            float* thresholds, void* stream) {
  const char* fn = "ssmq_softedge_calibrate_noalloc";
  Range nvtx_range(fn);
  CHECK(check_src(src, dtype, n, fn));
  CHECK(check_se_cal(q_lo, q_hi, alpha, thresholds, fn));
  void* ws = nullptr;
  CHECK(static_scratch(&ws, fn));
  return ssmq_softedge_calibrate(src, dtype, n, q_lo, q_hi, alpha, thresholds, ws,
                                 ssmq::percentile_workspace_bytes(), stream);
}

ssmq_status ssmq_softedge_decode(const uint8_t* codes, int64_t n, float scale, int32_t log2_ratio,
                                 float* out, void* stream) {
  const char* fn = "ssmq_softedge_decode";
  Range nvtx_range(fn);
  REQUIRE(n >= 0, SSMQ_ERR_INVALID_ARG, "%s: negative size", fn);
  REQUIRE(log2_ratio >= 0 && log2_ratio <= 8, SSMQ_ERR_INVALID_ARG,
          "%s: log2_ratio must be in [0, 8]", fn);
  if (n > 0) REQUIRE(codes && out, SSMQ_ERR_INVALID_ARG, "%s: NULL tensor", fn);
  REQUIRE(aligned16(codes) && aligned16(out), SSMQ_ERR_ALIGNMENT, "%s: 16-byte alignment", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_softedge_decode(codes, n, scale, log2_ratio, out,
                                             (cudaStream_t)stream),
                fn);
}

ssmq_status ssmq_conv_silu_quantize(const ssmq_conv_args* a, void* stream) {
  const char* fn = "ssmq_conv_silu_quantize";
  Range nvtx_range(fn);
  REQUIRE(a != nullptr, SSMQ_ERR_INVALID_ARG, "%s: args is NULL", fn);
  REQUIRE(a->batch >= 0 && a->seqlen >= 0 && a->dim >= 0, SSMQ_ERR_INVALID_ARG,
          "%s: negative size", fn);
  REQUIRE(a->width >= 1 && a->width <= 4, SSMQ_ERR_INVALID_ARG, "%s: width %d not in 1..4", fn,
          (int)a->width);
  REQUIRE(a->out_format == SSMQ_X_INT8_GROUP || a->out_format == SSMQ_X_SOFTEDGE,
          SSMQ_ERR_INVALID_ARG, "%s: out_format must be INT8_GROUP or SOFTEDGE", fn);
  if (a->out_format == SSMQ_X_INT8_GROUP) {
    REQUIRE(a->x_group && a->x_scale && a->n_x_groups >= 1, SSMQ_ERR_INVALID_ARG,
            "%s: x_group, x_scale and n_x_groups >= 1 required", fn);
  } else {
    REQUIRE(a->se_lo <= a->se_hi, SSMQ_ERR_INVALID_ARG, "%s: se_lo > se_hi", fn);
    REQUIRE(a->se_log2_ratio >= 0 && a->se_log2_ratio <= 8, SSMQ_ERR_INVALID_ARG,
            "%s: se_log2_ratio must be in [0, 8]", fn);
  }
  const int64_t n = a->batch * a->dim * a->seqlen;
  const int64_t ns = a->batch * a->dim * (a->width - 1);
  if (n > 0) REQUIRE(a->x && a->weight && a->codes, SSMQ_ERR_INVALID_ARG, "%s: NULL tensor", fn);
  if (a->x_prev_out && a->x_prev && ns > 0) {
    const uintptr_t p0 = (uintptr_t)a->x_prev, p1 = (uintptr_t)a->x_prev_out;
    const uintptr_t nb = (uintptr_t)ns * sizeof(uint16_t);
    REQUIRE(p0 + nb <= p1 || p1 + nb <= p0, SSMQ_ERR_INVALID_ARG,
            "%s: x_prev_out overlaps x_prev", fn);
  }
  if (a->x_prev_out && ns > 0 && a->seqlen > 0)
    REQUIRE(a->x != nullptr, SSMQ_ERR_INVALID_ARG, "%s: x is NULL", fn);
  REQUIRE(aligned16(a->x) && aligned16(a->codes) && aligned16(a->u), SSMQ_ERR_ALIGNMENT,
          "%s: x, codes and u must be 16-byte aligned", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_conv_silu_quantize(*a, (cudaStream_t)stream), fn);
}

ssmq_status ssmq_selective_scan_w8(const ssmq_scan_args* a, void* stream) {
  const char* fn = "ssmq_selective_scan_w8";
  Range nvtx_range(fn);
  REQUIRE(a != nullptr, SSMQ_ERR_INVALID_ARG, "%s: args is NULL", fn);
  REQUIRE(a->batch >= 0 && a->seqlen >= 0 && a->dim >= 0, SSMQ_ERR_INVALID_ARG,
          "%s: negative size", fn);
  REQUIRE(a->ngroups >= 1 && a->dim % a->ngroups == 0, SSMQ_ERR_INVALID_ARG,
          "%s: dim must be a multiple of ngroups >= 1", fn);
  REQUIRE(a->dstate == 4 || a->dstate == 8 || a->dstate == 16 || a->dstate == 32 ||
              a->dstate == 64,
          SSMQ_ERR_UNSUPPORTED, "%s: dstate %lld not in {4, 8, 16, 32, 64}", fn,
          (long long)a->dstate);
  REQUIRE(a->state_group_size >= 1 && a->dstate % a->state_group_size == 0,
          SSMQ_ERR_INVALID_ARG, "%s: dstate must be a multiple of state_group_size", fn);
  if (a->batch == 0 || a->dim == 0) return SSMQ_OK;
  REQUIRE(aligned16(a->x) && aligned16(a->dt) && aligned16(a->z) && aligned16(a->B) &&
              aligned16(a->C) && aligned16(a->y) && aligned16(a->h0) && aligned16(a->h_final) &&
              aligned16(a->A) && aligned16(a->dec_final),
          SSMQ_ERR_ALIGNMENT, "%s: tensors must be 16-byte aligned", fn);
  REQUIRE(a->batch <= 65535, SSMQ_ERR_UNSUPPORTED, "%s: batch > 65535", fn);
  if (a->seqlen > 0) {
    // an empty sequence reads no token tensor (they may be NULL); the final
    // state is then the initial state
    const ssmq_status xs = check_x(a->x_format, a->x, a->x_group, a->x_scale, a->n_x_groups,
                                   a->se_log2_ratio, fn, true);
    if (xs != SSMQ_OK) return xs;
    REQUIRE(a->x_format != SSMQ_X_F16_SOFTEDGE || a->se_lo <= a->se_hi, SSMQ_ERR_INVALID_ARG,
            "%s: se_lo must not exceed se_hi (as ssmq_softedge_encode)", fn);
    REQUIRE(a->dt && a->A && a->B && a->C && a->B_scale && a->C_scale && (a->y || a->y_q),
            SSMQ_ERR_INVALID_ARG,
            "%s: a required tensor (dt, A, B, C, B_scale, C_scale, y or y_q) is NULL", fn);
    const ssmq_status ys = check_yq(a->y_q, a->y_group, a->y_scale, a->n_y_groups, fn);
    if (ys != SSMQ_OK) return ys;
    if (ssmq_scan_time_segments(a) > 1) {
      const size_t need = ssmq_scan_workspace_size(a);
      REQUIRE(a->workspace && a->workspace_bytes >= need, SSMQ_ERR_INVALID_ARG,
              "%s: %d time segments need a workspace of %zu bytes", fn,
              (int)ssmq_scan_time_segments(a), need);
      REQUIRE(aligned16(a->workspace), SSMQ_ERR_ALIGNMENT,
              "%s: workspace must be 16-byte aligned", fn);
    }
  }
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_selective_scan(*a, (cudaStream_t)stream), fn);
}

ssmq_status ssmq_selective_scan_carry_in(const ssmq_scan_args* a, const float* h_carry,
                                         void* stream) {
  const char* fn = "ssmq_selective_scan_carry_in";
  Range nvtx_range(fn);
  REQUIRE(a != nullptr, SSMQ_ERR_INVALID_ARG, "%s: args is NULL", fn);
  REQUIRE(a->batch >= 0 && a->seqlen >= 0 && a->dim >= 0, SSMQ_ERR_INVALID_ARG,
          "%s: negative size", fn);
  REQUIRE(a->ngroups >= 1 && a->dim % a->ngroups == 0, SSMQ_ERR_INVALID_ARG,
          "%s: dim must be a multiple of ngroups >= 1", fn);
  REQUIRE(a->dstate == 4 || a->dstate == 8 || a->dstate == 16 || a->dstate == 32 ||
              a->dstate == 64,
          SSMQ_ERR_UNSUPPORTED, "%s: dstate %lld not in {4, 8, 16, 32, 64}", fn,
          (long long)a->dstate);
  REQUIRE(a->state_group_size >= 1 && a->dstate % a->state_group_size == 0,
          SSMQ_ERR_INVALID_ARG, "%s: dstate must be a multiple of state_group_size", fn);
  if (a->batch == 0 || a->dim == 0) return SSMQ_OK;
  REQUIRE(h_carry != nullptr, SSMQ_ERR_INVALID_ARG, "%s: h_carry is NULL", fn);
  if (a->seqlen > 0)
    REQUIRE(a->y && a->dt && a->A && a->C && a->C_scale, SSMQ_ERR_INVALID_ARG,
            "%s: a required tensor (y, dt, A, C, C_scale) is NULL", fn);
  REQUIRE(aligned16(a->dt) && aligned16(a->z) && aligned16(a->C) && aligned16(a->y) &&
              aligned16(a->h_final) && aligned16(a->A) && aligned16(h_carry),
          SSMQ_ERR_ALIGNMENT, "%s: tensors must be 16-byte aligned", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_selective_scan_carry_in(*a, h_carry, (cudaStream_t)stream), fn);
}

int32_t ssmq_scan_time_segments(const ssmq_scan_args* a) {
  if (!a) return 0;
  int64_t seg_len = 0;
  return (int32_t)ssmq::scan_time_segments(*a, &seg_len);
}

size_t ssmq_scan_workspace_size(const ssmq_scan_args* a) {
  if (!a) return 0;
  const int64_t k = ssmq_scan_time_segments(a);
  if (k <= 1 || a->batch <= 0 || a->dim <= 0 || a->dstate <= 0) return 0;
  return (size_t)k * (size_t)a->batch * (size_t)a->dim * (size_t)a->dstate * sizeof(float);
}

size_t ssmq_ssd_workspace_size(const ssmq_ssd_args* a) {
  if (!a) return 0;
  return ssmq::ssd_workspace_bytes(*a);
}

namespace {

// validation shared by the SSD scan and its carry-in; `batch` or `nheads` 0
// returns SSMQ_OK with *skip set (nothing to launch)
ssmq_status check_ssd(const ssmq_ssd_args* a, void* workspace, size_t ws_bytes, const char* fn,
                      bool* skip) {
  *skip = false;
  REQUIRE(a != nullptr, SSMQ_ERR_INVALID_ARG, "%s: args is NULL", fn);
  REQUIRE(a->batch >= 0 && a->seqlen >= 0 && a->nheads >= 0, SSMQ_ERR_INVALID_ARG,
          "%s: negative size", fn);
  REQUIRE(a->ngroups >= 1 && a->nheads % a->ngroups == 0, SSMQ_ERR_INVALID_ARG,
          "%s: nheads must be a multiple of ngroups >= 1", fn);
  REQUIRE(a->headdim == 64 && a->dstate == 128, SSMQ_ERR_UNSUPPORTED,
          "%s: the SSD kernel runs headdim 64, dstate 128", fn);
  REQUIRE(a->chunk == 64 || a->chunk == 128 || a->chunk == 256, SSMQ_ERR_UNSUPPORTED,
          "%s: chunk must be 64, 128 or 256", fn);
  REQUIRE(a->state_group_size >= 1 && a->dstate % a->state_group_size == 0,
          SSMQ_ERR_INVALID_ARG, "%s: dstate must be a multiple of state_group_size", fn);
  REQUIRE(a->max_segments >= 0, SSMQ_ERR_INVALID_ARG, "%s: max_segments must be >= 0", fn);
  if (a->batch == 0 || a->nheads == 0) {
    *skip = true;
    return SSMQ_OK;
  }
  if (a->seqlen == 0) {  // only the state passes through (h0 or zero to h_final)
    REQUIRE(aligned16(a->h0) && aligned16(a->h_final), SSMQ_ERR_ALIGNMENT,
            "%s: tensors must be 16-byte aligned", fn);
    return SSMQ_OK;
  }
  const ssmq_status xs = check_x(a->x_format, a->x, a->x_group, a->x_scale, a->n_x_groups,
                                 a->se_log2_ratio, fn);
  if (xs != SSMQ_OK) return xs;
  REQUIRE(a->dt && a->A && a->B && a->C && a->B_scale && a->C_scale && (a->y || a->y_q),
          SSMQ_ERR_INVALID_ARG,
          "%s: a required tensor (dt, A, B, C, B_scale, C_scale, y or y_q) is NULL", fn);
  REQUIRE(aligned16(a->x) && aligned16(a->dt) && aligned16(a->z) && aligned16(a->B) &&
              aligned16(a->C) && aligned16(a->y) && aligned16(a->h0) && aligned16(a->h_final),
          SSMQ_ERR_ALIGNMENT, "%s: tensors must be 16-byte aligned", fn);
  const ssmq_status ys = check_yq(a->y_q, a->y_group, a->y_scale, a->n_y_groups, fn);
  if (ys != SSMQ_OK) return ys;
  const size_t need = ssmq::ssd_workspace_bytes(*a);
  REQUIRE(need == 0 || (workspace && ws_bytes >= need), SSMQ_ERR_INVALID_ARG,
          "%s: workspace of %zu bytes required (got %zu)", fn, need, ws_bytes);
  REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, SSMQ_ERR_ALIGNMENT,
          "%s: workspace must be 256-byte aligned", fn);
  return SSMQ_OK;
}

}  // namespace

ssmq_status ssmq_ssd_chunk_scan_w8(const ssmq_ssd_args* a, void* workspace, size_t ws_bytes,
                                   void* stream) {
  const char* fn = "ssmq_ssd_chunk_scan_w8";
  Range nvtx_range(fn);
  bool skip;
  CHECK(check_ssd(a, workspace, ws_bytes, fn, &skip));
  if (skip) return SSMQ_OK;
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_ssd(*a, workspace, (cudaStream_t)stream), fn);
}

ssmq_status ssmq_ssd_carry_in(const ssmq_ssd_args* a, const float* h_carry, void* workspace,
                              size_t ws_bytes, void* stream) {
  const char* fn = "ssmq_ssd_carry_in";
  Range nvtx_range(fn);
  bool skip;
  CHECK(check_ssd(a, workspace, ws_bytes, fn, &skip));
  if (skip) return SSMQ_OK;
  REQUIRE((a->y != nullptr || a->seqlen == 0) && a->y_q == nullptr, SSMQ_ERR_INVALID_ARG,
          "%s: needs the binary16 y (and no int8 y)", fn);
  REQUIRE(h_carry != nullptr, SSMQ_ERR_INVALID_ARG, "%s: h_carry is NULL", fn);
  REQUIRE(aligned16(h_carry), SSMQ_ERR_ALIGNMENT, "%s: h_carry must be 16-byte aligned", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_ssd_carry_in(*a, h_carry, workspace, (cudaStream_t)stream), fn);
}

ssmq_status ssmq_state_chain(const float* h_end, const float* dec, int32_t n_parts,
                             int64_t units, int64_t elems, float* h_out, void* stream) {
  const char* fn = "ssmq_state_chain";
  Range nvtx_range(fn);
  REQUIRE(n_parts >= 1, SSMQ_ERR_INVALID_ARG, "%s: n_parts must be >= 1", fn);
  REQUIRE(units >= 0 && elems >= 0, SSMQ_ERR_INVALID_ARG, "%s: negative size", fn);
  if (units == 0 || elems == 0) return SSMQ_OK;
  REQUIRE(h_end && dec && h_out, SSMQ_ERR_INVALID_ARG, "%s: NULL tensor", fn);
  REQUIRE(units <= INT64_MAX / elems / n_parts, SSMQ_ERR_INVALID_ARG, "%s: size overflow", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_state_chain(h_end, dec, n_parts, units, elems, nullptr, h_out,
                                         (cudaStream_t)stream),
                fn);
}

ssmq_status ssmq_state_update_w8(const ssmq_decode_args* a, void* stream) {
  const char* fn = "ssmq_state_update_w8";
  Range nvtx_range(fn);
  REQUIRE(a != nullptr, SSMQ_ERR_INVALID_ARG, "%s: args is NULL", fn);
  REQUIRE(a->batch >= 0 && a->nheads >= 0 && a->headdim >= 0, SSMQ_ERR_INVALID_ARG,
          "%s: negative size", fn);
  REQUIRE(a->ngroups >= 1 && a->nheads % a->ngroups == 0, SSMQ_ERR_INVALID_ARG,
          "%s: nheads must be a multiple of ngroups >= 1", fn);
  REQUIRE(a->dstate == 16 || a->dstate == 32 || a->dstate == 64 || a->dstate == 128,
          SSMQ_ERR_UNSUPPORTED, "%s: dstate %lld not in {16, 32, 64, 128}", fn,
          (long long)a->dstate);
  REQUIRE(a->state_group_size >= 1 && a->dstate % a->state_group_size == 0,
          SSMQ_ERR_INVALID_ARG, "%s: dstate must be a multiple of state_group_size", fn);
  if (a->batch == 0 || a->nheads == 0 || a->headdim == 0) return SSMQ_OK;
  const ssmq_status xs = check_x(a->x_format, a->x, a->x_group, a->x_scale, a->n_x_groups,
                                 a->se_log2_ratio, fn);
  if (xs != SSMQ_OK) return xs;
  REQUIRE(a->dt && a->A && a->B && a->C && a->B_scale && a->C_scale && a->state && a->y,
          SSMQ_ERR_INVALID_ARG, "%s: a required tensor is NULL", fn);
  REQUIRE(aligned16(a->state) && aligned16(a->B) && aligned16(a->C), SSMQ_ERR_ALIGNMENT,
          "%s: state, B and C must be 16-byte aligned", fn);
  REQUIRE(a->batch * a->nheads <= 0x7fffffff, SSMQ_ERR_UNSUPPORTED, "%s: too many heads", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_state_update(*a, (cudaStream_t)stream), fn);
}

ssmq_status ssmq_selective_state_update_w8(const ssmq_m1_decode_args* a, void* stream) {
  const char* fn = "ssmq_selective_state_update_w8";
  Range nvtx_range(fn);
  REQUIRE(a != nullptr, SSMQ_ERR_INVALID_ARG, "%s: args is NULL", fn);
  REQUIRE(a->batch >= 0 && a->dim >= 0, SSMQ_ERR_INVALID_ARG, "%s: negative size", fn);
  REQUIRE(a->ngroups >= 1 && a->dim % a->ngroups == 0, SSMQ_ERR_INVALID_ARG,
          "%s: dim must be a multiple of ngroups >= 1", fn);
  REQUIRE(a->dstate == 4 || a->dstate == 8 || a->dstate == 16 || a->dstate == 32 ||
              a->dstate == 64 || a->dstate == 128,
          SSMQ_ERR_UNSUPPORTED, "%s: dstate %lld not in {4, 8, 16, 32, 64, 128}", fn,
          (long long)a->dstate);
  REQUIRE(a->state_group_size >= 1 && a->dstate % a->state_group_size == 0,
          SSMQ_ERR_INVALID_ARG, "%s: dstate must be a multiple of state_group_size", fn);
  if (a->batch == 0 || a->dim == 0) return SSMQ_OK;
  const ssmq_status xs = check_x(a->x_format, a->x, a->x_group, a->x_scale, a->n_x_groups,
                                 a->se_log2_ratio, fn);
  if (xs != SSMQ_OK) return xs;
  REQUIRE(a->dt && a->A && a->B && a->C && a->B_scale && a->C_scale && a->state && a->y,
          SSMQ_ERR_INVALID_ARG, "%s: a required tensor is NULL", fn);
  REQUIRE(aligned16(a->state) && aligned16(a->A) && aligned16(a->B) && aligned16(a->C),
          SSMQ_ERR_ALIGNMENT, "%s: state, A, B and C must be 16-byte aligned", fn);
  REQUIRE(a->batch * a->dim * (a->dstate / 4) <= 0x7fffffffLL * 256, SSMQ_ERR_UNSUPPORTED,
          "%s: too many channels", fn);
  if (injected(fn)) return fail(SSMQ_ERR_CUDA, "%s: injected launch failure", fn);
  return finish(ssmq::launch_m1_state_update(*a, (cudaStream_t)stream), fn);
}

}  // extern "C"
