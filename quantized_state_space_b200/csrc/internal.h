// Launchers behind the C ABI.  Each returns cudaSuccess or the launch error;
// arguments were validated by the caller (api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssmq.h"

namespace ssmq {

cudaError_t launch_quantize(const void* src, bool f16, int64_t outer, int64_t mid,
                            int64_t inner, const int32_t* gmap, int32_t n_groups,
                            bool absmax, float* scales, int8_t* q, uint32_t* status,
                            cudaStream_t st);

// one static quantization of a batch (validated by the API layer)
struct QuantJob {
  const void* src;
  bool f16;
  int64_t outer, mid, inner;
  const int32_t* gmap;
  int32_t n_groups;
  const float* scales;
  int8_t* q;
};
constexpr int kMaxQuantJobs = 8;
cudaError_t launch_quantize_batch(const QuantJob* jobs, int n_jobs, uint32_t* status,
                                  cudaStream_t st);
cudaError_t launch_softedge_encode(const void* src, bool f16, int64_t n, float scale,
                                   float lo, float hi, int log2_ratio, uint8_t* codes,
                                   uint32_t* status, cudaStream_t st);
cudaError_t launch_softedge_decode(const uint8_t* codes, int64_t n, float scale,
                                   int log2_ratio, float* out, cudaStream_t st);

// Time segments of a Mamba-1 scan call (1: one pass per row) and their
// length in steps (whole 32-step chunks).
int scan_time_segments(const ssmq_scan_args& a, int64_t* seg_len);
cudaError_t launch_selective_scan(const ssmq_scan_args& a, cudaStream_t st);
cudaError_t launch_selective_scan_carry_in(const ssmq_scan_args& a, const float* h_carry,
                                           cudaStream_t st);
cudaError_t launch_conv_silu_quantize(const ssmq_conv_args& a, cudaStream_t st);

cudaError_t launch_state_update(const ssmq_decode_args& a, cudaStream_t st);
cudaError_t launch_m1_state_update(const ssmq_m1_decode_args& a, cudaStream_t st);

cudaError_t launch_group_absmax(const void* src, bool f16, int64_t outer, int64_t mid,
                                int64_t inner, const int32_t* gmap, int32_t n_groups,
                                float* absmax, uint32_t* status, cudaStream_t st);
cudaError_t launch_cluster_by_absmax(const float* absmax, int n, int k, int32_t* cluster_of,
                                     float* scales, uint32_t* status, cudaStream_t st);
size_t percentile_workspace_bytes();
float* percentile_scratch_out(void* ws);
void* percentile_static_scratch(size_t need, cudaError_t* err);
int percentile_max_q();
cudaError_t launch_percentile_abs(const void* src, bool f16, int64_t n, const double* q, int nq,
                                  float* out, float* thr, float alpha, void* workspace,
                                  cudaStream_t st);

// diagnostics: base-2 exponentials on the special-function unit
cudaError_t launch_probe_ex2(int iters, float* sink, int64_t* n_ex2, cudaStream_t st);

// streaming multiprocessors of the current device
int sm_count();

size_t ssd_workspace_bytes(const ssmq_ssd_args& a);
cudaError_t launch_ssd(const ssmq_ssd_args& a, void* ws, cudaStream_t st);
cudaError_t launch_ssd_carry_in(const ssmq_ssd_args& a, const float* h_carry, void* ws,
                                cudaStream_t st);
cudaError_t launch_state_chain(const float* h_end, const float* dec, int n_parts, int64_t units,
                               int64_t elems, const float* h_init, float* h_out, cudaStream_t st);

}  // namespace ssmq
