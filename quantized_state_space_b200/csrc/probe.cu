// Diagnostics: the rate of the special-function unit's base-2 exponential.
//
// Every state update of the Mamba-1 scan evaluates one decay exp(delta A) on
// the special-function unit (MUFU.EX2), so at small state sizes that unit,
// not HBM, is the scan's compute roof.  This kernel measures the roof on the
// GPU at hand: each thread runs kChains independent chains y <- 2^-y (the
// negation is an operand modifier, so the loop body is exponentials only;
// the chains converge to y = 0.641..., no overflow or denormals), enough
// warps per SM to cover the unit's latency.  The host times it with CUDA
// events; rate = n_ex2 / time.
#include "common.cuh"
#include "internal.h"

namespace ssmq {
namespace {

constexpr int kChains = 8;
constexpr int kProbeThreads = 256;
constexpr int kProbeCtasPerSm = 8;  // 64 warps per SM

__global__ void __launch_bounds__(kProbeThreads) ex2_rate_kernel(int iters, float* sink) {
  float y[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) y[i] = 0.25f + 0.03125f * i + 1e-4f * (threadIdx.x & 31);
  for (int k = 0; k < iters; ++k) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) y[i] = ex2_sfu(-y[i]);
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += y[i];
  if (s < 0.0f) sink[0] = s;  // never true (every y > 0); keeps the chains live
}

}  // namespace

cudaError_t launch_probe_ex2(int iters, float* sink, int64_t* n_ex2, cudaStream_t st) {
  const int grid = sm_count() * kProbeCtasPerSm;
  *n_ex2 = (int64_t)grid * kProbeThreads * kChains * (int64_t)iters;
  ex2_rate_kernel<<<grid, kProbeThreads, 0, st>>>(iters, sink);
  return cudaGetLastError();
}

}  // namespace ssmq
