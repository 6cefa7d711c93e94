// Device helpers shared by the sm_100a kernels of the W8A8 scan library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssmq {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ uint16_t f2h(float v) { return __half_as_ushort(__float2half_rn(v)); }

// 2^x on the special-function unit (MUFU.EX2); ~2 ulp, subnormal results
// flushed to zero.
__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_sfu(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log(1 + u) for u in [0, 1] as 2 atanh(s), s = u / (2 + u) in [0, 1/3]:
// the odd series 2 s (1 + s^2/3 + ... + s^16/17) truncates below 2e-10
// relative on that range.
__device__ __forceinline__ float log1p_unit(float u) {
  const float s = u * rcp_sfu(2.0f + u);
  const float s2 = s * s;
  float p = 1.0f / 17.0f;
  p = fmaf(p, s2, 1.0f / 15.0f);
  p = fmaf(p, s2, 1.0f / 13.0f);
  p = fmaf(p, s2, 1.0f / 11.0f);
  p = fmaf(p, s2, 1.0f / 9.0f);
  p = fmaf(p, s2, 1.0f / 7.0f);
  p = fmaf(p, s2, 1.0f / 5.0f);
  p = fmaf(p, s2, 1.0f / 3.0f);
  p = fmaf(p, s2, 1.0f);
  return 2.0f * s * p;
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(e^-|v|)
__device__ __forceinline__ float softplus_f(float v) {
  const float e = ex2_sfu(-fabsf(v) * kLog2e);
  return fmaxf(v, 0.0f) + log1p_unit(e);
}

// silu(z) = z * sigmoid(z) = z / (1 + e^-z)
__device__ __forceinline__ float silu_f(float z) {
  return z * rcp_sfu(1.0f + ex2_sfu(-z * kLog2e));
}

// Symmetric quantization with binary32 semantics:
// clamp(round_half_even(fl32(v / step)), -lim, lim).  The quotient is the
// correctly rounded IEEE division (the library is built without fast-math).
__device__ __forceinline__ int quant_rne(float v, float step, int lim) {
  const float r = __fdiv_rn(v, step);
  const int k = __float2int_rn(r);  // saturates at the int range
  return max(-lim, min(lim, k));
}

// Soft-edge byte -> (payload, mode) with mode 0 standard, 1 small, 2 large.
__device__ __forceinline__ void se_split(uint32_t c, int& q, int& mode) {
  if ((c & 0x80u) == 0u) {
    const int v = (int)(c & 0x7Fu);
    q = v >= 64 ? v - 128 : v;
    mode = 0;
  } else {
    const int v = (int)(c & 0x3Fu);
    q = v >= 32 ? v - 64 : v;
    mode = (c & 0x40u) ? 2 : 1;
  }
}

// Step sizes of the three soft-edge modes: {scale, scale / 2^r, scale * 2^r},
// each one binary32 product.
struct SeSteps {
  float s[3];
};
__host__ __device__ inline SeSteps se_steps(float scale, int log2_ratio) {
  SeSteps st;
  const float f = (float)(1u << log2_ratio);
  st.s[0] = scale;
  st.s[1] = scale * (1.0f / f);
  st.s[2] = scale * f;
  return st;
}

__device__ __forceinline__ float se_decode(uint32_t c, const SeSteps& st) {
  int q, mode;
  se_split(c, q, mode);
  return (float)q * st.s[mode];
}

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bits) {
  if (bits && status) atomicOr(status, bits);
}

}  // namespace ssmq
