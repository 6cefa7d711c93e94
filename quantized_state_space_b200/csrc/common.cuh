// Device helpers shared by the sm_100a kernels of the W8A8 scan library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssmq.h"

namespace ssmq {

constexpr float kLog2e = 1.4426950408889634f;

// ---- packed fp32x2 arithmetic (sm_100: one instruction, two lanes) ---------
__device__ __forceinline__ uint64_t pk(float2 v) { return *reinterpret_cast<uint64_t*>(&v); }
__device__ __forceinline__ float2 upk(uint64_t v) { return *reinterpret_cast<float2*>(&v); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)));
  return upk(d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)));
  return upk(d);
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)));
  return upk(d);
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pk(a)), "l"(pk(b)), "l"(pk(c)));
  return upk(d);
}

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ uint16_t f2h(float v) { return __half_as_ushort(__float2half_rn(v)); }

// int8 byte i of w as an exact fp32 value without a conversion instruction:
// (q + 128) placed in the low mantissa of 2^23, then 2^23 + 128 subtracted.
// xw must be w ^ 0x80808080.
__device__ __forceinline__ float s8_to_f32(uint32_t xw, int i) {
  return __int_as_float((int)__byte_perm(xw, 0x4B000000u, 0x7650u + (uint32_t)i)) - 8388736.0f;
}
// int8 bytes i and j of w as an exact binary16 pair: (q + 128) in the low
// mantissa of 1024.0, then 1152 subtracted in half precision.  xw = w ^ 0x80808080.
__device__ __forceinline__ __half2 s8x2_to_h2(uint32_t xw, int i, int j) {
  const uint32_t bits = __byte_perm(xw, 0x64646464u, (uint32_t)(i | (4 << 4) | (j << 8) | (4 << 12)));
  return __hsub2(*reinterpret_cast<const __half2*>(&bits), __float2half2_rn(1152.0f));
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
// two fp32 values rounded to a packed binary16 pair (one instruction)
__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  return h2_bits(__floats2half2_rn(a, b));
}

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

// The same integer by a faster route.  rs is the correctly rounded binary32
// reciprocal of step (step normal, rs finite).  y = fl32(v * rs) differs from
// v / step by at most 2^-23 relative, i.e. by less than 2^-15 for |v / step|
// <= 128, and fl32(v / step) lies within 2^-18 of v / step there.  So unless
// y is within 2^-14 of a half-integer, y and fl32(v / step) round to the same
// integer, and clamping before rounding commutes with the rule (every value
// beyond +-lim rounds to at least lim).  Near a tie the exact division
// decides.  v must be finite.
__device__ __forceinline__ int quant_rne_fast(float v, float step, float rs, int lim) {
  const float flim = (float)lim;
  const float yc = fminf(fmaxf(v * rs, -flim), flim);
  const float m = yc + 12582912.0f;  // 1.5 * 2^23: the sum rounds yc to an integer, ties to even
  const float k = m - 12582912.0f;
  if (fabsf(fabsf(yc - k) - 0.5f) < (1.0f / 16384.0f)) return quant_rne(v, step, lim);
  return __float_as_int(m) - 0x4B400000;
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
// rs[] are the correctly rounded reciprocals of s[] when s[] is at least
// 2^-100 with a normal reciprocal, else 0 (which selects the exact division).
// fm[] are the quotient multipliers of the modes, {1, 2^r, 2^-r}: whenever
// rs[] are all usable, s[1] = s[0] / 2^r and s[2] = s[0] 2^r exactly, so
// fl32(v / s[m]) = fl32(v / s[0]) fm[m] up to underflow of tiny quotients.
struct SeSteps {
  float s[3];
  float rs[3];
  float fm[3];
};
// The bound 2^-100 keeps the residual of the packed routes' division
// correction (quant_fast.cuh) exact: for a quotient of magnitude at least
// 1/4 the residual is a multiple of 2^-149.
__host__ __device__ inline bool usable_recip(float s, float r) {
  return s >= 0x1p-100f && r > 0.0f && r <= 3.40282347e+38f && r >= 1.17549435e-38f;
}
__host__ inline SeSteps se_steps(float scale, int log2_ratio) {
  SeSteps st;
  const float f = (float)(1u << log2_ratio);
  st.s[0] = scale;
  st.s[1] = scale * (1.0f / f);
  st.s[2] = scale * f;
  st.fm[0] = 1.0f;
  st.fm[1] = f;
  st.fm[2] = 1.0f / f;
  for (int i = 0; i < 3; ++i) {
    const float r = 1.0f / st.s[i];
    st.rs[i] = usable_recip(st.s[i], r) ? r : 0.0f;
  }
  return st;
}

__device__ __forceinline__ float se_decode(uint32_t c, const SeSteps& st) {
  int q, mode;
  se_split(c, q, mode);
  // selects, not an indexed load: keeps the steps in registers
  return (float)q * (mode == 0 ? st.s[0] : (mode == 1 ? st.s[1] : st.s[2]));
}

// One element of the static quantizer; flags record device-side anomalies.
// rs: reciprocal of s for the fast route, 0 to force the exact division.
__device__ __forceinline__ int quant_elem(float v, float s, float rs, bool okg, uint32_t& flags) {
  if (!okg) {
    flags |= SSMQ_DEV_BAD_GROUP;
    return 0;
  }
  if (!isfinite(v)) {
    flags |= SSMQ_DEV_NONFINITE;
    return 0;
  }
  if (!(s > 0.0f) || !isfinite(s)) {
    if (s != 0.0f) flags |= SSMQ_DEV_BAD_SCALE;
    return 0;
  }
  return rs != 0.0f ? quant_rne_fast(v, s, rs, 127) : quant_rne(v, s, 127);
}

// One soft-edge code (Quamba-SE write-up 2.1-2.2): mode by |v| against the
// thresholds, payload by the quantizer at the mode's step and clamp.
__device__ __forceinline__ uint32_t se_encode1(float v, float lo, float hi, const SeSteps& st,
                                               uint32_t& flags) {
  if (!isfinite(v)) {
    flags |= SSMQ_DEV_NONFINITE;
    return 0u;
  }
  const float a = fabsf(v);
  const int mode = a < lo ? 1 : (a > hi ? 2 : 0);
  const float step = mode == 0 ? st.s[0] : (mode == 1 ? st.s[1] : st.s[2]);
  const int lim = mode == 0 ? 63 : 31;
  const float rs = mode == 0 ? st.rs[0] : (mode == 1 ? st.rs[1] : st.rs[2]);
  const int qv = (step > 0.0f && isfinite(step))
                     ? (rs != 0.0f ? quant_rne_fast(v, step, rs, lim) : quant_rne(v, step, lim))
                     : 0;
  if (mode == 0) return (uint32_t)(qv & 0x7F);
  return (mode == 1 ? 0x80u : 0xC0u) | (uint32_t)(qv & 0x3F);
}

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bits) {
  if (bits && status) atomicOr(status, bits);
}

}  // namespace ssmq
