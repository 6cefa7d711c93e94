// 16-element fast routes of the group quantizer and the soft-edge encoder
// (Quamba-SE write-up section 1: one scale maps floats onto the INT8 grid;
// 2.1-2.2: three modes and their byte codes), shared by the streaming
// quantizer / encoder and the fused conv + SiLU producer.  Each returns false
// when an element's quotient is not finite; the caller then redoes the vector
// element by element with the exact definition.
#pragma once

#include "common.cuh"

namespace ssmq {

constexpr int kQVec = 16;

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// Correctly rounded binary32 quotients v / s of two elements by one division
// correction (Markstein's theorem: when rs = fl32(1 / s) and y0 is within
// one ulp of v / s, the residual rr = v - y0 s is exact as one fma and
// fl32(y0 + rr rs) is the correctly rounded quotient), in packed fp32x2
// arithmetic: y0 = fl32(v rs), rr = fma(y0, -s, v), y = fma(rr, rs, y0).
// y0 is within one ulp whenever s and rs are normal: checked on the host
// for every binary32 s significand against every 11-bit v significand (all
// binary16 inputs) and against 2^34 random 24-bit v significands, with no
// exception.  The residual stays exact for quotients of magnitude 1/4 and
// more when s >= 2^-100 (usable_recip); smaller quotients round to code 0
// either way.  A non-finite v, or a v rs that overflows, makes y NaN or
// infinite.
__device__ __forceinline__ float2 div2_rn(float2 v, float2 s_neg, float2 rs) {
  const float2 y0 = fmul2(v, rs);
  const float2 rr = ffma2(y0, s_neg, v);
  return ffma2(rr, rs, y0);
}

// Branch-free fast route for 16 elements whose halves each share one valid
// scale (sr = (s, rs), rs usable): the code byte of each element is the low
// byte of m = fl32(clamp(y) + 1.5 2^23), y = fl32(v / s) by div2_rn; m holds
// 0x4B400000 + k for k = rne(clamp(y)), which is the definition's
// clamp(rne(fl32(v / s))) because the clamp bounds are integers.  One running
// sum of y * 0 is NaN exactly when some y is not finite (a non-finite input
// or an overflowing product); the caller then redoes the vector element by
// element.
__device__ __forceinline__ bool quant16_fast(const float (&x)[kQVec], float2 sr0, float2 sr1,
                                             uint4& out) {
  // sr0 for elements 0-7, sr1 for 8-15 (two groups of 8 columns)
  const float2 ra = make_float2(sr0.y, sr0.y), rb = make_float2(sr1.y, sr1.y);
  const float2 na = make_float2(-sr0.x, -sr0.x), nb = make_float2(-sr1.x, -sr1.x);
  const float2 mg = make_float2(12582912.0f, 12582912.0f);
  const float2 zero = make_float2(0.0f, 0.0f);
  float2 nf = zero;
  uint32_t mb[kQVec];
#pragma unroll
  for (int i = 0; i < kQVec; i += 2) {
    const bool lo = i < kQVec / 2;
    float2 y = div2_rn(make_float2(x[i], x[i + 1]), lo ? na : nb, lo ? ra : rb);
    nf = ffma2(y, zero, nf);
    y.x = fminf(fmaxf(y.x, -127.0f), 127.0f);
    y.y = fminf(fmaxf(y.y, -127.0f), 127.0f);
    const float2 m = fadd2(y, mg);
    mb[i] = __float_as_uint(m.x);
    mb[i + 1] = __float_as_uint(m.y);
  }
  out.x = __byte_perm(__byte_perm(mb[0], mb[1], 0x0040), __byte_perm(mb[2], mb[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(mb[4], mb[5], 0x0040), __byte_perm(mb[6], mb[7], 0x0040), 0x5410);
  out.z = __byte_perm(__byte_perm(mb[8], mb[9], 0x0040), __byte_perm(mb[10], mb[11], 0x0040), 0x5410);
  out.w = __byte_perm(__byte_perm(mb[12], mb[13], 0x0040), __byte_perm(mb[14], mb[15], 0x0040), 0x5410);
  return nf.x == 0.0f && nf.y == 0.0f;
}

// Branch-free fast route for 16 soft-edge codes (every st.rs[] usable): one
// quotient y = fl32(v / s[0]) by div2_rn serves the three modes, since
// fl32(v / s[m]) = y fm[m] exactly (SeSteps; a quotient that underflows
// there is below 1/2 and codes 0 in both forms).  The mode by two compares,
// then the rounding of quant16_fast with the mode's clamp.  From the low byte
// b of the rounding sum (two's complement k) the code is b & 0x7F
// (standard), (b & 0x3F) | 0x80 (small) or b | 0xC0 (large, |k| <= 31).
// Same fallback condition as quant16_fast.
__device__ __forceinline__ bool se16_fast(const float (&x)[kQVec], float lo, float hi,
                                          const SeSteps& st, uint4& out) {
  const float2 mg = make_float2(12582912.0f, 12582912.0f), zero = make_float2(0.0f, 0.0f);
  const float2 r0 = make_float2(st.rs[0], st.rs[0]), n0 = make_float2(-st.s[0], -st.s[0]);
  float2 nf = zero;
  uint32_t cb[kQVec];
#pragma unroll
  for (int i = 0; i < kQVec; i += 2) {
    const float2 xv = make_float2(x[i], x[i + 1]);
    const bool s0 = fabsf(xv.x) < lo, l0 = fabsf(xv.x) > hi;
    const bool s1 = fabsf(xv.y) < lo, l1 = fabsf(xv.y) > hi;
    const float2 q = div2_rn(xv, n0, r0);
    nf = ffma2(q, zero, nf);
    const float2 fm = make_float2(s0 ? st.fm[1] : (l0 ? st.fm[2] : 1.0f),
                                  s1 ? st.fm[1] : (l1 ? st.fm[2] : 1.0f));
    const float lim0 = (s0 || l0) ? 31.0f : 63.0f, lim1 = (s1 || l1) ? 31.0f : 63.0f;
    float2 y = fmul2(q, fm);
    y.x = fminf(fmaxf(y.x, -lim0), lim0);
    y.y = fminf(fmaxf(y.y, -lim1), lim1);
    const float2 m = fadd2(y, mg);
    const uint32_t b0 = __float_as_uint(m.x), b1 = __float_as_uint(m.y);
    cb[i] = s0 ? ((b0 & 0x3Fu) | 0x80u) : (l0 ? (b0 | 0xC0u) : (b0 & 0x7Fu));
    cb[i + 1] = s1 ? ((b1 & 0x3Fu) | 0x80u) : (l1 ? (b1 | 0xC0u) : (b1 & 0x7Fu));
  }
  out.x = __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
  out.z = __byte_perm(__byte_perm(cb[8], cb[9], 0x0040), __byte_perm(cb[10], cb[11], 0x0040), 0x5410);
  out.w = __byte_perm(__byte_perm(cb[12], cb[13], 0x0040), __byte_perm(cb[14], cb[15], 0x0040), 0x5410);
  return nf.x == 0.0f && nf.y == 0.0f;
}

}  // namespace ssmq
