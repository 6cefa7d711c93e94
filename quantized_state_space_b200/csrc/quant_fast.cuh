// 16-element fast routes of the group quantizer and the soft-edge encoder
// (Quamba-SE write-up section 1: one scale maps floats onto the INT8 grid;
// 2.1-2.2: three modes and their byte codes), shared by the streaming
// quantizer / encoder and the fused conv + SiLU producer.  Each returns false
// when an element lies near a rounding tie or is not finite; the caller then
// redoes the vector element by element with the exact definition.
#pragma once

#include "common.cuh"

namespace ssmq {

constexpr int kQVec = 16;

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// Branch-free fast route for 16 elements whose halves each share one valid
// (s, rs) (the argument of quant_rne_fast, in packed fp32x2 arithmetic): the code byte of
// each element is the low byte of m = fl32(clamp(v rs) + 1.5 2^23), which
// holds 0x4B400000 + k for the integer k = rne(clamp(v rs)).  Two running
// reductions replace per-element tests: the largest |y - (m - 1.5 2^23)|
// (at least 0.5 - 2^-14 only when some element lies within 2^-14 of a tie)
// and the sum of v * 0 (NaN exactly when some v is not finite).  Returns false
// in either case; the caller then redoes the vector element by element.
__device__ __forceinline__ bool quant16_fast(const float (&x)[kQVec], float rs0, float rs1,
                                             uint4& out) {
  // rs0 for elements 0-7, rs1 for 8-15 (two groups of 8 columns)
  const float2 ra = make_float2(rs0, rs0), rb = make_float2(rs1, rs1);
  const float2 mg = make_float2(12582912.0f, 12582912.0f);
  const float2 zero = make_float2(0.0f, 0.0f);
  float2 nf = zero;
  float dmax = 0.0f;
  uint32_t mb[kQVec];
#pragma unroll
  for (int i = 0; i < kQVec; i += 2) {
    const float2 xv = make_float2(x[i], x[i + 1]);
    float2 y = fmul2(xv, i < kQVec / 2 ? ra : rb);
    y.x = fminf(fmaxf(y.x, -127.0f), 127.0f);
    y.y = fminf(fmaxf(y.y, -127.0f), 127.0f);
    const float2 m = fadd2(y, mg);
    const float2 d = fsub2(y, fsub2(m, mg));
    dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
    nf = ffma2(xv, zero, nf);
    mb[i] = __float_as_uint(m.x);
    mb[i + 1] = __float_as_uint(m.y);
  }
  out.x = __byte_perm(__byte_perm(mb[0], mb[1], 0x0040), __byte_perm(mb[2], mb[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(mb[4], mb[5], 0x0040), __byte_perm(mb[6], mb[7], 0x0040), 0x5410);
  out.z = __byte_perm(__byte_perm(mb[8], mb[9], 0x0040), __byte_perm(mb[10], mb[11], 0x0040), 0x5410);
  out.w = __byte_perm(__byte_perm(mb[12], mb[13], 0x0040), __byte_perm(mb[14], mb[15], 0x0040), 0x5410);
  return dmax < 0.5f - 1.0f / 16384.0f && nf.x == 0.0f && nf.y == 0.0f;
}

// Branch-free fast route for 16 soft-edge codes (every st.rs[] usable):
// the mode by two compares, then quant16_fast's rounding with the mode's
// reciprocal and clamp.  From the low byte b of the rounding sum (two's
// complement k) the code is b & 0x7F (standard), (b & 0x3F) | 0x80 (small)
// or b | 0xC0 (large, |k| <= 31).  Same fallback conditions as quant16_fast.
__device__ __forceinline__ bool se16_fast(const float (&x)[kQVec], float lo, float hi,
                                          const SeSteps& st, uint4& out) {
  const float2 mg = make_float2(12582912.0f, 12582912.0f), zero = make_float2(0.0f, 0.0f);
  float2 nf = zero;
  float dmax = 0.0f;
  uint32_t cb[kQVec];
#pragma unroll
  for (int i = 0; i < kQVec; i += 2) {
    const float2 xv = make_float2(x[i], x[i + 1]);
    const bool s0 = fabsf(xv.x) < lo, l0 = fabsf(xv.x) > hi;
    const bool s1 = fabsf(xv.y) < lo, l1 = fabsf(xv.y) > hi;
    const float2 rs = make_float2(s0 ? st.rs[1] : (l0 ? st.rs[2] : st.rs[0]),
                                  s1 ? st.rs[1] : (l1 ? st.rs[2] : st.rs[0]));
    const float lim0 = (s0 || l0) ? 31.0f : 63.0f, lim1 = (s1 || l1) ? 31.0f : 63.0f;
    float2 y = fmul2(xv, rs);
    y.x = fminf(fmaxf(y.x, -lim0), lim0);
    y.y = fminf(fmaxf(y.y, -lim1), lim1);
    const float2 m = fadd2(y, mg);
    const float2 d = fsub2(y, fsub2(m, mg));
    dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
    nf = ffma2(xv, zero, nf);
    const uint32_t b0 = __float_as_uint(m.x), b1 = __float_as_uint(m.y);
    cb[i] = s0 ? ((b0 & 0x3Fu) | 0x80u) : (l0 ? (b0 | 0xC0u) : (b0 & 0x7Fu));
    cb[i + 1] = s1 ? ((b1 & 0x3Fu) | 0x80u) : (l1 ? (b1 | 0xC0u) : (b1 & 0x7Fu));
  }
  out.x = __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
  out.z = __byte_perm(__byte_perm(cb[8], cb[9], 0x0040), __byte_perm(cb[10], cb[11], 0x0040), 0x5410);
  out.w = __byte_perm(__byte_perm(cb[12], cb[13], 0x0040), __byte_perm(cb[14], cb[15], 0x0040), 0x5410);
  return dmax < 0.5f - 1.0f / 16384.0f && nf.x == 0.0f && nf.y == 0.0f;
}

}  // namespace ssmq
