// Exact unsigned 32-bit division by a run-time invariant divisor with one
// multiply-high, two adds and two shifts (Granlund and Montgomery, "Division
// by invariant integers using multiplication", PLDI 1994, section 4 and
// figure 4.1): for d >= 1 let l = ceil(log2 d) and
//     m = floor(2^32 (2^l - d) / d) + 1        (fits in 32 bits)
// then for every 0 <= n < 2^32
//     t = mulhi(m, n),   n / d = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0).
// Plain C++ (host and device) so it is tested exhaustively on the host.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define SSMQ_HD __host__ __device__ __forceinline__
#else
#define SSMQ_HD inline
#endif

namespace ssmq {

struct FastDiv {
  uint32_t d, m, s1, s2;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d ? d : 1u;
  uint32_t l = 0;
  while (l < 32 && (1ull << l) < (uint64_t)f.d) ++l;
  f.m = (uint32_t)((((1ull << l) - f.d) << 32) / f.d + 1ull);
  f.s1 = l < 1 ? l : 1u;
  f.s2 = l > 0 ? l - 1u : 0u;
  return f;
}

SSMQ_HD uint32_t mulhi32(uint32_t a, uint32_t b) {
#if defined(__CUDA_ARCH__)
  return __umulhi(a, b);
#else
  return (uint32_t)(((uint64_t)a * b) >> 32);
#endif
}

SSMQ_HD uint32_t fdiv(uint32_t n, const FastDiv& f) {
  const uint32_t t = mulhi32(f.m, n);
  return (t + ((n - t) >> f.s1)) >> f.s2;
}
SSMQ_HD uint32_t fmod_(uint32_t n, const FastDiv& f) { return n - fdiv(n, f) * f.d; }

}  // namespace ssmq
