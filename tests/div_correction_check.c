/* Host check of the packed quantizer routes' division (quant_fast.cuh,
 * div2_rn): with rs = fl32(1/s), y0 = fl32(v rs), rr = fma(y0, -s, v) and
 * y = fma(rr, rs, y0), y must equal the correctly rounded binary32 quotient
 * fl32(v / s) (Markstein's theorem; the quotient is exact-scaling invariant,
 * so significands suffice).
 *
 *   div_correction_check MODE STRIDE
 *   MODE 0: every 11-bit v significand (all binary16 inputs), v in [1, 4)
 *   MODE 1: 2048 pseudo-random 24-bit v significands per s
 *   s runs over the binary32 significands 1 + j 2^-23, j = 0, STRIDE, ...
 * Prints "pairs P mismatches M"; exit status 1 when M > 0. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

int main(int argc, char** argv) {
  const int mode = argc > 1 ? atoi(argv[1]) : 0;
  const int64_t stride = argc > 2 ? atoll(argv[2]) : 1;
  long long bad = 0, total = 0;
#pragma omp parallel for reduction(+ : bad, total) schedule(dynamic, 64)
  for (int64_t j = 0; j < (1 << 23); j += stride) {
    const float s = 1.0f + (float)j * 0x1p-23f;
    const float rs = 1.0f / s, ns = -s;
    float vs[2048];
    if (mode == 0) {
      for (int k = 0; k < 1024; ++k) {
        vs[k] = (float)(1024 + k) * 0x1p-10f;         /* [1, 2) */
        vs[1024 + k] = (float)(1024 + k) * 0x1p-9f;   /* [2, 4) */
      }
    } else {
      uint64_t h = (uint64_t)j * 0x9E3779B97F4A7C15ull + 12345u;
      for (int k = 0; k < 2048; ++k) {
        h ^= h >> 29;
        h *= 0xBF58476D1CE4E5B9ull;
        h ^= h >> 32;
        vs[k] = (1.0f + (float)(h & 0x7FFFFF) * 0x1p-23f) * ((k & 1) ? 2.0f : 1.0f);
      }
    }
    long long b = 0;
    for (int k = 0; k < 2048; ++k) {
      const float v = vs[k];
      const float y0 = v * rs;
      const float rr = fmaf(y0, ns, v);
      const float y = fmaf(rr, rs, y0);
      b += y != v / s;
    }
    bad += b;
    total += 2048;
  }
  printf("pairs %lld mismatches %lld\n", total, bad);
  return bad ? 1 : 0;
}
