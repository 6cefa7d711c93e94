"""Host check of the multiply-shift division used by the CUDA kernels for
group and row indices (csrc/fastdiv.h; Granlund and Montgomery, "Division by
invariant integers using multiplication", figure 4.1): compiled with g++ and
compared with the hardware division on edge and random dividends for edge and
random divisors."""
import os
import subprocess
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "quantized_state_space_b200", "csrc")

DRIVER = r"""
#include <stdio.h>
#include <stdint.h>
#include "fastdiv.h"
static uint64_t st = 0x9E3779B97F4A7C15ull;
static uint32_t rnd() { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return (uint32_t)st; }
static int check(uint32_t d) {
  const ssmq::FastDiv f = ssmq::make_fastdiv(d);
  uint32_t edge[] = {0u, 1u, 2u, d - 1u, d, d + 1u, 2u * d - 1u, 2u * d, 0x7FFFFFFFu, 0x80000000u,
                     0xFFFFFFFEu, 0xFFFFFFFFu, (0xFFFFFFFFu / d) * d, (0xFFFFFFFFu / d) * d - 1u};
  for (uint32_t n : edge)
    if (ssmq::fdiv(n, f) != n / d || ssmq::fmod_(n, f) != n % d) return 1;
  for (int i = 0; i < 4000; ++i) {
    const uint32_t n = rnd() >> (rnd() & 31);
    if (ssmq::fdiv(n, f) != n / d || ssmq::fmod_(n, f) != n % d) return 1;
  }
  return 0;
}
int main() {
  int bad = 0;
  for (uint32_t d = 1; d <= 5000; ++d) bad += check(d);
  for (int k = 0; k < 32; ++k) {
    const uint32_t p = 1u << k;
    bad += check(p);
    if (p > 1) bad += check(p - 1);
    if (p < 0x80000000u) bad += check(p + 1);
  }
  for (int i = 0; i < 3000; ++i) { uint32_t d = rnd() >> (rnd() & 31); if (d) bad += check(d); }
  bad += check(0xFFFFFFFFu) + check(0xFFFFFFFEu) + check(0x80000001u);
  printf("%d\n", bad);
  return bad != 0;
}
"""


def test_fastdiv_exact():
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "fd.cc")
        exe = os.path.join(td, "fd")
        with open(src, "w") as f:
            f.write(DRIVER)
        subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, src, "-o", exe], check=True)
        r = subprocess.run([exe], capture_output=True, text=True)
        assert r.returncode == 0 and r.stdout.strip() == "0", r.stdout + r.stderr
