"""The rotate+quantise kernel stores each token's scale absmax_u / (127 sqrt(g))
correctly rounded to float32. From 2^-100 up it forms the quotient without a
division: q0 = absmax_u * r (r the nearest float to the reciprocal of the
divisor), then one correction by the exact remainder, q = fma(fma(-q0, d, x), r, q0).
This test restates those three operations in C with the host's fused
multiply-add (IEEE single rounding, as on the GPU) and compares them with the
correctly rounded quotient for EVERY float32 from 2^-100 to the largest
finite value, for both divisors (g = 256: 2032; g = 128: the nearest float to
127 sqrt(128)). The quotient taken in double and rounded to float is the
correctly rounded float32 quotient (53 >= 2 * 24 + 2 bits). A negative control
(the uncorrected product) must show mismatches, so the checker can fail.
"""

import shutil
import subprocess

import pytest

C_SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
static inline float from_bits(uint32_t b) { float x; memcpy(&x, &b, 4); return x; }
int main(int argc, char** argv) {
  const float d = strtof(argv[1], NULL);
  const float r = 1.0f / d;               /* the nearest float to 1/d */
  const int corrected = atoi(argv[2]);
  const uint32_t lo = 0x0D800000u;        /* 2^-100 */
  const uint32_t hi = 0x7F7FFFFFu;        /* the largest finite float */
  unsigned long long bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
  for (long long b = lo; b <= (long long)hi; ++b) {
    const float x = from_bits((uint32_t)b);
    const float q0 = x * r;
    float q = q0;
    if (corrected) {
      const float e = fmaf(-q0, d, x);
      q = fmaf(e, r, q0);
    }
    const float ref = (float)((double)x / (double)d);
    bad += (q != ref);
  }
  printf("%llu %a\n", bad, (double)r);
  return 0;
}
"""

DIVISORS = {256: ("2032", float.fromhex("0x1.020408p-11")), 128: ("1436.8409423828125", float.fromhex("0x1.6ce3aep-11"))}


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    d = tmp_path_factory.mktemp("scale_div")
    src = d / "check.c"
    src.write_text(C_SRC)
    exe = d / "check"
    flags = ["-O2", "-ffp-contract=off", "-fopenmp"]
    if "fma" in open("/proc/cpuinfo").read():
        flags.append("-mfma")  # hardware fused multiply-add (glibc's fmaf is exact either way, only slower)
    subprocess.run([gcc, *flags, str(src), "-o", str(exe), "-lm"], check=True)
    return exe


def _run(exe, d: str, corrected: int):
    out = subprocess.run([str(exe), d, str(corrected)], check=True, capture_output=True, text=True, timeout=600)
    bad, r = out.stdout.split()
    return int(bad), float.fromhex(r)


@pytest.mark.parametrize("g", [256, 128])
def test_corrected_quotient_is_correctly_rounded_everywhere(checker, g):
    d, r_kernel = DIVISORS[g]
    bad, r = _run(checker, d, 1)
    assert r == r_kernel  # the reciprocal constant the kernel uses
    assert bad == 0


@pytest.mark.parametrize("g", [256, 128])
def test_uncorrected_product_is_caught(checker, g):
    bad, _ = _run(checker, DIVISORS[g][0], 0)
    assert bad > 1000
