/* Host check of the division the quantization kernels use: for a = every
 * bf16 significand (with an exponent and both signs), +-0 and a few bf16
 * subnormals, and b = every fp32 significand,
 *   y = RN(1/b), q0 = RN(a*y), r = RN(a - b*q0) (one FMA),
 *   q1 = q0 if r = 0, else RN(q0 + r*y)
 * equals the correctly rounded a/b bit for bit, sign of zero included
 * (Markstein's correction, P. Markstein, IBM J. Res. Dev. 34(1), 1990).
 * For subnormal a the steps may underflow and q1 may be off in its last
 * place; there the check is what the codes need when they differ: the same
 * sign, and both values below 2^-11 in magnitude (the code 0 in e4m3 and in
 * int8 alike).  Scaling a or b by a power of two scales
 * every step exactly while nothing underflows, so the significands cover
 * the normal range.  Usage: quotient_identity ea eb [bstep [plain]]; exit 1
 * on a mismatch.  A fourth argument checks the plain product q0 instead (the
 * test expects mismatches there: the check can fail). */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

int main(int argc, char **argv) {
  const int ea = argc > 1 ? atoi(argv[1]) : 0;
  const int eb = argc > 2 ? atoi(argv[2]) : 0;
  const uint32_t bstep = argc > 3 ? (uint32_t)atoi(argv[3]) : 1u;
  const int plain = argc > 4;
  long long bad = 0, n = 0;
  for (uint32_t bm = 0; bm < (1u << 23); bm += bstep) {
    const float b = from_bits(((uint32_t)(127 + eb) << 23) | bm);
    volatile float y = 1.0f / b;
    for (uint32_t am = 0; am < 256 + 8; ++am) {
      float a;
      if (am < 256) /* 7 fraction bits and the sign */
        a = from_bits(((am >> 7) << 31) | ((uint32_t)(127 + ea) << 23) | ((am & 127u) << 16));
      else /* +-0 and bf16 subnormals: 0x0000, 0x8000, 0x0001, 0x8001, 0x007f, 0x807f, 0x0040, 0x8040 */
        a = from_bits((uint32_t)((const uint16_t[]){0x0000, 0x8000, 0x0001, 0x8001, 0x007f, 0x807f, 0x0040,
                                                     0x8040})[am - 256] << 16);
      const float q0 = a * y;
      const float r = fmaf(-b, q0, a);
      const float q1 = plain ? q0 : (r == 0.0f ? q0 : fmaf(r, y, q0));
      const float want = a / b;
      uint32_t g, w;
      memcpy(&g, &q1, 4);
      memcpy(&w, &want, 4);
      ++n;
      const int subnormal_a = am >= 258;
      const int ok = g == w || (subnormal_a && (g >> 31) == (w >> 31) && fabsf(q1) < 0x1p-11f &&
                                fabsf(want) < 0x1p-11f);
      if (!ok) {
        if (bad < 5) printf("mismatch a=%a b=%a q1=%a want=%a\n", a, b, q1, want);
        ++bad;
      }
    }
  }
  printf("ea=%d eb=%d checked=%lld mismatches=%lld\n", ea, eb, n, bad);
  return bad != 0;
}
