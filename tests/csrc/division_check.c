/*
 * Exhaustive check of the quantizer's fast division against IEEE single division,
 * at the level that matters: the 4-bit code.
 *
 * The quantizer needs code(RN32(w / a)) = #{i : RN32(w/a) > T_i} for bf16 values
 * w, a with |w| <= a, a > 0, where T_0 < ... < T_14 are the decision thresholds
 * (midpoints of adjacent NF4 levels rounded down to fp32).  Its fast path
 * (blocks with 2^-64 <= a <= 2^64) replaces the division by Markstein's FMA
 * correction of a reciprocal quotient (P. Markstein, "Computation of elementary
 * functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
 *     y  = RN32(1/m) * 2^-e          (a = m * 2^e, m in [1, 2) with 7 fraction bits;
 *                                     RN32(1/m) from a 128-entry table, scaling exact)
 *     q0 = RN32(w * y)
 *     r  = fma(-q0, a, w)
 *     q  = fma(r, y, q0)
 * For every such pair of bf16 values (both signs of w, zeros and subnormals
 * included) this program checks that q and w/a (IEEE) give the same code, and
 * counts the pairs where the quotients differ at all (only tiny quotients, far
 * from any threshold, may).  Thresholds: 15 hex floats on the command line.
 * Exit status 0 iff every code agrees.
 * Build: gcc -O2 -ffp-contract=off division_check.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float bf16(uint32_t bits) {
  uint32_t u = bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static float T[15];

static int code_of(float x) {
  int c = 0;
  for (int i = 0; i < 15; ++i) c += x > T[i];
  return c;
}

int main(int argc, char **argv) {
  if (argc != 16) {
    fprintf(stderr, "usage: %s T0 ... T14 (hex floats)\n", argv[0]);
    return 2;
  }
  for (int i = 0; i < 15; ++i) T[i] = strtof(argv[i + 1], NULL);
  float table[128];
  for (int k = 0; k < 128; ++k) {
    volatile float m = 1.0f + (float)k / 128.0f;
    table[k] = 1.0f / m; /* IEEE RN */
  }
  unsigned long long pairs = 0, differ = 0, bad = 0;
  float max_abs_differ = 0.f;
  for (uint32_t ab = 0x0001; ab < 0x7F80; ++ab) {
    const float a = bf16(ab);
    if (!(a >= 0x1p-64f && a <= 0x1p64f)) continue;
    const int e = (int)((ab >> 7) & 0xFF) - 127;
    const float y = ldexpf(table[ab & 0x7F], -e);
    for (uint32_t wb = 0; wb < 0x7F80; ++wb) {
      const float wp = bf16(wb);
      if (wp > a) break; /* bf16 magnitudes increase with the bit pattern */
      for (int sgn = 0; sgn < 2; ++sgn) {
        const float w = sgn ? -wp : wp;
        volatile float q0 = w * y;
        volatile float r = fmaf(-q0, a, w);
        volatile float q = fmaf(r, y, q0);
        volatile float ref = w / a;
        ++pairs;
        if (q != ref) {
          ++differ;
          if (fabsf(ref) > max_abs_differ) max_abs_differ = fabsf(ref);
        }
        if (code_of(q) != code_of(ref)) {
          if (bad < 10)
            fprintf(stderr, "code mismatch a=%a w=%a fast=%a ieee=%a\n", (double)a, (double)w,
                    (double)q, (double)ref);
          ++bad;
        }
      }
    }
  }
  printf("pairs %llu quotient_differs %llu (max |w/a| among them %a) code_mismatches %llu\n", pairs,
         differ, (double)max_abs_differ, bad);
  return bad == 0 ? 0 : 1;
}
