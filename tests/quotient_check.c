/*
 * Checks, in IEEE binary32 with fused multiply-add, the quotient argument the
 * append kernel relies on (Markstein's correction step): with r = RN(1/s),
 *   q0 = RN(v r),  rem = RN(v - q0 s),  q1 = RN(q0 + rem r)
 * equals RN(v / s) for every bf16 significand of v and the float
 * significands of s given on the command line (both in [1, 2): powers of two
 * only shift every step while values stay normal).
 * Usage: quotient_check <first s significand> <count> <stride> [control]
 * Prints "n=<pairs> bad=<mismatches>"; with "control", q0 alone is compared
 * (it must differ somewhere, or the check would prove nothing).
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

int main(int argc, char** argv) {
  if (argc < 4) return 2;
  uint32_t first = (uint32_t)strtoul(argv[1], 0, 0);
  uint32_t count = (uint32_t)strtoul(argv[2], 0, 0);
  uint32_t stride = (uint32_t)strtoul(argv[3], 0, 0);
  int control = argc > 4;
  long n = 0, bad = 0;
  for (uint32_t c = 0; c < count; c++) {
    uint32_t m = (first + c * stride) & 0x7FFFFFu;
    volatile float s = u2f(0x3F800000u | m);
    volatile float r = 1.0f / s;
    for (uint32_t xm = 0; xm < 128; xm++) {
      volatile float v = u2f(0x3F800000u | (xm << 16));
      float want = v / s;
      float q0 = v * r;
      float rem = fmaf(-q0, s, v);
      float q1 = fmaf(rem, r, q0);
      n++;
      if (f2u(control ? q0 : q1) != f2u(want)) bad++;
    }
  }
  printf("n=%ld bad=%ld\n", n, bad);
  return 0;
}
