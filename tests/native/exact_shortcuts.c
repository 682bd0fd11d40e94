/* Exhaustive checks of two exact shortcuts the quantize kernels take instead of IEEE fp32
 * divisions (test code only; it shares nothing with the oracle or the kernels):
 *
 *   div6:  fl(x / 6) == q1 for x with a clear sign bit, where q0 = fl(x * fl(1/6)),
 *          rem = fma(-q0, 6, x), q1 = fma(rem, fl(1/6), q0), for +0 and every finite x >= 2^-125; infinity
 *          and NaN keep q0. Checked over all 2^31 such fp32 bit patterns.
 *   rtab:  g / value(c) == fl(g / k) * 2^(10 - max(e, 1)) (clamped to FLT_MAX) for every
 *          finite E4M3 code c = (e, m) with k = e ? 8 + m : m, and every g that the per-row
 *          global scale 2688 / amax yields from a bf16 or fp16 maximum (all 2^16 patterns).
 *
 * Built with -ffp-contract=off so every operation is one IEEE rounding; fmaf is the C99
 * fused multiply-add. Exit status 0 when every case agrees. */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static int same(float a, float b) { return (isnan(a) && isnan(b)) || bits(a) == bits(b); }

static float div6_shortcut(float x) {
  if (x > 0.0f && x < 0x1p-125f) return x / 6.0f;
  const float c = 0x1.555556p-3f;
  const float q0 = x * c;
  const float rem = fmaf(-q0, 6.0f, x);
  const float q1 = fmaf(rem, c, q0);
  return (rem == rem) ? q1 : q0;
}

static float e4m3_value(uint32_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  return e ? ldexpf(1.0f + m / 8.0f, e - 7) : ldexpf(m / 8.0f, -6);
}

static float f16_value(uint32_t h) {
  const int e = (h >> 10) & 31, m = h & 1023;
  float v = e == 31 ? (m ? NAN : INFINITY) : e ? ldexpf(1.0f + m / 1024.0f, e - 15) : ldexpf(m / 1024.0f, -14);
  return (h & 0x8000) ? -v : v;
}

static float row_scale(float amax) { return amax == 0.0f ? 1.0f : fminf(2688.0f / amax, FLT_MAX); }

int main(int argc, char **argv) {
  unsigned long long bad = 0, n = 0;
  const int skip_div6 = argc > 1 && strcmp(argv[1], "--rtab-only") == 0;
  if (!skip_div6) {
    for (uint64_t u = 0; u <= 0xFFFFFFFFull; ++u) {
      const float x = from_bits((uint32_t)u);
      if (u >> 31) continue; /* block maxima are magnitudes: the sign bit is clear */
      ++n;
      if (!same(x / 6.0f, div6_shortcut(x))) {
        if (bad < 5) printf("div6 mismatch at %08x\n", (uint32_t)u);
        ++bad;
      }
    }
  }
  for (int dt = 0; dt < 2; ++dt) {
    for (uint32_t h = 0; h < 0x10000; ++h) {
      const float amax = fabsf(dt == 0 ? from_bits(h << 16) : f16_value(h));
      const float g = row_scale(amax);
      float tab[16];
      tab[0] = 0.0f;
      for (int k = 1; k < 16; ++k) tab[k] = g / (float)k;
      for (uint32_t c = 0; c < 127; ++c) {
        const float sd = e4m3_value(c);
        const float direct = sd == 0.0f ? 0.0f : fminf(g / sd, FLT_MAX);
        const uint32_t e = c >> 3, m = c & 7;
        const float p2 = from_bits((137u - (e ? e : 1u)) << 23);
        const float via = fminf(tab[e ? (8 | m) : m] * p2, FLT_MAX);
        ++n;
        if (!same(direct, via)) {
          if (bad < 10) printf("rtab mismatch dtype %d amax bits %04x code %02x\n", dt, h, c);
          ++bad;
        }
      }
    }
  }
  printf("checked %llu cases, %llu mismatches\n", n, bad);
  return bad != 0;
}
