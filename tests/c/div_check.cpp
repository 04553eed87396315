// Host check of the quantizers' division (csrc/quant_div.h) against IEEE
// fp32 division, bit for bit, over the inputs the pre-pass can give it:
//   int8 quantizers: delta = RN(absmax / 127), x in [-absmax, absmax];
//   E4M3 quantizer:  delta = RN(colmax / V_r) for V_r in {448, 9}, colmax a
//                    finite fp16 magnitude, x an fp16 value with |x| <= colmax.
// Divisors include every positive finite fp16 absmax, fp32 absmax values
// whose delta has an all-ones significand, powers of two and random fp32
// values.  Prints "ok <count>" or the first mismatches and exits non-zero.
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "quant_div.h"

static float bits_f(uint32_t b) {
  float f;
  memcpy(&f, &b, 4);
  return f;
}
static uint32_t f_bits(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  return b;
}
static float half_to_float(uint16_t h) {  // exact widening of an fp16 code
  const uint32_t s = (h >> 15) & 1u, e = (h >> 10) & 31u, m = h & 1023u;
  float v;
  if (e == 0)
    v = ldexpf(static_cast<float>(m), -24);
  else
    v = ldexpf(static_cast<float>(m | 1024u), static_cast<int>(e) - 25);
  return s ? -v : v;
}

static uint64_t g_checked = 0, g_bad = 0;
static uint32_t g_rng = 12345u;
static uint32_t rnd() {
  g_rng = g_rng * 1664525u + 1013904223u;
  return g_rng;
}

// checks one (x, d) pair with both helpers
static void check(float x, float d) {
  const float r = 1.0f / d;  // RN(1/d), as __frcp_rn on the device
  const float want = x / d;  // IEEE fp32 division
  const float got = sage::div_rn_by(x, d, r);
  const float got2 = sage::div_rn_nosign(x, d, r);
  ++g_checked;
  if (f_bits(got) != f_bits(want) || !(got2 == want)) {
    if (g_bad < 10)
      printf("mismatch x=%a d=%a want=%a div_rn_by=%a div_rn_nosign=%a\n", x, d, want, got, got2);
    ++g_bad;
  }
}

// every finite fp16 x within [-lim, lim], plus `extra` random fp32 x in it
static void sweep_x(float d, float lim, int extra) {
  for (uint32_t h = 0; h < 65536u; ++h) {
    if (((h >> 10) & 31u) == 31u) continue;  // inf / nan
    const float x = half_to_float(static_cast<uint16_t>(h));
    if (fabsf(x) <= lim) check(x, d);
  }
  for (int i = 0; i < extra; ++i) {
    const float u = static_cast<float>(rnd() >> 8) * 0x1p-24f;  // [0, 1)
    const float x = (rnd() & 1u ? -1.0f : 1.0f) * u * lim;
    check(x, d);
  }
  check(lim, d);
  check(-lim, d);
}

int main() {
  // int8 quantizers: absmax = every positive finite fp16 magnitude (sampled
  // x), and a few hundred with every fp16 x
  for (uint32_t h = 1; h < 0x7C00u; ++h) {
    const float amax = half_to_float(static_cast<uint16_t>(h));
    const float d = amax / 127.0f;
    if ((h % 97u) == 0) {
      sweep_x(d, amax, 2000);
    } else {
      for (int i = 0; i < 24; ++i) {
        const float u = static_cast<float>(rnd() >> 8) * 0x1p-24f;
        check((rnd() & 1u ? -1.0f : 1.0f) * u * amax, d);
      }
      check(amax, d);
      check(-amax, d);
    }
  }
  // divisors with an all-ones significand and powers of two, at many scales
  for (int e = -40; e <= 8; ++e) {
    const float ones = ldexpf(bits_f(0x3FFFFFFFu), e);  // 1.11...1 (binary) * 2^e
    const float pow2 = ldexpf(1.0f, e);
    sweep_x(ones, 127.0f * ones, 20000);
    sweep_x(pow2, 127.0f * pow2, 2000);
  }
  // random fp32 divisors (the smoothed K block maxima are fp32)
  for (int i = 0; i < 4000; ++i) {
    const float d = ldexpf(1.0f + static_cast<float>(rnd() >> 9) * 0x1p-23f, static_cast<int>(rnd() % 60u) - 40);
    sweep_x(d, 127.0f * d, 200);
  }
  // E4M3 quantizer: delta_v = colmax / V_r
  const float vrs[2] = {448.0f, 9.0f};
  for (int k = 0; k < 2; ++k) {
    for (uint32_t h = 1; h < 0x7C00u; ++h) {
      const float cm = half_to_float(static_cast<uint16_t>(h));
      const float d = cm / vrs[k];
      if ((h % 61u) == 0) {
        sweep_x(d, cm, 0);
      } else {
        for (int i = 0; i < 16; ++i) {
          const uint16_t xh = static_cast<uint16_t>(rnd() % (h + 1));  // |x| <= colmax
          const float x = half_to_float(xh);
          check(rnd() & 1u ? -x : x, d);
        }
        check(cm, d);
        check(-cm, d);
      }
    }
  }
  if (g_bad) {
    printf("FAIL %llu of %llu\n", static_cast<unsigned long long>(g_bad),
           static_cast<unsigned long long>(g_checked));
    return 1;
  }
  printf("ok %llu\n", static_cast<unsigned long long>(g_checked));
  return 0;
}
