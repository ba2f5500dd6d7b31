/*
 * Exhaustive check of the quantizers' division-free E4M3 cast (test harness,
 * not part of the library or of the oracle).
 *
 * Claim checked: for every BF16 value x and every BF16 tile maximum
 * amax >= |x| (amax = 0 and both signed zeros included), with
 *   s  = max(fl32(amax / 448), fl32(1e-12))      (the tile scale)
 *   nr = -fl32(1 / s)
 *   n  = fl32(x * nr),  e = fma(n, s, x),  t = fma(e, nr, n)
 * the E4M3 code of -t equals the E4M3 code of fl32(x / s), the quotient the
 * pages' scaling rule defines ("Fine-Grained FP8 Quantization in DeepSeek",
 * section 2: scale = tile max / 448, value / scale cast to E4M3).  The FMA
 * correction step is Markstein's (IBM J. Res. Develop. 34(1), 1990).
 *
 * The same walk is run for the E5M2 gradient variant, with 57344 (the E5M2
 * maximum) in place of 448 and the E5M2 code in place of the E4M3 one.
 *
 * The encoders here are independent of the library; the Python side checks
 * them against the oracle's encoders before trusting the counts.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float bf16_value(uint32_t bits) {
  uint32_t u = bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* E4M3 (bias 7, max 448, no infinities): round to nearest even, saturate. */
int cfc_e4m3(float v) {
  const int sign = signbit(v) ? 0x80 : 0;
  const double a = fabs((double)v);
  int code;
  if (a < 0.015625) {                 /* below 2^-6: subnormal grid 2^-9 */
    code = (int)nearbyint(a * 512.0);
  } else {
    int e;
    frexp(a, &e);
    e -= 1;                           /* a in [2^e, 2^(e+1)) */
    const double n = nearbyint(a / ldexp(1.0, e - 3));
    code = ((e + 7) << 3) + (int)n - 8;
  }
  if (code > 0x7E) code = 0x7E;
  return sign | code;
}

void cfc_encode(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)cfc_e4m3(v[i]);
}

/*
 * Walk every pair; return the number of pairs (through *pairs) and the number
 * of mismatches of the corrected formula (return value).  plain_mismatches
 * receives the count for the uncorrected product fl32(x * fl32(1/s)), which
 * must be non-zero: it shows that the walk can see a difference at all.
 */
long long cfc_check(long long* pairs, long long* plain_mismatches) {
  long long bad = 0, bad_plain = 0, tot = 0;
  const float tiny = 1e-12f;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad, bad_plain, tot)
  for (int ab = 0; ab < 0x7F80; ++ab) {
    const float amax = bf16_value((uint32_t)ab);
    volatile float t0 = amax / 448.0f;
    const float s = t0 > tiny ? t0 : tiny;
    volatile float r0 = 1.0f / s;
    const float r = r0;
    const float nr = -r;
    for (uint32_t k = 0; k <= 2u * (uint32_t)ab + 1u; ++k) {
      const uint32_t xb = (k >> 1) | ((k & 1u) ? 0x8000u : 0u);
      const float x = bf16_value(xb);
      volatile float quot = x / s;
      const int ref = cfc_e4m3(quot);
      volatile float n = x * nr;
      volatile float e = fmaf(n, s, x);
      volatile float t = fmaf(e, nr, n);
      const int got = cfc_e4m3(t) ^ 0x80;
      volatile float plain = x * r;
      tot++;
      if (got != ref) bad++;
      if (cfc_e4m3(plain) != ref) bad_plain++;
    }
  }
  *pairs = tot;
  *plain_mismatches = bad_plain;
  return bad;
}

/* E5M2 (bias 15, max 57344): round to nearest even, saturate finite. */
int cfc_e5m2(float v) {
  const int sign = signbit(v) ? 0x80 : 0;
  const double a = fabs((double)v);
  int code;
  if (a < ldexp(1.0, -14)) {          /* subnormal grid 2^-16 */
    code = (int)nearbyint(a * 65536.0);
  } else {
    int e;
    frexp(a, &e);
    e -= 1;
    const double n = nearbyint(a / ldexp(1.0, e - 2));
    code = ((e + 15) << 2) + (int)n - 4;
  }
  if (code > 0x7B) code = 0x7B;
  return sign | code;
}

void cfc_encode_e5m2(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)cfc_e5m2(v[i]);
}

long long cfc_check_e5m2(long long* pairs, long long* plain_mismatches) {
  long long bad = 0, bad_plain = 0, tot = 0;
  const float tiny = 1e-12f;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad, bad_plain, tot)
  for (int ab = 0; ab < 0x7F80; ++ab) {
    const float amax = bf16_value((uint32_t)ab);
    volatile float t0 = amax / 57344.0f;
    const float s = t0 > tiny ? t0 : tiny;
    volatile float r0 = 1.0f / s;
    const float r = r0;
    const float nr = -r;
    for (uint32_t k = 0; k <= 2u * (uint32_t)ab + 1u; ++k) {
      const uint32_t xb = (k >> 1) | ((k & 1u) ? 0x8000u : 0u);
      const float x = bf16_value(xb);
      volatile float quot = x / s;
      const int ref = cfc_e5m2(quot);
      volatile float n = x * nr;
      volatile float e = fmaf(n, s, x);
      volatile float t = fmaf(e, nr, n);
      const int got = cfc_e5m2(t) ^ 0x80;
      volatile float plain = x * r;
      tot++;
      if (got != ref) bad++;
      if (cfc_e5m2(plain) != ref) bad_plain++;
    }
  }
  *pairs = tot;
  *plain_mismatches = bad_plain;
  return bad;
}
