// fp8q oracle: a plain, slow, obviously correct CPU statement of the
// fine-grained FP8 path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check
// and the bench's CPU-baseline leg may call it; the product path never does.
//
// It shares no code, table or helper with the CUDA library.  Every function
// cites the passage it follows, as "page title, section/equation":
//   [P1] "Online Quantization During Training" (shivam2003.com)
//   [P2] "Fine-Grained FP8 Quantization in DeepSeek" (shivam2003.com)
//   [P3] "FP8 Mixed Precision: DeepSeek-V3 Training Architecture" (aifetchly)
//   [P4] "Making Low Precision Work" (sahipadhai.cc)
//   [P5] "Introduction to LLM Quantization" (medium)
// and, for the bit-level FP8 formats, the public OCP / Micikevicius et al.
// "FP8 Formats for Deep Learning" definition that [P1] and [P2] list among
// their primary sources.
//
// Readings of points the pages leave open (each restated where it is used):
//  * The cast written as clip(round(W/s), -448, 448) in [P3] eq. W_FP8 is read
//    as a round-to-nearest-even cast to E4M3 with saturation at +-448 (the
//    page names E4M3 as the format).  The integer-grid model the page's code
//    simulates is kept as a separate mode (orc_quant_tiles_intgrid) only to
//    reproduce that page's error comparison.
//  * q = e4m3(fl32(x / s)): IEEE float division, then the E4M3 rounding.
//  * s = max(fl32(amax / 448), fl32(1e-12)); the 1e-12 floor is the one the
//    [P3] "Step 1" listing applies.  s (the dequantisation multiplier) is stored.
//  * GEMM: D = sum over 128-wide K chunks of (sa*sb) * (sum of the chunk's FP8
//    products), evaluated in FP64, then rounded once to BF16 or FP32.
//
// Parity pins for every function live in tests/ (codec enumeration, library
// cross-checks, worked examples of the pages, closed forms, brute force).
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math -fPIC -shared -pthread.
// -ffp-contract=off keeps every float product and sum individually rounded.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Threading: split [0, n) over the host cores.  Used only for speed; every
// per-item computation is independent, so the result does not depend on it.
// ---------------------------------------------------------------------------
std::atomic<int> g_threads_used{1};

int host_threads() {
  unsigned h = std::thread::hardware_concurrency();
  return h == 0 ? 1 : static_cast<int>(h);
}

template <class F>
void parallel_for(int64_t n, F fn) {
  int nt = host_threads();
  if (n < 2 || nt < 2) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  if (nt > n) nt = static_cast<int>(n);
  int prev = g_threads_used.load();
  while (nt > prev && !g_threads_used.compare_exchange_weak(prev, nt)) {
  }
  std::atomic<int64_t> next{0};
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int t = 0; t < nt; ++t) {
    pool.emplace_back([&]() {
      for (;;) {
        int64_t i = next.fetch_add(1);
        if (i >= n) break;
        fn(i);
      }
    });
  }
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------------------
// BF16 <-> float.  A BF16 value is the upper half of an IEEE binary32.
// ---------------------------------------------------------------------------
float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round a double to the nearest value with `bits` significant bits
// (round-half-to-even), with the exponent range of binary32 / bfloat16
// (normal exponents -126..127, subnormal quantum 2^(-126 - (bits - 1))).
// Returns the rounded value as a double (exact).  Overflow -> +-inf.
double round_to_precision(double v, int bits) {
  if (v == 0.0 || !std::isfinite(v)) return v;
  double a = std::fabs(v);
  int e;
  std::frexp(a, &e);            // a = f * 2^e, f in [0.5, 1)
  int exp_unbiased = e - 1;     // a in [2^exp, 2^(exp+1))
  if (exp_unbiased < -126) exp_unbiased = -126;  // subnormal range: fixed quantum
  double quantum = std::ldexp(1.0, exp_unbiased - (bits - 1));
  double n = a / quantum;       // exact: quantum is a power of two
  double fl = std::floor(n);
  double frac = n - fl;
  double r;
  if (frac > 0.5) r = fl + 1.0;
  else if (frac < 0.5) r = fl;
  else r = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  double out = r * quantum;
  // binary32 and bfloat16 share the exponent range; largest finite value is
  // (2 - 2^(1-bits)) * 2^127.
  double maxfin = (2.0 - std::ldexp(1.0, 1 - bits)) * std::ldexp(1.0, 127);
  if (out > maxfin) out = INFINITY;
  return std::copysign(out, v);
}

// ---------------------------------------------------------------------------
// E4M3 (OCP "E4M3FN"): 1 sign, 4 exponent (bias 7), 3 mantissa bits.
// No infinities; S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448.
// [P3] "3. Why Naive FP8 Training Suffers Precision Collapse": E4M3 max ~448.
// ---------------------------------------------------------------------------
double e4m3_decode(uint8_t c) {
  int s = c >> 7;
  int e = (c >> 3) & 0xF;
  int m = c & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0) v = m * std::ldexp(1.0, -9);                 // subnormal m * 2^-9
  else v = (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);        // normal
  return s ? -v : v;
}

// Encode a float to E4M3, round-to-nearest-even, saturating to +-448
// ("satfinite").  The sign is kept on zero and on values that round to zero.
uint8_t e4m3_encode(float x) {
  if (std::isnan(x)) return 0x7F;
  uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double a = std::fabs(static_cast<double>(x));
  if (a >= 448.0) return sign | 0x7E;           // at or above max: saturate
  // quantum (spacing) of the E4M3 grid around a
  double quantum;
  if (a < std::ldexp(1.0, -6)) {
    quantum = std::ldexp(1.0, -9);              // subnormal binade
  } else {
    int e;
    std::frexp(a, &e);                          // a in [2^(e-1), 2^e)
    quantum = std::ldexp(1.0, (e - 1) - 3);     // 3 fraction bits
  }
  double n = a / quantum;                       // exact
  double fl = std::floor(n);
  double frac = n - fl;
  double r;
  if (frac > 0.5) r = fl + 1.0;
  else if (frac < 0.5) r = fl;
  else r = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  double v = r * quantum;                       // an exact E4M3 value, <= 448
  if (v > 448.0) v = 448.0;                     // cannot happen below 448, kept for clarity
  // value -> code
  uint8_t mag;
  if (v < std::ldexp(1.0, -6)) {
    mag = static_cast<uint8_t>(v / std::ldexp(1.0, -9));   // 0..7 (8 would be 2^-6)
  } else {
    int e;
    double f = std::frexp(v, &e);               // v = f * 2^e, f in [0.5,1)
    int E = e - 1;                              // v = (2f) * 2^E, 2f in [1,2)
    int m = static_cast<int>((2.0 * f - 1.0) * 8.0);
    mag = static_cast<uint8_t>(((E + 7) << 3) | m);
  }
  return sign | mag;
}

// ---------------------------------------------------------------------------
// E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa bits, IEEE-like
// (S.11111.00 = inf, S.11111.xx = NaN); largest finite 1.75 * 2^15 = 57344.
// [P3] same section and [P5] "E4M3 vs E5M2": wider range, 2-bit mantissa.
// Used by the oracle's format pins only; the method uses E4M3 everywhere.
// ---------------------------------------------------------------------------
double e5m2_decode(uint8_t c) {
  int s = c >> 7;
  int e = (c >> 2) & 0x1F;
  int m = c & 0x3;
  double v;
  if (e == 0x1F) v = (m == 0) ? INFINITY : NAN;
  else if (e == 0) v = m * std::ldexp(1.0, -16);
  else v = (1.0 + m / 4.0) * std::ldexp(1.0, e - 15);
  return s ? -v : v;
}

uint8_t e5m2_encode_sat(float x) {
  if (std::isnan(x)) return 0x7F;
  uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double a = std::fabs(static_cast<double>(x));
  if (a >= 57344.0) return sign | 0x7B;         // satfinite
  double quantum;
  if (a < std::ldexp(1.0, -14)) {
    quantum = std::ldexp(1.0, -16);
  } else {
    int e;
    std::frexp(a, &e);
    quantum = std::ldexp(1.0, (e - 1) - 2);
  }
  double n = a / quantum;
  double fl = std::floor(n);
  double frac = n - fl;
  double r;
  if (frac > 0.5) r = fl + 1.0;
  else if (frac < 0.5) r = fl;
  else r = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  double v = r * quantum;
  uint8_t mag;
  if (v < std::ldexp(1.0, -14)) {
    mag = static_cast<uint8_t>(v / std::ldexp(1.0, -16));
  } else {
    int e;
    double f = std::frexp(v, &e);
    int E = e - 1;
    int m = static_cast<int>((2.0 * f - 1.0) * 4.0);
    mag = static_cast<uint8_t>(((E + 15) << 2) | m);
  }
  return sign | mag;
}

}  // namespace

// ===========================================================================
// Exported C interface (ctypes).  All pointers are host memory owned by the
// caller; sizes are element counts; leading dimensions are in elements.
// ===========================================================================
extern "C" {

int orc_version(void) { return 1; }

// Most threads any call used since the last reset (for reporting).
int orc_threads_used(void) { return g_threads_used.load(); }
void orc_reset_threads_used(void) { g_threads_used.store(1); }
int orc_host_threads(void) { return host_threads(); }

// ---- codecs ---------------------------------------------------------------
uint8_t orc_e4m3_encode(float x) { return e4m3_encode(x); }
double orc_e4m3_decode(uint8_t c) { return e4m3_decode(c); }
uint8_t orc_e5m2_encode(float x) { return e5m2_encode_sat(x); }
double orc_e5m2_decode(uint8_t c) { return e5m2_decode(c); }

void orc_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
  int64_t chunk = 1 << 16;
  int64_t nchunks = (n + chunk - 1) / chunk;
  parallel_for(nchunks, [&](int64_t c) {
    int64_t lo = c * chunk, hi = std::min(n, lo + chunk);
    for (int64_t i = lo; i < hi; ++i) out[i] = e4m3_encode(x[i]);
  });
}

void orc_e5m2_encode_array(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e5m2_encode_sat(x[i]);
}

// Round doubles to BF16 / FP32 (single rounding, RNE).  Output as double.
void orc_round_bf16(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_to_precision(x[i], 8);
}
void orc_round_f32(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_to_precision(x[i], 24);
}

// ---- tile scale ------------------------------------------------------------
// [P3] "1. Fine-Grained Tile and Block-Wise Scaling", eq. s = max|block| / 448,
// with the 1e-12 floor of the [P3] "Step 1" listing.  Float (IEEE) division.
float orc_tile_scale(float amax) {
  float s = amax / 448.0f;
  const float floor_s = 1e-12f;
  return s < floor_s ? floor_s : s;
}

// ---- 1x128 activation tiles -----------------------------------------------
// [P2] "2. Activations use 1x128 tiles"; [P3] "Activation Tile Scaling (1x128)";
// [P5] "5) Online Quantization": per token, per 128 contiguous channels:
// amax, s = amax/448, q = e4m3(x / s).
// x: bf16 bits [M][ldx]; q: [M][ldq]; sf: [M][K/128] row-major (logical).
int orc_quant_act_1x128(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                        uint8_t* q, int64_t ldq, float* sf) {
  if (K % 128 != 0 || ldx < K || ldq < K || M < 0) return 1;
  const int64_t KB = K / 128;
  parallel_for(M, [&](int64_t m) {
    for (int64_t kb = 0; kb < KB; ++kb) {
      const uint16_t* t = x + m * ldx + kb * 128;
      float amax = 0.0f;
      for (int i = 0; i < 128; ++i) amax = std::max(amax, std::fabs(bf16_to_float(t[i])));
      float s = orc_tile_scale(amax);
      sf[m * KB + kb] = s;
      for (int i = 0; i < 128; ++i) {
        float v = bf16_to_float(t[i]) / s;
        q[m * ldq + kb * 128 + i] = e4m3_encode(v);
      }
    }
  });
  return 0;
}

// ---- 128x1 tiles along the token dimension, written transposed --------------
// The same online rule with tiles of 128 consecutive tokens of one channel.
// Wgrad needs x^T (d L/d z) ([P5] "3) Backward propagation"), so both operands
// are quantised along the token dimension and stored K(token)-major.
// x: bf16 [T][ldx]; qt: [C][ldqt] (qt[c][t]); sf: [T/128][C] row-major.
int orc_quant_act_128x1(const uint16_t* x, int64_t T, int64_t C, int64_t ldx,
                        uint8_t* qt, int64_t ldqt, float* sf) {
  if (T % 128 != 0 || ldx < C || ldqt < T || C < 0) return 1;
  const int64_t TB = T / 128;
  parallel_for(C, [&](int64_t c) {
    for (int64_t tb = 0; tb < TB; ++tb) {
      float amax = 0.0f;
      for (int i = 0; i < 128; ++i)
        amax = std::max(amax, std::fabs(bf16_to_float(x[(tb * 128 + i) * ldx + c])));
      float s = orc_tile_scale(amax);
      sf[tb * C + c] = s;
      for (int i = 0; i < 128; ++i) {
        float v = bf16_to_float(x[(tb * 128 + i) * ldx + c]) / s;
        qt[c * ldqt + tb * 128 + i] = e4m3_encode(v);
      }
    }
  });
  return 0;
}

// ---- 128x128 weight blocks ---------------------------------------------------
// [P2] "3. Weights use 128x128 blocks"; [P3] eq. s_W = max|W_block| / 448 and
// eq. W_FP8 (read as the E4M3 cast).  w: bf16 [N][ldw]; q: [N][ldq];
// sf: [N/128][K/128] row-major.
int orc_quant_w_128x128(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                        uint8_t* q, int64_t ldq, float* sf) {
  if (N % 128 != 0 || K % 128 != 0 || ldw < K || ldq < K) return 1;
  const int64_t NB = N / 128, KB = K / 128;
  parallel_for(NB * KB, [&](int64_t b) {
    int64_t nb = b / KB, kb = b % KB;
    float amax = 0.0f;
    for (int r = 0; r < 128; ++r)
      for (int c = 0; c < 128; ++c)
        amax = std::max(amax, std::fabs(bf16_to_float(w[(nb * 128 + r) * ldw + kb * 128 + c])));
    float s = orc_tile_scale(amax);
    sf[nb * KB + kb] = s;
    for (int r = 0; r < 128; ++r)
      for (int c = 0; c < 128; ++c) {
        int64_t n = nb * 128 + r, k = kb * 128 + c;
        q[n * ldq + k] = e4m3_encode(bf16_to_float(w[n * ldw + k]) / s);
      }
  });
  return 0;
}

// ---- power-of-two (UE8M0) scales: a throughput study beside the method ---------
// The pages fix the scale as s = amax/448 ([P3] eq. s_W), a full FP32 value.
// Block-scaled tensor-core MMAs take scales that are powers of two, stored as
// UE8M0 bytes (an 8-bit biased exponent: byte b stands for 2^(b - 127)).  The
// pages do not define such a scale; the reading taken here keeps the method's
// tiles (1x128 activations, 128x128 weight blocks) and rounds the method's
// scale UP to the next power of two, so no element saturates:
//   t  = max(fl32(amax / 448), fl32(1e-12))      (the method's scale)
//   s2 = 2^ceil(log2 t)                          (smallest power of two >= t)
//   q  = e4m3(fl32(x / s2))
// The GEMM over such operands is the block-scaled GEMM above with these scales.
float orc_pow2_scale(float t) {
  int e = 0;
  const float m = std::frexp(t, &e);      // t = m * 2^e, 0.5 <= m < 1
  return m == 0.5f ? t : std::ldexp(1.0f, e);
}

// UE8M0 byte of a power of two s = 2^p (p in [-127, 127]): p + 127.
int orc_ue8m0_encode(float s) {
  int e = 0;
  const float m = std::frexp(s, &e);      // s = 0.5 * 2^e
  if (m != 0.5f) return -1;               // not a power of two
  const int b = (e - 1) + 127;
  return (b < 0 || b > 254) ? -1 : b;
}

// 1x128 tiles with power-of-two scales.  x: bf16 [M][ldx]; q: [M][ldq];
// sf: [M][K/128] row-major (the scale values s2).
int orc_quant_act_1x128_pow2(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                             uint8_t* q, int64_t ldq, float* sf) {
  if (K % 128 != 0 || ldx < K || ldq < K || M < 0) return 1;
  const int64_t KB = K / 128;
  parallel_for(M, [&](int64_t m) {
    for (int64_t kb = 0; kb < KB; ++kb) {
      const uint16_t* t = x + m * ldx + kb * 128;
      float amax = 0.0f;
      for (int i = 0; i < 128; ++i) amax = std::max(amax, std::fabs(bf16_to_float(t[i])));
      const float s = orc_pow2_scale(orc_tile_scale(amax));
      sf[m * KB + kb] = s;
      for (int i = 0; i < 128; ++i) q[m * ldq + kb * 128 + i] = e4m3_encode(bf16_to_float(t[i]) / s);
    }
  });
  return 0;
}

// 128x128 weight blocks with power-of-two scales.  w: bf16 [N][ldw];
// q: [N][ldq]; sf: [N/128][K/128] row-major.
int orc_quant_w_128x128_pow2(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                             uint8_t* q, int64_t ldq, float* sf) {
  if (N % 128 != 0 || K % 128 != 0 || ldw < K || ldq < K) return 1;
  const int64_t NB = N / 128, KB = K / 128;
  parallel_for(NB * KB, [&](int64_t b) {
    const int64_t nb = b / KB, kb = b % KB;
    float amax = 0.0f;
    for (int r = 0; r < 128; ++r)
      for (int c = 0; c < 128; ++c)
        amax = std::max(amax, std::fabs(bf16_to_float(w[(nb * 128 + r) * ldw + kb * 128 + c])));
    const float s = orc_pow2_scale(orc_tile_scale(amax));
    sf[nb * KB + kb] = s;
    for (int r = 0; r < 128; ++r)
      for (int c = 0; c < 128; ++c) {
        const int64_t n = nb * 128 + r, k = kb * 128 + c;
        q[n * ldq + k] = e4m3_encode(bf16_to_float(w[n * ldw + k]) / s);
      }
  });
  return 0;
}

// ---- the [P3] listing's integer-grid simulation --------------------------------
// [P3] "Step 1": q = clip(round(x/s), -448, 448) with numpy's round-half-even,
// s = max(amax/448, 1e-12), here in double like the listing.  Groups are
// `count` runs of `len` values with stride 1 (rows of tiles).  Output is the
// dequantised value q*s.  Only used to reproduce the page's comparison.
void orc_quant_tiles_intgrid(const double* x, int64_t count, int64_t len, double* deq) {
  for (int64_t g = 0; g < count; ++g) {
    const double* t = x + g * len;
    double amax = 0.0;
    for (int64_t i = 0; i < len; ++i) amax = std::max(amax, std::fabs(t[i]));
    double s = std::max(amax / 448.0, 1e-12);
    for (int64_t i = 0; i < len; ++i) {
      double v = t[i] / s;
      double fl = std::floor(v), frac = v - fl, r;
      if (frac > 0.5) r = fl + 1.0;
      else if (frac < 0.5) r = fl;
      else r = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
      r = std::min(448.0, std::max(-448.0, r));
      deq[g * len + i] = r * s;
    }
  }
}

// ---- symmetric absmax INT8 --------------------------------------------------
// [P5] "INT8": divide every value by the largest magnitude alpha and multiply
// by 127; round half to even; clamp to [-127, 127].  scale_out = alpha / 127.
void orc_int8_absmax(const double* x, int64_t n, int8_t* q, double* scale_out) {
  double alpha = 0.0;
  for (int64_t i = 0; i < n; ++i) alpha = std::max(alpha, std::fabs(x[i]));
  *scale_out = alpha / 127.0;
  for (int64_t i = 0; i < n; ++i) {
    double v = alpha > 0.0 ? x[i] / alpha * 127.0 : 0.0;
    double fl = std::floor(v), frac = v - fl, r;
    if (frac > 0.5) r = fl + 1.0;
    else if (frac < 0.5) r = fl;
    else r = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    r = std::min(127.0, std::max(-127.0, r));
    q[i] = static_cast<int8_t>(r);
  }
}

// ---- block-scaled GEMM over the dequantised operands --------------------------
// [P3] "3. Decoupled Accumulation in Tensor Core GEMMs", eq. C_ij, read per
// 128-wide K chunk; [P5] "Fine-grained Quantization" Steps 1-4 (multiply the
// FP8 blocks, then rescale by the blocks' factors) and "3) Backward
// propagation" (Dgrad / Wgrad).  For every requested (m, n):
//     D[m,n] = sum_kb (sa[m,kb] * sb(n,kb)) * (sum_{k in chunk kb} qa[m,k] * qb[n,k])
// in FP64.  The chunk sum is exact in FP64: E4M3 values are multiples of 2^-9
// below 2^9, so each product is a multiple of 2^-18 below 2^18 and 128 of them
// stay below 2^25 (a 43-bit span).  sa*sb (two 24-bit significands) is exact
// too, so each chunk contributes its true value with one rounding.
// This equals P3's "Step 2" X_fine @ W_fine.T on the dequantised operands.
//
// a: [M][lda] E4M3 codes (K-major); sfa: [M][K/128] row-major.
// b: [N][ldb] E4M3 codes (K-major).
// sfb_mode 0: sfb [N/128][K/128] row-major (128x128 weight blocks).
// sfb_mode 1: sfb [N][K/128] row-major (per-row 1x128 / 128x1 tiles).
// rows[nr], cols[nc]: the outputs wanted; out: [nr][nc] FP64.
int orc_gemm_sampled_fmt(const uint8_t* a, int64_t lda, const float* sfa,
                         const uint8_t* b, int64_t ldb, const float* sfb, int sfb_mode,
                         int64_t M, int64_t N, int64_t K,
                         const int64_t* rows, int64_t nr, const int64_t* cols, int64_t nc,
                         int a_fmt, int b_fmt, double* out) {
  if (K % 128 != 0 || (sfb_mode == 0 && N % 128 != 0)) return 1;
  if (sfb_mode != 0 && sfb_mode != 1) return 1;
  if (a_fmt < 0 || a_fmt > 1 || b_fmt < 0 || b_fmt > 1) return 1;
  const int64_t KB = K / 128;
  // operand codes -> values: format 0 E4M3, format 1 E5M2
  double lut_a[256], lut_b[256];
  for (int c = 0; c < 256; ++c) {
    lut_a[c] = a_fmt == 0 ? e4m3_decode(static_cast<uint8_t>(c)) : e5m2_decode(static_cast<uint8_t>(c));
    lut_b[c] = b_fmt == 0 ? e4m3_decode(static_cast<uint8_t>(c)) : e5m2_decode(static_cast<uint8_t>(c));
  }
  for (int64_t i = 0; i < nr; ++i) if (rows[i] < 0 || rows[i] >= M) return 2;
  for (int64_t j = 0; j < nc; ++j) if (cols[j] < 0 || cols[j] >= N) return 2;
  parallel_for(nr, [&](int64_t i) {
    const int64_t m = rows[i];
    std::vector<double> arow(K);
    for (int64_t k = 0; k < K; ++k) arow[k] = lut_a[a[m * lda + k]];
    for (int64_t j = 0; j < nc; ++j) {
      const int64_t n = cols[j];
      const uint8_t* brow = b + n * ldb;
      double acc = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        double chunk = 0.0;
        for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) chunk += arow[k] * lut_b[brow[k]];
        double sa = sfa[m * KB + kb];
        double sb = (sfb_mode == 0) ? sfb[(n / 128) * KB + kb] : sfb[n * KB + kb];
        acc += (sa * sb) * chunk;
      }
      out[i * nc + j] = acc;
    }
  });
  return 0;
}

// Both operands E4M3 (the method's format).
int orc_gemm_sampled(const uint8_t* a, int64_t lda, const float* sfa,
                     const uint8_t* b, int64_t ldb, const float* sfb, int sfb_mode,
                     int64_t M, int64_t N, int64_t K,
                     const int64_t* rows, int64_t nr, const int64_t* cols, int64_t nc,
                     double* out) {
  return orc_gemm_sampled_fmt(a, lda, sfa, b, ldb, sfb, sfb_mode, M, N, K, rows, nr, cols, nc, 0, 0, out);
}

// ---- grouped (MoE) GEMM ---------------------------------------------------------
// One block-scaled GEMM per expert g over its packed rows
// [offsets[g], offsets[g+1]) with that expert's weight w[g] and block scales.
// The per-expert semantics are those of orc_gemm_sampled (sfb_mode 0).
// a: [M_total][lda]; sfa: [M_total][K/128]; w: [G][N][K]; sfw: [G][N/128][K/128];
// offsets: [G+1] nondecreasing, offsets[0] = 0, offsets[G] = M_total.
int orc_grouped_gemm_sampled(const uint8_t* a, int64_t lda, const float* sfa,
                             const uint8_t* w, const float* sfw,
                             const int64_t* offsets, int64_t G, int64_t N, int64_t K,
                             const int64_t* rows, int64_t nr, const int64_t* cols, int64_t nc,
                             double* out) {
  if (K % 128 != 0 || N % 128 != 0 || G < 1 || offsets[0] != 0) return 1;
  for (int64_t g = 0; g < G; ++g) if (offsets[g + 1] < offsets[g]) return 1;
  const int64_t M_total = offsets[G];
  const int64_t KB = K / 128, NB = N / 128;
  for (int64_t i = 0; i < nr; ++i) if (rows[i] < 0 || rows[i] >= M_total) return 2;
  for (int64_t j = 0; j < nc; ++j) if (cols[j] < 0 || cols[j] >= N) return 2;
  double lut[256];
  for (int c = 0; c < 256; ++c) lut[c] = e4m3_decode(static_cast<uint8_t>(c));
  parallel_for(nr, [&](int64_t i) {
    const int64_t m = rows[i];
    int64_t g = 0;
    while (!(offsets[g] <= m && m < offsets[g + 1])) ++g;  // expert owning row m
    const uint8_t* wg = w + g * N * K;
    const float* sg = sfw + g * NB * KB;
    for (int64_t j = 0; j < nc; ++j) {
      const int64_t n = cols[j];
      double acc = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        double chunk = 0.0;
        for (int64_t k = kb * 128; k < kb * 128 + 128; ++k)
          chunk += lut[a[m * lda + k]] * lut[wg[n * K + k]];
        acc += (static_cast<double>(sfa[m * KB + kb]) * sg[(n / 128) * KB + kb]) * chunk;
      }
      out[i * nc + j] = acc;
    }
  });
  return 0;
}

// ---- per-tensor FP8 baseline ---------------------------------------------------
// [P3] "Step 2": the per-tensor baseline: one scale amax/448 for the whole
// tensor, then the same E4M3 cast.  Output: dequantised values (double).
void orc_quant_pertensor_e4m3(const uint16_t* x, int64_t n, double* deq, float* scale_out) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(bf16_to_float(x[i])));
  float s = orc_tile_scale(amax);
  *scale_out = s;
  for (int64_t i = 0; i < n; ++i) deq[i] = e4m3_decode(e4m3_encode(bf16_to_float(x[i]) / s)) * s;
}

// The same per-tensor rule on a BF16 matrix x [M][ldx], returning the codes:
// amax over all M x K values, s = max(fl32(amax / 448), fl32(1e-12)),
// q = e4m3(fl32(x / s)).  *amax_out and *scale_out receive amax and s.
int orc_quant_pertensor(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                        float* amax_out, float* scale_out) {
  if (K % 8 != 0 || ldx < K || ldq < K || M < 0) return 1;
  float amax = 0.0f;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) amax = std::max(amax, std::fabs(bf16_to_float(x[m * ldx + k])));
  const float s = orc_tile_scale(amax);
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) q[m * ldq + k] = e4m3_encode(bf16_to_float(x[m * ldx + k]) / s);
  *amax_out = amax;
  *scale_out = s;
  return 0;
}

// ---- scale policies: quantizing with given scales, and history updates -------
// [P1] "4. Max scaling is robust but noisy": percentile clipping, delayed
// scaling or amax histories trade clipping against stability, and any smoother
// lags; [P1] "Worked example": fixed calibration, current-max and an
// exponential amax history compared on clipping rate and mean error; [P5]
// "5) Online Quantization", "Delayed Quantization (Previous Method)": the scale
// of the current tensor comes from past maxima, so a range change overflows.
//
// Readings: a policy supplies one scale per 1x128 tile; the tile is cast as the
// online rule casts it, q = e4m3(fl32(x / s)) with IEEE division, and an
// element is "clipped" when the cast saturates it: |fl32(x / s)| > 464, the
// point above which round-to-nearest-even would leave 448, the E4M3 maximum
// (448 < v <= 464 rounds to 448 by itself).
// x: bf16 [M][ldx]; sf: [M][K/128] given scales; q: [M][ldq];
// amax: [M][K/128] the tiles' current maxima (for the history update; may be
// NULL); *clipped += the number of clipped elements (may be NULL).
int orc_quant_act_1x128_scaled(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const float* sf,
                               uint8_t* q, int64_t ldq, float* amax, int64_t* clipped) {
  if (K % 128 != 0 || ldx < K || ldq < K || M < 0) return 1;
  const int64_t KB = K / 128;
  int64_t total = 0;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t kb = 0; kb < KB; ++kb) {
      const uint16_t* t = x + m * ldx + kb * 128;
      const float s = sf[m * KB + kb];
      float mx = 0.0f;
      for (int i = 0; i < 128; ++i) {
        const float xv = bf16_to_float(t[i]);
        mx = std::max(mx, std::fabs(xv));
        const float v = xv / s;
        if (std::fabs(v) > 464.0f) ++total;
        q[m * ldq + kb * 128 + i] = e4m3_encode(v);
      }
      if (amax != nullptr) amax[m * KB + kb] = mx;
    }
  }
  if (clipped != nullptr) *clipped += total;
  return 0;
}

// One step of a tile-scale history ([P1] section 4 and worked example), for n
// tiles: the state h is updated from the step's tile maxima a, and the next
// step's scale is s = max(fl32(h / 448), fl32(1e-12)), the online rule applied
// to the history instead of the current tile.
//   policy 0, previous step (delayed):   h = a
//   policy 1, exponential history:       h = fl32(fl32(alpha * h) + fl32(fl32(1 - alpha) * a))
//   policy 2, decaying maximum:          h = max(a, fl32(alpha * h))
// Every product and sum is rounded to FP32 on its own (the build disables
// contraction), which fixes the result bit for bit.
int orc_scale_history_update(int policy, float alpha, const float* a, float* h, float* sf, int64_t n) {
  if (policy < 0 || policy > 2 || n < 0) return 1;
  const float beta = 1.0f - alpha;
  for (int64_t i = 0; i < n; ++i) {
    float nh;
    if (policy == 0) {
      nh = a[i];
    } else if (policy == 1) {
      const float p = alpha * h[i];
      const float r = beta * a[i];
      nh = p + r;
    } else {
      const float d = alpha * h[i];
      nh = std::max(a[i], d);
    }
    h[i] = nh;
    sf[i] = orc_tile_scale(nh);
  }
  return 0;
}

// ---- E5M2 gradient variant ------------------------------------------------------
// [P3] "2. Universal E4M3" and [P5] "E4M3 vs E5M2": conventional FP8 recipes
// store gradients in E5M2 (wider range, 2 mantissa bits), which DeepSeek drops
// for E4M3 everywhere.  Reading: the same online tile rule with the E5M2
// maximum in place of 448: s = max(fl32(amax / 57344), fl32(1e-12)),
// q = e5m2(fl32(x / s)), round-to-nearest-even, saturating at +-57344.
static float tile_scale_e5m2(float amax) {
  const float s = amax / 57344.0f;
  const float floor_s = 1e-12f;
  return s < floor_s ? floor_s : s;
}

float orc_tile_scale_e5m2(float amax) { return tile_scale_e5m2(amax); }

// 1x128 tiles (as orc_quant_act_1x128): x [M][ldx] -> q [M][ldq], sf [M][K/128].
int orc_quant_act_1x128_e5m2(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                             float* sf) {
  if (K % 128 != 0 || ldx < K || ldq < K || M < 0) return 1;
  const int64_t KB = K / 128;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t kb = 0; kb < KB; ++kb) {
      const uint16_t* t = x + m * ldx + kb * 128;
      float amax = 0.0f;
      for (int i = 0; i < 128; ++i) amax = std::max(amax, std::fabs(bf16_to_float(t[i])));
      const float s = tile_scale_e5m2(amax);
      sf[m * KB + kb] = s;
      for (int i = 0; i < 128; ++i) q[m * ldq + kb * 128 + i] = e5m2_encode_sat(bf16_to_float(t[i]) / s);
    }
  }
  return 0;
}

// 128x1 tiles along tokens, transposed (as orc_quant_act_128x1):
// x [T][ldx] -> qt [C][ldqt], sf [T/128][C].
int orc_quant_act_128x1_e5m2(const uint16_t* x, int64_t T, int64_t C, int64_t ldx, uint8_t* qt, int64_t ldqt,
                             float* sf) {
  if (T % 128 != 0 || ldx < C || ldqt < T || C < 0) return 1;
  for (int64_t tb = 0; tb < T / 128; ++tb) {
    for (int64_t c = 0; c < C; ++c) {
      float amax = 0.0f;
      for (int i = 0; i < 128; ++i) amax = std::max(amax, std::fabs(bf16_to_float(x[(tb * 128 + i) * ldx + c])));
      const float s = tile_scale_e5m2(amax);
      sf[tb * C + c] = s;
      for (int i = 0; i < 128; ++i)
        qt[c * ldqt + tb * 128 + i] = e5m2_encode_sat(bf16_to_float(x[(tb * 128 + i) * ldx + c]) / s);
    }
  }
  return 0;
}

// Percentile clipping ([P1] "4. Max scaling is robust but noisy" names it
// beside delayed scaling and amax histories): the tile's scale comes from an
// upper percentile of its magnitudes instead of their maximum, so the few
// values above it saturate.  Reading: the p-th percentile of the tile's 128
// magnitudes by the nearest-rank rule, i.e. the r-th largest magnitude with
// r = 128 - ceil(p * 128) + 1; the call takes r (1 <= r <= 128) and r = 1 is
// the online rule.  s = max(fl32(v / 448), fl32(1e-12)) with v that magnitude;
// the cast, the IEEE division and the clip rule are those of the given-scale
// quantizer above.
// x: bf16 [M][ldx]; q: [M][ldq]; sf: [M][K/128]; *clipped += clipped count.
int orc_quant_act_1x128_percentile(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int rank,
                                   uint8_t* q, int64_t ldq, float* sf, int64_t* clipped) {
  if (K % 128 != 0 || ldx < K || ldq < K || M < 0 || rank < 1 || rank > 128) return 1;
  const int64_t KB = K / 128;
  int64_t total = 0;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t kb = 0; kb < KB; ++kb) {
      const uint16_t* t = x + m * ldx + kb * 128;
      float mags[128];
      for (int i = 0; i < 128; ++i) mags[i] = std::fabs(bf16_to_float(t[i]));
      std::sort(mags, mags + 128, [](float a, float b) { return a > b; });   // descending
      const float s = orc_tile_scale(mags[rank - 1]);
      sf[m * KB + kb] = s;
      for (int i = 0; i < 128; ++i) {
        const float v = bf16_to_float(t[i]) / s;
        if (std::fabs(v) > 464.0f) ++total;
        q[m * ldq + kb * 128 + i] = e4m3_encode(v);
      }
    }
  }
  if (clipped != nullptr) *clipped += total;
  return 0;
}

}  // extern "C"
