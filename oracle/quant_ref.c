/*
 * Oracle for the per-token INT8 KV quantiser — TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load
 * this file's library. It shares no code with the CUDA path.
 *
 * What it computes: Eq. 3 of "KV-Cache Optimization Techniques", section
 * "KV-Cache Quantization": code = round((x - z) / s) with x ~= s * code + z,
 * calibrated per token (one scale/zero per row of K or V).  The section names
 * s and z but does not define them; this oracle takes the plain asymmetric
 * min/max reading for an 8-bit unsigned code:
 *     z = min over the row, s = (max - min) / 255,
 *     code = clamp(round_half_even((x - z) / s), 0, 255),
 * with every step in IEEE fp32, round-to-nearest-even, in exactly this order,
 * and a row whose max equals its min stored as s = 0, z = min, codes 0.
 * Signed zero is left open by the pages; -0 and +0 are the same number, so
 * each input is read as x + 0.0f (which turns -0 into +0 and changes nothing
 * else) and the stored (s, z) have a single bit pattern.
 * Build with -ffp-contract=off and no fast-math so the compiler keeps the
 * subtraction and the division as two rounded fp32 operations.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f + 0.0f; /* -0 -> +0 */
}

/* x: [n_rows][d] bf16 bits.  codes: [n_rows][d].  sz: [n_rows][2] (s, z). */
void oracle_quantize_rows(const uint16_t *x, int64_t n_rows, int d,
                          uint8_t *codes, float *sz) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    const uint16_t *row = x + r * d;
    float mn = bf16_bits_to_f32(row[0]);
    float mx = mn;
    for (int j = 1; j < d; ++j) {
      const float v = bf16_bits_to_f32(row[j]);
      if (v < mn) mn = v;
      if (v > mx) mx = v;
    }
    const float range = mx - mn;
    const float s = range / 255.0f;
    const float z = mn;
    for (int j = 0; j < d; ++j) {
      uint8_t c = 0;
      if (s != 0.0f) {
        const float v = bf16_bits_to_f32(row[j]);
        const float diff = v - z;
        const float ratio = diff / s;
        float rq = nearbyintf(ratio); /* default rounding mode: half to even */
        if (rq < 0.0f) rq = 0.0f;
        if (rq > 255.0f) rq = 255.0f;
        c = (uint8_t)rq;
      }
      codes[r * d + j] = c;
    }
    sz[2 * r + 0] = s;
    sz[2 * r + 1] = z;
  }
}

/*
 * FP8 per-token KV quantiser. The pages recommend FP8 KV caches ("Understanding
 * KV-Cache Optimization in Modern LLM Serving", "Practical Takeaways"; the
 * "KV Cache" glossary page: "INT8 or FP8 formats ... per-token quantization
 * granularity") without fixing the encoding. Reading taken here: the OCP
 * E4M3 format (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, S.1111.111 = NaN, largest finite 448) with one fp32 scale
 * per row: s = max|x| / 448 (IEEE fp32), code = E4M3(x / s) rounded to
 * nearest, ties to even, saturating at +-448; a row of zeros stores s = 0 and
 * codes 0. Dequantisation is s * value(code). Inputs are read as x + 0.0f.
 */
static double e4m3_value(uint8_t c) {
  const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m / 8.0, -6);
  else v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* round-to-nearest-even onto the E4M3 grid, saturating; r is an fp32 value */
static uint8_t e4m3_encode(float r) {
  const int sign = signbit(r) ? 1 : 0;
  double a = fabs((double)r);
  if (a >= 448.0) return (uint8_t)((sign << 7) | 0x7E);
  /* quantum of the binade holding a (subnormal binade below 2^-6) */
  int e = a > 0.0 ? (int)floor(log2(a)) : -6;
  if (e < -6) e = -6;
  if (a > 0.0 && ldexp(1.0, e) > a) e -= 1;        /* guard log2 rounding */
  if (a > 0.0 && ldexp(1.0, e + 1) <= a) e += 1;
  if (e < -6) e = -6;
  const double q = ldexp(1.0, e - 3);
  double m = a / q; /* exact: q is a power of two */
  double fl = floor(m);
  double frac = m - fl;
  double mi = fl;
  if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0)) mi = fl + 1.0;
  double v = mi * q;
  if (v >= 448.0) return (uint8_t)((sign << 7) | 0x7E);
  if (v == 0.0) return (uint8_t)(sign << 7);
  /* encode v exactly */
  int ev = (int)floor(log2(v));
  if (ldexp(1.0, ev) > v) ev -= 1;
  if (ldexp(1.0, ev + 1) <= v) ev += 1;
  uint8_t bits;
  if (ev < -6) { /* subnormal: v = mant/8 * 2^-6 */
    bits = (uint8_t)(v / ldexp(1.0, -9));
  } else {
    const int mant = (int)(v / ldexp(1.0, ev - 3)) - 8;
    bits = (uint8_t)(((ev + 7) << 3) | mant);
  }
  return (uint8_t)((sign << 7) | bits);
}

double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }
uint8_t oracle_e4m3_encode(float r) { return e4m3_encode(r); }

void oracle_quantize_rows_fp8(const uint16_t *x, int64_t n_rows, int d, uint8_t *codes,
                              float *sz) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    const uint16_t *row = x + r * d;
    float amax = 0.0f;
    for (int j = 0; j < d; ++j) {
      const float v = fabsf(bf16_bits_to_f32(row[j]));
      if (v > amax) amax = v;
    }
    const float s = amax / 448.0f;
    for (int j = 0; j < d; ++j) {
      uint8_t c = 0;
      if (s != 0.0f) {
        const float ratio = bf16_bits_to_f32(row[j]) / s;
        c = e4m3_encode(ratio);
      }
      codes[r * d + j] = c;
    }
    sz[2 * r + 0] = s;
    sz[2 * r + 1] = 0.0f;
  }
}

/*
 * INT4 per-token quantiser: Eq. 3 with 16 levels ("KV-Cache Quantization",
 * "FP16 -> INT4: 4x reduction"): z = min, s = (max - min) / 15, code =
 * clamp(round_half_even((x - z) / s), 0, 15), every step in IEEE fp32 as for
 * INT8; a constant row stores s = 0 and codes 0. Two codes per byte: element
 * 2i in the low nibble of byte i, element 2i + 1 in the high nibble.
 */
void oracle_quantize_rows_int4(const uint16_t *x, int64_t n_rows, int d, uint8_t *packed,
                               float *sz) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    const uint16_t *row = x + r * d;
    float mn = bf16_bits_to_f32(row[0]);
    float mx = mn;
    for (int j = 1; j < d; ++j) {
      const float v = bf16_bits_to_f32(row[j]);
      if (v < mn) mn = v;
      if (v > mx) mx = v;
    }
    const float range = mx - mn;
    const float s = range / 15.0f;
    const float z = mn;
    for (int j = 0; j < d; j += 2) {
      uint8_t c[2] = {0, 0};
      for (int k = 0; k < 2; ++k) {
        if (s != 0.0f) {
          const float diff = bf16_bits_to_f32(row[j + k]) - z;
          float rq = nearbyintf(diff / s);
          if (rq < 0.0f) rq = 0.0f;
          if (rq > 15.0f) rq = 15.0f;
          c[k] = (uint8_t)rq;
        }
      }
      packed[r * (d / 2) + j / 2] = (uint8_t)(c[0] | (c[1] << 4));
    }
    sz[2 * r + 0] = s;
    sz[2 * r + 1] = z;
  }
}
