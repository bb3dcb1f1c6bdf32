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
