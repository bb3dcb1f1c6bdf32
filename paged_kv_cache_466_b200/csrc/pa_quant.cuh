// Per-row quantisers of the cache write (Eq. 3 of "KV-Cache Optimization
// Techniques", section "KV-Cache Quantization", and its FP8 and INT4
// variants). One warp quantises one (token, KV head) row of D bf16 values:
// lane l holds elements [l * D / 32, (l + 1) * D / 32). Every step is an IEEE
// fp32 operation in a fixed order (explicit _rn intrinsics, no contraction),
// so every kernel that includes this header stores the same bits.
#pragma once

#include "pa_device.cuh"

namespace pa {
namespace {

template <int D>
__device__ __forceinline__ void quantise_row(const unsigned char *src_row, unsigned char *dst_codes,
                                             float *dst_sz, int lane) {
  constexpr int E = D / 32;  // elements per lane
  const __nv_bfloat16 *x16 = reinterpret_cast<const __nv_bfloat16 *>(src_row) + lane * E;
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = __fadd_rn(__bfloat162float(x16[e]), 0.0f);
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int e = 1; e < E; ++e) {
    mn = fminf(mn, x[e]);
    mx = fmaxf(mx, x[e]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float s = __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
  const float z = mn;
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    uint32_t c = 0;
    if (s != 0.0f) {
      float r = rintf(__fdiv_rn(__fsub_rn(x[e], z), s));
      r = fminf(fmaxf(r, 0.0f), 255.0f);
      c = static_cast<uint32_t>(r);
    }
    packed |= c << (8 * e);
  }
  if constexpr (E == 4) {
    *reinterpret_cast<uint32_t *>(dst_codes + lane * 4) = packed;
  } else {
    *reinterpret_cast<uint16_t *>(dst_codes + lane * 2) = static_cast<uint16_t>(packed);
  }
  if (lane == 0) *reinterpret_cast<float2 *>(dst_sz) = make_float2(s, z);
}

// FP8 (E4M3) per-token quantiser: s = max|x| / 448 (IEEE fp32), code =
// E4M3(x / s) rounded to nearest even and saturated; an all-zero row stores
// s = 0 and codes 0. The zero point is stored as 0.
template <int D>
__device__ __forceinline__ void quantise_row_fp8(const unsigned char *src_row,
                                                 unsigned char *dst_codes, float *dst_sz,
                                                 int lane) {
  constexpr int E = D / 32;  // elements per lane (even)
  const __nv_bfloat16 *x16 = reinterpret_cast<const __nv_bfloat16 *>(src_row) + lane * E;
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = __fadd_rn(__bfloat162float(x16[e]), 0.0f);
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 448.0f);
  uint32_t packed = 0;
  if (s != 0.0f) {
#pragma unroll
    for (int e = 0; e < E; e += 2)
      packed |= f32x2_to_e4m3x2(__fdiv_rn(x[e], s), __fdiv_rn(x[e + 1], s)) << (8 * e);
  }
  if constexpr (E == 4) {
    *reinterpret_cast<uint32_t *>(dst_codes + lane * 4) = packed;
  } else {
    *reinterpret_cast<uint16_t *>(dst_codes + lane * 2) = static_cast<uint16_t>(packed);
  }
  if (lane == 0) *reinterpret_cast<float2 *>(dst_sz) = make_float2(s, 0.f);
}

// INT4: Eq. 3 with 16 levels, the INT8 arithmetic with 15 in place of 255;
// element 2i goes to the low nibble of byte i.
template <int D>
__device__ __forceinline__ void quantise_row_u4(const unsigned char *src_row,
                                                unsigned char *dst_codes, float *dst_sz,
                                                int lane) {
  constexpr int E = D / 32;  // elements per lane (even)
  const __nv_bfloat16 *x16 = reinterpret_cast<const __nv_bfloat16 *>(src_row) + lane * E;
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = __fadd_rn(__bfloat162float(x16[e]), 0.0f);
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int e = 1; e < E; ++e) {
    mn = fminf(mn, x[e]);
    mx = fmaxf(mx, x[e]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  const float z = mn;
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    uint32_t c = 0;
    if (s != 0.0f) {
      float r = rintf(__fdiv_rn(__fsub_rn(x[e], z), s));
      r = fminf(fmaxf(r, 0.0f), 15.0f);
      c = static_cast<uint32_t>(r);
    }
    packed |= c << (4 * e);
  }
  if constexpr (E == 4) {
    *reinterpret_cast<uint16_t *>(dst_codes + lane * 2) = static_cast<uint16_t>(packed);
  } else {
    dst_codes[lane] = static_cast<unsigned char>(packed);
  }
  if (lane == 0) *reinterpret_cast<float2 *>(dst_sz) = make_float2(s, z);
}

}  // namespace
}  // namespace pa
