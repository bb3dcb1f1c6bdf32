// Device-side helpers shared by the pagedattn kernels (sm_100a).
//
// Thin inline-PTX wrappers for the handful of instructions the kernels use:
// 16-byte cp.async with zero-fill, warp-level mma.sync on bf16/f16 operands
// with fp32 accumulators, packed conversions, ex2, and programmatic
// dependent launch controls.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pagedattn.h"

namespace pa {

// ------------------------------------------------------------------ errors
__device__ __forceinline__ void flag_error(int32_t *d_err, int32_t bits) {
  if (d_err != nullptr) atomicOr(d_err, bits);
}

// ------------------------------------------------------------- async copy
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy that bypasses L1. Only the first `src_bytes`
// (0, 8 or 16) bytes are read; the rest of the 16 are zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src,
                                           uint32_t src_bytes) {
  asm volatile(
      "cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;\n" ::"r"(dst),
      "l"(src), "r"(src_bytes)
      : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 ldg_nc128(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Four 8x8 b16 matrices from shared memory; lane l supplies the address of
// row (l % 8) of matrix (l / 8). The .trans form transposes each matrix.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                        uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                              uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose of an 8x8 matrix of 16-bit elements held in the mma fragment layout
// (lane l holds row l / 4, columns 2 (l % 4) and 2 (l % 4) + 1): afterwards
// lane l holds the same positions of the transposed matrix.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

// ------------------------------------------------------------ tensor cores
// D = A(16x16, row) * B(16x8, col) + D, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0,
                                               uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0,
                                              uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------ conversions
// Pack two fp32 into bf16x2 / f16x2 (round to nearest even); `lo` lands in
// bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t v) {
  return __uint_as_float(v << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t v) {
  return __uint_as_float(v & 0xffff0000u);
}
__device__ __forceinline__ float f16_lo(uint32_t v) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xffffu)));
}
__device__ __forceinline__ float f16_hi(uint32_t v) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
}

// Split p into hi + lo, both representable in the 16-bit operand type, so that
// a tensor-core product with hi and with lo sums to p * x within ~2^-16 of p.
__device__ __forceinline__ void split_bf16(float p0, float p1, uint32_t &hi,
                                           uint32_t &lo) {
  hi = pack_bf16(p0, p1);
  lo = pack_bf16(p0 - bf16_lo(hi), p1 - bf16_hi(hi));
}
__device__ __forceinline__ void split_f16(float p0, float p1, uint32_t &hi,
                                          uint32_t &lo) {
  hi = pack_f16(p0, p1);
  lo = pack_f16(p0 - f16_lo(hi), p1 - f16_hi(hi));
}

// Two uint8 codes -> f16x2 holding exactly (code_a * 2^-24, code_b * 2^-24):
// a byte under a zero high byte is the f16 subnormal c * 2^-24, so one byte
// permute builds the pair and nothing is added or subtracted. The caller
// puts the exact 2^24 back into the row scale.
__device__ __forceinline__ uint32_t u8x2_to_f16x2(uint32_t word, uint32_t sel) {
  return __byte_perm(word, 0u, sel);
}

// Two E4M3 codes (bits 0..7 and 8..15 of `pair`) -> f16x2 with the first code in
// the low half. Exact: every E4M3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair) {
  uint32_t r;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n}\n"
      : "=r"(r)
      : "r"(pair));
  return r;
}
// The same for the two codes in bits 16..31 (the upper half of the register,
// read in place: no shift).
__device__ __forceinline__ uint32_t e4m3x2_hi_to_f16x2(uint32_t pair) {
  uint32_t r;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.rn.f16x2.e4m3x2 %0, hi;\n}\n"
      : "=r"(r)
      : "r"(pair));
  return r;
}

// Two fp32 -> two E4M3 codes (round to nearest even, saturate to +-448), the
// code of `lo` in bits 0..7.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint32_t r;
  asm("{\n .reg .b16 c;\n cvt.rn.satfinite.e4m3x2.f32 c, %1, %2;\n cvt.u32.u16 %0, c;\n}\n"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------- bounded waits
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait until the phase of the mbarrier at shared address `bar` with this
// parity has completed. Gives up and returns false once `limit_ns` of wall
// time (the global timer) has passed, or after 2^26 polls, so that a wait
// that can never be satisfied ends in an error status instead of a hang.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  for (int i = 0; i < (1 << 26); ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity));
    if (done) return true;
    if ((i & 15) == 15 && global_ns() - t0 > limit_ns) return false;
  }
  return false;
}

// ------------------------------------------------- programmatic dependent launch
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_primary() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

}  // namespace pa
