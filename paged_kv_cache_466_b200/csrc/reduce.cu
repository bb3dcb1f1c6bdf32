// Split-KV merge: combine per-split attention results by their log-sum-exp.
//
// Softmax over a union of disjoint token ranges equals the per-range results
// weighted by exp(lse_s - M) and renormalised (M = max_s lse_s). This is the
// exact identity that lets pa_decode spread one long context over several
// CTAs; the pages do not describe it, it is the plain algebra of Eq. 1's
// softmax. One warp merges one (sequence, query head) row; splits are visited
// in index order, so the result is deterministic.
#include <cmath>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32) splitkv_reduce_kernel(
    const float *__restrict__ o_part, const float *__restrict__ lse, int rows, int S, int D,
    float *__restrict__ out) {
  pdl_wait_primary();  // partials come from the kernel just before us
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + warp;
  if (row >= rows) return;
  const float *ls = lse + (size_t)row * S;
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, ls[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float4 *op = reinterpret_cast<const float4 *>(o_part + (size_t)row * S * D);
  float4 *dst = reinterpret_cast<float4 *>(out + (size_t)row * D);
  const int D4 = D / 4;
  for (int i0 = 0; i0 < D4; i0 += 32) {
    const int i = i0 + lane;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    // splits in chunks of 32: lane s holds the weight of split s0 + s, and
    // every lane then issues its loads for the whole chunk back to back
    for (int s0 = 0; s0 < S; s0 += 32) {
      const int n = min(32, S - s0);
      const float wl =
          (lane < n && M != -INFINITY) ? expf(ls[s0 + lane] - M) : 0.f;  // -inf -> 0
      den += wl;
#pragma unroll 8
      for (int s = 0; s < n; ++s) {
        const float w = __shfl_sync(0xffffffffu, wl, s);
        if (i < D4 && w != 0.f) {  // weight-0 (empty) splits are never read
          const float4 v = op[(size_t)(s0 + s) * D4 + i];
          acc.x = fmaf(w, v.x, acc.x);
          acc.y = fmaf(w, v.y, acc.y);
          acc.z = fmaf(w, v.z, acc.z);
          acc.w = fmaf(w, v.w, acc.w);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (i < D4) {
      const float r = den > 0.f ? 1.f / den : 0.f;
      dst[i] = make_float4(acc.x * r, acc.y * r, acc.z * r, acc.w * r);
    }
  }
}

}  // namespace

cudaError_t launch_splitkv_reduce(const float *o_part, const float *lse, int B, int hq, int S,
                                  int D, float *out, bool programmatic, cudaStream_t stream) {
  const int rows = B * hq;
  if (rows == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((rows + kWarps - 1) / kWarps);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = programmatic ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, splitkv_reduce_kernel, o_part, lse, rows, S, D, out);
}

}  // namespace pa
