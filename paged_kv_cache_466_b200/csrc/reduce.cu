// Split-KV merge: combine per-split attention results by their log-sum-exp.
//
// Softmax over a union of disjoint token ranges equals the per-range results
// weighted by exp(lse_s - M) and renormalised (M = max_s lse_s). This is the
// exact identity that lets pa_decode spread one long context over several
// CTAs; the pages do not describe it, it is the plain algebra of Eq. 1's
// softmax. One warp merges one (sequence, query head) row; splits are visited
// in index order, so the result is deterministic (the order of the sum is
// fixed, whichever path a row takes).
#include <cmath>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kWarps = 4;
constexpr int kFast = 16;  // rows of at most this many partials take the one-round path

// Partials i < S are the row's own (o_part[row][i], lse[row][i]); i >= S are
// prior partials p = i - S (prior_o + p * po_stride + row * D,
// prior_lse[p * pl_stride + row]); the strides are in floats.
__global__ void __launch_bounds__(kWarps * 32) splitkv_reduce_kernel(
    const float *__restrict__ o_part, const float *__restrict__ lse, int rows, int S, int D,
    float *__restrict__ out, const float *__restrict__ prior_o,
    const float *__restrict__ prior_lse, int n_prior, size_t po_stride, size_t pl_stride,
    float *__restrict__ lse_out) {
  pdl_wait_primary();  // partials come from the kernel just before us
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + warp;
  if (row >= rows) return;
  const int n_all = S + n_prior;
  const float *ls = lse + (size_t)row * S;
  auto lse_at = [&](int i) { return i < S ? ls[i] : prior_lse[(size_t)(i - S) * pl_stride + row]; };
  const int D4 = D / 4;
  const float4 *op = reinterpret_cast<const float4 *>(o_part + (size_t)row * S * D);
  auto o_at = [&](int i) {
    return i < S ? op + (size_t)i * D4
                 : reinterpret_cast<const float4 *>(prior_o + (size_t)(i - S) * po_stride +
                                                    (size_t)row * D);
  };
  float4 *dst = reinterpret_cast<float4 *>(out + (size_t)row * D);
  if (n_all <= kFast && D4 <= 32) {
    // Every load of the row goes out at once — lane s's log-sum-exp and each
    // lane's four outputs of every partial — so the merge waits for one round
    // trip instead of one for the log-sum-exps and more for the partials.
    const float lv = lane < n_all ? lse_at(lane) : -INFINITY;
    // (partials past n_all re-read the last one, and lanes past D4 their
    // row's first chunk: valid addresses whose values get weight 0 / no store)
    const int li = lane < D4 ? lane : 0;
    float4 v[kFast];
#pragma unroll
    for (int k = 0; k < kFast; ++k) v[k] = o_at(min(k, n_all - 1))[li];
    float M = lv;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float wl = (lane < n_all && M != -INFINITY) ? expf(lv - M) : 0.f;  // -inf -> 0
    float den = wl;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kFast; ++k) {
      const float w = __shfl_sync(0xffffffffu, wl, k);
      // a weight-0 (empty) partial is loaded but never used
      if (k < n_all && w != 0.f) {
        acc.x = fmaf(w, v[k].x, acc.x);
        acc.y = fmaf(w, v[k].y, acc.y);
        acc.z = fmaf(w, v[k].z, acc.z);
        acc.w = fmaf(w, v[k].w, acc.w);
      }
    }
    if (lane < D4) {
      const float r = den > 0.f ? 1.f / den : 0.f;
      dst[lane] = make_float4(acc.x * r, acc.y * r, acc.z * r, acc.w * r);
    }
    if (lse_out != nullptr && lane == 0) lse_out[row] = den > 0.f ? M + logf(den) : -INFINITY;
    return;
  }
  float M = -INFINITY;
  for (int s = lane; s < n_all; s += 32) M = fmaxf(M, lse_at(s));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  for (int i0 = 0; i0 < D4; i0 += 32) {
    const int i = i0 + lane;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    // partials in chunks of 32: lane s holds the weight of partial s0 + s,
    // and every lane then issues its loads for the whole chunk back to back
    for (int s0 = 0; s0 < n_all; s0 += 32) {
      const int n = min(32, n_all - s0);
      const float wl =
          (lane < n && M != -INFINITY) ? expf(lse_at(s0 + lane) - M) : 0.f;  // -inf -> 0
      den += wl;
      // eight loads in flight per lane; a weight-0 (empty) partial is loaded
      // but never used, so whatever its slot holds cannot reach the sum
      for (int b0 = 0; b0 < n; b0 += 8) {
        float4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (b0 + k < n && i < D4) v[k] = o_at(s0 + b0 + k)[i];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float w = __shfl_sync(0xffffffffu, wl, (b0 + k) & 31);
          if (b0 + k < n && i < D4 && w != 0.f) {
            acc.x = fmaf(w, v[k].x, acc.x);
            acc.y = fmaf(w, v[k].y, acc.y);
            acc.z = fmaf(w, v[k].z, acc.z);
            acc.w = fmaf(w, v[k].w, acc.w);
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (i < D4) {
      const float r = den > 0.f ? 1.f / den : 0.f;
      dst[i] = make_float4(acc.x * r, acc.y * r, acc.z * r, acc.w * r);
    }
    // the merged log-sum-exp: M + ln(sum_s exp(lse_s - M))
    if (lse_out != nullptr && i0 == 0 && lane == 0)
      lse_out[row] = den > 0.f ? M + logf(den) : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_splitkv_reduce(const float *o_part, const float *lse, int B, int hq, int S,
                                  int D, float *out, bool programmatic, cudaStream_t stream,
                                  const float *prior_o, const float *prior_lse, int n_prior,
                                  float *lse_out, size_t prior_o_stride,
                                  size_t prior_lse_stride) {
  const int rows = B * hq;
  if (prior_o_stride == 0) prior_o_stride = (size_t)rows * D;
  if (prior_lse_stride == 0) prior_lse_stride = (size_t)rows;
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
  return cudaLaunchKernelEx(&cfg, splitkv_reduce_kernel, o_part, lse, rows, S, D, out, prior_o,
                            prior_lse, n_prior, prior_o_stride, prior_lse_stride, lse_out);
}

}  // namespace pa
