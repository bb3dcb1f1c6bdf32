// Shared-prefix attention: the prefix half of a cascade decode.
//
// "KV-Cache Optimization Techniques", section "Prefix Caching" (Eq. 2): when
// many requests share a prompt prefix, its KV pages are stored once and every
// request's page table points at them. Eq. 1 over [prefix; own tokens] splits
// exactly into attention over the prefix and attention over the request's own
// tokens, merged by log-sum-exp. This kernel does the prefix part for all
// requests at once: per KV head, the B*G query rows that read that head form
// an [rows x D] x [D x prefix] contraction, so each prefix K/V row is read once
// per CTA row-tile instead of once per request, and the work runs as dense
// tensor-core tiles (FlashAttention-2-style online softmax).
//
// CTA: 4 warps x 16 query rows = 64 rows of one KV head; it walks a range of
// 64-token prefix tiles (a prefix split) and writes, per row, the normalised
// partial output and its natural-log log-sum-exp. K/V tiles are staged by all
// threads with cp.async into a 2-stage ring (16-byte chunks XOR-swizzled by
// row so ldmatrix reads are conflict free); per tile each warp computes
// S = Q K^T (m16n8k16, K via ldmatrix), the online softmax, and O += P V with
// P split into bf16 hi + lo halves (V via ldmatrix.trans).
#include <cmath>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr float kLn2 = 0.693147180559945309f;
constexpr int kRowsPerCta = 64;
constexpr int kTileTok = 64;
constexpr int kWarps = 4;

template <int D>
struct PTile {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunks = kRowBytes / 16;
  static constexpr int kTileBytes = kTileTok * kRowBytes;  // one tensor
  static constexpr int kStageBytes = 2 * kTileBytes;       // K and V
  static constexpr int kKSteps = D / 16;
  static constexpr int kNTilesD = D / 8;
};

__device__ __forceinline__ int swz_off(int row, int chunk, int row_bytes) {
  return row * row_bytes + ((chunk ^ (row & 7)) << 4);
}

template <int D, int P>
__global__ void __launch_bounds__(kWarps * 32, 2) prefix_kernel(const PrefixArgs a) {
  using T = PTile<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  pdl_wait_primary();

  const int mt = blockIdx.x;
  const int h = blockIdx.y;
  const int ps = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int G = a.hq / a.hkv;
  const int rows = a.B * G;

  const int n_tiles = (a.prefix_len + kTileTok - 1) / kTileTok;
  const int tile0 = ps * a.tiles_per_split;
  const int tile1 = min(tile0 + a.tiles_per_split, n_tiles);
  const int tok_lo = tile0 * kTileTok;
  const int tok_hi = min(tile1 * kTileTok, a.prefix_len);

  // prefix page ids of this split, bounds-checked
  int *pages = reinterpret_cast<int *>(smem + 2 * T::kStageBytes);
  const int pg0 = tok_lo / P;
  const int npg = tok_hi > tok_lo ? (tok_hi - 1) / P - pg0 + 1 : 0;
  for (int i = threadIdx.x; i < npg; i += kWarps * 32) {
    int pg = __ldg(a.prefix_pages + pg0 + i);
    if (pg < 0 || pg >= a.num_pages) {
      flag_error(a.d_err, PA_DERR_BAD_PAGE);
      pg = -1;
    }
    pages[i] = pg;
  }

  // query rows g and g + 8 of this warp -> (sequence, query head)
  int qrow[2];
  bool qok[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = mt * kRowsPerCta + warp * 16 + g + 8 * i;
    qok[i] = r < rows;
    const int rr = qok[i] ? r : 0;
    qrow[i] = (rr / G) * a.hq + h * G + rr % G;
  }
  uint32_t qa[T::kKSteps][4];
  {
    const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(a.q);
#pragma unroll
    for (int j = 0; j < T::kKSteps; ++j) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t *qr = reinterpret_cast<const uint32_t *>(qb + (size_t)qrow[i] * D);
        qa[j][i] = qok[i] ? __ldg(qr + 8 * j + t) : 0u;          // k = 16j + 2t
        qa[j][2 + i] = qok[i] ? __ldg(qr + 8 * j + 4 + t) : 0u;  // k = 16j + 8 + 2t
      }
    }
  }
  __syncthreads();  // page ids visible

  const unsigned char *kbase = static_cast<const unsigned char *>(a.k_pool);
  const unsigned char *vbase = static_cast<const unsigned char *>(a.v_pool);
  const uint32_t sbase = smem_u32(smem);
  const int ntl = tile1 - tile0;

  // all threads copy one 64-token tile of K and V (each copy instruction of the
  // CTA moves 2 KB: 8 whole rows)
  auto load_tile = [&](int k, int st) {
    const int ttok = tok_lo + k * kTileTok;
    const uint32_t dst = sbase + st * T::kStageBytes;
    constexpr int kCopies = T::kTileBytes / (kWarps * 32 * 16);
#pragma unroll
    for (int i = 0; i < kCopies; ++i) {
      const int c = threadIdx.x + i * kWarps * 32;
      const int row = c / T::kChunks;
      const int chunk = c % T::kChunks;
      const int tok = ttok + row;
      int page = -1;
      if (tok < tok_hi) page = pages[tok / P - pg0];
      const bool ok = page >= 0;
      const size_t grow = ((size_t)(ok ? page : 0) * a.hkv + h) * P + (ok ? tok % P : 0);
      const int so = swz_off(row, chunk, T::kRowBytes);
      cp_async16(dst + so, kbase + grow * T::kRowBytes + chunk * 16, ok ? 16u : 0u);
      cp_async16(dst + T::kTileBytes + so, vbase + grow * T::kRowBytes + chunk * 16,
                 ok ? 16u : 0u);
    }
  };

  float o[T::kNTilesD][4];
#pragma unroll
  for (int n = 0; n < T::kNTilesD; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  if (ntl > 0) load_tile(0, 0);
  cp_async_commit();
  for (int k = 0; k < ntl; ++k) {
    if (k + 1 < ntl) load_tile(k + 1, (k + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t ks = sbase + (k & 1) * T::kStageBytes;
    const uint32_t vs = ks + T::kTileBytes;
    const int ttok = tok_lo + k * kTileTok;

    // ---- S = Q K^T: 8 n-tiles of 8 tokens
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
      for (int j = 0; j < T::kKSteps; j += 2) {
        const int row = nt * 8 + (lane & 7);
        const int chunk = 2 * j + (lane >> 3);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(ks + swz_off(row, chunk, T::kRowBytes), b0, b1, b2, b3);
        mma_bf16_16816(s[nt], qa[j][0], qa[j][1], qa[j][2], qa[j][3], b0, b1);
        mma_bf16_16816(s[nt], qa[j + 1][0], qa[j + 1][1], qa[j + 1][2], qa[j + 1][3], b2, b3);
      }
    }
    // ---- online softmax for rows g (c0, c1) and g + 8 (c2, c3)
    const bool full = ttok + kTileTok <= tok_hi;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int tok = ttok + nt * 8 + 2 * t + (c & 1);
        float v = s[nt][c] * a.scale_log2;
        if (!full && tok >= tok_hi) v = -INFINITY;
        s[nt][c] = v;
        mx[c >> 1] = fmaxf(mx[c >> 1], v);
      }
    }
    float alpha[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
      const float m_new = fmaxf(m_run[i], mx[i]);
      alpha[i] = m_new == -INFINITY ? 1.f : fast_exp2(m_run[i] - m_new);
      m_run[i] = m_new;
      l_run[i] *= alpha[i];
    }
#pragma unroll
    for (int n = 0; n < T::kNTilesD; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    const float mref[2] = {m_run[0] == -INFINITY ? 0.f : m_run[0],
                           m_run[1] == -INFINITY ? 0.f : m_run[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = fast_exp2(s[nt][c] - mref[c >> 1]);
        s[nt][c] = p;
        l_run[c >> 1] += p;
      }
    }
    // ---- O += P V: 4 k-steps of 16 tokens; P from the score fragments
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ah[4], al[4];
      split_bf16(s[2 * kk][0], s[2 * kk][1], ah[0], al[0]);
      split_bf16(s[2 * kk][2], s[2 * kk][3], ah[1], al[1]);
      split_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1], ah[2], al[2]);
      split_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3], ah[3], al[3]);
#pragma unroll
      for (int n = 0; n < T::kNTilesD; n += 2) {
        const int mi = lane >> 3;
        const int row = 16 * kk + (lane & 7) + 8 * (mi & 1);
        const int chunk = n + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(vs + swz_off(row, chunk, T::kRowBytes), b0, b1, b2, b3);
        mma_bf16_16816(o[n], ah[0], ah[1], ah[2], ah[3], b0, b1);
        mma_bf16_16816(o[n], al[0], al[1], al[2], al[3], b0, b1);
        mma_bf16_16816(o[n + 1], ah[0], ah[1], ah[2], ah[3], b2, b3);
        mma_bf16_16816(o[n + 1], al[0], al[1], al[2], al[3], b2, b3);
      }
    }
    __syncthreads();  // stage (k & 1) is refilled next iteration
  }
  cp_async_wait<0>();

  // ---- normalise and write this split's partial for rows g and g + 8
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 1);
    l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 2);
  }
  const size_t R = (size_t)a.B * a.hq;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (!qok[i]) continue;
    const float inv = l_run[i] > 0.f ? 1.f / l_run[i] : 0.f;
    float *orow = a.o_pre + ((size_t)ps * R + qrow[i]) * D;
#pragma unroll
    for (int n = 0; n < T::kNTilesD; ++n)
      *reinterpret_cast<float2 *>(orow + 8 * n + 2 * t) =
          make_float2(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
    if (t == 0)
      a.lse_pre[(size_t)ps * R + qrow[i]] =
          l_run[i] > 0.f ? (m_run[i] + log2f(l_run[i])) * kLn2 : -INFINITY;
  }
}

template <int D, int P>
cudaError_t launch_prefix_t(const PrefixArgs &a, cudaStream_t stream) {
  using T = PTile<D>;
  const int max_pages_per_split = a.tiles_per_split * kTileTok / P + 2;
  const size_t smem = 2 * T::kStageBytes + (size_t)max_pages_per_split * 4;
  static_assert(2 * PTile<D>::kStageBytes + 4 * 4096 <= 227 * 1024, "shared memory");
  if (max_pages_per_split > 4096) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(prefix_kernel<D, P>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(2 * T::kStageBytes + 4 * 4096));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.B * (a.hq / a.hkv) + kRowsPerCta - 1) / kRowsPerCta, a.hkv, a.n_psplits);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefix_kernel<D, P>, a);
}

}  // namespace

int prefix_rows_per_cta() { return kRowsPerCta; }
int prefix_tile_tokens() { return kTileTok; }

cudaError_t launch_prefix(int D, int P, const PrefixArgs &a, cudaStream_t stream) {
  if (D == 128 && P == 16) return launch_prefix_t<128, 16>(a, stream);
  if (D == 128 && P == 32) return launch_prefix_t<128, 32>(a, stream);
  if (D == 64 && P == 16) return launch_prefix_t<64, 16>(a, stream);
  if (D == 64 && P == 32) return launch_prefix_t<64, 32>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
