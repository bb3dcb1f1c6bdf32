// Cache write: scatter new tokens' K/V rows into their page slots.
//
// "KV-Cache Optimization Techniques", section "PagedAttention (vLLM)",
// "Architecture": each request's page table maps a logical KV position to a
// physical page of P tokens; position pos lives in page table[pos / P], slot
// pos % P. For an INT8 pool every (token, KV head) row is quantised on the way
// in by Eq. 3 ("KV-Cache Quantization", per-token calibration; an FP8 pool
// uses E4M3 codes with an absmax scale, see quantise_row_fp8):
//   z = min(row), s = (max(row) - min(row)) / 255,
//   code = clamp(round_half_even((x - z) / s), 0, 255)   (s == 0 -> code 0),
// every step an IEEE fp32 operation in that order (explicit _rn intrinsics,
// no contraction), inputs read as x + 0 so that -0 is stored as +0.
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_quant.cuh"

namespace pa {
namespace {

struct AppendArgs {
  const unsigned char *k_new;
  const unsigned char *v_new;
  const int32_t *seq_idx;
  const int32_t *pos;
  const int32_t *block_tables;
  int32_t n;
  int32_t num_seqs;
  int32_t max_pages;
  int32_t num_pages;
  int32_t hkv;
  int32_t P;
  int32_t D;
  unsigned char *k_pool;
  unsigned char *v_pool;
  float *k_sz;
  float *v_sz;
  int32_t *d_err;
};

// Physical row index (page * Hkv + h) * P + slot of token i, KV head h; -1 and
// an error bit if the token's sequence, position or page is out of range.
__device__ __forceinline__ long long slot_row(const AppendArgs &a, int i, int h) {
  const int seq = __ldg(a.seq_idx + i);
  const int p = __ldg(a.pos + i);
  if (seq < 0 || seq >= a.num_seqs) {
    flag_error(a.d_err, PA_DERR_BAD_SEQ);
    return -1;
  }
  if (p < 0 || p / a.P >= a.max_pages) {
    flag_error(a.d_err, PA_DERR_BAD_POS);
    return -1;
  }
  const int page = __ldg(a.block_tables + (size_t)seq * a.max_pages + p / a.P);
  if (page < 0 || page >= a.num_pages) {
    flag_error(a.d_err, PA_DERR_BAD_PAGE);
    return -1;
  }
  return ((long long)page * a.hkv + h) * a.P + p % a.P;
}

// bf16: one thread per 16-byte chunk of a (token, head) row, K and V.
__global__ void append_bf16_kernel(const AppendArgs a) {
  pdl_launch_dependents();  // the decode that follows may be scheduled now;
                            // it waits for this grid before reading anything
  const int chunks = a.D / 8;
  const long long total = (long long)a.n * a.hkv * chunks;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(idx % chunks);
    const long long r = idx / chunks;  // token * hkv + h
    const int h = (int)(r % a.hkv);
    const int i = (int)(r / a.hkv);
    const long long row = slot_row(a, i, h);
    if (row < 0) continue;
    const size_t src = ((size_t)r * a.D + c * 8) * 2;
    const size_t dst = ((size_t)row * a.D + c * 8) * 2;
    *reinterpret_cast<uint4 *>(a.k_pool + dst) = ldg_nc128(a.k_new + src);
    *reinterpret_cast<uint4 *>(a.v_pool + dst) = ldg_nc128(a.v_new + src);
  }
}

// INT8 / FP8 / INT4: one warp per (token, head) row; K then V.
template <int D, int kFmt>  // kFmt: the pool's pa_kv_dtype_t
__global__ void append_u8_kernel(const AppendArgs a) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)a.n * a.hkv;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const int h = (int)(r % a.hkv);
    const int i = (int)(r / a.hkv);
    long long row = 0;
    if (lane == 0) row = slot_row(a, i, h);
    row = __shfl_sync(0xffffffffu, row, 0);
    if (row < 0) continue;
    const size_t src = (size_t)r * D * 2;
    if constexpr (kFmt == PA_KV_U4_PER_TOKEN) {
      quantise_row_u4<D>(a.k_new + src, a.k_pool + (size_t)row * (D / 2),
                              a.k_sz + (size_t)row * 2, lane);
      quantise_row_u4<D>(a.v_new + src, a.v_pool + (size_t)row * (D / 2),
                              a.v_sz + (size_t)row * 2, lane);
    } else if constexpr (kFmt == PA_KV_FP8_PER_TOKEN) {
      quantise_row_fp8<D>(a.k_new + src, a.k_pool + (size_t)row * D,
                               a.k_sz + (size_t)row * 2, lane);
      quantise_row_fp8<D>(a.v_new + src, a.v_pool + (size_t)row * D,
                               a.v_sz + (size_t)row * 2, lane);
    } else {
      quantise_row<D>(a.k_new + src, a.k_pool + (size_t)row * D, a.k_sz + (size_t)row * 2,
                           lane);
      quantise_row<D>(a.v_new + src, a.v_pool + (size_t)row * D, a.v_sz + (size_t)row * 2,
                           lane);
    }
  }
}

}  // namespace

cudaError_t launch_kv_append(const pa_kv_pool_t &pool, const void *k_new, const void *v_new,
                             const int32_t *seq_idx, const int32_t *pos, int32_t n,
                             const int32_t *block_tables, int32_t num_seqs, int32_t max_pages,
                             int32_t *d_err, cudaStream_t stream) {
  AppendArgs a;
  a.k_new = static_cast<const unsigned char *>(k_new);
  a.v_new = static_cast<const unsigned char *>(v_new);
  a.seq_idx = seq_idx;
  a.pos = pos;
  a.block_tables = block_tables;
  a.n = n;
  a.num_seqs = num_seqs;
  a.max_pages = max_pages;
  a.num_pages = pool.num_pages;
  a.hkv = pool.num_kv_heads;
  a.P = pool.page_size;
  a.D = pool.head_dim;
  a.k_pool = static_cast<unsigned char *>(pool.k_pool);
  a.v_pool = static_cast<unsigned char *>(pool.v_pool);
  a.k_sz = pool.k_sz;
  a.v_sz = pool.v_sz;
  a.d_err = d_err;
  const int sms = device_sm_count();
  if (pool.dtype == PA_KV_BF16) {
    const long long work = (long long)n * a.hkv * (a.D / 8);
    long long blocks = (work + 255) / 256;
    blocks = blocks < 1 ? 1 : (blocks > 16LL * sms ? 16LL * sms : blocks);
    append_bf16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(a);
  } else {
    const long long rows = (long long)n * a.hkv;
    long long blocks = (rows + 7) / 8;
    blocks = blocks < 1 ? 1 : (blocks > 16LL * sms ? 16LL * sms : blocks);
#define PA_APPEND(D_, F_)                                                  \
  if (a.D == D_ && pool.dtype == F_) {                                     \
    append_u8_kernel<D_, F_><<<(unsigned)blocks, 256, 0, stream>>>(a);     \
    return cudaGetLastError();                                             \
  }
    PA_APPEND(128, PA_KV_U8_PER_TOKEN)
    PA_APPEND(64, PA_KV_U8_PER_TOKEN)
    PA_APPEND(128, PA_KV_FP8_PER_TOKEN)
    PA_APPEND(64, PA_KV_FP8_PER_TOKEN)
    PA_APPEND(128, PA_KV_U4_PER_TOKEN)
    PA_APPEND(64, PA_KV_U4_PER_TOKEN)
#undef PA_APPEND
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pa
