// pa_decode_noalloc: the split-KV decode for callers that cannot allocate
// device memory. Its scratch (partial outputs and their log-sum-exps) lives in
// a library-owned device array instead of a caller-provided workspace; the
// computation is pa_decode's, unchanged.
#include <atomic>
#include <cstdio>

#include "pa_internal.h"

namespace pa {

// Records a message for pa_last_error() (defined with the other entry points).
void set_last_error_message(const char *msg);

namespace {

constexpr size_t kScratchBytes = PA_NOALLOC_SCRATCH_BYTES;

// The scratch itself. In host code this name is only a stand-in for the
// symbol, not a device address: kernels get the address looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];

pa_status_t noalloc_fail(pa_status_t st, const char *msg) {
  set_last_error_message(msg);
  return st;
}

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (with that device current) and cached.
pa_status_t scratch_address(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char buf[256];
    snprintf(buf, sizeof buf, "pa_decode_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    return noalloc_fail(PA_ERR_CUDA, buf);
  }
  if (dev < 0 || dev >= kMaxDevices)
    return noalloc_fail(PA_ERR_UNSUPPORTED, "pa_decode_noalloc: device index out of range");
  void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char buf[256];
      snprintf(buf, sizeof buf, "pa_decode_noalloc: cudaGetSymbolAddress: %s",
               cudaGetErrorString(e));
      return noalloc_fail(PA_ERR_CUDA, buf);
    }
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" pa_status_t pa_decode_noalloc(const pa_kv_pool_t *pool, const void *q,
                                         int32_t num_seqs, int32_t num_q_heads,
                                         const int32_t *block_tables, int32_t max_pages,
                                         const int32_t *context_lens, float scale, float *out,
                                         int32_t num_splits, int32_t *d_err, void *stream) {
  using namespace pa;
  int32_t S = num_splits;
  if (pool != nullptr && num_seqs > 0 && num_q_heads > 0 && max_pages > 0 && num_splits >= 0) {
    S = pa_decode_num_splits(pool, num_seqs, max_pages, num_splits);
    if (S > 0) {
      size_t need = pa_decode_workspace_bytes(num_seqs, num_q_heads, pool->head_dim, S);
      if (need > kScratchBytes && num_splits == 0) {
        // automatic: take the largest split count whose partials fit
        for (int32_t s = S - 1; s >= 1 && need > kScratchBytes; --s) {
          S = pa_decode_num_splits(pool, num_seqs, max_pages, s);
          need = pa_decode_workspace_bytes(num_seqs, num_q_heads, pool->head_dim, S);
        }
      }
      if (need > kScratchBytes) {
        char buf[320];
        snprintf(buf, sizeof buf,
                 "pa_decode_noalloc: %d splits need %zu bytes of scratch, more than the "
                 "library's static %zu bytes; use fewer splits or pa_decode with a workspace",
                 (int)S, need, kScratchBytes);
        return noalloc_fail(PA_ERR_WORKSPACE, buf);
      }
    }
  }
  void *ws = nullptr;
  if (S > 1) {
    const pa_status_t st = scratch_address(&ws);
    if (st != PA_OK) return st;
  }
  return pa_decode(pool, q, num_seqs, num_q_heads, block_tables, max_pages, context_lens, scale,
                   out, ws, ws ? kScratchBytes : 0, S, d_err, stream);
}
