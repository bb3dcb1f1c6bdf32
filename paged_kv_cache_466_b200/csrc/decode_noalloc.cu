// pa_decode_noalloc: the split-KV decode for callers that cannot allocate
// device memory. Its scratch (partial outputs and their log-sum-exps) lives in
// a library-owned device array instead of a caller-provided workspace; the
// computation is pa_decode's, unchanged.
#include <cuda.h>

#include <cstdio>
#include <mutex>

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

pa_status_t noalloc_fail(pa_status_t st, const char *msg) {
  set_last_error_message(msg);
  return st;
}

// The array's device address is a property of the CUDA context that loaded
// the library's module, not of the device alone: after cudaDeviceReset (or
// anything else that destroys and re-creates the primary context) the module
// is loaded again and the array may sit elsewhere. The cache is therefore
// keyed by the context's id, which CUDA never reuses within a process. The
// two driver calls that read it come through the runtime's entry-point
// lookup, so the library needs no link against the driver library.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

struct CtxCalls {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const CtxCalls &ctx_calls() {
  static const CtxCalls calls = [] {
    CtxCalls c;
    void *f1 = nullptr, *f2 = nullptr;
    cudaDriverEntryPointQueryResult r1 = cudaDriverEntryPointSymbolNotFound;
    cudaDriverEntryPointQueryResult r2 = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &r1) == cudaSuccess &&
        r1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &r2) == cudaSuccess &&
        r2 == cudaDriverEntryPointSuccess && f1 != nullptr && f2 != nullptr) {
      c.get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
      c.get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    return c;
  }();
  return calls;
}

// Id of the context current on the calling thread, 0 if there is none or it
// cannot be read (then nothing is cached and every call looks the address up).
unsigned long long current_ctx_id() {
  const CtxCalls &c = ctx_calls();
  if (c.get_current == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (c.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (c.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

struct ScratchSlot {
  unsigned long long ctx_id = 0;
  void *addr = nullptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch_addr[kMaxDevices];

// Device address of g_noalloc_scratch for the current device and context:
// looked up with cudaGetSymbolAddress (with that device current) the first
// time a context is seen, then cached under the context's id.
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
  unsigned long long id = current_ctx_id();
  if (id != 0) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev].ctx_id == id && g_scratch_addr[dev].addr != nullptr) {
      *out = g_scratch_addr[dev].addr;
      return PA_OK;
    }
  }
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    char buf[256];
    snprintf(buf, sizeof buf, "pa_decode_noalloc: cudaGetSymbolAddress: %s",
             cudaGetErrorString(e));
    return noalloc_fail(PA_ERR_CUDA, buf);
  }
  // the lookup itself makes the device's primary context current if no
  // context was yet, so read the id again before caching
  id = current_ctx_id();
  if (id != 0) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    g_scratch_addr[dev].ctx_id = id;
    g_scratch_addr[dev].addr = p;
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
    // a pool or shape the planner rejects goes to pa_decode with the caller's
    // own split count, so that its error message names the real problem
    if (S <= 0) {
      S = num_splits;
    } else {
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
