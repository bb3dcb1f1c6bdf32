// Self-test of the failure path of the bounded waits: one thread waits on an
// mbarrier that nothing ever arrives at, through the same bounded wait the
// tensor-core kernels use, and must give up with PA_DERR_TIMEOUT once its
// time limit has passed. Nothing else is pending in the CTA (no copies, no
// tensor memory), so giving up leaves nothing behind.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

__global__ void wait_timeout_kernel(uint64_t limit_ns, int32_t *d_err) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b), "r"(1));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // expected arrivals: 1, arrivals made: none; phase 0 never completes
  if (threadIdx.x == 0 && !mbar_wait_bounded(b, 0, limit_ns)) flag_error(d_err, PA_DERR_TIMEOUT);
}

}  // namespace
}  // namespace pa

extern "C" pa_status_t pa_selftest_wait_timeout(int32_t limit_us, int32_t *d_err, void *stream) {
  if (limit_us < 1 || limit_us > 1000000 || d_err == nullptr) return PA_ERR_INVALID_ARG;
  pa::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (uint64_t)limit_us * 1000ull, d_err);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
