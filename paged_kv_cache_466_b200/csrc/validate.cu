// Page-table check: every table entry a decode would dereference must name a
// page of the pool ("PagedAttention (vLLM)", "Architecture"), and every
// context length must fit its table. Violations are reported through an
// error word; nothing traps.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

__global__ void validate_tables_kernel(const int32_t *bt, int B, int max_pages,
                                       const int32_t *ctx, int num_pages, int P,
                                       int32_t *d_err) {
  const long long total = (long long)B * max_pages;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int b = (int)(idx / max_pages);
    const int lp = (int)(idx % max_pages);
    const int c = __ldg(ctx + b);
    if (c < 0 || c > max_pages * P) {
      if (lp == 0) flag_error(d_err, PA_DERR_BAD_CTX);
      continue;
    }
    if (lp < (c + P - 1) / P) {
      const int pg = __ldg(bt + idx);
      if (pg < 0 || pg >= num_pages) flag_error(d_err, PA_DERR_BAD_PAGE);
    }
  }
}

}  // namespace

cudaError_t launch_validate_tables(const int32_t *block_tables, int32_t B, int32_t max_pages,
                                   const int32_t *ctx, int32_t num_pages, int32_t page_size,
                                   int32_t *d_err, cudaStream_t stream) {
  const long long total = (long long)B * max_pages;
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  const long long cap = 8LL * device_sm_count();
  if (blocks > cap) blocks = cap;
  validate_tables_kernel<<<(unsigned)blocks, 256, 0, stream>>>(block_tables, B, max_pages, ctx,
                                                               num_pages, page_size, d_err);
  return cudaGetLastError();
}

}  // namespace pa
