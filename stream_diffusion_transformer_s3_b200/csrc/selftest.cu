// Health check of the library's bounded waits: a kernel waits on an mbarrier that
// nothing will ever arrive on, through the same mbar_wait the pipelines use, and must
// give up after the wait limit with ZDIT_ERR_DEVICE_TIMEOUT latched, leaving the
// context usable.  No fault, trap or unbounded loop is involved.
#include "internal.h"
#include "ptx.cuh"

namespace zdit {
namespace {

__global__ void wait_timeout_kernel(int* err, int* result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag, err);  // phase 0 never completes
    *result = ok ? 1 : (abort_flag ? 2 : 3);
  }
}

}  // namespace
}  // namespace zdit

using namespace zdit;

extern "C" ZDIT_API zdit_status zdit_selftest_wait_timeout(int32_t* result_dev, void* stream) {
  if (result_dev == nullptr) return ZDIT_ERR_INVALID_ARG;
  ProfScope ps(PROF_MISC, 0.0, 0.0, static_cast<cudaStream_t>(stream));
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(device_error_ptr(), result_dev);
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}
