// Diagnostic entry point for the failure-detection path of the library's
// kernels: every wait on an mbarrier is bounded in time, and a wait that runs
// out sets HSTU_DEVICE_TIMEOUT in the device status word and lets the kernel
// return instead of hanging.  The kernel here waits on a barrier that nothing
// ever arrives on, with a caller-chosen limit, so the limit is what ends it.
// It issues no copy and no tensor-core instruction, and holds no TMEM.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hstu {
namespace {

__global__ void wait_timeout_kernel(uint64_t limit_ns, uint32_t* status, int32_t* result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 of a fresh barrier with one expected arrival never completes
    const bool done = tc::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    if (result) *result = done ? 1 : 0;
  }
  __syncthreads();
}

}  // namespace
}  // namespace hstu

extern "C" hstu_status hstu_selftest_wait_timeout(uint64_t limit_ns, int32_t* d_result,
                                                  cudaStream_t stream) {
  if (limit_ns == 0 || limit_ns > 100000000ull) return HSTU_ERR_INVALID;  // at most 0.1 s
  uint32_t* status = hstu::device_status();
  if (!status) return HSTU_ERR_CUDA;
  hstu::wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns, status, d_result);
  hstu::count_launch();
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}
