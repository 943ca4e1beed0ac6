// selftest.cu -- diffattn_selftest_timeout: drives the bounded-wait path of the kernels on
// purpose, so that tests can check that a wait which never completes ends in a status
// code and leaves the CUDA context usable (no fault, no hang).
#include "../../include/diffattn.h"
#include "common.cuh"

namespace diffattn {
namespace {

// One block: thread 0 initialises an mbarrier expecting one arrival that never comes;
// every thread waits for its first phase with the kernels' wait routine, bounded by
// limit_ns. All waits give up; thread 0 reports the timeout.
__global__ void __launch_bounds__(128, 1) selftest_timeout_kernel(int* dev_status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(&bar, 0, &abort_flag, limit_ns);
  __syncthreads();
  if (threadIdx.x == 0 && (!ok || abort_flag)) report_status(dev_status, DIFFATTN_ERR_TIMEOUT);
}

}  // namespace
}  // namespace diffattn

extern "C" int diffattn_selftest_timeout(int* dev_status, int timeout_ms, void* stream) {
  if (!dev_status || timeout_ms < 1 || timeout_ms > 10000) return DIFFATTN_ERR_INVALID_ARG;
  diffattn::selftest_timeout_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      dev_status, (uint64_t)timeout_ms * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? DIFFATTN_OK : DIFFATTN_ERR_CUDA;
}
