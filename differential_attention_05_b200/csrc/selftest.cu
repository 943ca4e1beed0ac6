// selftest.cu -- diagnostics of this library's device code, for tests:
//   diffattn_selftest_timeout drives the bounded-wait path of the kernels on purpose, so
//   that tests can check that a wait which never completes ends in a status code and
//   leaves the CUDA context usable (no fault, no hang);
//   diffattn_selftest_exp2 evaluates the FMA-pipe 2^x that the V2 prefill uses for part of
//   its exponentials beside CUDA's exp2f, so that tests can bound its error.
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

// y[i] = exp2_fma2(x[i]) (the prefill's polynomial 2^x, evaluated on pairs as the kernel
// does), y_ref[i] = exp2f(x[i]).
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y,
                                     float* __restrict__ y_ref, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = (i + 1 < n) ? x[i + 1] : 0.f;
  float y0, y1;
  exp2_fma2(y0, y1, x0, x1);
  y[i] = y0;
  y_ref[i] = exp2f(x0);
  if (i + 1 < n) {
    y[i + 1] = y1;
    y_ref[i + 1] = exp2f(x1);
  }
}

}  // namespace
}  // namespace diffattn

extern "C" int diffattn_selftest_timeout(int* dev_status, int timeout_ms, void* stream) {
  if (!dev_status || timeout_ms < 1 || timeout_ms > 10000) return DIFFATTN_ERR_INVALID_ARG;
  diffattn::selftest_timeout_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      dev_status, (uint64_t)timeout_ms * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? DIFFATTN_OK : DIFFATTN_ERR_CUDA;
}

extern "C" int diffattn_selftest_exp2(const float* x, float* y, float* y_ref, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y || !y_ref))) return DIFFATTN_ERR_INVALID_ARG;
  if (n == 0) return DIFFATTN_OK;
  const int pairs = (n + 1) / 2;
  diffattn::selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y, y_ref, n);
  return cudaGetLastError() == cudaSuccess ? DIFFATTN_OK : DIFFATTN_ERR_CUDA;
}
