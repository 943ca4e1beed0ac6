// lambda.cu -- the lambda re-parameterisation on the device.
//
//   lambda_h = exp(lq1_h . lk1_h) - exp(lq2_h . lk2_h) + lambda_init
//   ("Differential Attention (V2)", The Concept, "The difference idea"; Key Terms, "lambda")
//   lambda_init = 0.8 - 0.6 * exp(-0.3 * (depth - 1))
//   (skill-diff-attention-integrator, "Architecture diff")
//
// One warp per head: lanes stride over the vector, the warp reduces with a fixed xor tree
// (so the result does not depend on scheduling), lane 0 applies exp and writes.
#include "common.cuh"
#include "kernels.h"

namespace diffattn {

__global__ void __launch_bounds__(256) lambda_kernel(const float* __restrict__ lq1,
                                                     const float* __restrict__ lk1,
                                                     const float* __restrict__ lq2,
                                                     const float* __restrict__ lk2, int n_heads,
                                                     int dim, int depth, float* __restrict__ lam,
                                                     float* __restrict__ lam_init) {
  const float li = 0.8f - 0.6f * expf(-0.3f * (float)(depth - 1));
  if (lam_init && blockIdx.x == 0 && threadIdx.x == 0) lam_init[0] = li;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_heads) return;
  const size_t base = (size_t)warp * dim;
  float d1 = 0.f, d2 = 0.f;
  for (int c = lane; c < dim; c += 32) {
    d1 = fmaf(lq1[base + c], lk1[base + c], d1);
    d2 = fmaf(lq2[base + c], lk2[base + c], d2);
  }
  d1 = warp_sum(d1);
  d2 = warp_sum(d2);
  if (lane == 0) lam[warp] = expf(d1) - expf(d2) + li;
}

cudaError_t launch_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                          int n_heads, int dim, int depth, float* lam, float* lam_init,
                          cudaStream_t stream) {
  const int threads = 256, warps_per_block = threads / 32;
  const int blocks = (n_heads + warps_per_block - 1) / warps_per_block;
  lambda_kernel<<<blocks, threads, 0, stream>>>(lq1, lk1, lq2, lk2, n_heads, dim, depth, lam,
                                                lam_init);
  return cudaGetLastError();
}

// Gradients of the four vectors from dL/dlambda (one warp per head; the dot products in
// the forward's order): d lambda / d lq1 = e1 lk1, / d lk1 = e1 lq1, / d lq2 = -e2 lk2,
// / d lk2 = -e2 lq2 with e_b = exp(lq_b . lk_b).
__global__ void __launch_bounds__(256) lambda_bwd_kernel(
    const float* __restrict__ lq1, const float* __restrict__ lk1, const float* __restrict__ lq2,
    const float* __restrict__ lk2, int n_heads, int dim, const float* __restrict__ dlam,
    float* __restrict__ dlq1, float* __restrict__ dlk1, float* __restrict__ dlq2,
    float* __restrict__ dlk2) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_heads) return;
  const size_t base = (size_t)warp * dim;
  float d1 = 0.f, d2 = 0.f;
  for (int c = lane; c < dim; c += 32) {
    d1 = fmaf(lq1[base + c], lk1[base + c], d1);
    d2 = fmaf(lq2[base + c], lk2[base + c], d2);
  }
  d1 = warp_sum(d1);
  d2 = warp_sum(d2);
  const float g1 = dlam[warp] * expf(d1), g2 = -dlam[warp] * expf(d2);
  for (int c = lane; c < dim; c += 32) {
    dlq1[base + c] = g1 * lk1[base + c];
    dlk1[base + c] = g1 * lq1[base + c];
    dlq2[base + c] = g2 * lk2[base + c];
    dlk2[base + c] = g2 * lq2[base + c];
  }
}

cudaError_t launch_lambda_bwd(const float* lq1, const float* lk1, const float* lq2,
                              const float* lk2, int n_heads, int dim, const float* dlam,
                              float* dlq1, float* dlk1, float* dlq2, float* dlk2,
                              cudaStream_t stream) {
  const int threads = 256, warps_per_block = threads / 32;
  const int blocks = (n_heads + warps_per_block - 1) / warps_per_block;
  lambda_bwd_kernel<<<blocks, threads, 0, stream>>>(lq1, lk1, lq2, lk2, n_heads, dim, dlam, dlq1,
                                                    dlk1, dlq2, dlk2);
  return cudaGetLastError();
}

}  // namespace diffattn
