// kernels.h -- internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace diffattn {

// Resolved prefill problem (validated by the API layer).
struct PrefillArgs {
  int variant;       // DIFFATTN_V1 / DIFFATTN_V2
  int B, N;          // N queries (the last N of the Nk key positions)
  int Nk;            // keys; Nk >= N
  int window;        // causal sliding window in keys (0: none)
  int units;         // V1 heads / V2 pairs
  int Hq, Hkv;       // head counts as given
  int group;         // V2: Hq / Hkv (query heads per KV head); V1: 1
  int d, dv;         // branch width, value width
  int causal, apply_norm;
  float eps;
  int64_t qs[3], ks[3], vs[3], os[3];  // element strides {batch, token, head}
  const void* q;
  const void* k;
  const void* v;
  const float* lambda;
  const float* lambda_init;
  void* out;
  int* dev_status;
};

struct DecodeArgs {
  int B, L, Hq, Hkv, d;   // V1: Hq = Hkv = H differential heads, d = branch width
  int splits, split_len;  // keys per split (multiple of the chunk size)
  int64_t qs[2], kvs[3], os[2];
  const void* q;
  const void* k;
  const void* v;
  const int32_t* kv_len;
  const float* lambda;
  const float* lambda_init;  // V1, read when apply_norm
  int apply_norm;            // V1
  float eps;                 // V1
  void* out;
  float* ws_o;   // V2: [B, Hq, splits, d]; V1: [B, H, splits, 2 branches, 2d]
  float* ws_ml;  // V2: [B, Hq, splits, 2];  V1: [B, H, splits, 2 branches, 2]
  int* dev_status;
};

cudaError_t launch_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                          int n_heads, int dim, int depth, float* lam, float* lam_init,
                          cudaStream_t stream);

cudaError_t launch_prefill_f32(const PrefillArgs& a, cudaStream_t stream);

// bf16 prefill on tcgen05, single pass with the (p1 - c p2, p2) operand split: V1 with
// d = 64 (prefill_v1.cu), V2 with d = 128 and an even number of query heads per KV head
// (prefill_v2.cu); each returns cudaErrorNotSupported for shapes it does not handle.
cudaError_t launch_prefill_v1(const PrefillArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_v2(const PrefillArgs& a, cudaStream_t stream);

// split-KV decode (V2, bf16, d = 128, 8 query heads per KV head)
constexpr int kDecodeChunk = 64;  // keys per pipeline stage
int decode_default_splits(int B, int L, int Hkv);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// split-KV decode, V1 (bf16, d = 64: K rows K_1 | K_2, value rows of 2d), fp32 on the CUDA
// cores; per-head RMSNorm and (1 - lambda_init) scale in the merge
int decode_v1_default_splits(int B, int L, int H);
cudaError_t launch_decode_v1(const DecodeArgs& a, cudaStream_t stream);

}  // namespace diffattn
