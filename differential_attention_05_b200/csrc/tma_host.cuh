// tma_host.cuh -- host-side TMA descriptor creation shared by the prefill kernels.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace diffattn {

struct TcMaps {
  CUtensorMap q, k, v;
};

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 4-D bf16 map {C (contiguous), heads, tokens, batch}, box {64, 1, box_rows, 1}, 128-byte
// swizzle, zero fill outside the tensor. Loads start at x in {0, 64}: 16-byte aligned.
inline bool make_map(CUtensorMap* m, const void* ptr, int C, int heads, int N, int B,
                     const int64_t* strides /* batch, token, head (elements) */,
                     int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)heads, (cuuint64_t)N, (cuuint64_t)B};
  int64_t hs = strides[2], ts = strides[1], bs = strides[0];
  // extents of 1 may carry any stride; give TMA a well-formed one
  if (heads == 1) hs = C;
  if (N == 1) ts = hs * heads;
  if (B == 1) bs = ts * N;
  cuuint64_t gstr[3] = {(cuuint64_t)hs * 2, (cuuint64_t)ts * 2, (cuuint64_t)bs * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, gstr, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace diffattn
