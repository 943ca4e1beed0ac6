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
  // variable-length batch (cu_q != nullptr): sequence b is rows cu_q[b] .. cu_q[b+1] of
  // q / out and rows cu_k[b] .. cu_k[b+1] of k / v (packed, batch stride unused); N is then
  // the longest query count the grid covers and total_q / total_k the packed row counts
  const int32_t* cu_q;
  const int32_t* cu_k;
  int total_q, total_k;
  // statistics pass of the backward (launch_prefill_v2_stats, launch_prefill_v1_stats):
  // instead of the output, per (query, unit) the log2-domain log-sum-exps of both branches
  // and delta_b = dO . (A_b V) go to st[((b * units + u) * st_rows + i) * 4 + 0..3], and
  // the row's dlambda share -dO . (A_2 V) to dl[(b * units + u) * N + i]. V2: dO = dy. V1:
  // dO is dy taken back through the per-head norm, written in bf16 to
  // st_do[((b * N + i) * units + u) * 2d + ..] (dense [B, N, H, 2d]); the deltas take that
  // bf16 dO, the dlambda share the fp32 one
  const void* st_dy;
  int64_t st_dys[3];
  float* st;
  float* st_dl;
  int st_rows;
  void* st_do;
  // training forward (launch_prefill_v2_train): the branch-2 output O_2 / l_2 of every
  // (query, pair) in out's layout and dtype, and lse[((b * units + u) * N + i) * 2 + 0..1],
  // the log2-domain log-sum-exps of both branches
  void* tr_o2;
  float* tr_lse;
  // element extents (one past the largest element offset the shapes and strides reach) of
  // q, k, v, out and the statistics-pass tensors, and the bounds-checked build's own status
  // word (see in_bounds in common.cuh; unused by the normal build)
  int64_t ext_q, ext_k, ext_v, ext_out, ext_st_dy, ext_st, ext_st_dl, ext_st_do, ext_tr_lse;
  int* dbg_status;
};

// Resolved backward problem: the forward's arguments plus the incoming gradient dy (the
// layout of out) and the fp32 gradients, dense in the shapes of q, k, v; the workspace
// pointers are set by launch_backward.
struct BwdArgs {
  PrefillArgs f;
  int bf16;                  // q, k, v, dy are bf16 (else fp32)
  const void* dy;
  int64_t dys[3];            // dy strides {batch, token, unit}
  float* dq;
  float* dk;
  float* dv;
  float* dlambda;            // [units]
  float* w_do;               // [B, N, units, dv] gradient reaching O
  float* w_st;               // [B, N, units, 4] lse_1, lse_2, delta_1, delta_2
  float* w_dl;               // [B, units, N] per-row dlambda shares
  void* w_do16;              // V1 tensor-core path: dO in bf16 [B, N, H, 2d]
  // element extents of dq, dk, dv (dense) and of the workspace in floats, which starts at
  // w_base (bounds-checked build, see in_bounds in common.cuh)
  int64_t ext_dq, ext_dk, ext_dv, ext_ws;
  const float* w_base;
};

#ifdef __CUDACC__
// The sequence a tile of batch index b works on: its query and key counts, its first rows
// in the tensors and its batch coordinate. ok = false for inconsistent varlen offsets.
struct SeqRange {
  int nq, nk, qrow0, krow0, bc;
  bool ok;
};

template <bool VARLEN = true>
__device__ __forceinline__ SeqRange seq_range(const PrefillArgs& a, int b) {
  SeqRange r;
  if (!VARLEN || !a.cu_q) {
    r.nq = a.N; r.nk = a.Nk; r.qrow0 = 0; r.krow0 = 0; r.bc = b; r.ok = true;
    return r;
  }
  r.qrow0 = a.cu_q[b];
  r.nq = a.cu_q[b + 1] - r.qrow0;
  r.krow0 = a.cu_k[b];
  r.nk = a.cu_k[b + 1] - r.krow0;
  r.bc = 0;
  r.ok = r.qrow0 >= 0 && r.nq >= 0 && r.nq <= a.N && r.qrow0 <= a.total_q - r.nq &&
         r.krow0 >= 0 && r.nk >= r.nq && r.krow0 <= a.total_k - r.nk;
  return r;
}
#endif

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
  // paged cache (block_table != nullptr): token t of batch entry b is row t % page_size of
  // page block_table[b * bt_stride + t / page_size]; kvs = {page, token, head} strides
  const int32_t* block_table;
  int64_t bt_stride;
  int page_shift;            // log2(page_size)
  int num_pages;
  void* out;
  float* ws_o;   // V2: [B, Hq, splits, d]; V1: [B, H, splits, 2 branches, 2d]
  float* ws_ml;  // V2: [B, Hq, splits, 2];  V1: [B, H, splits, 2 branches, 2]
  int* dev_status;
  // element extents of q, the caches (or page pools), out, the two workspace parts and the
  // block table, and the bounds-checked build's status word (see in_bounds in common.cuh)
  int64_t ext_q, ext_kv, ext_out, ext_ws_o, ext_ws_ml, ext_bt;
  int* dbg_status;
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
cudaError_t launch_prefill_v2_stats(const PrefillArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_v1_stats(const PrefillArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_v2_train(const PrefillArgs& a, cudaStream_t stream);

// split-KV decode (V2, bf16, d = 128, 8 query heads per KV head)
constexpr int kDecodeChunk = 64;  // keys per pipeline stage
int decode_default_splits(int B, int L, int Hkv);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// split-KV decode, V1 (bf16, d = 64: K rows K_1 | K_2, value rows of 2d), fp32 on the CUDA
// cores; per-head RMSNorm and (1 - lambda_init) scale in the merge
int decode_v1_default_splits(int B, int L, int H);
cudaError_t launch_decode_v1(const DecodeArgs& a, cudaStream_t stream);
size_t bwd_workspace_bytes(int B, int N, int units, int dv);
cudaError_t launch_backward(BwdArgs g, void* workspace, cudaStream_t stream);
cudaError_t launch_dlambda_reduce(const BwdArgs& g, cudaStream_t stream);
size_t bwd_tc_workspace_bytes(int variant, int B, int N, int units);
cudaError_t launch_backward_tc(BwdArgs g, void* workspace, cudaStream_t stream);
// the same from a training forward's saved O_2 / l_2 and log-sum-exps (no recompute)
cudaError_t launch_backward_tc_saved(BwdArgs g, const void* out, const void* o2, const float* lse,
                                     void* workspace, cudaStream_t stream);
cudaError_t launch_lambda_bwd(const float* lq1, const float* lk1, const float* lq2,
                              const float* lk2, int n_heads, int dim, const float* dlam,
                              float* dlq1, float* dlk1, float* dlq2, float* dlk2,
                              cudaStream_t stream);

}  // namespace diffattn
