// api.cu -- the C ABI (include/diffattn.h): host-side validation and dispatch.
// Nothing is launched unless every argument passes; no entry point allocates memory.
#include <math.h>
#include <string.h>

#include "../../include/diffattn.h"
#include "kernels.h"

using namespace diffattn;

namespace {

constexpr int kAbiVersion = 100;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return DIFFATTN_OK;
  if (e == cudaErrorNotSupported) return DIFFATTN_ERR_UNSUPPORTED;
  return DIFFATTN_ERR_CUDA;
}

// The first n strides are non-negative (the kernels address rows as base + index * stride;
// alignment of the strides is checked separately, where the kernel needs it).
inline bool strides_ok(const int64_t* s, int n) {
  for (int i = 0; i < n; ++i)
    if (s[i] < 0) return false;
  return true;
}

// One past the largest element offset of a [nb, rows, heads, width] view with element
// strides {batch, token, head}; 0 for an empty view.
inline int64_t extent(int64_t nb, int64_t rows, int64_t heads, int64_t width, const int64_t* s) {
  if (nb <= 0 || rows <= 0 || heads <= 0 || width <= 0) return 0;
  return (nb - 1) * s[0] + (rows - 1) * s[1] + (heads - 1) * s[2] + width;
}

#ifdef DIFFATTN_DEBUG
// the bounds-checked build's own status word: the number of accesses its checks skipped
__device__ int g_bounds_violations;
int* debug_status_word() {
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_bounds_violations) == cudaSuccess ? static_cast<int*>(p) : nullptr;
}
#else
int* debug_status_word() { return nullptr; }
#endif

}  // namespace

extern "C" {

int diffattn_version(void) { return kAbiVersion; }

int diffattn_debug_bounds_violations(int* count) {
  if (!count) return DIFFATTN_ERR_INVALID_ARG;
  *count = 0;
#ifdef DIFFATTN_DEBUG
  int* p = debug_status_word();
  if (!p) return DIFFATTN_ERR_CUDA;
  if (cudaMemcpy(count, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return DIFFATTN_ERR_CUDA;
  return DIFFATTN_OK;
#else
  return DIFFATTN_ERR_UNSUPPORTED;
#endif
}

const char* diffattn_status_string(int status) {
  switch (status) {
    case DIFFATTN_OK: return "ok";
    case DIFFATTN_ERR_INVALID_ARG: return "invalid argument";
    case DIFFATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case DIFFATTN_ERR_MISALIGNED: return "misaligned pointer or stride";
    case DIFFATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case DIFFATTN_ERR_CUDA: return "CUDA error";
    case DIFFATTN_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int diffattn_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                    int n_heads, int dim, int depth, float* lambda_out, float* lambda_init_out,
                    void* stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !lambda_out) return DIFFATTN_ERR_INVALID_ARG;
  if (n_heads < 1 || n_heads > 65535 || dim < 1 || dim > 4096 || depth < 1)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(lq1) || !aligned16(lk1) || !aligned16(lq2) || !aligned16(lk2))
    return DIFFATTN_ERR_MISALIGNED;
  return from_cuda(launch_lambda(lq1, lk1, lq2, lk2, n_heads, dim, depth, lambda_out,
                                 lambda_init_out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// The body shared by the fixed-length and the variable-length prefill. cu_q = nullptr:
// p->batch sequences of p->seqlen queries and kv_seqlen keys. Otherwise p->batch packed
// sequences with offsets cu_q / cu_k (device), p->seqlen / kv_seqlen the packed row counts
// and max_q the longest query count.
// Checks shared by the forward and the backward and the resolved arguments; *empty is set
// when there is nothing to launch.
static int prefill_setup(const diffattn_prefill_params* p, const int32_t* cu_q, const int32_t* cu_k,
                         int max_q, const void* q, const void* k, const void* v,
                         const float* lambda, const float* lambda_init, const void* out,
                         int* dev_status, PrefillArgs* pa, bool* empty) {
  *empty = false;
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->seqlen < 0 || p->head_dim < 1) return DIFFATTN_ERR_INVALID_ARG;
  if (p->variant != DIFFATTN_V1 && p->variant != DIFFATTN_V2) return DIFFATTN_ERR_INVALID_ARG;
  if (p->dtype != DIFFATTN_F32 && p->dtype != DIFFATTN_BF16) return DIFFATTN_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return DIFFATTN_ERR_INVALID_ARG;
  if (p->apply_norm != 0 && p->apply_norm != 1) return DIFFATTN_ERR_INVALID_ARG;
  const bool varlen = cu_q != nullptr;
  // keys: kv_seqlen (0 reads as seqlen); fixed length needs at least as many keys as
  // queries (chunked prefill); a window only when causal
  const int nk = p->kv_seqlen == 0 ? p->seqlen : p->kv_seqlen;
  if (nk < 0 || (!varlen && nk < p->seqlen) || p->window < 0 || (p->window > 0 && !p->causal))
    return DIFFATTN_ERR_INVALID_ARG;
  if (varlen && (max_q < 0 || !cu_k)) return DIFFATTN_ERR_INVALID_ARG;
  if (!strides_ok(p->q_strides, 3) || !strides_ok(p->k_strides, 3) ||
      !strides_ok(p->v_strides, 3) || !strides_ok(p->o_strides, 3))
    return DIFFATTN_ERR_INVALID_ARG;

  PrefillArgs& a = *pa;
  memset(&a, 0, sizeof(a));
  a.variant = p->variant;
  a.B = p->batch;
  a.N = varlen ? max_q : p->seqlen;
  a.Nk = nk;
  a.window = p->window;
  a.d = p->head_dim;
  a.causal = p->causal;
  a.apply_norm = p->apply_norm;
  a.eps = p->norm_eps;
  if (varlen) {
    a.cu_q = cu_q;
    a.cu_k = cu_k;
    a.total_q = p->seqlen;
    a.total_k = nk;
  }
  if (p->variant == DIFFATTN_V1) {
    if (p->n_q_heads < 1 || p->n_kv_heads != p->n_q_heads) return DIFFATTN_ERR_INVALID_ARG;
    a.units = p->n_q_heads;
    a.Hq = a.Hkv = p->n_q_heads;
    a.group = 1;
    a.dv = 2 * a.d;
  } else {
    if (p->n_q_heads < 2 || p->n_kv_heads < 1 || p->n_q_heads % p->n_kv_heads != 0 ||
        (p->n_q_heads / p->n_kv_heads) % 2 != 0)
      return DIFFATTN_ERR_INVALID_ARG;
    if (p->apply_norm) return DIFFATTN_ERR_INVALID_ARG;  // V2 has no per-head norm
    a.units = p->n_q_heads / 2;
    a.Hq = p->n_q_heads;
    a.Hkv = p->n_kv_heads;
    a.group = p->n_q_heads / p->n_kv_heads;
    a.dv = a.d;
  }
  if (a.apply_norm && !(p->norm_eps >= 0.f && isfinite(p->norm_eps))) return DIFFATTN_ERR_INVALID_ARG;
  if (a.units > 65535 || a.B > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  if (a.B == 0 || a.N == 0 || (varlen && p->seqlen == 0)) {
    *empty = true;
    return DIFFATTN_OK;
  }
  if (!q || !k || !v || !lambda || !out) return DIFFATTN_ERR_INVALID_ARG;
  if (a.apply_norm && !lambda_init) return DIFFATTN_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return DIFFATTN_ERR_MISALIGNED;
  if (varlen && ((reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u)))
    return DIFFATTN_ERR_MISALIGNED;
  const int vec = p->dtype == DIFFATTN_BF16 ? 8 : 4;  // elements per 16 bytes
  for (int i = 0; i < 3; ++i) {
    if (p->q_strides[i] % vec || p->k_strides[i] % vec || p->v_strides[i] % vec ||
        p->o_strides[i] % vec)
      return DIFFATTN_ERR_MISALIGNED;
  }
  memcpy(a.qs, p->q_strides, sizeof(a.qs));
  memcpy(a.ks, p->k_strides, sizeof(a.ks));
  memcpy(a.vs, p->v_strides, sizeof(a.vs));
  memcpy(a.os, p->o_strides, sizeof(a.os));
  a.q = q;
  a.k = k;
  a.v = v;
  a.lambda = lambda;
  a.lambda_init = lambda_init;
  a.out = const_cast<void*>(out);
  a.dev_status = dev_status;
  // element extents (checked by the bounds-checked build): a variable-length batch is one
  // packed sequence of rows
  {
    const int64_t nb = varlen ? 1 : a.B;
    const int64_t rq = varlen ? p->seqlen : a.N, rk = varlen ? nk : a.Nk;
    const int v1 = a.variant == DIFFATTN_V1;
    a.ext_q = extent(nb, rq, v1 ? a.units : a.Hq, v1 ? 2 * a.d : a.d, a.qs);
    a.ext_k = extent(nb, rk, a.Hkv, v1 ? 2 * a.d : a.d, a.ks);
    a.ext_v = extent(nb, rk, a.Hkv, a.dv, a.vs);
    a.ext_out = extent(nb, rq, a.units, a.dv, a.os);
    a.dbg_status = debug_status_word();
  }
  return DIFFATTN_OK;
}

static int prefill_run(const diffattn_prefill_params* p, const int32_t* cu_q, const int32_t* cu_k,
                       int max_q, const void* q, const void* k, const void* v, const float* lambda,
                       const float* lambda_init, void* out, int* dev_status, void* stream) {
  PrefillArgs a;
  bool empty = false;
  const int rc = prefill_setup(p, cu_q, cu_k, max_q, q, k, v, lambda, lambda_init, out, dev_status,
                               &a, &empty);
  if (rc != DIFFATTN_OK || empty) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p->dtype == DIFFATTN_F32) {
    if (a.d > 128 || a.d % 4 != 0) return DIFFATTN_ERR_UNSUPPORTED;
    return from_cuda(launch_prefill_f32(a, s));
  }
  // bf16: tcgen05 kernel (V1: d = 64; V2: d = 128)
  if (p->variant == DIFFATTN_V1 && a.d != 64) return DIFFATTN_ERR_UNSUPPORTED;
  if (p->variant == DIFFATTN_V2 && a.d != 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (a.Nk > (1 << 24) || p->seqlen > (1 << 24)) return DIFFATTN_ERR_UNSUPPORTED;
  return from_cuda(a.variant == DIFFATTN_V1 ? launch_prefill_v1(a, s) : launch_prefill_v2(a, s));
}

extern "C" {

int diffattn_fwd_prefill(const diffattn_prefill_params* p, const void* q, const void* k,
                         const void* v, const float* lambda, const float* lambda_init, void* out,
                         int* dev_status, void* stream) {
  return prefill_run(p, nullptr, nullptr, 0, q, k, v, lambda, lambda_init, out, dev_status, stream);
}

int diffattn_fwd_prefill_varlen(const diffattn_prefill_params* p, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k, int max_seqlen_q, const void* q,
                                const void* k, const void* v, const float* lambda,
                                const float* lambda_init, void* out, int* dev_status,
                                void* stream) {
  if (!cu_seqlens_q || !cu_seqlens_k) return DIFFATTN_ERR_INVALID_ARG;
  return prefill_run(p, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, q, k, v, lambda, lambda_init,
                     out, dev_status, stream);
}

// the tensor-core backward serves bf16 V2 with d = 128 and bf16 V1 with d = 64; everything
// else (fp32 inputs, other d) runs on the exact-fp32 SIMT kernels
static bool bwd_tensor_core(const diffattn_prefill_params* p) {
  return p->dtype == DIFFATTN_BF16 &&
         ((p->variant == DIFFATTN_V2 && p->head_dim == 128) || (p->variant == DIFFATTN_V1 && p->head_dim == 64));
}

// backward: any d <= 128 with d % 4 == 0, f32 or bf16 inputs, fixed-length batches
static int bwd_check(const diffattn_prefill_params* p) {
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  if (p->head_dim > 128 || p->head_dim % 4 != 0) return DIFFATTN_ERR_UNSUPPORTED;
  return DIFFATTN_OK;
}

int diffattn_bwd_workspace_size(const diffattn_prefill_params* p, size_t* bytes) {
  if (!bytes) return DIFFATTN_ERR_INVALID_ARG;
  const int rc = bwd_check(p);
  if (rc != DIFFATTN_OK) return rc;
  if (p->batch < 0 || p->seqlen < 0 || p->head_dim < 1) return DIFFATTN_ERR_INVALID_ARG;
  int units, dv;
  if (p->variant == DIFFATTN_V1) {
    if (p->n_q_heads < 1 || p->n_kv_heads != p->n_q_heads) return DIFFATTN_ERR_INVALID_ARG;
    units = p->n_q_heads;
    dv = 2 * p->head_dim;
  } else if (p->variant == DIFFATTN_V2) {
    if (p->n_q_heads < 2 || p->n_kv_heads < 1 || p->n_q_heads % p->n_kv_heads != 0 ||
        (p->n_q_heads / p->n_kv_heads) % 2 != 0)
      return DIFFATTN_ERR_INVALID_ARG;
    units = p->n_q_heads / 2;
    dv = p->head_dim;
  } else {
    return DIFFATTN_ERR_INVALID_ARG;
  }
  *bytes = bwd_tensor_core(p) ? bwd_tc_workspace_bytes(p->variant, p->batch, p->seqlen, units)
                              : bwd_workspace_bytes(p->batch, p->seqlen, units, dv);
  return DIFFATTN_OK;
}

int diffattn_bwd_prefill(const diffattn_prefill_params* p, const void* q, const void* k,
                         const void* v, const float* lambda, const float* lambda_init,
                         const void* dout, float* dq, float* dk, float* dv, float* dlambda,
                         void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  int rc = bwd_check(p);
  if (rc != DIFFATTN_OK) return rc;
  BwdArgs g;
  memset(&g, 0, sizeof(g));
  bool empty = false;
  rc = prefill_setup(p, nullptr, nullptr, 0, q, k, v, lambda, lambda_init, dout, dev_status, &g.f,
                     &empty);
  if (rc != DIFFATTN_OK || empty) return rc;
  if (!dout || !dq || !dk || !dv || !dlambda) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return DIFFATTN_ERR_MISALIGNED;
  const PrefillArgs& a = g.f;
  const bool tc = bwd_tensor_core(p);
  const size_t need = tc ? bwd_tc_workspace_bytes(a.variant, a.B, a.N, a.units)
                         : bwd_workspace_bytes(a.B, a.N, a.units, a.dv);
  if (!workspace || workspace_bytes < need) return DIFFATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DIFFATTN_ERR_MISALIGNED;
  g.bf16 = p->dtype == DIFFATTN_BF16;
  g.dy = dout;
  memcpy(g.dys, p->o_strides, sizeof(g.dys));
  g.dq = dq;
  g.dk = dk;
  g.dv = dv;
  g.dlambda = dlambda;
  {
    const int v1 = a.variant == DIFFATTN_V1;
    g.ext_dq = (int64_t)a.B * a.N * (v1 ? a.units * 2 * a.d : a.Hq * a.d);
    g.ext_dk = (int64_t)a.B * a.Nk * a.Hkv * (v1 ? 2 * a.d : a.d);
    g.ext_dv = (int64_t)a.B * a.Nk * a.Hkv * a.dv;
    g.ext_ws = (int64_t)(workspace_bytes / sizeof(float));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return from_cuda(tc ? launch_backward_tc(g, workspace, s) : launch_backward(g, workspace, s));
}

int diffattn_fwd_prefill_train(const diffattn_prefill_params* p, const void* q, const void* k,
                               const void* v, const float* lambda, void* out, void* o2, float* lse,
                               int* dev_status, void* stream) {
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  if (p->variant != DIFFATTN_V2 || p->dtype != DIFFATTN_BF16 || p->head_dim != 128)
    return DIFFATTN_ERR_UNSUPPORTED;
  PrefillArgs a;
  bool empty = false;
  int rc = prefill_setup(p, nullptr, nullptr, 0, q, k, v, lambda, nullptr, out, dev_status, &a, &empty);
  if (rc != DIFFATTN_OK || empty) return rc;
  if (!o2 || !lse) return DIFFATTN_ERR_INVALID_ARG;
  if (o2 == out || o2 == q || o2 == k || o2 == v) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(o2) || !aligned16(lse)) return DIFFATTN_ERR_MISALIGNED;
  if (a.Nk > (1 << 24) || p->seqlen > (1 << 24)) return DIFFATTN_ERR_UNSUPPORTED;
  a.tr_o2 = o2;
  a.tr_lse = lse;
  a.ext_tr_lse = (int64_t)a.B * a.units * a.N * 2;
  return from_cuda(launch_prefill_v2_train(a, static_cast<cudaStream_t>(stream)));
}

int diffattn_bwd_prefill_saved(const diffattn_prefill_params* p, const void* q, const void* k,
                               const void* v, const float* lambda, const void* out, const void* o2,
                               const float* lse, const void* dout, float* dq, float* dk, float* dv,
                               float* dlambda, void* workspace, size_t workspace_bytes,
                               int* dev_status, void* stream) {
  int rc = bwd_check(p);
  if (rc != DIFFATTN_OK) return rc;
  if (p->variant != DIFFATTN_V2 || p->dtype != DIFFATTN_BF16 || p->head_dim != 128)
    return DIFFATTN_ERR_UNSUPPORTED;
  BwdArgs g;
  memset(&g, 0, sizeof(g));
  bool empty = false;
  rc = prefill_setup(p, nullptr, nullptr, 0, q, k, v, lambda, nullptr, dout, dev_status, &g.f, &empty);
  if (rc != DIFFATTN_OK || empty) return rc;
  if (!out || !o2 || !lse || !dout || !dq || !dk || !dv || !dlambda) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(o2) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return DIFFATTN_ERR_MISALIGNED;
  const PrefillArgs& a = g.f;
  const size_t need = bwd_tc_workspace_bytes(DIFFATTN_V2, a.B, a.N, a.units);
  if (!workspace || workspace_bytes < need) return DIFFATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DIFFATTN_ERR_MISALIGNED;
  g.bf16 = 1;
  g.dy = dout;
  memcpy(g.dys, p->o_strides, sizeof(g.dys));
  g.dq = dq;
  g.dk = dk;
  g.dv = dv;
  g.dlambda = dlambda;
  g.ext_dq = (int64_t)a.B * a.N * a.Hq * a.d;
  g.ext_dk = (int64_t)a.B * a.Nk * a.Hkv * a.d;
  g.ext_dv = (int64_t)a.B * a.Nk * a.Hkv * a.dv;
  g.ext_ws = (int64_t)(workspace_bytes / sizeof(float));
  return from_cuda(launch_backward_tc_saved(g, out, o2, lse, workspace, static_cast<cudaStream_t>(stream)));
}

int diffattn_lambda_bwd(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                        int n_heads, int dim, const float* dlambda, float* dlq1, float* dlk1,
                        float* dlq2, float* dlk2, void* stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !dlambda || !dlq1 || !dlk1 || !dlq2 || !dlk2)
    return DIFFATTN_ERR_INVALID_ARG;
  if (n_heads < 1 || n_heads > 65535 || dim < 1 || dim > 4096) return DIFFATTN_ERR_INVALID_ARG;
  return from_cuda(launch_lambda_bwd(lq1, lk1, lq2, lk2, n_heads, dim, dlambda, dlq1, dlk1, dlq2,
                                     dlk2, static_cast<cudaStream_t>(stream)));
}

static int decode_check(const diffattn_decode_params* p, int* splits, int* split_len) {
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->max_kv_len < 0 || p->n_q_heads < 1 || p->n_kv_heads < 1 ||
      p->head_dim < 1 || p->num_splits < 0)
    return DIFFATTN_ERR_INVALID_ARG;
  if (p->variant != DIFFATTN_V2) return p->variant == DIFFATTN_V1 ? DIFFATTN_ERR_UNSUPPORTED
                                                                  : DIFFATTN_ERR_INVALID_ARG;
  if (p->dtype != DIFFATTN_BF16) return p->dtype == DIFFATTN_F32 ? DIFFATTN_ERR_UNSUPPORTED
                                                                 : DIFFATTN_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0 || (p->n_q_heads / p->n_kv_heads) % 2 != 0)
    return DIFFATTN_ERR_INVALID_ARG;
  if (p->n_q_heads / p->n_kv_heads != 8 || p->head_dim != 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (!strides_ok(p->q_strides, 2) || !strides_ok(p->kv_strides, 3) || !strides_ok(p->o_strides, 2))
    return DIFFATTN_ERR_INVALID_ARG;
  if (p->batch > 65535 || p->n_kv_heads > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  int s = p->num_splits ? p->num_splits : decode_default_splits(p->batch, p->max_kv_len, p->n_kv_heads);
  const int L = p->max_kv_len;
  int len = (L + s - 1) / (s > 0 ? s : 1);
  len = ((len + kDecodeChunk - 1) / kDecodeChunk) * kDecodeChunk;
  if (len < kDecodeChunk) len = kDecodeChunk;
  s = (L + len - 1) / len;
  if (s < 1) s = 1;
  if (s > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  *splits = s;
  *split_len = len;
  return DIFFATTN_OK;
}

// V1 decode: one (K_1 | K_2, V) cache per differential head, d = 64.
static int decode_v1_check(const diffattn_decode_params* p, int* splits, int* split_len) {
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->max_kv_len < 0 || p->n_q_heads < 1 || p->n_kv_heads < 1 ||
      p->head_dim < 1 || p->num_splits < 0)
    return DIFFATTN_ERR_INVALID_ARG;
  if (p->variant != DIFFATTN_V1) return DIFFATTN_ERR_INVALID_ARG;
  if (p->dtype != DIFFATTN_BF16) return p->dtype == DIFFATTN_F32 ? DIFFATTN_ERR_UNSUPPORTED
                                                                 : DIFFATTN_ERR_INVALID_ARG;
  if (p->n_q_heads != p->n_kv_heads) return DIFFATTN_ERR_INVALID_ARG;  // one cache per head
  if (p->head_dim != 64) return DIFFATTN_ERR_UNSUPPORTED;
  if (!strides_ok(p->q_strides, 2) || !strides_ok(p->kv_strides, 3) || !strides_ok(p->o_strides, 2))
    return DIFFATTN_ERR_INVALID_ARG;
  if (p->batch > 65535 || p->n_q_heads > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  int s = p->num_splits ? p->num_splits
                        : decode_v1_default_splits(p->batch, p->max_kv_len, p->n_q_heads);
  const int L = p->max_kv_len;
  int len = (L + s - 1) / (s > 0 ? s : 1);
  len = ((len + kDecodeChunk - 1) / kDecodeChunk) * kDecodeChunk;
  if (len < kDecodeChunk) len = kDecodeChunk;
  s = (L + len - 1) / len;
  if (s < 1) s = 1;
  if (s > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  *splits = s;
  *split_len = len;
  return DIFFATTN_OK;
}

static size_t decode_ws_bytes(const diffattn_decode_params* p, int splits) {
  if (p->variant == DIFFATTN_V1) {
    // per (b, h, split) and branch: 2d partial outputs, then (max, sum)
    const size_t recs = (size_t)p->batch * p->n_q_heads * splits * 2;
    const size_t o_bytes = ((recs * 2 * p->head_dim * sizeof(float)) + 255) & ~(size_t)255;
    return o_bytes + recs * 2 * sizeof(float);
  }
  const size_t recs = (size_t)p->batch * p->n_q_heads * splits;
  const size_t o_bytes = ((recs * p->head_dim * sizeof(float)) + 255) & ~(size_t)255;
  return o_bytes + recs * 2 * sizeof(float);
}

int diffattn_decode_workspace_size(const diffattn_decode_params* p, size_t* bytes) {
  if (!bytes) return DIFFATTN_ERR_INVALID_ARG;
  int splits = 0, len = 0;
  int rc = (p && p->variant == DIFFATTN_V1) ? decode_v1_check(p, &splits, &len)
                                            : decode_check(p, &splits, &len);
  if (rc != DIFFATTN_OK) return rc;
  *bytes = decode_ws_bytes(p, splits);
  return DIFFATTN_OK;
}

}  // extern "C"

// The body shared by the decode entry points: checks by variant, the paged-cache checks
// when pk is given, then the launch.
static int decode_run(const diffattn_decode_params* p, const diffattn_paged_kv* pk,
                      const void* q, const void* k, const void* v, const int32_t* block_table,
                      const int32_t* kv_len, const float* lambda, const float* lambda_init,
                      int apply_norm, float norm_eps, void* out, void* workspace,
                      size_t workspace_bytes, int* dev_status, void* stream) {
  int splits = 0, len = 0;
  const bool v1 = p->variant == DIFFATTN_V1;
  int rc = v1 ? decode_v1_check(p, &splits, &len) : decode_check(p, &splits, &len);
  if (rc != DIFFATTN_OK) return rc;
  if (apply_norm != 0 && apply_norm != 1) return DIFFATTN_ERR_INVALID_ARG;
  if (!v1 && apply_norm) return DIFFATTN_ERR_INVALID_ARG;  // V2 has no per-head norm
  if (apply_norm && !(norm_eps >= 0.f && isfinite(norm_eps))) return DIFFATTN_ERR_INVALID_ARG;
  int page_shift = 0;
  if (pk) {
    if (pk->page_size < 1 || pk->page_size > 65536 || (pk->page_size & (pk->page_size - 1)))
      return DIFFATTN_ERR_INVALID_ARG;
    if (pk->num_pages < 1 || pk->max_pages_per_seq < 1 || pk->reserved != 0 ||
        !strides_ok(pk->page_strides, 3))
      return DIFFATTN_ERR_INVALID_ARG;
    if ((int64_t)pk->max_pages_per_seq * pk->page_size < p->max_kv_len) return DIFFATTN_ERR_INVALID_ARG;
    while ((1 << page_shift) < pk->page_size) ++page_shift;
  }
  if (p->batch == 0) return DIFFATTN_OK;
  if (!q || !k || !v || !lambda || !out) return DIFFATTN_ERR_INVALID_ARG;
  if (pk && !block_table) return DIFFATTN_ERR_INVALID_ARG;
  if (apply_norm && !lambda_init) return DIFFATTN_ERR_INVALID_ARG;
  const size_t need = decode_ws_bytes(p, splits);
  if (!workspace || workspace_bytes < need) return DIFFATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DIFFATTN_ERR_MISALIGNED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return DIFFATTN_ERR_MISALIGNED;
  const int64_t* kvs = pk ? pk->page_strides : p->kv_strides;
  if (p->q_strides[0] % 8 || p->q_strides[1] % 8 || kvs[0] % 8 || kvs[1] % 8 || kvs[2] % 8 ||
      p->o_strides[0] % 8 || p->o_strides[1] % 8)
    return DIFFATTN_ERR_MISALIGNED;
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.B = p->batch;
  a.L = p->max_kv_len;
  a.Hq = p->n_q_heads;
  a.Hkv = p->n_kv_heads;
  a.d = p->head_dim;
  a.splits = splits;
  a.split_len = len;
  memcpy(a.qs, p->q_strides, sizeof(a.qs));
  memcpy(a.kvs, kvs, sizeof(a.kvs));
  memcpy(a.os, p->o_strides, sizeof(a.os));
  a.q = q;
  a.k = k;
  a.v = v;
  a.kv_len = kv_len;
  a.lambda = lambda;
  a.lambda_init = lambda_init;
  a.apply_norm = apply_norm;
  a.eps = norm_eps;
  a.out = out;
  if (pk) {
    a.block_table = block_table;
    a.bt_stride = pk->max_pages_per_seq;
    a.page_shift = page_shift;
    a.num_pages = pk->num_pages;
  }
  // per (b, head, split): V2 one record of d floats; V1 two (one per branch) of 2d
  const size_t recs = (size_t)a.B * a.Hq * splits * (v1 ? 2 : 1);
  const size_t rec_floats = v1 ? 2 * (size_t)a.d : (size_t)a.d;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                     (((recs * rec_floats * sizeof(float)) + 255) & ~(size_t)255));
  a.dev_status = dev_status;
  // element extents (checked by the bounds-checked build)
  {
    const int64_t qh[3] = {p->q_strides[0], 0, p->q_strides[1]};  // [B, 1, heads, width]
    const int64_t oh[3] = {p->o_strides[0], 0, p->o_strides[1]};
    const int width = v1 ? 2 * a.d : a.d;
    a.ext_q = extent(a.B, 1, a.Hq, width, qh);
    a.ext_kv = pk ? extent(pk->num_pages, pk->page_size, a.Hkv, width, kvs)
                  : extent(a.B, a.L, a.Hkv, width, kvs);
    a.ext_out = extent(a.B, 1, v1 ? a.Hq : a.Hq / 2, width, oh);
    a.ext_ws_o = (int64_t)(recs * rec_floats);
    a.ext_ws_ml = (int64_t)(recs * 2);
    a.ext_bt = pk ? (int64_t)a.B * pk->max_pages_per_seq : 0;
    a.dbg_status = debug_status_word();
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return from_cuda(v1 ? launch_decode_v1(a, s) : launch_decode(a, s));
}

extern "C" {

int diffattn_fwd_decode(const diffattn_decode_params* p, const void* q, const void* k_cache,
                        const void* v_cache, const int32_t* kv_len, const float* lambda, void* out,
                        void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  if (p->variant != DIFFATTN_V2) return p->variant == DIFFATTN_V1 ? DIFFATTN_ERR_UNSUPPORTED
                                                                  : DIFFATTN_ERR_INVALID_ARG;
  return decode_run(p, nullptr, q, k_cache, v_cache, nullptr, kv_len, lambda, nullptr, 0, 0.f, out,
                    workspace, workspace_bytes, dev_status, stream);
}

int diffattn_fwd_decode_v1(const diffattn_decode_params* p, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* kv_len, const float* lambda,
                           const float* lambda_init, int apply_norm, float norm_eps, void* out,
                           void* workspace, size_t workspace_bytes, int* dev_status,
                           void* stream) {
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  if (p->variant != DIFFATTN_V1) return DIFFATTN_ERR_INVALID_ARG;
  return decode_run(p, nullptr, q, k_cache, v_cache, nullptr, kv_len, lambda, lambda_init,
                    apply_norm, norm_eps, out, workspace, workspace_bytes, dev_status, stream);
}

int diffattn_fwd_decode_paged(const diffattn_decode_params* p, const diffattn_paged_kv* pk,
                              const void* q, const void* k_pages, const void* v_pages,
                              const int32_t* block_table, const int32_t* kv_len,
                              const float* lambda, const float* lambda_init, int apply_norm,
                              float norm_eps, void* out, void* workspace, size_t workspace_bytes,
                              int* dev_status, void* stream) {
  if (!p || !pk) return DIFFATTN_ERR_INVALID_ARG;
  if (p->variant != DIFFATTN_V1 && p->variant != DIFFATTN_V2) return DIFFATTN_ERR_INVALID_ARG;
  return decode_run(p, pk, q, k_pages, v_pages, block_table, kv_len, lambda, lambda_init,
                    apply_norm, norm_eps, out, workspace, workspace_bytes, dev_status, stream);
}

}  // extern "C"
