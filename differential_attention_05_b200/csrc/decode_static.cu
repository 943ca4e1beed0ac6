// decode_static.cu -- the split-KV decode for callers that cannot allocate device memory.
//
// diffattn_fwd_decode needs a caller-provided workspace for its per-split partial softmax
// states. Some callers have no way to provide one at call time: a serving loop that
// works from a device-memory budget fixed at start-up and must not allocate per request,
// or a plugin whose host application owns every device allocation through its own pool.
// This entry point runs the same two decode kernels with the partial states kept in a
// library-owned, file-scope device array instead.
//
// The array is statically sized (kStaticScratchBytes, 16 MiB), so every GPU on which the
// library is loaded holds it until the process exits. Host code may not pass the array's
// symbol to a kernel (in host code that name stands for a host-side shadow, not a device
// address); the device address is looked up once per device with cudaGetSymbolAddress on
// the first call made with that device current, and cached.
#include <mutex>

#include "../../include/diffattn.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

// workspace of diffattn_fwd_decode_static: partial (max, sum, output) per split and head
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DIFFATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return DIFFATTN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DIFFATTN_OK;
}

}  // namespace

extern "C" int diffattn_fwd_decode_static(const diffattn_decode_params* p, const void* q,
                                          const void* k_cache, const void* v_cache,
                                          const int32_t* kv_len, const float* lambda, void* out,
                                          int* dev_status, void* stream) {
  if (!p) return DIFFATTN_ERR_INVALID_ARG;
  // Pick the split count so the partial states fit the static array: the automatic choice
  // when it fits, otherwise fewer splits; an explicit num_splits must fit as given.
  diffattn_decode_params pp = *p;
  size_t need = 0;
  int rc = diffattn_decode_workspace_size(&pp, &need);
  if (rc != DIFFATTN_OK) return rc;
  if (need > kStaticScratchBytes) {
    if (p->num_splits != 0) return DIFFATTN_ERR_WORKSPACE;
    const int cap = p->max_kv_len > 0 ? (p->max_kv_len + diffattn::kDecodeChunk - 1) / diffattn::kDecodeChunk : 1;
    int s = diffattn::decode_default_splits(p->batch, p->max_kv_len, p->n_kv_heads);
    if (s > cap) s = cap;
    for (; s >= 1; --s) {
      pp.num_splits = s;
      rc = diffattn_decode_workspace_size(&pp, &need);
      if (rc != DIFFATTN_OK) return rc;
      if (need <= kStaticScratchBytes) break;
    }
    if (need > kStaticScratchBytes) return DIFFATTN_ERR_WORKSPACE;  // too large even unsplit
  }
  if (p->batch == 0) return DIFFATTN_OK;
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != DIFFATTN_OK) return rc;
  return diffattn_fwd_decode(&pp, q, k_cache, v_cache, kv_len, lambda, out, scratch,
                             kStaticScratchBytes, dev_status, stream);
}
