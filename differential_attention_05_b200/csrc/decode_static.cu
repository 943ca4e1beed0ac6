// decode_static.cu -- the split-KV decode for callers that cannot allocate device memory.
//
// diffattn_fwd_decode needs a caller-provided workspace for its per-split partial softmax
// states. Some callers have no way to provide one at call time: a serving loop that
// works from a device-memory budget fixed at start-up and must not allocate per request,
// or a plugin whose host application owns every device allocation through its own pool.
// This entry point runs the same two decode kernels with the partial states kept in a
// library-owned, file-scope device array instead.
//
// The array is statically sized (kStaticScratchBytes, 16 MiB). CUDA loads a library's
// device code lazily by default (CUDA_MODULE_LOADING=LAZY), so the array's device memory is
// committed when this file's module is first loaded on a device -- by the first call of this
// entry point there -- and is held until the process exits (with
// CUDA_MODULE_LOADING=EAGER, when the library's context starts). Host code may not pass the
// array's symbol to a kernel (in host code that name stands for a host-side shadow, not a
// device address); the device address is looked up with cudaGetSymbolAddress on the first
// call made with a device current, and cached per device together with the identity of the
// device's current context, so that a context created after a device reset gets a fresh
// lookup instead of a stale address.
#include <cudaTypedefs.h>

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
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context the cached address belongs to

// Unique id of the calling thread's current CUDA context (the driver's cuCtxGetId, reached
// through the runtime's driver entry points); false if it cannot be read.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  if (!get_current || !get_id) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_decode_scratch on the current device: looked up once per device and
// context (cudaGetSymbolAddress, with that device current), then taken from the cache.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DIFFATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long ctx = 0;
  const bool have_ctx = g_scratch_addr[dev] && current_context_id(&ctx);
  if (!have_ctx || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);  // makes the context current
    if (e != cudaSuccess || p == nullptr) return DIFFATTN_ERR_CUDA;
    if (!current_context_id(&ctx)) ctx = 0;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx;
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
