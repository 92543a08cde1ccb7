// score_noalloc.cu -- bkv_score for callers that cannot allocate device memory.
//
// bkv_score keeps its intermediate results (each observation row's softmax
// normaliser and the per-group partial maxima) in a workspace the caller
// allocates.  Some callers have no way to do that where they score: code that
// runs inside another runtime's execute callback, which hands over only the
// tensors it was asked for; or a serving loop that must not allocate once it
// has started, because a pool allocator has reserved the device's memory.
// For them this file holds one fixed scratch array, compiled into the library,
// and an entry point that runs bkv_score on it.  Every GPU that loads the
// library keeps the array (BKV_SCORE_NOALLOC_SCRATCH_BYTES) until the process
// exits.  Nothing here allocates: the array is part of the loaded module.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "bkv_internal.h"

namespace {

constexpr size_t kScratchBytes = BKV_SCORE_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only a handle for the CUDA
// runtime, not a device address: a kernel must be given the address looked up
// below, never the symbol.
static __device__ __align__(256) unsigned char g_score_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[64];                 // device address of g_score_scratch per device
unsigned long long g_scratch_ctx[64];     // the context that address belongs to

// Unique id of the calling thread's current CUDA context (0 when there is
// none yet or the driver cannot say).  A device reset replaces the context,
// and with it the module that holds the scratch array, so a cached address is
// only good while the id is unchanged.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch on the current device.  It is looked up with
// that device current on the first call, and again whenever the device's
// context has changed since (after a cudaDeviceReset, for one).
bkv_status scratch_on_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long ctx = current_context_id();
  if (g_scratch_addr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // do not leave the error for the caller's next call
      return BKV_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();  // the lookup made the context current
  }
  *out = g_scratch_addr[dev];
  return BKV_OK;
}

}  // namespace

extern "C" bkv_status bkv_score_noalloc(const bkv_cache_desc *desc, const void *k, int64_t L,
                                        const void *recent_q, int32_t R, const void *beacons,
                                        int32_t n_beacons, int32_t M, float scale,
                                        float *scores, void *stream) {
  void *scratch = nullptr;
  const bkv_status st = scratch_on_current_device(&scratch);
  if (st != BKV_OK) return st;
  // bkv_score checks every argument on the host and returns BKV_ERR_WORKSPACE,
  // before launching anything, when the problem needs more scratch than the
  // array holds.  Every scratch element it reads was written earlier in the
  // same call, so the previous call's contents never need clearing.
  return bkv_score(desc, k, L, recent_q, R, beacons, n_beacons, M, scale, scores, scratch,
                   kScratchBytes, stream);
}
