// bkv_device_status.cuh -- the device-side status word of one translation unit.
//
// A kernel that gives up (a bounded wait that ran out, a failed consistency
// check) records a code here instead of trapping; the host reads and clears it
// through bkv_read_device_status().  Each translation unit that includes this
// header owns one copy of the word and exports one host accessor, declared with
// BKV_DEFINE_STATUS_ACCESSOR(name).
#pragma once

#include <cuda_runtime.h>

namespace bkv {

enum : int { BKV_DEV_OK = 0, BKV_DEV_TIMEOUT = 5, BKV_DEV_ASSERT = 6 };

static __device__ int g_bkv_dev_status = 0;
static __device__ int g_bkv_dev_where = 0;

__device__ __forceinline__ void record_device_status(int code, int where) {
  if (atomicCAS(&g_bkv_dev_status, 0, code) == 0) g_bkv_dev_where = where;
}

}  // namespace bkv

// Host accessor: waits for `stream`, returns the recorded code (0 if none) and
// its location tag, and clears both.
#define BKV_DEFINE_STATUS_ACCESSOR(name)                                             \
  namespace bkv {                                                                    \
  int name(cudaStream_t stream, int *where) {                                        \
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;                     \
    int code = 0, loc = 0;                                                           \
    if (cudaMemcpyFromSymbol(&code, g_bkv_dev_status, sizeof(int)) != cudaSuccess)   \
      return -1;                                                                     \
    if (cudaMemcpyFromSymbol(&loc, g_bkv_dev_where, sizeof(int)) != cudaSuccess)     \
      return -1;                                                                     \
    if (code != 0) {                                                                 \
      const int zero = 0;                                                            \
      cudaMemcpyToSymbol(g_bkv_dev_status, &zero, sizeof(int));                      \
      cudaMemcpyToSymbol(g_bkv_dev_where, &zero, sizeof(int));                       \
    }                                                                                \
    if (where) *where = loc;                                                         \
    return code;                                                                     \
  }                                                                                  \
  }
