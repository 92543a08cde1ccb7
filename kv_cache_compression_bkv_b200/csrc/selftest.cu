// selftest.cu -- a diagnostic of the library's bounded device-side waits.
//
// Every wait in the kernels (sm100.cuh, mbar_wait) gives up after a
// wall-clock limit, records BKV_ERR_TIMEOUT in the device status word and
// lets the kernel wind down, so that a wait that can never be satisfied ends
// instead of hanging the GPU.  bkv_selftest_wait_timeout makes such a wait
// happen on purpose, safely: one warp initialises an mbarrier that nothing
// will ever arrive on, with no TMA load or MMA in flight, and waits on it with
// a short limit through the same wait routine the kernels use.
#include <cuda_runtime.h>

#include "bkv_device_status.cuh"
#include "bkv_internal.h"
#include "sm100.cuh"

BKV_DEFINE_STATUS_ACCESSOR(take_status_selftest)

namespace bkv {
namespace {

using namespace sm100;

constexpr int kWhereSelfTest = 901;

__global__ void selftest_wait_kernel(unsigned long long limit_ns, int *outcome) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);  // one arrival expected; none is ever made
    fence_barrier_init();
  }
  __syncwarp();
  const bool done = mbar_wait_warp_for(b, 0, kWhereSelfTest, limit_ns);
  if (threadIdx.x == 0) *outcome = done ? 1 : 0;
}

}  // namespace
}  // namespace bkv

using namespace bkv;

extern "C" bkv_status bkv_selftest_wait_timeout(int64_t limit_ns, int32_t *outcome,
                                                void *stream) {
  if (limit_ns < 1000 || limit_ns > 100000000 || !outcome ||
      (reinterpret_cast<uintptr_t>(outcome) & 3u))
    return BKV_ERR_INVALID_ARG;
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_ns), outcome);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}
