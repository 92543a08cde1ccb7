// compact.cu -- eviction of the unselected KV pairs (BeaconKV abstract and
// Fig. 5(a)): the kept K and V rows are gathered into a dense new cache.
//
// A pure byte copy, bound by HBM bandwidth.  Each thread moves 16-byte
// vectors; consecutive threads cover consecutive 16-byte chunks of a row, so
// every row is read and written by full, aligned 32-byte sectors.  Each thread
// keeps several rows' loads in flight before storing (kUnroll) so that enough
// bytes are outstanding per SM to cover HBM latency.
#include <cuda_runtime.h>

#include <algorithm>

#include "bkv_internal.h"

namespace bkv {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(uint4 *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

template <bool kHasK, bool kHasV>
__global__ void __launch_bounds__(kThreads) compact_kernel(const CompactArgs a) {
  const int chunks = a.row_bytes >> 4;
  const long long total = static_cast<long long>(a.n_heads) * a.n_keep * chunks;
  const long long stride = static_cast<long long>(gridDim.x) * kThreads;
  for (long long e0 = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x; e0 < total;
       e0 += stride * kUnroll) {
    uint4 kv[kUnroll], vv[kUnroll];
    long long dst_off[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = e0 + u * stride;
      dst_off[u] = -1;
      if (e < total) {
        const long long row = e / chunks;
        const int c = static_cast<int>(e - row * chunks);
        const long long h = row / a.n_keep;
        const long long i = row - h * a.n_keep;
        const long long src_row = a.idx ? static_cast<long long>(a.idx[row]) : i;
        const long long src_off = (h * a.src_cap + src_row) * a.row_bytes + c * 16;
        dst_off[u] = (h * a.dst_cap + i) * a.row_bytes + c * 16;
        if (kHasK) kv[u] = ld_stream(reinterpret_cast<const uint4 *>(a.k_src + src_off));
        if (kHasV) vv[u] = ld_stream(reinterpret_cast<const uint4 *>(a.v_src + src_off));
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (dst_off[u] < 0) continue;
      if (kHasK) st_stream(reinterpret_cast<uint4 *>(a.k_dst + dst_off[u]), kv[u]);
      if (kHasV) st_stream(reinterpret_cast<uint4 *>(a.v_dst + dst_off[u]), vv[u]);
    }
  }
}

}  // namespace

bkv_status launch_compact(const CompactArgs &a, cudaStream_t stream) {
  const long long total = static_cast<long long>(a.n_heads) * a.n_keep * (a.row_bytes >> 4);
  if (total == 0) return BKV_OK;
  const long long want = (total + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  const unsigned blocks = static_cast<unsigned>(std::min<long long>(want, 148LL * 8));
  const bool hk = a.k_src != nullptr, hv = a.v_src != nullptr;
  if (hk && hv)
    compact_kernel<true, true><<<blocks, kThreads, 0, stream>>>(a);
  else if (hk)
    compact_kernel<true, false><<<blocks, kThreads, 0, stream>>>(a);
  else if (hv)
    compact_kernel<false, true><<<blocks, kThreads, 0, stream>>>(a);
  else
    return BKV_OK;
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace bkv
