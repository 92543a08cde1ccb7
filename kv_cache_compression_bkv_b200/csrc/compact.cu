// compact.cu -- eviction of the unselected KV pairs (BeaconKV abstract and
// Fig. 5(a)): the kept K and V rows are gathered into a dense new cache.
//
// A pure byte copy, bound by HBM bandwidth.  A kept position outside the
// source cache is never followed: its row is skipped and reported as a failed
// device-side check.  Each thread moves 16-byte
// vectors; consecutive threads cover consecutive 16-byte chunks of a row, so
// every row is read and written by full, aligned 32-byte sectors.  Each thread
// keeps several rows' loads in flight before storing (kUnroll) so that enough
// bytes are outstanding per SM to cover HBM latency.
//
// In place (the destination is the source cache): row i takes row idx_i with
// idx_i >= i, which holds for any ascending list of kept positions.  One CTA
// per (head, K or V) walks its rows in chunks in increasing i; a chunk is
// read whole into registers, the CTA synchronises, then it is written.  A
// row read by chunk c lies at or past the chunk's
// first row, so it is either in chunk c (written only after the barrier) or
// in a later chunk (written only after chunk c's reads have returned); rows
// written by chunk c lie before every row a later chunk reads.  Rows already
// in place are skipped.  A chunk is at most 32 KB (128 rows of 256 bytes).
#include <cuda_runtime.h>

#include <algorithm>

#include "bkv_device_status.cuh"
#include "bkv_internal.h"

BKV_DEFINE_STATUS_ACCESSOR(take_status_compact)

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
        if (src_row < 0 || src_row >= a.src_cap) {
          // a position outside the source cache: report it and leave the
          // destination row as it is rather than read out of bounds
          if (c == 0) record_device_status(BKV_DEV_ASSERT, 502);
          continue;
        }
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

constexpr int kInplaceThreads = 256;
constexpr int kInplacePer = 8;  // 16-byte pieces per thread and chunk (32 KB chunks)
constexpr int kInplaceMaxRows = kInplacePer * kInplaceThreads;  // rows per chunk, 16-byte rows
// CTAs resident per SM: every (head, K or V) of a step runs at once up to
// 5 x 148 = 740 of them (640 at the 14B shape).  A CTA walks its head's
// chunks in order, so a CTA left for a second wave would take the whole
// head's time again; at 4 per SM (62 registers) the 14B shape's 640 CTAs
// took 0.59 ms against 0.33 ms for the out-of-place copy.
constexpr int kInplaceCtasPerSm = 5;

// Each chunk is read whole into registers, the CTA synchronises, and the
// chunk is written.  The kept positions of the next chunk are fetched into
// shared memory while the chunk's rows are in flight, so a chunk waits for
// one load latency rather than two (position, then row).  kChunks: the
// number of 16-byte pieces per row when the kernel is built for it (it
// divides the CTA's threads, so each thread keeps one piece column and its
// rows are a fixed stride apart, and a head's slice is below 4 GB, so byte
// offsets within it take 32 bits); 0 for any row size.
template <int kChunks>
__global__ void __launch_bounds__(kInplaceThreads, kInplaceCtasPerSm)
    compact_inplace_kernel(const CompactArgs a) {
  constexpr bool kEven = kChunks > 0;
  static_assert(!kEven || kInplaceThreads % kChunks == 0, "pieces must divide the threads");
  __shared__ int32_t s_idx[2][kInplaceMaxRows];
  const int head = blockIdx.x;
  uint8_t *base = (blockIdx.y == 0 ? a.k_dst : a.v_dst) + static_cast<size_t>(head) * a.dst_cap * a.row_bytes;
  const int32_t *idx = a.idx + static_cast<size_t>(head) * a.n_keep;
  // kept positions are int32, so every row index fits in 32 bits (the
  // launcher checks n_keep and the capacity)
  const int n_keep = static_cast<int>(a.n_keep), cap = static_cast<int>(a.dst_cap);
  const int chunks = kEven ? kChunks : a.row_bytes >> 4;  // 16-byte pieces per row
  const int rows = kInplacePer * kInplaceThreads / chunks;  // rows per chunk
  const int per_chunk = rows * chunks;
  // piece u of this thread: row ri(u) of the chunk, 16-byte column col(u)
  auto ri = [&](int u) {
    return kEven ? static_cast<int>(threadIdx.x) / kChunks + u * (kInplaceThreads / kChunks)
                 : (static_cast<int>(threadIdx.x) + u * kInplaceThreads) / chunks;
  };
  auto col = [&](int u) {
    return kEven ? static_cast<int>(threadIdx.x) % kChunks
                 : (static_cast<int>(threadIdx.x) + u * kInplaceThreads) % chunks;
  };
  for (int r = threadIdx.x; r < rows; r += kInplaceThreads)
    if (r < n_keep) s_idx[0][r] = idx[r];
  __syncthreads();
  int buf = 0;
  for (int i0 = 0; i0 < n_keep; i0 += rows, buf ^= 1) {
    uint4 v[kInplacePer];
    uint32_t moved = 0u;  // bit u: piece u is read here and written below
    bool bad = false;     // a kept position below its slot or past the cache
#pragma unroll
    for (int u = 0; u < kInplacePer; ++u) {
      if (!kEven && static_cast<int>(threadIdx.x) + u * kInplaceThreads >= per_chunk) continue;
      const int i = i0 + ri(u);
      if (i >= n_keep) continue;
      const int src = s_idx[buf][ri(u)];
      if (src < i || src >= cap) {
        bad = true;
        continue;
      }
      if (src == i) continue;  // already in place
      // L2-coherent load: this kernel writes the same buffer
      const size_t off =
          kEven ? static_cast<size_t>(static_cast<uint32_t>(src) * (kChunks * 16u) +
                                      static_cast<uint32_t>(col(u) * 16))
                : static_cast<size_t>(src) * a.row_bytes + col(u) * 16;
      v[u] = __ldcg(reinterpret_cast<const uint4 *>(base + off));
      moved |= 1u << u;
    }
    // the next chunk's positions (the other buffer was last read before the
    // previous barrier)
    for (int r = threadIdx.x; r < rows; r += kInplaceThreads)
      if (i0 + rows + r < n_keep) s_idx[buf ^ 1][r] = idx[i0 + rows + r];
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kInplacePer; ++u) {
      if (!((moved >> u) & 1u)) continue;
      const int i = i0 + ri(u);
      const size_t off =
          kEven ? static_cast<size_t>(static_cast<uint32_t>(i) * (kChunks * 16u) +
                                      static_cast<uint32_t>(col(u) * 16))
                : static_cast<size_t>(i) * a.row_bytes + col(u) * 16;
      __stcg(reinterpret_cast<uint4 *>(base + off), v[u]);
    }
    // reported once the chunk's data is out of registers
    if (bad) record_device_status(BKV_DEV_ASSERT, 501);
  }
}

}  // namespace

bkv_status launch_compact_inplace(const CompactArgs &a, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  if (a.n_keep == 0 || a.n_heads == 0) return BKV_OK;
  if (a.row_bytes < 16 || a.row_bytes > 16 * kInplacePer * kInplaceThreads) return BKV_ERR_UNSUPPORTED;
  if (a.dst_cap > INT32_MAX || a.n_keep > a.dst_cap) return BKV_ERR_INVALID_ARG;
  dim3 grid(static_cast<unsigned>(a.n_heads), a.v_dst != nullptr ? 2u : 1u);
  if (a.k_dst == nullptr) return BKV_ERR_INVALID_ARG;
  const bool off32 = static_cast<unsigned long long>(a.dst_cap) * a.row_bytes <= 0xffffffffull;
  switch (off32 ? a.row_bytes : 0) {
    case 128: compact_inplace_kernel<8><<<grid, kInplaceThreads, 0, stream>>>(a); break;
    case 256: compact_inplace_kernel<16><<<grid, kInplaceThreads, 0, stream>>>(a); break;
    case 512: compact_inplace_kernel<32><<<grid, kInplaceThreads, 0, stream>>>(a); break;
    case 1024: compact_inplace_kernel<64><<<grid, kInplaceThreads, 0, stream>>>(a); break;
    default: compact_inplace_kernel<0><<<grid, kInplaceThreads, 0, stream>>>(a); break;
  }
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

bkv_status launch_compact(const CompactArgs &a, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
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
