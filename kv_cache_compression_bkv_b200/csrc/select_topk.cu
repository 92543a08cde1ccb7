// select_topk.cu -- top-K budget selection (BeaconKV Fig. 5(c); Table 1's
// "maximum KV cache budget").
//
// One CTA of 512 threads per row, all rows resident at once (a few CTAs per
// SM, ~8 KB of shared memory each).  Scores become order-preserving unsigned
// keys (larger score -> larger key; -0 and +0 map to one key).  The row is
// never staged: every pass re-reads it (from L2 after the first) and rebuilds
// the keys, which for the step's max form also merges the observation
// groups' partial maxima.  Three MSB-first radix passes with 11-, 11- and
// 10-bit digits (one shared histogram, block-wide scan of its bins) find the
// K-th largest key T and how many keys equal to T are kept; two more passes
// write the kept positions in ascending order: each warp owns a contiguous
// slice of the row, counts its keys above T and equal to T, the warps' slices
// are placed by a prefix sum, and each warp then emits its kept positions in
// order with ballots -- every key > T, plus the first `need_eq` keys equal to
// T (ties go to the lower position).
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "bkv_device_status.cuh"
#include "bkv_internal.h"

BKV_DEFINE_STATUS_ACCESSOR(take_status_select)

namespace bkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBins = 2048;  // 11-bit digits

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;  // -0 -> +0
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float load_key_value(const SelectInput &in, size_t off) {
  float v = in.src[off];
  if (in.mean) {
    for (int p = 1; p < in.n_parts; ++p) v += in.src[p * in.part_stride + off];
    return v * in.inv_count;
  }
  for (int p = 1; p < in.n_parts; ++p) v = fmaxf(v, in.src[p * in.part_stride + off]);
  return v;
}

// The score a key stands for: the max form keeps log-domain maxima.
__device__ __forceinline__ float score_of_key(const SelectInput &in, float v) {
  return in.mean ? v : expf(v);
}

// Exclusive prefix sum over the block of one value per thread; returns the
// thread's exclusive prefix and leaves the total in *total (all threads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *wsum,
                                                         uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t wpre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t x = wsum[w];
    if (w < warp) wpre += x;
    tot += x;
  }
  __syncthreads();  // wsum is reused by the caller's next scan
  *total = tot;
  return wpre + incl - v;
}

__global__ void __launch_bounds__(kThreads)
    select_topk_kernel(const SelectInput in, long long L, long long K, int32_t *__restrict__ idx,
                       float *__restrict__ s_out) {
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t wcnt[2][kWarps];
  __shared__ long long sel[2];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t rbase = static_cast<size_t>(row) * static_cast<size_t>(L);

  // ---- radix select of the K-th largest key: bits [lo, hi) per pass
  uint32_t prefix = 0, mask = 0;
  long long krem = K;  // rank of the wanted key among those matching the prefix
  for (int hi = 32; hi > 0;) {
    const int lo = hi > 11 ? hi - 11 : 0;
    const int nbits = hi - lo;
    const uint32_t dmask = (1u << nbits) - 1u;
    const int nb = 1 << nbits;
    for (int b = tid; b < nb; b += kThreads) hist[b] = 0u;
    __syncthreads();
    for (long long j = tid; j < L; j += kThreads) {
      const float v = load_key_value(in, rbase + j);
      if (hi == 32 && s_out) s_out[rbase + j] = score_of_key(in, v);
      const uint32_t key = order_key(v);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> lo) & dmask], 1u);
    }
    __syncthreads();
    // bins in descending digit order, 4 per thread: thread t holds digits
    // nb-1-4t .. nb-4-4t
    uint32_t c4[4], local = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int d = nb - 1 - 4 * tid - q;
      c4[q] = d >= 0 ? hist[d] : 0u;
      local += c4[q];
    }
    uint32_t total;
    const uint32_t excl = block_exclusive_scan(local, wsum, &total);
    if (static_cast<long long>(excl) < krem && krem <= static_cast<long long>(excl + local)) {
      uint32_t acc = excl;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (static_cast<long long>(acc + c4[q]) >= krem) {
          sel[0] = nb - 1 - 4 * tid - q;
          sel[1] = acc;
          break;
        }
        acc += c4[q];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel[0]) << lo;
    mask |= dmask << lo;
    krem -= sel[1];
    hi = lo;
    __syncthreads();  // sel and hist are rewritten by the next pass
  }
  const uint32_t T = prefix;
  const long long need_eq = krem;  // keys equal to T that are kept

  // ---- ordered emission: warp w owns positions [w * chunk, (w + 1) * chunk)
  const long long chunk = (L + 32 * kWarps - 1) / (32 * kWarps) * 32;
  const long long j0 = warp * chunk, j1 = min(L, j0 + chunk);
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t n_gt = 0, n_eq = 0;
  for (long long base = j0; base < j1; base += 32) {
    const long long j = base + lane;
    const uint32_t key = j < j1 ? order_key(load_key_value(in, rbase + j)) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, j < j1 && key > T));
    n_eq += __popc(__ballot_sync(0xffffffffu, j < j1 && key == T));
  }
  if (lane == 0) {
    wcnt[0][warp] = n_gt;
    wcnt[1][warp] = n_eq;
  }
  __syncthreads();
  // eq_off: equal keys in the warps before this one (the rank of this warp's
  // first equal key); out_off: keys those warps keep (this warp's first slot)
  long long eq_off = 0, out_off = 0, total_kept = 0, eo = 0;
  for (int w = 0; w < kWarps; ++w) {
    const long long e = wcnt[1][w];
    const long long k = wcnt[0][w] + max(0LL, min(e, need_eq - eo));
    if (w < warp) {
      eq_off += e;
      out_off += k;
    }
    total_kept += k;
    eo += e;
  }
  int32_t *out = idx + static_cast<size_t>(row) * static_cast<size_t>(K);
  long long run_eq = eq_off, run_out = out_off;
  for (long long base = j0; base < j1; base += 32) {
    const long long j = base + lane;
    const uint32_t key = j < j1 ? order_key(load_key_value(in, rbase + j)) : 0u;
    const bool gt = j < j1 && key > T;
    const bool eq = j < j1 && key == T;
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    const bool kept = gt || (eq && run_eq + __popc(eb & lt) < need_eq);
    const uint32_t kb = __ballot_sync(0xffffffffu, kept);
    if (kept) {
      const long long pos = run_out + __popc(kb & lt);
      if (pos < K) out[pos] = static_cast<int32_t>(j);
      else record_device_status(BKV_DEV_ASSERT, 301);
    }
    run_eq += __popc(eb);
    run_out += __popc(kb);
  }
  if (tid == 0 && total_kept != K) record_device_status(BKV_DEV_ASSERT, 302);
}

__global__ void finalize_scores_kernel(const SelectInput in, size_t total, float *__restrict__ s) {
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * blockDim.x)
    s[e] = score_of_key(in, load_key_value(in, e));
}

__global__ void iota_rows_kernel(int32_t *idx, size_t total, long long n) {
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * blockDim.x)
    idx[e] = static_cast<int32_t>(e % static_cast<size_t>(n));
}

unsigned grid_for(size_t total, int threads) {
  const size_t blocks = (total + threads - 1) / threads;
  return static_cast<unsigned>(std::min<size_t>(blocks, 148 * 16));
}

}  // namespace

size_t select_workspace_bytes(int, long long) { return 0; }

bkv_status launch_select_topk(const SelectInput &in, int n_rows, long long L, long long K,
                              int32_t *idx, float *s_out, void *, size_t, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  if (n_rows <= 0) return BKV_OK;
  select_topk_kernel<<<n_rows, kThreads, 0, stream>>>(in, L, K, idx, s_out);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

bkv_status launch_finalize_scores(const SelectInput &in, int n_rows, long long L, float *s,
                                  cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  const size_t total = static_cast<size_t>(n_rows) * static_cast<size_t>(L);
  finalize_scores_kernel<<<grid_for(total, 256), 256, 0, stream>>>(in, total, s);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

bkv_status launch_iota_rows(int32_t *idx, int n_rows, long long n, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  const size_t total = static_cast<size_t>(n_rows) * static_cast<size_t>(n);
  iota_rows_kernel<<<grid_for(total, 256), 256, 0, stream>>>(idx, total, n);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace bkv
