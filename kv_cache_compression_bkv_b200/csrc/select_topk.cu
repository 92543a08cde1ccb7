// select_topk.cu -- top-K budget selection (BeaconKV Fig. 5(c); Table 1's
// "maximum KV cache budget").
//
// One CTA per row.  Scores become order-preserving unsigned keys (larger score
// -> larger key; -0 and +0 map to one key), staged in shared memory when the
// row fits (else in the caller's workspace).  An MSB-first radix select with
// 8-bit digits finds the K-th largest key T and how many of the keys equal to
// T are kept; a block-wide ballot/prefix-sum scan then writes the kept
// positions in ascending order: every key > T, plus the first `need_eq` keys
// equal to T (ties go to the lower position).
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "bkv_device_status.cuh"
#include "bkv_internal.h"

BKV_DEFINE_STATUS_ACCESSOR(take_status_select)

namespace bkv {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
// histogram, per-warp histograms, warp counts and offsets, scalars
constexpr int kSmallWords = 256 + kWarps * 256 + 4 * kWarps + 8;
constexpr int kSmemLimit = 232448;
constexpr long long kMaxSmemKeys = (kSmemLimit - kSmallWords * 4) / 4;

// Exclusive prefix sums of the per-warp counts cnt[0..kWarps) into off[], and
// their total into *total (warp 0 only; the caller synchronises).
__device__ __forceinline__ void scan_warp_counts(const uint32_t *cnt, uint32_t *off,
                                                 uint32_t *total, int lane) {
  const uint32_t c = cnt[lane];
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  off[lane] = incl - c;
  if (lane == 31) *total = incl;
}

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

__global__ void __launch_bounds__(kThreads, 1)
    select_topk_kernel(const SelectInput in, long long L, long long K, int32_t *__restrict__ idx,
                       float *__restrict__ s_out, uint32_t *__restrict__ gkeys, int keys_in_smem) {
  extern __shared__ uint32_t sh[];
  uint32_t *hist = sh;                           // [256]
  uint32_t *whist = sh + 256;                    // [kWarps][256]
  uint32_t *wcnt = whist + kWarps * 256;         // [2][kWarps] counts
  uint32_t *woff = wcnt + 2 * kWarps;            // [2][kWarps] offsets
  uint32_t *scal = woff + 2 * kWarps;            // [8]
  const int row = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t *keys = keys_in_smem ? sh + kSmallWords : gkeys + static_cast<size_t>(row) * L;
  const size_t rbase = static_cast<size_t>(row) * L;

  for (long long j = tid; j < L; j += kThreads) {
    const float v = load_key_value(in, rbase + j);
    if (s_out) s_out[rbase + j] = score_of_key(in, v);
    keys[j] = order_key(v);
  }
  __syncthreads();

  // ---- radix select of the K-th largest key
  uint32_t prefix = 0, mask = 0;
  long long krem = K;  // rank of the wanted key among those matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    // per-warp histograms (atomics contend only inside a warp), then summed
    uint32_t *mine = whist + warp * 256;
    for (int b = lane; b < 256; b += 32) mine[b] = 0;
    __syncwarp();
    for (long long j = tid; j < L; j += kThreads) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&mine[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    for (int b = tid; b < 256; b += kThreads) {
      uint32_t sum = 0;
#pragma unroll 8
      for (int w = 0; w < kWarps; ++w) sum += whist[w * 256 + b];
      hist[b] = sum;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255-8l .. 248-8l (descending digits)
      uint32_t cnt[8];
      uint32_t local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - 8 * lane - i];
        local += cnt[i];
      }
      uint32_t incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const uint32_t excl = incl - local;
      if (static_cast<long long>(excl) < krem && krem <= static_cast<long long>(incl)) {
        uint32_t acc = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc + cnt[i] >= krem) {
            scal[0] = 255u - 8u * lane - i;
            scal[1] = acc;
            break;
          }
          acc += cnt[i];
        }
      }
    }
    __syncthreads();
    const uint32_t digit = scal[0];
    krem -= scal[1];
    prefix |= digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const long long need_eq = krem;  // keys equal to T that are kept

  // ---- ordered emission
  int32_t *out = idx + static_cast<size_t>(row) * K;
  long long kept_so_far = 0, eq_so_far = 0;
  for (long long base = 0; base < L; base += kThreads) {
    const long long j = base + tid;
    const uint32_t key = j < L ? keys[j] : 0u;
    const bool gt = j < L && key > T;
    const bool eq = j < L && key == T;
    const uint32_t eq_bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) wcnt[warp] = __popc(eq_bal);
    __syncthreads();
    if (warp == 0) scan_warp_counts(wcnt, woff, &scal[4], lane);
    __syncthreads();
    const uint32_t eq_before = woff[warp] + __popc(eq_bal & ((1u << lane) - 1u));
    const uint32_t eq_total = scal[4];
    const bool kept = gt || (eq && eq_so_far + eq_before < need_eq);
    const uint32_t k_bal = __ballot_sync(0xffffffffu, kept);
    if (lane == 0) wcnt[kWarps + warp] = __popc(k_bal);
    __syncthreads();
    if (warp == 0) scan_warp_counts(wcnt + kWarps, woff + kWarps, &scal[5], lane);
    __syncthreads();
    const uint32_t k_before = woff[kWarps + warp] + __popc(k_bal & ((1u << lane) - 1u));
    const uint32_t k_total = scal[5];
    if (kept) {
      const long long pos = kept_so_far + k_before;
      if (pos < K) out[pos] = static_cast<int32_t>(j);
      else record_device_status(BKV_DEV_ASSERT, 301);
    }
    kept_so_far += k_total;
    eq_so_far += eq_total;
    __syncthreads();
  }
  if (tid == 0 && kept_so_far != K) record_device_status(BKV_DEV_ASSERT, 302);
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

size_t select_workspace_bytes(int n_rows, long long L) {
  if (L <= kMaxSmemKeys) return 0;
  return static_cast<size_t>(n_rows) * static_cast<size_t>(L) * sizeof(uint32_t);
}

bkv_status launch_select_topk(const SelectInput &in, int n_rows, long long L, long long K,
                              int32_t *idx, float *s_out, void *ws, size_t ws_bytes,
                              cudaStream_t stream) {
  const bool in_smem = L <= kMaxSmemKeys;
  if (!in_smem && ws_bytes < select_workspace_bytes(n_rows, L)) return BKV_ERR_WORKSPACE;
  static int attr_done[64];
  if (!ensure_smem_limit(select_topk_kernel, kSmemLimit, attr_done)) return BKV_ERR_CUDA;
  const size_t smem = (kSmallWords + (in_smem ? static_cast<size_t>(L) : 0)) * sizeof(uint32_t);
  select_topk_kernel<<<n_rows, kThreads, smem, stream>>>(
      in, L, K, idx, s_out, static_cast<uint32_t *>(ws), in_smem ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

bkv_status launch_finalize_scores(const SelectInput &in, int n_rows, long long L, float *s,
                                  cudaStream_t stream) {
  const size_t total = static_cast<size_t>(n_rows) * static_cast<size_t>(L);
  finalize_scores_kernel<<<grid_for(total, 256), 256, 0, stream>>>(in, total, s);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

bkv_status launch_iota_rows(int32_t *idx, int n_rows, long long n, cudaStream_t stream) {
  const size_t total = static_cast<size_t>(n_rows) * static_cast<size_t>(n);
  iota_rows_kernel<<<grid_for(total, 256), 256, 0, stream>>>(idx, total, n);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace bkv
