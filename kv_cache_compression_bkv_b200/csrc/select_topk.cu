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

// Four consecutive values of a row (off a multiple of 4, the row 16-byte
// aligned), merged over the parts like load_key_value.
__device__ __forceinline__ float4 load_key_value4(const SelectInput &in, size_t off) {
  float4 v = *reinterpret_cast<const float4 *>(in.src + off);
  for (int p = 1; p < in.n_parts; ++p) {
    const float4 w = *reinterpret_cast<const float4 *>(in.src + p * in.part_stride + off);
    if (in.mean) {
      v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
    } else {
      v.x = fmaxf(v.x, w.x); v.y = fmaxf(v.y, w.y); v.z = fmaxf(v.z, w.z); v.w = fmaxf(v.w, w.w);
    }
  }
  if (in.mean) {
    v.x *= in.inv_count; v.y *= in.inv_count; v.z *= in.inv_count; v.w *= in.inv_count;
  }
  return v;
}

// Inclusive prefix sum across the warp.
__device__ __forceinline__ uint32_t warp_inclusive_scan(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// kVec: the row length is a multiple of 4 and rows are 16-byte aligned, so
// every pass reads float4s (four keys per thread and load).
template <bool kVec>
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
    auto count = [&](uint32_t key) {
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> lo) & dmask], 1u);
    };
    if (kVec) {
      // two float4 loads in flight per thread before their keys are counted
      const long long L4 = L >> 2;
      for (long long q = tid; q < L4; q += 2 * kThreads) {
        const long long q2 = q + kThreads;
        const float4 a = load_key_value4(in, rbase + 4 * q);
        float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
        if (q2 < L4) b = load_key_value4(in, rbase + 4 * q2);
        if (hi == 32 && s_out) {
          *reinterpret_cast<float4 *>(s_out + rbase + 4 * q) =
              make_float4(score_of_key(in, a.x), score_of_key(in, a.y), score_of_key(in, a.z),
                          score_of_key(in, a.w));
          if (q2 < L4)
            *reinterpret_cast<float4 *>(s_out + rbase + 4 * q2) =
                make_float4(score_of_key(in, b.x), score_of_key(in, b.y), score_of_key(in, b.z),
                            score_of_key(in, b.w));
        }
        count(order_key(a.x)); count(order_key(a.y)); count(order_key(a.z)); count(order_key(a.w));
        if (q2 < L4) {
          count(order_key(b.x)); count(order_key(b.y)); count(order_key(b.z)); count(order_key(b.w));
        }
      }
    } else {
      for (long long j = tid; j < L; j += kThreads) {
        const float v = load_key_value(in, rbase + j);
        if (hi == 32 && s_out) s_out[rbase + j] = score_of_key(in, v);
        count(order_key(v));
      }
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

  // ---- ordered emission: warp w owns positions [w * chunk, (w + 1) * chunk);
  // a warp step covers 32 * V consecutive positions, lane l the V positions
  // from V * l (so lane order is position order)
  constexpr int V = kVec ? 4 : 1;
  const long long chunk = (L + 32 * V * kWarps - 1) / (32 * V * kWarps) * (32 * V);
  const long long j0 = warp * chunk, j1 = min(L, j0 + chunk);
  auto keys_at = [&](long long base, uint32_t (&k)[V]) {
    const long long j = base + V * lane;
    if (kVec) {
      if (j < j1) {
        const float4 v = load_key_value4(in, rbase + j);
        k[0] = order_key(v.x);
        k[V > 1 ? 1 : 0] = order_key(v.y);
        k[V > 2 ? 2 : 0] = order_key(v.z);
        k[V > 3 ? 3 : 0] = order_key(v.w);
      } else {
#pragma unroll
        for (int u = 0; u < V; ++u) k[u] = 0u;
      }
    } else {
      k[0] = j < j1 ? order_key(load_key_value(in, rbase + j)) : 0u;
    }
  };
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t n_gt = 0, n_eq = 0;
  for (long long base = j0; base < j1; base += 32 * V) {
    uint32_t k[V];
    keys_at(base, k);
    const long long j = base + V * lane;
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const bool in_range = j + u < j1;
      n_gt += (in_range && k[u] > T) ? 1u : 0u;
      n_eq += (in_range && k[u] == T) ? 1u : 0u;
    }
  }
  n_gt = __reduce_add_sync(0xffffffffu, n_gt);
  n_eq = __reduce_add_sync(0xffffffffu, n_eq);
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
  for (long long base = j0; base < j1; base += 32 * V) {
    uint32_t k[V];
    keys_at(base, k);
    const long long j = base + V * lane;
    bool gt[V], eq[V];
    uint32_t my_eq = 0;
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const bool in_range = j + u < j1;
      gt[u] = in_range && k[u] > T;
      eq[u] = in_range && k[u] == T;
      my_eq += eq[u] ? 1u : 0u;
    }
    const uint32_t eq_incl = warp_inclusive_scan(my_eq, lane);
    long long eq_rank = run_eq + eq_incl - my_eq;  // rank of this lane's first equal key
    bool kept[V];
    uint32_t my_kept = 0;
#pragma unroll
    for (int u = 0; u < V; ++u) {
      kept[u] = gt[u] || (eq[u] && eq_rank < need_eq);
      if (eq[u]) ++eq_rank;
      my_kept += kept[u] ? 1u : 0u;
    }
    const uint32_t kept_incl = warp_inclusive_scan(my_kept, lane);
    long long pos = run_out + kept_incl - my_kept;
#pragma unroll
    for (int u = 0; u < V; ++u) {
      if (kept[u]) {
        if (pos < K) out[pos] = static_cast<int32_t>(j + u);
        else record_device_status(BKV_DEV_ASSERT, 301);
        ++pos;
      }
    }
    run_eq += __shfl_sync(0xffffffffu, eq_incl, 31);
    run_out += __shfl_sync(0xffffffffu, kept_incl, 31);
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
  // float4 passes when every row (and every part) starts on a 16-byte boundary
  const bool vec = (L & 3) == 0 && (in.part_stride & 3) == 0 &&
                   (reinterpret_cast<uintptr_t>(in.src) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(s_out) & 15u) == 0;
  if (vec)
    select_topk_kernel<true><<<n_rows, kThreads, 0, stream>>>(in, L, K, idx, s_out);
  else
    select_topk_kernel<false><<<n_rows, kThreads, 0, stream>>>(in, L, K, idx, s_out);
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
