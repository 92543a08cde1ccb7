// select_topk.cu -- top-K budget selection (BeaconKV Fig. 5(c); Table 1's
// "maximum KV cache budget").
//
// One CTA per row (a (layer, KV head)); scores become order-preserving
// unsigned keys (larger score -> larger key; -0 and +0 map to one key).  The
// row is never staged whole: each pass re-reads it (from HBM the first time,
// L2 after) and rebuilds the keys -- for a mean, or for partials of several
// observation groups, that also merges the groups.  The tensor-core max
// aggregation hands over the keys already merged (one word per position).
//
// The common path (rows of a multiple of 4 keys, 16-byte aligned, at most
// 65536 of them) reads the row twice and does the rest in shared memory:
//   1. (HBM) a histogram of the keys' top 12 bits finds the bin holding the
//      K-th largest key (and the step's scores are written);
//   2. (L2) every key above that bin is certainly kept: it is marked in a
//      bitmask of the row's positions (each 8 lanes of a warp assemble one
//      32-position word with three shuffles); the keys of the bin itself are
//      collected, with their positions, in a list;
//   3. a radix select over the listed keys' low 20 bits finds the K-th largest
//      key T and how many keys equal to T are kept; listed keys above T are
//      marked, and the first `need_eq` keys equal to T (ties to the lower
//      position: a prefix count over a second bitmask) too;
//   4. the marked positions are written in ascending order, each thread
//      taking a run of mask words at its prefix-sum offset.
// A row whose threshold bin holds more keys than the list can take (scores
// piled into a narrow range), longer rows, and rows not laid out for 16-byte
// loads take the general path: MSB-first radix passes over the streamed row
// for the remaining bits, then a counting pass and a writing pass in which
// each warp emits the kept positions of its slice of the row.
#include <cuda_runtime.h>

#include <algorithm>

#include "bkv_check.cuh"
#include "bkv_device_status.cuh"
#include "bkv_internal.h"
#include "order_key.cuh"

BKV_DEFINE_STATUS_ACCESSOR(take_status_select)

namespace bkv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTopBits = 12;                 // the first pass's digit
constexpr int kTopBins = 1 << kTopBits;      // 4096
constexpr int kListCap = 6144;               // threshold-bin keys held in shared memory
constexpr int kMaskMaxL = 65536;             // longest row whose bitmasks are held
// histogram (4096 words) + list keys and positions + two bitmasks of L bits
constexpr int mask_smem_bytes(long long L) {
  return static_cast<int>((kTopBins + 2 * kListCap + 2 * ((L + 127) / 128 * 4)) * 4);
}

__device__ __forceinline__ float load_key_value(const SelectInput &in, size_t off) {
  if (in.keys) return key_value(reinterpret_cast<const uint32_t *>(in.src)[off]);
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
  return in.mean ? v : __expf(v);
}

// Four consecutive values of a row (off a multiple of 4, the row 16-byte
// aligned), merged over the parts like load_key_value.
__device__ __forceinline__ float4 load_key_value4(const SelectInput &in, size_t off) {
  if (in.keys) {
    const uint4 k = *reinterpret_cast<const uint4 *>(in.src + off);
    return make_float4(key_value(k.x), key_value(k.y), key_value(k.z), key_value(k.w));
  }
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

__device__ __forceinline__ uint4 keys_of(float4 v) {
  return make_uint4(order_key(v.x), order_key(v.y), order_key(v.z), order_key(v.w));
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

// Inclusive prefix sum across the warp.
__device__ __forceinline__ uint32_t warp_inclusive_scan(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// The digit of `hist` (nb bins, highest digit first, nb / kThreads per
// thread) holding the krem-th key: sel[0] = the digit, sel[1] = the keys in
// higher digits.  Every thread calls it; it synchronises.
template <int kPer>
__device__ __forceinline__ void find_digit(const uint32_t *hist, int nb, long long krem,
                                           uint32_t *wsum, long long *sel) {
  const int tid = threadIdx.x;
  uint32_t c[kPer], local = 0;
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int d = nb - 1 - kPer * tid - q;
    c[q] = d >= 0 ? hist[d] : 0u;
    local += c[q];
  }
  uint32_t total;
  const uint32_t excl = block_exclusive_scan(local, wsum, &total);
  if (static_cast<long long>(excl) < krem && krem <= static_cast<long long>(excl + local)) {
    uint32_t acc = excl;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      if (static_cast<long long>(acc + c[q]) >= krem) {
        sel[0] = nb - 1 - kPer * tid - q;
        sel[1] = acc;
        break;
      }
      acc += c[q];
    }
  }
  __syncthreads();
}

// Ordered emission of row `row`'s kept positions given the threshold key T:
// warp w owns positions [w * chunk, (w + 1) * chunk); cnt_gt[w] / cnt_eq[w]
// (shared) hold the keys > T and == T of each slice.  Writes idx[row][..].
template <bool kVec>
__device__ void emit_kept(const SelectInput &in, long long L, long long K, int32_t *idx,
                          size_t rbase, int row, uint32_t T, long long need_eq, long long chunk,
                          const uint32_t *cnt_gt, const uint32_t *cnt_eq) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int V = kVec ? 4 : 1;
  const long long j0 = warp * chunk, j1 = min(L, j0 + chunk);
  // eq_off: equal keys in the slices before this one (the rank of this
  // slice's first equal key); out_off: keys those slices keep
  long long eq_off = 0, out_off = 0, total_kept = 0, eo = 0;
  for (int w = 0; w < kWarps; ++w) {
    const long long e = cnt_eq[w];
    const long long k = cnt_gt[w] + max(0LL, min(e, need_eq - eo));
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
    const long long j = base + V * lane;
    if constexpr (kVec) {
      const uint4 kk = j < j1 ? keys_of(load_key_value4(in, rbase + j)) : make_uint4(0u, 0u, 0u, 0u);
      k[0] = kk.x;
      k[1] = kk.y;
      k[2] = kk.z;
      k[3] = kk.w;
    } else {
      k[0] = j < j1 ? order_key(load_key_value(in, rbase + j)) : 0u;
    }
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

// The general path from a known prefix: MSB-first radix passes over the
// streamed row for bits [0, hi) (11 bits at a time) with the keys matching
// `prefix` under `mask`, then a counting pass and the ordered emission.
// s_out is written by the first pass when hi == 32.
template <bool kVec>
__device__ void stream_select(const SelectInput &in, long long L, long long K, int32_t *idx,
                              float *s_out, int row, uint32_t prefix, uint32_t mask,
                              long long krem, int hi, uint32_t *hist, uint32_t *wsum,
                              long long *sel, uint32_t *cnt_gt, uint32_t *cnt_eq) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t rbase = static_cast<size_t>(row) * static_cast<size_t>(L);
  while (hi > 0) {
    const int lo = hi > 11 ? hi - 11 : 0;
    const int nbits = hi - lo;
    const uint32_t dmask = (1u << nbits) - 1u;
    const int nb = 1 << nbits;
    for (int b = tid; b < nb; b += kThreads) hist[b] = 0u;
    __syncthreads();
    auto count = [&](uint32_t key) {
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> lo) & dmask], 1u);
    };
    if constexpr (kVec) {
      const long long L4 = L >> 2;
      for (long long q = tid; q < L4; q += kThreads) {
        const float4 a = load_key_value4(in, rbase + 4 * q);
        if (hi == 32 && s_out)
          *reinterpret_cast<float4 *>(s_out + rbase + 4 * q) =
              make_float4(score_of_key(in, a.x), score_of_key(in, a.y), score_of_key(in, a.z),
                          score_of_key(in, a.w));
        const uint4 k = keys_of(a);
        count(k.x); count(k.y); count(k.z); count(k.w);
      }
    } else {
      for (long long j = tid; j < L; j += kThreads) {
        const float v = load_key_value(in, rbase + j);
        if (hi == 32 && s_out) s_out[rbase + j] = score_of_key(in, v);
        count(order_key(v));
      }
    }
    __syncthreads();
    find_digit<(1 << 11) / kThreads>(hist, nb, krem, wsum, sel);
    prefix |= static_cast<uint32_t>(sel[0]) << lo;
    mask |= dmask << lo;
    krem -= sel[1];
    hi = lo;
    __syncthreads();  // sel and hist are rewritten by the next pass
  }
  const uint32_t T = prefix;
  const long long need_eq = krem;  // keys equal to T that are kept
  constexpr int V = kVec ? 4 : 1;
  const long long chunk = (L + 32 * V * kWarps - 1) / (32 * V * kWarps) * (32 * V);
  const long long j0 = warp * chunk, j1 = min(L, j0 + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (long long base = j0; base < j1; base += 32 * V) {
    const long long j = base + V * lane;
    if constexpr (kVec) {
      if (j < j1) {
        const uint4 k = keys_of(load_key_value4(in, rbase + j));
        n_gt += (k.x > T) + (k.y > T) + (k.z > T) + (k.w > T);
        n_eq += (k.x == T) + (k.y == T) + (k.z == T) + (k.w == T);
      }
    } else if (j < j1) {
      const uint32_t k = order_key(load_key_value(in, rbase + j));
      n_gt += k > T;
      n_eq += k == T;
    }
  }
  n_gt = __reduce_add_sync(0xffffffffu, n_gt);
  n_eq = __reduce_add_sync(0xffffffffu, n_eq);
  if (lane == 0) {
    cnt_gt[warp] = n_gt;
    cnt_eq[warp] = n_eq;
  }
  __syncthreads();
  emit_kept<kVec>(in, L, K, idx, rbase, row, T, need_eq, chunk, cnt_gt, cnt_eq);
}

// The general path for a whole row.
template <bool kVec>
__global__ void __launch_bounds__(kThreads)
    select_topk_kernel(const SelectInput in, long long L, long long K, int32_t *__restrict__ idx,
                       float *__restrict__ s_out) {
  __shared__ uint32_t hist[1 << 11];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t cnt[2][kWarps];
  __shared__ long long sel[2];
  stream_select<kVec>(in, L, K, idx, s_out, blockIdx.x, 0u, 0u, K, 32, hist, wsum, sel, cnt[0],
                      cnt[1]);
}

// Four consecutive merged values at p (16-byte aligned), with the part count
// fixed at compile time (kP > 0) or read from the input (kP == 0); kP < 0:
// the row holds the merged order keys themselves.
template <int kP, bool kMean>
__device__ __forceinline__ float4 merged4(const SelectInput &in, const float *p) {
  if constexpr (kP < 0) {
    const uint4 k = *reinterpret_cast<const uint4 *>(p);
    return make_float4(key_value(k.x), key_value(k.y), key_value(k.z), key_value(k.w));
  } else {
    float4 v = *reinterpret_cast<const float4 *>(p);
    const int np = kP > 0 ? kP : in.n_parts;
#pragma unroll
    for (int q = 1; q < (kP > 0 ? kP : 64); ++q) {
      if (kP == 0 && q >= np) break;
      const float4 w = *reinterpret_cast<const float4 *>(p + q * in.part_stride);
      if constexpr (kMean) {
        v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
      } else {
        v.x = fmaxf(v.x, w.x); v.y = fmaxf(v.y, w.y); v.z = fmaxf(v.z, w.z); v.w = fmaxf(v.w, w.w);
      }
    }
    if constexpr (kMean) {
      v.x *= in.inv_count; v.y *= in.inv_count; v.z *= in.inv_count; v.w *= in.inv_count;
    }
    return v;
  }
}

// The common path: two streaming passes, then shared memory only (see the
// file comment).  Shared memory: the histogram, the threshold bin's list, and
// two bitmasks of the row's positions (kept; equal to T).
template <int kP, bool kMean>
__global__ void __launch_bounds__(kThreads, 3)
    select_topk_mask_kernel(const SelectInput in, int L, int K, int32_t *__restrict__ idx,
                            float *__restrict__ s_out) {
  extern __shared__ uint32_t sm[];
  const int n_words = (L + 127) / 128 * 4;  // mask words, whole 128-position groups
  uint32_t *hist = sm;                      // [kTopBins]
  uint32_t *lkey = hist + kTopBins;         // [kListCap]
  uint32_t *lpos = lkey + kListCap;         // [kListCap]
  uint32_t *mask = lpos + kListCap;         // [n_words] kept positions
  uint32_t *eqm = mask + n_words;           // [n_words] positions of keys equal to T
  __shared__ uint32_t wsum[kWarps];
  __shared__ long long sel[2];
  __shared__ int n_list;
  const int row = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float *src = in.src + static_cast<size_t>(row) * static_cast<size_t>(L);
  float *so = s_out ? s_out + static_cast<size_t>(row) * static_cast<size_t>(L) : nullptr;
  const int L4 = L >> 2;
  constexpr int U = 4;  // float4 loads in flight per thread

  for (int b = tid; b < kTopBins; b += kThreads) hist[b] = 0u;
  for (int w = tid; w < 2 * n_words; w += kThreads) mask[w] = 0u;  // mask and eqm
  if (tid == 0) n_list = 0;
  __syncthreads();

  // ---- pass 1 (HBM): histogram of the top 12 bits, and the scores
  for (int q0 = tid; q0 < L4; q0 += U * kThreads) {
    float4 a[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (q0 + u * kThreads < L4) a[u] = merged4<kP, kMean>(in, src + 4 * (q0 + u * kThreads));
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int q = q0 + u * kThreads;
      if (q < L4) {
        if (so) {
          const float4 v = a[u];
          *reinterpret_cast<float4 *>(so + 4 * q) =
              kMean ? v : make_float4(__expf(v.x), __expf(v.y), __expf(v.z), __expf(v.w));
        }
        const uint4 k = keys_of(a[u]);
        atomicAdd(&hist[k.x >> (32 - kTopBits)], 1u);
        atomicAdd(&hist[k.y >> (32 - kTopBits)], 1u);
        atomicAdd(&hist[k.z >> (32 - kTopBits)], 1u);
        atomicAdd(&hist[k.w >> (32 - kTopBits)], 1u);
      }
    }
  }
  __syncthreads();
  find_digit<kTopBins / kThreads>(hist, kTopBins, K, wsum, sel);
  const uint32_t b1 = static_cast<uint32_t>(sel[0]);
  const long long need1 = K - sel[1];
  const uint32_t in_bin = hist[b1];
  __syncthreads();
  if (in_bin > static_cast<uint32_t>(kListCap)) {
    // scores piled into one bin: the general path for the remaining bits
    stream_select<true>(in, L, K, idx, nullptr, row, b1 << (32 - kTopBits),
                        0xffffffffu << (32 - kTopBits), need1, 32 - kTopBits, hist, wsum, sel,
                        lkey, lkey + kWarps);
    return;
  }

  const uint32_t key_lo = b1 << (32 - kTopBits);
  const uint32_t key_top = key_lo | ((1u << (32 - kTopBits)) - 1u);  // the bin's largest key
  // ---- pass 2 (L2): keys above the bin -> mask bits; the bin's keys -> list.
  // Lane l of a warp holds positions 4q .. 4q+3 with q = base + l, so lanes
  // 8m .. 8m+7 cover one 32-position mask word; base is warp-uniform.
  for (int base = warp * 32; base < L4; base += U * kThreads) {
    float4 a[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int q = base + u * kThreads + lane;
      if (q < L4) a[u] = merged4<kP, kMean>(in, src + 4 * q);
    }
    // the mask words of all U steps first (no branch between them, so their
    // shuffles overlap), then one vote for the rare listing of the bin's keys
    uint32_t kq[U][4];
    uint32_t inb = 0u;  // bit 4u + e: key e of step u lies in the threshold bin
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int q = base + u * kThreads + lane;
      const uint4 k4 = q < L4 ? keys_of(a[u]) : make_uint4(0u, 0u, 0u, 0u);
      kq[u][0] = k4.x; kq[u][1] = k4.y; kq[u][2] = k4.z; kq[u][3] = k4.w;
      uint32_t nib = 0u;
      // above the bin: key > key_top; in it: key - key_lo < bin width
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        nib |= (kq[u][e] > key_top ? 1u : 0u) << e;
        if (q < L4 && kq[u][e] - key_lo < (1u << (32 - kTopBits))) inb |= 1u << (4 * u + e);
      }
      uint32_t word = nib << (4 * (lane & 7));
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      word |= __shfl_xor_sync(0xffffffffu, word, 2);
      word |= __shfl_xor_sync(0xffffffffu, word, 4);
      const int wi = (base + u * kThreads + lane) >> 3;
      if ((lane & 7) == 0 && wi < n_words) mask[wi] = word;
    }
    if (inb != 0u) {  // the threshold bin's keys: a few percent of a row, up to ~11%
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((inb >> (4 * u + e)) & 1u) {
            const int p = atomicAdd(&n_list, 1);
            if (p < kListCap) {
              lkey[p] = kq[u][e];
              lpos[p] = static_cast<uint32_t>(4 * (base + u * kThreads + lane) + e);
            }
          }
        }
      }
    }
  }
  __syncthreads();
  const int listed = min(n_list, kListCap);

  // ---- the K-th key within the collected bin: bits 19..0 in two 10-bit
  // digits over the list
  uint32_t prefix = b1 << (32 - kTopBits), pmask = 0xffffffffu << (32 - kTopBits);
  long long krem = need1;
  for (int hi = 32 - kTopBits; hi > 0;) {
    const int lo = hi > 10 ? hi - 10 : 0;
    const uint32_t dmask = (1u << (hi - lo)) - 1u;
    const int nb = 1 << (hi - lo);
    for (int b = tid; b < nb; b += kThreads) hist[b] = 0u;
    __syncthreads();
    for (int e = tid; e < listed; e += kThreads) {
      const uint32_t key = lkey[e];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> lo) & dmask], 1u);
    }
    __syncthreads();
    find_digit<(1 << 10) / kThreads>(hist, nb, krem, wsum, sel);
    prefix |= static_cast<uint32_t>(sel[0]) << lo;
    pmask |= dmask << lo;
    krem -= sel[1];
    hi = lo;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int need_eq = static_cast<int>(krem);  // keys equal to T that are kept

  // ---- listed keys above T are kept; those equal to T are marked
  for (int e = tid; e < listed; e += kThreads) {
    const uint32_t key = lkey[e], pos = lpos[e];
    if (!BKV_CHECK(pos < static_cast<uint32_t>(L), 711)) continue;
    if (key > T) atomicOr(&mask[pos >> 5], 1u << (pos & 31));
    else if (key == T) atomicOr(&eqm[pos >> 5], 1u << (pos & 31));
  }
  __syncthreads();

  // ---- the first need_eq keys equal to T (lowest positions), then the
  // kept positions in ascending order; thread t owns a run of words
  const int wpt = (n_words + kThreads - 1) / kThreads;
  const int w0 = min(n_words, tid * wpt), w1 = min(n_words, w0 + wpt);
  uint32_t n_eq = 0;
  for (int w = w0; w < w1; ++w) n_eq += __popc(eqm[w]);
  uint32_t total;
  uint32_t rank = block_exclusive_scan(n_eq, wsum, &total);
  uint32_t n_kept = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t e = eqm[w];
    const uint32_t c = __popc(e);
    if (rank >= static_cast<uint32_t>(need_eq)) {
      e = 0u;
    } else if (rank + c > static_cast<uint32_t>(need_eq)) {
      uint32_t keep = 0u;  // the lowest need_eq - rank set bits
      for (uint32_t r = rank; r < static_cast<uint32_t>(need_eq); ++r) {
        const uint32_t low = e & (0u - e);
        keep |= low;
        e ^= low;
      }
      e = keep;
    }
    rank += c;
    const uint32_t m = mask[w] | e;
    mask[w] = m;
    n_kept += __popc(m);
  }
  uint32_t out = block_exclusive_scan(n_kept, wsum, &total);
  int32_t *dst = idx + static_cast<size_t>(row) * static_cast<size_t>(K);
  for (int w = w0; w < w1; ++w) {
    uint32_t m = mask[w];
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1u;
      if (out < static_cast<uint32_t>(K)) dst[out] = 32 * w + b;
      ++out;
    }
  }
  if (tid == 0 && total != static_cast<uint32_t>(K)) record_device_status(BKV_DEV_ASSERT, 303);
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
  if (vec && L <= kMaskMaxL) {
    const int smem = mask_smem_bytes(L);
    const int parts = in.keys ? -1 : in.n_parts >= 1 && in.n_parts <= 4 ? in.n_parts : 0;
    bkv_status st = BKV_OK;
    auto run = [&](auto kernel, int *attr_done) {
      if (!ensure_smem_limit(kernel, mask_smem_bytes(kMaskMaxL), attr_done)) {
        st = BKV_ERR_CUDA;
        return;
      }
      kernel<<<n_rows, kThreads, smem, stream>>>(in, static_cast<int>(L), static_cast<int>(K),
                                                 idx, s_out);
    };
    static int done[11][64];
    if (in.mean) {
      switch (parts) {
        case 1: run(select_topk_mask_kernel<1, true>, done[0]); break;
        case 2: run(select_topk_mask_kernel<2, true>, done[1]); break;
        case 3: run(select_topk_mask_kernel<3, true>, done[2]); break;
        case 4: run(select_topk_mask_kernel<4, true>, done[3]); break;
        default: run(select_topk_mask_kernel<0, true>, done[4]); break;
      }
    } else {
      switch (parts) {
        case -1: run(select_topk_mask_kernel<-1, false>, done[10]); break;
        case 1: run(select_topk_mask_kernel<1, false>, done[5]); break;
        case 2: run(select_topk_mask_kernel<2, false>, done[6]); break;
        case 3: run(select_topk_mask_kernel<3, false>, done[7]); break;
        case 4: run(select_topk_mask_kernel<4, false>, done[8]); break;
        default: run(select_topk_mask_kernel<0, false>, done[9]); break;
      }
    }
    if (st != BKV_OK) return st;
  } else if (vec) {
    select_topk_kernel<true><<<n_rows, kThreads, 0, stream>>>(in, L, K, idx, s_out);
  } else {
    select_topk_kernel<false><<<n_rows, kThreads, 0, stream>>>(in, L, K, idx, s_out);
  }
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
