// fps_common.cuh -- arithmetic shared by the FPS kernels (fps.cu, fps_tc.cu):
// element loads, the f32 dot-product step, the cosine distance, and the
// (distance desc, index asc) order of the greedy choice.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bkv {
namespace fpsk {

// ---- element access: 8 consecutive elements as f32
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&u)[8]) {
  const uint4 w = *reinterpret_cast<const uint4 *>(p);
  u[0] = __uint_as_float(w.x << 16); u[1] = __uint_as_float(w.x & 0xffff0000u);
  u[2] = __uint_as_float(w.y << 16); u[3] = __uint_as_float(w.y & 0xffff0000u);
  u[4] = __uint_as_float(w.z << 16); u[5] = __uint_as_float(w.z & 0xffff0000u);
  u[6] = __uint_as_float(w.w << 16); u[7] = __uint_as_float(w.w & 0xffff0000u);
}
__device__ __forceinline__ void load8(const float *p, float (&u)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p);
  const float4 b = *reinterpret_cast<const float4 *>(p + 4);
  u[0] = a.x; u[1] = a.y; u[2] = a.z; u[3] = a.w;
  u[4] = b.x; u[5] = b.y; u[6] = b.z; u[7] = b.w;
}

// One 8-element step of a dot product, the same operation sequence wherever a
// dot product is formed (point pass and Gram block), so both agree bit for bit.
__device__ __forceinline__ float2 dot8_step(float2 acc, const float (&u)[8], const float *s) {
  const float4 s0 = *reinterpret_cast<const float4 *>(s);
  const float4 s1 = *reinterpret_cast<const float4 *>(s + 4);
  acc = __ffma2_rn(make_float2(u[0], u[1]), make_float2(s0.x, s0.y), acc);
  acc = __ffma2_rn(make_float2(u[2], u[3]), make_float2(s0.z, s0.w), acc);
  acc = __ffma2_rn(make_float2(u[4], u[5]), make_float2(s1.x, s1.y), acc);
  acc = __ffma2_rn(make_float2(u[6], u[7]), make_float2(s1.z, s1.w), acc);
  return acc;
}

__device__ __forceinline__ float cos_dist(float2 acc, float inv_a, float inv_b) {
  const float dot = __fadd_rn(acc.x, acc.y);
  const float dd = __fmaf_rn(-__fmul_rn(dot, inv_a), inv_b, 1.0f);
  return fminf(fmaxf(dd, 0.f), 2.f);
}

// Order key of a distance: larger distance -> larger key; selected points
// (distance -1) -> 0, below every unselected point.
__device__ __forceinline__ uint32_t dist_key(float d) {
  return d < 0.f ? 0u : (__float_as_uint(d) | 0x80000000u);
}

// (distance desc, index asc): true if (da, ia) comes before (db, ib).
__device__ __forceinline__ bool before(float da, int ia, float db, int ib) {
  return da > db || (da == db && ia < ib);
}


// The `want` best unselected points by (distance desc, index asc), written
// unordered to cidx/cdist (want <= number of unselected points).  An MSB-first
// radix select over the distance keys: a min/max reduction first finds the
// leading bits that every key shares, so the histogram passes start at the
// first bit that differs (distances of one head tend to share their exponent,
// which would otherwise pile every key into one or two bins); each warp counts
// into its own histogram.  Then every key above the threshold and the
// lowest-index keys equal to it are emitted.
// Once the bin still to be resolved holds at most kRankMax keys, the
// remaining digit passes are replaced by ranking those keys against each
// other (key desc, index asc).
// Scratch: whist[kThreads / 32 * 256] (>= 2 * kRankMax words), hist[256], scal[>= 8].
constexpr int kRankMax = 256;

// With have_range, scal[6] and scal[7] already hold (as unsigned) a lower
// bound of the live keys' minimum and their maximum, and the first pass over
// the keys is skipped.
template <int kThreads>
__device__ void select_best(const float *dist, int n, int n_live, int want, uint32_t *whist,
                            uint32_t *hist, int *scal, int *cidx, float *cdist,
                            bool have_range = false) {
  constexpr int kWarps = kThreads / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (!have_range) {
  // common prefix of the live keys
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int i = tid; i < n; i += kThreads) {
    const uint32_t key = dist_key(dist[i]);
    if (key != 0u) {
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    hist[2 * warp] = kmin;
    hist[2 * warp + 1] = kmax;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t a = 0xffffffffu, b = 0u;
    for (int w = 0; w < kWarps; ++w) {
      a = min(a, hist[2 * w]);
      b = max(b, hist[2 * w + 1]);
    }
    scal[6] = static_cast<int>(a);
    scal[7] = static_cast<int>(b);
  }
  __syncthreads();
  }
  const uint32_t gmin = static_cast<uint32_t>(scal[7]) == 0u ? 0u : static_cast<uint32_t>(scal[6]);
  const uint32_t diff = gmin ^ static_cast<uint32_t>(scal[7]);
  int hi = diff == 0u ? 0 : 32 - __clz(diff);  // bits [hi, 32) are shared
  uint32_t mask = hi >= 32 ? 0u : ~((1u << hi) - 1u);
  uint32_t prefix = gmin & mask;
  int krem = want;
  int n_eq = n_live;  // live keys matching the prefix
  for (; hi > 0; hi -= 8) {
    if (n_eq <= kRankMax) break;  // few enough to rank directly
    const int lo = hi > 8 ? hi - 8 : 0;
    uint32_t *mine = whist + warp * 256;
    for (int b = lane; b < 256; b += 32) mine[b] = 0;
    __syncwarp();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t key = dist_key(dist[i]);
      if (key != 0u && (key & mask) == prefix) atomicAdd(&mine[(key >> lo) & 255u], 1u);
    }
    __syncthreads();
    for (int b = tid; b < 256; b += kThreads) {
      uint32_t sum = 0;
      for (int w = 0; w < kWarps; ++w) sum += whist[w * 256 + b];
      hist[b] = sum;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t cnt[8], local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[255 - 8 * lane - j];
        local += cnt[j];
      }
      uint32_t incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const uint32_t excl = incl - local;
      if (static_cast<int>(excl) < krem && krem <= static_cast<int>(incl)) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (static_cast<int>(acc + cnt[j]) >= krem) {
            scal[0] = 255 - 8 * lane - j;
            scal[1] = static_cast<int>(acc);
            break;
          }
          acc += cnt[j];
        }
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(scal[0]) << lo;
    mask |= ((hi - lo) >= 32 ? 0xffffffffu : ((1u << (hi - lo)) - 1u)) << lo;
    krem -= scal[1];
    n_eq = static_cast<int>(hist[scal[0]]);
    __syncthreads();
  }
  if (tid == 0) scal[2] = 0;
  __syncthreads();
  if (n_eq == krem) {
    // every key equal to the threshold is kept: the selection is the keys
    // >= threshold, emitted in any order (one atomic per warp)
    for (int base = 0; base < n; base += kThreads) {
      const int i = base + tid;
      const uint32_t key = i < n ? dist_key(dist[i]) : 0u;
      const bool keep = key != 0u && key >= prefix;
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      int wbase = 0;
      if (lane == 0 && bal) wbase = atomicAdd(&scal[2], __popc(bal));
      wbase = __shfl_sync(0xffffffffu, wbase, 0);
      if (keep) {
        const int pos = wbase + __popc(bal & ((1u << lane) - 1u));
        if (pos < want) {
          cidx[pos] = i;
          cdist[pos] = dist[i];
        }
      }
    }
    return;
  }
  if (hi > 0) {
    // the bin (key & mask) == prefix holds n_eq <= kRankMax keys, of which
    // the krem best are kept, with every key above the bin.  Keys above are
    // emitted as found; the bin's keys are listed, then each is kept when
    // fewer than krem listed keys come before it in (key desc, index asc).
    static_assert(kThreads / 32 * 256 >= 2 * kRankMax, "rank list does not fit");
    uint32_t *lkey = whist;
    int *lidx = reinterpret_cast<int *>(whist + kRankMax);
    if (tid == 0) scal[3] = 0;
    __syncthreads();
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < n; base += kThreads) {
      const int i = base + tid;
      const uint32_t key = i < n ? dist_key(dist[i]) : 0u;
      const bool live = key != 0u;
      const bool above = live && (key & mask) > prefix;
      const bool inbin = live && (key & mask) == prefix;
      const uint32_t ba = __ballot_sync(0xffffffffu, above);
      const uint32_t bb = __ballot_sync(0xffffffffu, inbin);
      int pa = 0, pb = 0;
      if (lane == 0) {
        if (ba) pa = atomicAdd(&scal[2], __popc(ba));
        if (bb) pb = atomicAdd(&scal[3], __popc(bb));
      }
      pa = __shfl_sync(0xffffffffu, pa, 0) + __popc(ba & lt_mask);
      pb = __shfl_sync(0xffffffffu, pb, 0) + __popc(bb & lt_mask);
      if (above && pa < want) {
        cidx[pa] = i;
        cdist[pa] = dist[i];
      }
      if (inbin && pb < kRankMax) {
        lkey[pb] = key;
        lidx[pb] = i;
      }
    }
    __syncthreads();
    const int listed = min(scal[3], kRankMax);
    for (int e = tid; e < listed; e += kThreads) {
      const uint32_t ke = lkey[e];
      const int ie = lidx[e];
      int rank = 0;
      for (int f = 0; f < listed; ++f) {
        const uint32_t kf = lkey[f];
        rank += (kf > ke || (kf == ke && lidx[f] < ie)) ? 1 : 0;
      }
      if (rank < krem) {
        const int pos = atomicAdd(&scal[2], 1);
        if (pos < want) {
          cidx[pos] = ie;
          cdist[pos] = dist[ie];
        }
      }
    }
    return;
  }
  // emission: keys above the threshold, and the lowest-index krem keys equal
  // to it in index order
  int eq_base = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + tid;
    const uint32_t key = i < n ? dist_key(dist[i]) : 0u;
    const bool gt = key > prefix;
    const bool eq = key == prefix && key != 0u;
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) hist[warp] = __popc(eb);
    __syncthreads();
    int before_me = 0, total = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int c = static_cast<int>(hist[w]);
      if (w < warp) before_me += c;
      total += c;
    }
    before_me += __popc(eb & ((1u << lane) - 1u));
    if (gt || (eq && eq_base + before_me < krem)) {
      const int pos = atomicAdd(&scal[2], 1);
      if (pos < want) {
        cidx[pos] = i;
        cdist[pos] = dist[i];
      }
    }
    eq_base += total;
    __syncthreads();
  }
}

}  // namespace fpsk
}  // namespace bkv
