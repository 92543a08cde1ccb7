// fps.cu -- Continual farthest-point sampling of the beacon queries
// (BeaconKV, Fig. 7) in cosine distance.
//
// For each (layer, query head) the union U = [current beacons; newest window]
// is sampled greedily: seed U[0]; each further pick is the unselected point
// with the largest distance to the selected set (ties to the lowest index);
// dist(a, b) = 1 - (u_a . u_b) / (|u_a| |u_b|), clamped to [0, 2], and 1 when a
// norm is zero.  One CTA per query head keeps the running distances and the
// inverse norms in shared memory; each pick rereads the points (L2-resident)
// to take their dot products with the newly picked point in f32.  bf16 inputs
// make every product exact in f32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "bkv_internal.h"

namespace bkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemLimit = 232448;
constexpr int kMaxDim = 128;

template <typename T>
struct Vec;

template <>
struct Vec<float> {
  // 4 elements per 16-byte load
  static constexpr int kPer = 4;
  __device__ static float dot16(const float *p, const float *s) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    const float4 y = *reinterpret_cast<const float4 *>(s);
    return fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, x.w * y.w)));
  }
  __device__ static float sq16(const float *p) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    return fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, x.w * x.w)));
  }
  __device__ static float to_f(float v) { return v; }
};

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kPer = 8;
  __device__ static float dot16(const __nv_bfloat16 *p, const float *s) {
    const uint4 x = *reinterpret_cast<const uint4 *>(p);
    const float4 s0 = *reinterpret_cast<const float4 *>(s);
    const float4 s1 = *reinterpret_cast<const float4 *>(s + 4);
    float a = bf_lo(x.x) * s0.x;
    a = fmaf(bf_hi(x.x), s0.y, a);
    a = fmaf(bf_lo(x.y), s0.z, a);
    a = fmaf(bf_hi(x.y), s0.w, a);
    a = fmaf(bf_lo(x.z), s1.x, a);
    a = fmaf(bf_hi(x.z), s1.y, a);
    a = fmaf(bf_lo(x.w), s1.z, a);
    a = fmaf(bf_hi(x.w), s1.w, a);
    return a;
  }
  __device__ static float sq16(const __nv_bfloat16 *p) {
    const uint4 x = *reinterpret_cast<const uint4 *>(p);
    float a = bf_lo(x.x) * bf_lo(x.x);
    a = fmaf(bf_hi(x.x), bf_hi(x.x), a);
    a = fmaf(bf_lo(x.y), bf_lo(x.y), a);
    a = fmaf(bf_hi(x.y), bf_hi(x.y), a);
    a = fmaf(bf_lo(x.z), bf_lo(x.z), a);
    a = fmaf(bf_hi(x.z), bf_hi(x.z), a);
    a = fmaf(bf_lo(x.w), bf_lo(x.w), a);
    a = fmaf(bf_hi(x.w), bf_hi(x.w), a);
    return a;
  }
  __device__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
};

// (distance, index) order of the argmax: larger distance wins, then lower index.
__device__ __forceinline__ bool better(float d1, int i1, float d2, int i2) {
  return d1 > d2 || (d1 == d2 && i1 < i2);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    fps_kernel(const FpsGeom g, const T *__restrict__ beacons_in, const T *__restrict__ window,
               T *__restrict__ beacons_out) {
  extern __shared__ __align__(16) float sm[];
  const int d = g.head_dim;
  const int n = g.nb_in + g.W;
  float *sv = sm;                 // [kMaxDim] picked point, f32
  float *inv = sv + kMaxDim;      // [n] inverse norms (0 for a zero vector)
  float *dist = inv + n;          // [n] distance to the selected set; -1 = selected
  __shared__ float red_d[kWarps];
  __shared__ int red_i[kWarps];
  __shared__ int pick_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t qh = blockIdx.x;  // layer * n_q_heads + query head
  const T *B = beacons_in + qh * static_cast<size_t>(g.M) * d;
  const T *Wp = window + qh * static_cast<size_t>(g.W) * d;
  T *out = beacons_out + qh * static_cast<size_t>(g.M) * d;
  auto point = [&](int i) -> const T * {
    return i < g.nb_in ? B + static_cast<size_t>(i) * d : Wp + static_cast<size_t>(i - g.nb_in) * d;
  };

  for (int i = tid; i < n; i += kThreads) {
    const T *p = point(i);
    float ss = 0.f;
    for (int t = 0; t < d; t += Vec<T>::kPer) ss += Vec<T>::sq16(p + t);
    inv[i] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
  }
  int pick = 0;
  for (int step = 0; step < g.n_pick; ++step) {
    const T *pp = point(pick);
    for (int t = tid; t < d; t += kThreads) {
      out[static_cast<size_t>(step) * d + t] = pp[t];
      sv[t] = Vec<T>::to_f(pp[t]);
    }
    __syncthreads();  // sv and (first step) inv are ready
    if (step + 1 == g.n_pick) break;
    const float inv_s = inv[pick];
    float best_d = -2.f;
    int best_i = n;
    for (int i = tid; i < n; i += kThreads) {
      float di;
      if (i == pick || (step > 0 && dist[i] < 0.f)) {
        di = -1.f;
      } else {
        const T *p = point(i);
        float dot = 0.f;
        for (int t = 0; t < d; t += Vec<T>::kPer) dot += Vec<T>::dot16(p + t, sv + t);
        float dd = 1.0f - dot * inv[i] * inv_s;
        dd = fminf(fmaxf(dd, 0.f), 2.f);
        di = step > 0 ? fminf(dist[i], dd) : dd;
      }
      dist[i] = di;
      if (better(di, i, best_d, best_i)) {
        best_d = di;
        best_i = i;
      }
    }
    for (int off = 16; off > 0; off >>= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, best_d, off);
      const int oi = __shfl_xor_sync(0xffffffffu, best_i, off);
      if (better(od, oi, best_d, best_i)) {
        best_d = od;
        best_i = oi;
      }
    }
    if (lane == 0) {
      red_d[warp] = best_d;
      red_i[warp] = best_i;
    }
    __syncthreads();
    if (warp == 0) {
      best_d = lane < kWarps ? red_d[lane] : -2.f;
      best_i = lane < kWarps ? red_i[lane] : n;
      for (int off = 16; off > 0; off >>= 1) {
        const float od = __shfl_xor_sync(0xffffffffu, best_d, off);
        const int oi = __shfl_xor_sync(0xffffffffu, best_i, off);
        if (better(od, oi, best_d, best_i)) {
          best_d = od;
          best_i = oi;
        }
      }
      if (lane == 0) pick_sh = best_i;
    }
    __syncthreads();
    pick = pick_sh;
  }
}

size_t fps_smem_bytes(const FpsGeom &g) {
  return (kMaxDim + 2 * static_cast<size_t>(g.nb_in + g.W)) * sizeof(float);
}

template <typename T>
bkv_status launch_typed(const FpsGeom &g, const void *bin, const void *win, void *bout,
                        cudaStream_t stream) {
  static int attr_done[64];
  if (!ensure_smem_limit(fps_kernel<T>, kSmemLimit - 1024, attr_done)) return BKV_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(g.n_layers) * static_cast<unsigned>(g.n_q_heads);
  fps_kernel<T><<<grid, kThreads, fps_smem_bytes(g), stream>>>(
      g, static_cast<const T *>(bin), static_cast<const T *>(win), static_cast<T *>(bout));
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace

size_t fps_workspace_bytes(const FpsGeom &) { return 0; }

bool fps_supported(const FpsGeom &g) {
  return g.head_dim <= kMaxDim && fps_smem_bytes(g) <= static_cast<size_t>(kSmemLimit - 1024);
}

bkv_status launch_fps(const FpsGeom &g, const void *beacons_in, const void *window,
                      void *beacons_out, void *, size_t, cudaStream_t stream) {
  if (!fps_supported(g)) return BKV_ERR_UNSUPPORTED;
  if (g.n_pick <= 0) return BKV_OK;
  if (g.dtype == BKV_BF16)
    return launch_typed<__nv_bfloat16>(g, beacons_in, window, beacons_out, stream);
  return launch_typed<float>(g, beacons_in, window, beacons_out, stream);
}

}  // namespace bkv
