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

}  // namespace fpsk
}  // namespace bkv
