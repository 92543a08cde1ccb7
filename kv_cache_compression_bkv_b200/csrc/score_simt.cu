// score_simt.cu -- attention-based scores with max (or mean) aggregation on
// the CUDA cores, for f32 caches (small correctness workloads; BeaconKV
// Fig. 5(b)/(c), Table 2).  Same two passes as the tensor-core path:
//   pass 1: c_o = log sum_j exp(scale * q_o . k_j), one warp per observation
//           row, an online (max, sum) per lane, merged across the warp;
//   pass 2: y_j = max_o (scale * q_o . k_j - c_o), one thread per key (for
//           the mean: y_j = sum_o exp(scale * q_o . k_j - c_o)).
#include <cuda_runtime.h>

#include "bkv_internal.h"

namespace bkv {
namespace {

constexpr int kMaxDim = 128;

__device__ __forceinline__ const float *obs_row_f32(const ScoreGeom &g, const float *recent,
                                                    const float *beacons, int layer, int kvh,
                                                    int o) {
  const int per = g.R + g.nb;
  const int gq = o / per;
  const int i = o - gq * per;
  const long long qh = static_cast<long long>(layer) * g.n_q_heads +
                       static_cast<long long>(kvh) * g.group + gq;
  if (i < g.R)  // row (recent_start + i) mod recent_cap of the head's block (a ring or dense)
    return recent + (qh * g.recent_cap + (g.recent_start + i) % g.recent_cap) * g.head_dim;
  return beacons + (qh * g.M + (i - g.R)) * g.head_dim;
}

__device__ __forceinline__ float dot_f32(const float *a, const float *b, int d) {
  float acc0 = 0.f, acc1 = 0.f;
  for (int t = 0; t < d; t += 4) {
    const float4 x = *reinterpret_cast<const float4 *>(a + t);
    const float4 y = *reinterpret_cast<const float4 *>(b + t);
    acc0 = fmaf(x.x, y.x, acc0);
    acc1 = fmaf(x.y, y.y, acc1);
    acc0 = fmaf(x.z, y.z, acc0);
    acc1 = fmaf(x.w, y.w, acc1);
  }
  return acc0 + acc1;
}

constexpr int kRowsPerBlock = 8;

__global__ void __launch_bounds__(256) rowstats_simt_kernel(const ScoreGeom g,
                                                            const float *__restrict__ k,
                                                            const float *__restrict__ recent,
                                                            const float *__restrict__ beacons,
                                                            float *__restrict__ c_out) {
  __shared__ __align__(16) float q_sh[kRowsPerBlock][kMaxDim];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int layer = head / g.n_kv_heads, kvh = head - layer * g.n_kv_heads;
  const int o = blockIdx.x * kRowsPerBlock + warp;
  const int d = g.head_dim;
  if (o < g.n_obs) {
    const float *q = obs_row_f32(g, recent, beacons, layer, kvh, o);
    for (int t = lane; t < d; t += 32) q_sh[warp][t] = q[t];
  }
  __syncwarp();
  if (o >= g.n_obs) return;
  const float *kh = k + static_cast<size_t>(head) * g.cap * d;
  float m = -INFINITY, s = 0.f;
  for (long long j = lane; j < g.L; j += 32) {
    const float x = g.scale * dot_f32(q_sh[warp], kh + j * d, d);
    if (x > m) {
      s = s * expf(m - x) + 1.f;
      m = x;
    } else {
      s += expf(x - m);
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
    const float M = fmaxf(m, m2);
    s = (m == -INFINITY ? 0.f : s * expf(m - M)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - M));
    m = M;
  }
  if (lane == 0) c_out[static_cast<size_t>(head) * g.n_obs_pad + o] = m + logf(s);
}

constexpr int kKeysPerBlock = 128;
constexpr int kObsChunk = 32;

// Per key j: max over the rows of (x_oj - c_o), or with kMean the sum over
// the rows of exp(x_oj - c_o).
template <bool kMean>
__global__ void __launch_bounds__(kKeysPerBlock) colmax_simt_kernel(
    const ScoreGeom g, const float *__restrict__ k, const float *__restrict__ recent,
    const float *__restrict__ beacons, const float *__restrict__ c_in,
    float *__restrict__ ypart) {
  __shared__ __align__(16) float q_sh[kObsChunk][kMaxDim];
  __shared__ float c_sh[kObsChunk];
  const int head = blockIdx.y;
  const int layer = head / g.n_kv_heads, kvh = head - layer * g.n_kv_heads;
  const int d = g.head_dim;
  const long long j = static_cast<long long>(blockIdx.x) * kKeysPerBlock + threadIdx.x;
  const float *kj = k + (static_cast<size_t>(head) * g.cap + (j < g.L ? j : 0)) * d;
  float y = kMean ? 0.f : -INFINITY;
  for (int o0 = 0; o0 < g.n_obs; o0 += kObsChunk) {
    const int n = min(kObsChunk, g.n_obs - o0);
    __syncthreads();
    for (int e = threadIdx.x; e < n * d; e += blockDim.x) {
      const int r = e / d, t = e - r * d;
      q_sh[r][t] = obs_row_f32(g, recent, beacons, layer, kvh, o0 + r)[t];
    }
    for (int r = threadIdx.x; r < n; r += blockDim.x)
      c_sh[r] = c_in[static_cast<size_t>(head) * g.n_obs_pad + o0 + r];
    __syncthreads();
    for (int r = 0; r < n; ++r) {
      const float a = g.scale * dot_f32(q_sh[r], kj, d) - c_sh[r];
      y = kMean ? y + expf(a) : fmaxf(y, a);
    }
  }
  if (j < g.L) ypart[static_cast<size_t>(head) * g.L + j] = y;
}

}  // namespace

bkv_status launch_score_rowstats_simt(const ScoreGeom &g, const float *k, const float *recent,
                                      const float *beacons, float *c, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  dim3 grid((g.n_obs + kRowsPerBlock - 1) / kRowsPerBlock, g.n_heads());
  rowstats_simt_kernel<<<grid, 256, 0, stream>>>(g, k, recent, beacons, c);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

bkv_status launch_score_colmax_simt(const ScoreGeom &g, const float *k, const float *recent,
                                    const float *beacons, const float *c, float *ypart,
                                    bool mean, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  dim3 grid(static_cast<unsigned>((g.L + kKeysPerBlock - 1) / kKeysPerBlock), g.n_heads());
  if (mean)
    colmax_simt_kernel<true><<<grid, kKeysPerBlock, 0, stream>>>(g, k, recent, beacons, c, ypart);
  else
    colmax_simt_kernel<false><<<grid, kKeysPerBlock, 0, stream>>>(g, k, recent, beacons, c, ypart);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace bkv
