// fps.cu -- Continual farthest-point sampling of the beacon queries
// (BeaconKV, Fig. 7) in cosine distance.
//
// For each (layer, query head) the union U = [current beacons; newest window]
// is sampled greedily: seed U[0]; each further pick is the unselected point
// with the largest distance to the selected set (ties to the lowest index);
// dist(a, b) = 1 - (u_a . u_b) / (|u_a| |u_b|), clamped to [0, 2], and 1 when a
// norm is zero.
//
// The greedy picks are found in exact speculative rounds, so that the points
// are streamed once per round rather than once per pick:
//   1. the T+1 best unselected points by (distance desc, index asc) are found
//      by a radix select over the shared-memory distance array; the first T
//      are the candidates, the last bounds every other point (distances only
//      ever decrease);
//   2. the candidates' Gram block is formed (same arithmetic as step 4);
//   3. one warp replays the greedy choice among the candidates alone: the best
//      remaining candidate is the true argmax while it beats that bound, so it
//      is picked and the other candidates' distances are lowered with the Gram
//      block; the round stops at the first candidate that does not;
//   4. one pass over the points lowers every distance by the round's picks
//      (packed FFMA2 dot products, the point loaded and converted once per
//      round and reused for every pick).
// The result is exactly the greedy sequence (no approximation); bf16 products
// are exact in f32, the sums are f32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "bkv_device_status.cuh"
#include "bkv_internal.h"
#include "fps_common.cuh"

BKV_DEFINE_STATUS_ACCESSOR(take_status_fps)

namespace bkv {
namespace {

using namespace fpsk;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kCand = 32;        // candidates per round (T)
constexpr int kMaxDim = 128;
constexpr int kCStride = kMaxDim + 4;  // candidate rows, padded against bank conflicts
constexpr int kSmemLimit = 232448;

struct Smem {
  float *dist;       // [n]
  float *inv;        // [n]
  float *cvec;       // [kCand][kCStride] candidate vectors (f32)
  float *pvec;       // [kCand][d] this round's picks (f32)
  float *gram;       // [kCand][kCand]
  uint32_t *hist;    // [256]
  uint32_t *whist;   // [kWarps][256]
  int *cidx;         // [kCand + 1] candidates, then the bound
  float *cdist;      // [kCand + 1]
  int *pick;         // [kCand] candidate slots picked this round
  float *pinv;       // [kCand]
  int *scal;         // [8]
};

// Union point i: beacon i, or window row i - nb, which is row
// (w_start + i - nb) mod w_cap of the head's window block (dense or a ring).
template <typename T>
struct Points {
  const T *B, *Wp;
  int nb, d;
  long long w_cap, w_start;
  __device__ const T *operator()(int i) const {
    return i < nb ? B + static_cast<size_t>(i) * d
                  : Wp + static_cast<size_t>((w_start + (i - nb)) % w_cap) * d;
  }
};

// Lower every unselected point's distance by the picks pvec[0..np) (or set it,
// for the seed).  NP >= np accumulators are carried; the extra ones are not used.
template <int NP, int D, typename T>
__device__ void point_pass(const Smem &s, const Points<T> &pt, int n, int np, bool first) {
  for (int i = threadIdx.x; i < n; i += kThreads) {
    float di = s.dist[i];
    if (!first && di < 0.f) continue;
    const T *p = pt(i);
    float2 acc[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < D; t += 8) {
      float u[8];
      load8(p + t, u);
#pragma unroll
      for (int k = 0; k < NP; ++k) acc[k] = dot8_step(acc[k], u, s.pvec + k * kMaxDim + t);
    }
    const float inv_i = s.inv[i];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      if (k < np) {
        const float dd = cos_dist(acc[k], inv_i, s.pinv[k]);
        di = (first && k == 0) ? dd : fminf(di, dd);
      }
    }
    s.dist[i] = di;
  }
}

template <int D, typename T>
__device__ void point_pass_dispatch(const Smem &s, const Points<T> &pt, int n, int np,
                                    bool first) {
  switch ((np + 3) >> 2) {
    case 1: point_pass<4, D>(s, pt, n, np, first); break;
    case 2: point_pass<8, D>(s, pt, n, np, first); break;
    case 3: point_pass<12, D>(s, pt, n, np, first); break;
    case 4: point_pass<16, D>(s, pt, n, np, first); break;
    case 5: point_pass<20, D>(s, pt, n, np, first); break;
    case 6: point_pass<24, D>(s, pt, n, np, first); break;
    case 7: point_pass<28, D>(s, pt, n, np, first); break;
    default: point_pass<32, D>(s, pt, n, np, first); break;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    fps_kernel(const FpsGeom g, const T *__restrict__ beacons_in, const T *__restrict__ window,
               T *__restrict__ beacons_out) {
  extern __shared__ __align__(16) float sm[];
  constexpr int d = D;
  const int n = g.nb_in + g.W;
  const int m = g.n_pick;
  Smem s;
  s.cvec = sm;
  s.pvec = s.cvec + kCand * kCStride;
  s.gram = s.pvec + kCand * kMaxDim;
  s.pinv = s.gram + kCand * kCand;
  s.cdist = s.pinv + kCand;
  s.dist = s.cdist + (kCand + 4);
  s.inv = s.dist + n;
  s.hist = reinterpret_cast<uint32_t *>(s.inv + n);
  s.whist = s.hist + 256;
  s.cidx = reinterpret_cast<int *>(s.whist + kWarps * 256);
  s.pick = s.cidx + (kCand + 4);
  s.scal = s.pick + kCand;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t qh = blockIdx.x;  // layer * n_q_heads + query head
  Points<T> pt{beacons_in + qh * static_cast<size_t>(g.M) * d,
               window + qh * static_cast<size_t>(g.w_cap) * d, g.nb_in, d,
               g.w_cap > 0 ? g.w_cap : 1, g.w_start};
  T *out = beacons_out + qh * static_cast<size_t>(g.M) * d;

  // inverse norms (0 for a zero vector, which makes its distance 1)
  for (int i = tid; i < n; i += kThreads) {
    const T *p = pt(i);
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < D; t += 8) {
      float u[8];
      load8(p + t, u);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(u[j], u[j], ss);
    }
    s.inv[i] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
  }
  // the seed, U[0], is the first pick
  for (int t = tid; t < d; t += kThreads) {
    s.pvec[t] = static_cast<float>(pt(0)[t]);
    out[t] = pt(0)[t];
  }
  __syncthreads();
  if (tid == 0) s.pinv[0] = s.inv[0];
  __syncthreads();
  point_pass_dispatch<D>(s, pt, n, 1, true);
  __syncthreads();
  if (tid == 0) s.dist[0] = -1.f;
  __syncthreads();

  int picked = 1;
  while (picked < m) {
    const int unsel = n - picked;
    const int nc = min(kCand, unsel);           // candidates this round
    const bool bounded = unsel > kCand;         // a (kCand+1)-th point exists
    select_best<kThreads>(s.dist, n, unsel, bounded ? kCand + 1 : nc, s.whist, s.hist, s.scal,
                          s.cidx, s.cdist);
    __syncthreads();
    // order the selected points: rank by (distance desc, index asc)
    const int want = bounded ? kCand + 1 : nc;
    int my_i = 0;
    float my_d = 0.f;
    int my_rank = 0;
    if (tid < want) {
      my_i = s.cidx[tid];
      my_d = s.cdist[tid];
      for (int j = 0; j < want; ++j)
        if (j != tid && before(s.cdist[j], s.cidx[j], my_d, my_i)) ++my_rank;
    }
    __syncthreads();
    if (tid < want) {
      s.cidx[my_rank] = my_i;
      s.cdist[my_rank] = my_d;
    }
    __syncthreads();
    // candidate vectors, f32
    for (int e = tid; e < nc * (d / 8); e += kThreads) {
      const int a = e / (d / 8), t = (e - a * (d / 8)) * 8;
      float u[8];
      load8(pt(s.cidx[a]) + t, u);
#pragma unroll
      for (int j = 0; j < 8; ++j) s.cvec[a * kCStride + t + j] = u[j];
    }
    __syncthreads();
    // Gram block: gram[a][b] = u_a . u_b with a as the point and b as the pick
    // (lanes take consecutive points a of one pick b: the b row is a broadcast
    // and the a rows fall in distinct banks)
    for (int e = tid; e < nc * nc; e += kThreads) {
      const int b = e / nc, a = e - b * nc;
      float2 acc = make_float2(0.f, 0.f);
      for (int t = 0; t < D; t += 8) {
        float u[8];
        load8(s.cvec + a * kCStride + t, u);
        acc = dot8_step(acc, u, s.cvec + b * kCStride + t);
      }
      s.gram[a * kCand + b] = __fadd_rn(acc.x, acc.y);
    }
    __syncthreads();
    // replay the greedy choice among the candidates (warp 0; lane a = candidate a)
    if (warp == 0) {
      const bool live = lane < nc;
      float cd = live ? s.cdist[lane] : -3.f;
      const int ci = live ? s.cidx[lane] : 0x7fffffff;
      const float cinv = live ? s.inv[ci] : 0.f;
      const float bd = bounded ? s.cdist[kCand] : -3.f;
      const int bi = bounded ? s.cidx[kCand] : 0x7fffffff;
      bool taken = !live;
      int np = 0;
      while (picked + np < m) {
        float best_d = taken ? -3.f : cd;
        int best_i = taken ? 0x7fffffff : ci;
        int best_a = lane;
        for (int off = 16; off > 0; off >>= 1) {
          const float od = __shfl_xor_sync(0xffffffffu, best_d, off);
          const int oi = __shfl_xor_sync(0xffffffffu, best_i, off);
          const int oa = __shfl_xor_sync(0xffffffffu, best_a, off);
          if (before(od, oi, best_d, best_i)) {
            best_d = od;
            best_i = oi;
            best_a = oa;
          }
        }
        if (best_d < 0.f) break;                       // no candidate left
        if (bounded && !before(best_d, best_i, bd, bi)) break;
        if (lane == 0) s.pick[np] = best_a;
        ++np;
        if (lane == best_a) taken = true;
        if (!taken) {
          const float2 dotv = make_float2(s.gram[lane * kCand + best_a], 0.f);
          cd = fminf(cd, cos_dist(dotv, cinv, s.inv[best_i]));
        }
      }
      if (lane == 0) s.scal[4] = np;
    }
    __syncthreads();
    const int np = s.scal[4];
    if (np == 0) {
      // only distances that are not numbers (NaN input rows) can stop the
      // replay before its first pick; report instead of looping
      if (tid == 0) record_device_status(BKV_DEV_ASSERT, 406);
      break;
    }
    // this round's picks: outputs, vectors, inverse norms
    for (int e = tid; e < np * d; e += kThreads) {
      const int k = e / d, t = e - k * d;
      const int a = s.pick[k];
      s.pvec[k * kMaxDim + t] = s.cvec[a * kCStride + t];
      out[static_cast<size_t>(picked + k) * d + t] = pt(s.cidx[a])[t];
    }
    if (tid < np) s.pinv[tid] = s.inv[s.cidx[s.pick[tid]]];
    __syncthreads();
    if (tid < np) s.dist[s.cidx[s.pick[tid]]] = -1.f;
    __syncthreads();
    point_pass_dispatch<D>(s, pt, n, np, false);
    __syncthreads();
    picked += np;
  }
}

size_t fps_smem_bytes(const FpsGeom &g) {
  const size_t n = static_cast<size_t>(g.nb_in) + g.W;
  return sizeof(float) * (kCand * kCStride + kCand * kMaxDim + kCand * kCand + kCand + kCand +
                          4 + 2 * n) +
         sizeof(uint32_t) * (256 + kWarps * 256) + sizeof(int) * (kCand + 4 + kCand + 8);
}

template <typename T, int D>
bkv_status launch_typed(const FpsGeom &g, const void *bin, const void *win, void *bout,
                        cudaStream_t stream) {
  static int attr_done[64];
  if (!ensure_smem_limit(fps_kernel<T, D>, kSmemLimit, attr_done)) return BKV_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(g.n_layers) * static_cast<unsigned>(g.n_q_heads);
  fps_kernel<T, D><<<grid, kThreads, fps_smem_bytes(g), stream>>>(
      g, static_cast<const T *>(bin), static_cast<const T *>(win), static_cast<T *>(bout));
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

template <typename T>
bkv_status launch_dim(const FpsGeom &g, const void *bin, const void *win, void *bout,
                      cudaStream_t stream) {
  switch (g.head_dim) {
    case 32: return launch_typed<T, 32>(g, bin, win, bout, stream);
    case 64: return launch_typed<T, 64>(g, bin, win, bout, stream);
    case 96: return launch_typed<T, 96>(g, bin, win, bout, stream);
    case 128: return launch_typed<T, 128>(g, bin, win, bout, stream);
    default: return BKV_ERR_UNSUPPORTED;
  }
}

}  // namespace

size_t fps_workspace_bytes(const FpsGeom &g) {
  return fps_tc_supported(g) ? fps_tc_workspace_bytes(g) : 0;
}

namespace {
bool fps_simt_supported(const FpsGeom &g) {
  return (g.head_dim == 32 || g.head_dim == 64 || g.head_dim == 96 || g.head_dim == 128) &&
         fps_smem_bytes(g) <= static_cast<size_t>(kSmemLimit);
}
}  // namespace

bool fps_supported(const FpsGeom &g) { return fps_tc_supported(g) || fps_simt_supported(g); }

// bf16 queries with head_dim 128 take the tensor-core kernel (fps_tc.cu);
// f32 inputs and other head sizes take the CUDA-core kernel above.
bkv_status launch_fps(const FpsGeom &g, const void *beacons_in, const void *window,
                      void *beacons_out, void *ws, size_t ws_bytes, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  if (g.n_pick <= 0) return BKV_OK;
  if (fps_tc_supported(g))
    return launch_fps_tc(g, beacons_in, window, beacons_out, ws, ws_bytes, stream);
  if (!fps_simt_supported(g)) return BKV_ERR_UNSUPPORTED;
  if (g.dtype == BKV_BF16)
    return launch_dim<__nv_bfloat16>(g, beacons_in, window, beacons_out, stream);
  return launch_dim<float>(g, beacons_in, window, beacons_out, stream);
}

}  // namespace bkv
