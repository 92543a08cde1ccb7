// fps_tc.cu -- Continual farthest-point sampling (BeaconKV, Fig. 7) of bf16
// queries with head_dim 128, the distance pass of every round on tcgen05.
//
// Same exact speculative rounds as fps.cu (select the T+1 best unselected
// points; Gram block of the T candidates; replay the greedy choice among
// them while the best one provably beats every other point; lower all
// distances by the round's picks), with T = 64 and the contractions on the
// tensor cores:
//   * the distance pass streams the union [beacons; window] of a query head
//     by TMA in tiles of 128 points (128-byte swizzle, no multicast) through a
//     4-stage ring and forms D[128 points][N] = tile . picks^T (M = 128, N =
//     picks rounded up to 16, K = 128) in one of two TMEM accumulators.  Two
//     threads issue the MMAs, warp 1 for the even tiles of the sequence
//     (stages 0 and 2, accumulator 0) and warp 2 for the odd ones, so their
//     instruction latencies overlap and every stage and accumulator keeps a
//     single consumer.  Two epilogue warpgroups (TMEM lane = point) turn the
//     dot products into cosine distances and lower the distance array;
//   * the candidates' rows are staged in the MMA's swizzled layout and one
//     M = 128 x N = 64 MMA forms their Gram block, the same f32 sums of exact
//     bf16 products as the distance pass.
// While a round selects, the first tiles of its coming pass are already
// loaded into the ring.  After the seed pass (whose epilogue also reads the
// staged tiles for the norms) a stage is released by the MMA's commit.
//
// The grid is persistent: one CTA per SM loops over the query heads.  The
// distance and inverse-norm arrays live in shared memory, or for a union too
// large for it in the caller's workspace (one slice per CTA).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "bkv_internal.h"
#include "fps_common.cuh"
#include "sm100.cuh"
#include "tma_host.h"

BKV_DEFINE_STATUS_ACCESSOR(take_status_fps_tc)

namespace bkv {
namespace {

using namespace sm100;
using namespace fpsk;

constexpr int kThreads = 384;  // warp 0 TMA, warps 1-2 MMA, warps 4..11 distance epilogue
constexpr int kWarps = kThreads / 32;
constexpr int kCand = 64;      // candidates per round (T)
constexpr int kDim = 128;
constexpr int kTileRows = 128;
constexpr int kStages = 4;  // even tiles use stages 0 and 2, odd tiles 1 and 3
constexpr int kTileBytes = kTileRows * kDim * 2;  // 32 KB
constexpr int kBBlock = kCand * 128;              // one 64-element K block of the picks
constexpr int kBBytes = 2 * kBBlock;              // 16 KB
constexpr int kCRows = kCand;                     // candidate operand rows
constexpr int kCBlock = kCRows * 128;             // one 64-element K block of the candidates
constexpr int kCBytes = 2 * kCBlock;              // 16 KB
constexpr int kSmallBytes = 4096;
constexpr int kFixedBytes = kSmallBytes + 1024 + kStages * kTileBytes + kBBytes +
                            kCBytes + kCand * kCand * 4 + kWarps * 256 * 4;
constexpr int kSmemLimit = 232448;
// two accumulators of up to 64 columns, then the candidates' Gram block
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kGramCol = 128;
constexpr int kAbort = 15;           // index of the abort flag in scal[]

enum { kWhereProd = 401, kWhereMma = 402, kWhereEpi = 403, kWhereDrain = 404 };

// Barriers: full[4] empty[4] tfull[2] tempty[2], the two MMA threads' drain
// barriers, the Gram block's.
constexpr int kBarFull = 0, kBarEmpty = 4, kBarTfull = 8, kBarTempty = 10, kBarDone = 12,
              kBarGram = 14;

struct Layout {
  uint64_t *bars;   // see kBarFull ..
  uint32_t *tmem_slot;
  int *scal;        // [16]
  uint32_t *hist;   // [256]
  int *cidx;        // [kCand + 1]
  float *cdist;     // [kCand + 1]
  int *pick;        // [kCand]
  float *pinv;      // [kCand]
  uint8_t *stages;  // [kStages][kTileBytes]
  uint8_t *bop;     // picks, K-major 128-byte swizzle: [2][kCand rows][128 B]
  uint8_t *cop;     // candidates, K-major 128-byte swizzle: [2][kCRows rows][128 B]
  float *gram;      // [kCand][kCand]
  uint32_t *whist;  // [kWarps][256] per-warp histograms of the selection
  float *dist;      // [n]
  float *inv;       // [n]
};

struct Head {
  const __nv_bfloat16 *B, *Wp;
  int nb, W;
  __device__ const __nv_bfloat16 *point(int i) const {
    return i < nb ? B + static_cast<size_t>(i) * kDim : Wp + static_cast<size_t>(i - nb) * kDim;
  }
};

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Issue the TMA loads of tiles [j0, j1) of the pass that starts at `seq`
// (producer thread only).  Returns false after a timeout.
__device__ bool issue_tiles(const Layout &s, const CUtensorMap *bmap, const CUtensorMap *wmap,
                            int qh, const FpsGeom &g, int n_btiles, uint32_t seq, int j0,
                            int j1) {
  const uint32_t full0 = smem_u32(&s.bars[kBarFull]), empty0 = smem_u32(&s.bars[kBarEmpty]);
  for (int j = j0; j < j1; ++j) {
    const uint32_t q = seq + j, st = q % kStages;
    if (!mbar_wait(empty0 + 8 * st, ((q / kStages) & 1) ^ 1, kWhereProd)) return false;
    mbar_arrive_expect_tx(full0 + 8 * st, kTileBytes);
    const uint32_t dst = smem_u32(s.stages + st * kTileBytes);
    const CUtensorMap *map = j < n_btiles ? bmap : wmap;
    const int y = j < n_btiles ? qh * g.M + j * kTileRows : qh * g.W + (j - n_btiles) * kTileRows;
    tma_load_2d(dst, map, full0 + 8 * st, 0, y);
    tma_load_2d(dst + kTileRows * 128, map, full0 + 8 * st, 64, y);
  }
  return true;
}

// One distance pass over every tile of the head: the producer (warp 0), the
// two MMA threads (warps 1 and 2) and the epilogue warpgroups (warps 4..11)
// run their own loops; `seq` is the number of tiles all passes so far have
// moved through the ring, so every role derives the same stage, accumulator
// and barrier phase for each tile.
__device__ void distance_pass(const Layout &s, const CUtensorMap *bmap, const CUtensorMap *wmap,
                              uint32_t tmem, int qh, const FpsGeom &g, int n_btiles, int n_tiles,
                              uint32_t seq, int np, bool first, int prefetched) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(&s.bars[kBarFull]), empty0 = smem_u32(&s.bars[kBarEmpty]);
  const uint32_t tfull0 = smem_u32(&s.bars[kBarTfull]), tempty0 = smem_u32(&s.bars[kBarTempty]);
  if (warp == 0) {
    if (lane == 0 &&
        !issue_tiles(s, bmap, wmap, qh, g, n_btiles, seq, prefetched, n_tiles))
      s.scal[kAbort] = 1;
  } else if (warp == 1 || warp == 2) {
    // two MMA threads, one per accumulator: warp 1 takes the even tiles of
    // the sequence (stages 0, 2, accumulator 0), warp 2 the odd ones, so the
    // issue latencies of their tcgen05 instructions and barrier waits overlap
    if (lane == 0) {
      const int npad = (np + 15) & ~15;
      const uint32_t idesc = idesc_bf16_f32(kTileRows, npad);
      const uint32_t b_base = smem_u32(s.bop);
      const uint32_t mine = static_cast<uint32_t>(warp - 1);
      for (int j = 0; j < n_tiles; ++j) {
        const uint32_t q = seq + j, st = q % kStages, a = q & 1;
        if (a != mine) continue;
        if (!mbar_wait(full0 + 8 * st, (q / kStages) & 1, kWhereMma) ||
            !mbar_wait(tempty0 + 8 * a, ((q >> 1) & 1) ^ 1, kWhereMma)) {
          s.scal[kAbort] = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(s.stages + st * kTileBytes);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_k_sw128(a_base + kb * (kTileRows * 128) + kk * 32);
            const uint64_t bd = smem_desc_k_sw128(b_base + kb * kBBlock + kk * 32);
            umma_f16(tmem + a * 64, ad, bd, idesc, (kb | kk) != 0);
          }
        }
        // the stage is free once these MMAs complete (in the seed pass the
        // epilogue still reads it for the norms and releases it itself)
        if (!first) umma_commit(empty0 + 8 * st);
        umma_commit(tfull0 + 8 * a);
      }
    }
  } else if (warp >= 4) {
    // epilogue warpgroup w consumes accumulator w, i.e. every other tile
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int npad = (np + 15) & ~15;
    bool ok = true;  // warp-uniform; after a timeout the warp keeps only the barriers
    for (int j = 0; j < n_tiles; ++j) {
      const uint32_t q = seq + j, a = q & 1;
      if (static_cast<int>(a) != wg) continue;
      if (ok && !mbar_wait_warp(tfull0 + 8 * a, (q >> 1) & 1, kWhereEpi)) {
        s.scal[kAbort] = 1;
        ok = false;
      }
      float v0[32], v1[32];
      if (ok) {
        tc_fence_after();
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + a * 64;
        tmem_ld_32x32b_x32(taddr, v0);
        if (npad > 32) tmem_ld_32x32b_x32(taddr + 32, v1);
        tmem_ld_wait_regs(v0);
        tmem_reg_fence(v1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty0 + 8 * a);
      }
      int i;
      bool valid;
      if (j < n_btiles) {
        i = j * kTileRows + r;
        valid = i < g.nb_in;
      } else {
        const int w = (j - n_btiles) * kTileRows + r;
        i = g.nb_in + w;
        valid = w < g.W;
      }
      const uint32_t st = q % kStages;
      if (first) {
        // the seed pass also takes every point's inverse norm from its row of
        // the staged tile (0 for a zero vector, whose distance is then 1)
        if (ok && !mbar_wait_warp(full0 + 8 * st, (q / kStages) & 1, kWhereEpi)) {
          s.scal[kAbort] = 1;
          ok = false;
        }
        if (ok) {
          const uint8_t *row = s.stages + st * kTileBytes;
          float ss = 0.f;
#pragma unroll
          for (int c16 = 0; c16 < 16; ++c16) {
            float u[8];
            load8(reinterpret_cast<const __nv_bfloat16 *>(
                      row + (c16 >> 3) * (kTileRows * 128) + sw128_offset(r, c16 & 7)),
                  u);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(u[e], u[e], ss);
          }
          if (valid) s.inv[i] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
        }
        named_barrier_sync(2 + wg, 128);
      }
      if (first && ok && warp == 4 + 4 * wg && lane == 0) mbar_arrive(empty0 + 8 * st);
      if (!ok) continue;
      const float di = !valid ? -1.f : first ? 2.f : s.dist[i];
      // the range of the new keys, which the next selection starts from
      uint32_t kmn = 0xffffffffu, kmx = 0u;
      if (di >= 0.f) {  // a point not yet selected
        // x_k = 1 - dot_k * inv_i * inv_k, as cos_dist computes it; padded
        // picks carry a NaN inverse norm, which min ignores
        const float inv_i = s.inv[i];
        const float2 ninv = make_float2(-inv_i, -inv_i);
        float mn = INFINITY;
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          if (k < npad) {
            const float4 pv = *reinterpret_cast<const float4 *>(s.pinv + k);
            const float2 x0 = __ffma2_rn(__fmul2_rn(make_float2(v0[k], v0[k + 1]), ninv),
                                         make_float2(pv.x, pv.y), make_float2(1.f, 1.f));
            const float2 x1 = __ffma2_rn(__fmul2_rn(make_float2(v0[k + 2], v0[k + 3]), ninv),
                                         make_float2(pv.z, pv.w), make_float2(1.f, 1.f));
            mn = fminf(mn, fminf(fminf(x0.x, x0.y), fminf(x1.x, x1.y)));
          }
        }
        if (npad > 32) {
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            if (k + 32 < npad) {
              const float4 pv = *reinterpret_cast<const float4 *>(s.pinv + 32 + k);
              const float2 x0 = __ffma2_rn(__fmul2_rn(make_float2(v1[k], v1[k + 1]), ninv),
                                           make_float2(pv.x, pv.y), make_float2(1.f, 1.f));
              const float2 x1 = __ffma2_rn(__fmul2_rn(make_float2(v1[k + 2], v1[k + 3]), ninv),
                                           make_float2(pv.z, pv.w), make_float2(1.f, 1.f));
              mn = fminf(mn, fminf(fminf(x0.x, x0.y), fminf(x1.x, x1.y)));
            }
          }
        }
        // min(di, clamp(x, 0, 2)) == max(min(di, x), 0) for di in [0, 2]
        const float nd = fmaxf(fminf(di, mn), 0.f);
        s.dist[i] = nd;
        kmn = kmx = dist_key(nd);
      }
      kmn = __reduce_min_sync(0xffffffffu, kmn);
      kmx = __reduce_max_sync(0xffffffffu, kmx);
      if (lane == 0) {
        atomicMin(reinterpret_cast<unsigned int *>(&s.scal[6]), kmn);
        atomicMax(reinterpret_cast<unsigned int *>(&s.scal[7]), kmx);
      }
    }
  }
}

// The picks of this round into the B operand (rows padded with zeros to a
// multiple of 16) and the output beacons: the seed's row from global memory,
// a round's picks from the staged candidate rows.
__device__ void stage_picks(const Layout &s, const Head &h, __nv_bfloat16 *out, int picked,
                            int np, bool seed) {
  const int npad = (np + 15) & ~15;
  for (int e = threadIdx.x; e < npad * 16; e += kThreads) {
    const int k = e >> 4, c16 = e & 15, kb = c16 >> 3, c = c16 & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k < np) {
      v = seed ? *reinterpret_cast<const uint4 *>(h.point(s.cidx[s.pick[k]]) + c16 * 8)
               : *reinterpret_cast<const uint4 *>(s.cop + kb * kCBlock + sw128_offset(s.pick[k], c));
      *reinterpret_cast<uint4 *>(out + static_cast<size_t>(picked + k) * kDim + c16 * 8) = v;
    }
    *reinterpret_cast<uint4 *>(s.bop + kb * kBBlock + sw128_offset(k, c)) = v;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    fps_tc_kernel(const __grid_constant__ CUtensorMap bmap, const __grid_constant__ CUtensorMap wmap,
                  const FpsGeom g, const __nv_bfloat16 *__restrict__ beacons_in,
                  const __nv_bfloat16 *__restrict__ window, __nv_bfloat16 *__restrict__ beacons_out,
                  int n_qheads, float *__restrict__ gdist) {
  extern __shared__ uint8_t smem_raw[];
  const int n = g.nb_in + g.W;
  const int m = g.n_pick;
  Layout s;
  s.bars = reinterpret_cast<uint64_t *>(smem_raw);
  s.tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + 128);
  s.scal = reinterpret_cast<int *>(smem_raw + 192);
  s.hist = reinterpret_cast<uint32_t *>(smem_raw + 256);
  s.cidx = reinterpret_cast<int *>(smem_raw + 1280);
  s.cdist = reinterpret_cast<float *>(smem_raw + 1552);
  s.pick = reinterpret_cast<int *>(smem_raw + 1824);
  s.pinv = reinterpret_cast<float *>(smem_raw + 2096);
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t big = (raw_base + kSmallBytes + 1023u) & ~1023u;
  s.stages = smem_raw + (big - raw_base);
  s.bop = s.stages + kStages * kTileBytes;
  s.cop = s.bop + kBBytes;
  s.gram = reinterpret_cast<float *>(s.cop + kCBytes);
  s.whist = reinterpret_cast<uint32_t *>(s.gram + kCand * kCand);
  // the distance and inverse-norm arrays: in shared memory, or this CTA's
  // slice of the workspace for a union too large for it
  s.dist = gdist ? gdist + static_cast<size_t>(blockIdx.x) * 2 * n
                 : reinterpret_cast<float *>(s.whist + kWarps * 256);
  s.inv = s.dist + n;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_btiles = (g.nb_in + kTileRows - 1) / kTileRows;
  const int n_tiles = n_btiles + (g.W + kTileRows - 1) / kTileRows;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&s.bars[kBarFull + i]), 1);
      mbar_init(smem_u32(&s.bars[kBarEmpty + i]), 1);  // the MMA's commit (seed pass: the epilogue)
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&s.bars[kBarTfull + a]), 1);
      mbar_init(smem_u32(&s.bars[kBarTempty + a]), 4);  // one arrive per warp of its warpgroup
      mbar_init(smem_u32(&s.bars[kBarDone + a]), 1);
    }
    mbar_init(smem_u32(&s.bars[kBarGram]), 1);  // the Gram block's MMA
    fence_barrier_init();
    prefetch_tensormap(&bmap);
    prefetch_tensormap(&wmap);
    s.scal[kAbort] = 0;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s.tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_slot;
  uint32_t seq = 0;
  uint32_t gram_phase = 0;
  bool stuck = false;  // uniform: set by every thread from the same shared value

  for (int qh = blockIdx.x; qh < n_qheads; qh += gridDim.x) {
    Head h{beacons_in + static_cast<size_t>(qh) * g.M * kDim,
           window + static_cast<size_t>(qh) * g.W * kDim, g.nb_in, g.W};
    __nv_bfloat16 *out = beacons_out + static_cast<size_t>(qh) * g.M * kDim;
    if (tid == 0) {
      s.cidx[0] = 0;  // the seed U[0] is the first pick
      s.pick[0] = 0;
      // its inverse norm, summed in the order the seed pass uses for every point
      float ss = 0.f;
      for (int t = 0; t < kDim; t += 8) {
        float u[8];
        load8(h.point(0) + t, u);
        for (int e = 0; e < 8; ++e) ss = fmaf(u[e], u[e], ss);
      }
      s.pinv[0] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
    }
    if (tid > 0 && tid < 16) s.pinv[tid] = __int_as_float(0x7fc00000);
    if (tid == 0) {  // the seed pass gathers the range of its keys (the seed's
      s.scal[6] = -1;  // own 0 among them: a lower bound is all it needs)
      s.scal[7] = 0;
    }
    __syncthreads();
    stage_picks(s, h, out, 0, 1, true);
    fence_proxy_async_smem();
    __syncthreads();
    distance_pass(s, &bmap, &wmap, tmem, qh, g, n_btiles, n_tiles, seq, 1, true, 0);
    seq += n_tiles;
    __syncthreads();
    if (s.scal[kAbort]) break;
    if (tid == 0) s.dist[0] = -1.f;
    __syncthreads();

    int picked = 1;
    while (picked < m) {
      const int unsel = n - picked;
      const int nc = min(kCand, unsel);
      const bool bounded = unsel > kCand;
      const int want = bounded ? kCand + 1 : nc;
      // the next distance pass streams the same tiles whatever this round
      // picks: start its first loads now, behind the round's selection work
      const int pre = min(kStages, n_tiles);
      if (tid == 0 && !issue_tiles(s, &bmap, &wmap, qh, g, n_btiles, seq, 0, pre))
        s.scal[kAbort] = 1;
      select_best<kThreads>(s.dist, n, unsel, want, s.whist, s.hist, s.scal, s.cidx, s.cdist,
                            true);  // the pass left the key range in scal[6..7]
      __syncthreads();
      // the candidates need no order; only the bound (the last of the kCand+1
      // selected in (distance desc, index asc) order) moves to slot kCand
      if (bounded && warp == 0) {
        float wd = 3.f;
        int wi = -1, ws = -1;
        for (int j = lane; j < want; j += 32) {
          const float dj = s.cdist[j];
          const int ij = s.cidx[j];
          if (ws < 0 || before(wd, wi, dj, ij)) {
            wd = dj;
            wi = ij;
            ws = j;
          }
        }
        for (int off = 16; off > 0; off >>= 1) {
          const float od = __shfl_xor_sync(0xffffffffu, wd, off);
          const int oi = __shfl_xor_sync(0xffffffffu, wi, off);
          const int os = __shfl_xor_sync(0xffffffffu, ws, off);
          if (os >= 0 && (ws < 0 || before(wd, wi, od, oi))) {
            wd = od;
            wi = oi;
            ws = os;
          }
        }
        if (lane == 0 && ws != kCand) {
          s.cidx[ws] = s.cidx[kCand];
          s.cdist[ws] = s.cdist[kCand];
          s.cidx[kCand] = wi;
          s.cdist[kCand] = wd;
        }
      }
      __syncthreads();
      // the candidates' rows into the swizzled operand (rows past nc keep
      // whatever an earlier round left; their Gram entries are never read)
      for (int e = tid; e < nc * 16; e += kThreads) {
        const int a = e >> 4, c16 = e & 15, kb = c16 >> 3, c = c16 & 7;
        *reinterpret_cast<uint4 *>(s.cop + kb * kCBlock + sw128_offset(a, c)) =
            *reinterpret_cast<const uint4 *>(h.point(s.cidx[a]) + c16 * 8);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // Gram block on the tensor cores: D[a][b] = cand_a . cand_b, N = kCand,
      // K = 128, the same f32 accumulation of exact bf16 products as the
      // distance pass.  M = 128: rows a >= kCand of A run on into the next
      // 8 KB of shared memory (the other K block, then the Gram buffer), and
      // those rows of D are never read.
      if (warp == 1 && lane == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, kCand);
        const uint32_t c_base = smem_u32(s.cop);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_k_sw128(c_base + kb * kCBlock + kk * 32);
            umma_f16(tmem + kGramCol, ad, ad, idesc, (kb | kk) != 0);
          }
        }
        umma_commit(smem_u32(&s.bars[kBarGram]));
      }
      if (warp == 4 || warp == 5) {
        // TMEM lane = candidate a: warp 4 reads rows 0..31, warp 5 rows 32..63
        if (mbar_wait_warp(smem_u32(&s.bars[kBarGram]), gram_phase & 1, kWhereEpi)) {
          tc_fence_after();
          const uint32_t taddr = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16) + kGramCol;
          float *row = s.gram + ((warp - 4) * 32 + lane) * kCand;
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            float x[32];
            tmem_ld_32x32b_x32(taddr + half * 32, x);
            tmem_ld_wait_regs(x);
#pragma unroll
            for (int b = 0; b < 32; b += 4)
              *reinterpret_cast<float4 *>(row + half * 32 + b) =
                  make_float4(x[b], x[b + 1], x[b + 2], x[b + 3]);
          }
        } else {
          s.scal[kAbort] = 1;
        }
        tc_fence_before();
      }
      ++gram_phase;
      __syncthreads();
      // replay the greedy choice among the candidates (warp 0, two per lane).
      // The argmax in (distance desc, index asc) order takes two warp
      // reductions: the largest distance key, then the lowest index holding it.
      if (warp == 0) {
        const int a0 = lane, a1 = lane + 32;
        bool t0 = a0 >= nc, t1 = a1 >= nc;  // taken or absent
        float c0 = t0 ? 0.f : s.cdist[a0], c1 = t1 ? 0.f : s.cdist[a1];
        const int i0 = t0 ? 0x7fffffff : s.cidx[a0], i1 = t1 ? 0x7fffffff : s.cidx[a1];
        const float inv0 = t0 ? 0.f : s.inv[i0], inv1 = t1 ? 0.f : s.inv[i1];
        const float bd = bounded ? s.cdist[kCand] : -3.f;
        const int bi = bounded ? s.cidx[kCand] : 0x7fffffff;
        int np = 0;
        while (picked + np < m) {
          // distances are >= 0, so their bits order like the values; +1 keeps
          // 0 free for "taken"
          const uint32_t k0 = t0 ? 0u : __float_as_uint(c0) + 1u;
          const uint32_t k1 = t1 ? 0u : __float_as_uint(c1) + 1u;
          const uint32_t kbest = __reduce_max_sync(0xffffffffu, max(k0, k1));
          if (kbest == 0u) break;  // no candidate left
          const uint32_t mine = min(k0 == kbest ? static_cast<uint32_t>(i0) : 0xffffffffu,
                                    k1 == kbest ? static_cast<uint32_t>(i1) : 0xffffffffu);
          const int best_i = static_cast<int>(__reduce_min_sync(0xffffffffu, mine));
          const float best_d = __uint_as_float(kbest - 1u);
          if (bounded && !before(best_d, best_i, bd, bi)) break;
          const bool own0 = k0 == kbest && i0 == best_i, own1 = k1 == kbest && i1 == best_i;
          const uint32_t owners = __ballot_sync(0xffffffffu, own0 || own1);
          const int src = __ffs(owners) - 1;
          const int best_a = __shfl_sync(0xffffffffu, own0 ? a0 : a1, src);
          if (lane == 0) s.pick[np] = best_a;
          ++np;
          if (own0) t0 = true;
          if (own1) t1 = true;
          const float inv_b = s.inv[best_i];
          if (!t0) c0 = fminf(c0, cos_dist(make_float2(s.gram[best_a * kCand + a0], 0.f), inv0, inv_b));
          if (!t1) c1 = fminf(c1, cos_dist(make_float2(s.gram[best_a * kCand + a1], 0.f), inv1, inv_b));
        }
        if (lane == 0) s.scal[4] = np;
      }
      __syncthreads();
      const int np = s.scal[4];
      if (np == 0) {
        // only distances that are not numbers (NaN input rows) can stop the
        // replay before its first pick; report and stop instead of looping
        if (tid == 0) record_device_status(BKV_DEV_ASSERT, 405);
        stuck = true;
        seq += pre;  // the coming pass's first tiles are in flight: drain them
        break;
      }
      if (tid < ((np + 15) & ~15))
        s.pinv[tid] = tid < np ? s.inv[s.cidx[s.pick[tid]]] : __int_as_float(0x7fc00000);
      stage_picks(s, h, out, picked, np, false);
      __syncthreads();
      if (tid < np) s.dist[s.cidx[s.pick[tid]]] = -1.f;
      if (tid == 0) {  // the coming pass gathers the range of its new keys
        s.scal[6] = -1;
        s.scal[7] = 0;
      }
      fence_proxy_async_smem();
      __syncthreads();
      distance_pass(s, &bmap, &wmap, tmem, qh, g, n_btiles, n_tiles, seq, np, false, pre);
      seq += n_tiles;
      __syncthreads();
      if (s.scal[kAbort]) break;
      picked += np;
    }
    if (s.scal[kAbort] || stuck) break;
  }

  // drain: every TMA load and MMA issued by this CTA has completed before the
  // CTA exits and frees its TMEM
  if (warp == 0 && lane == 0 && seq > 0) {
    const uint32_t first = seq > kStages ? seq - kStages : 0;
    for (uint32_t q = first; q < seq; ++q)
      mbar_wait(smem_u32(&s.bars[kBarFull + q % kStages]), (q / kStages) & 1, kWhereDrain);
  }
  if ((warp == 1 || warp == 2) && lane == 0) {
    umma_commit(smem_u32(&s.bars[kBarDone + warp - 1]));
    mbar_wait(smem_u32(&s.bars[kBarDone + warp - 1]), 0, kWhereDrain);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

namespace {

// The persistent grid never exceeds this many CTAs (the workspace holds one
// distance slice per CTA when the arrays live there).
constexpr int kMaxCtas = 148;

size_t union_array_bytes(const FpsGeom &g) { return 8 * (static_cast<size_t>(g.nb_in) + g.W); }

bool arrays_in_smem(const FpsGeom &g) {
  return static_cast<size_t>(kFixedBytes) + union_array_bytes(g) <= static_cast<size_t>(kSmemLimit);
}

size_t smem_bytes(const FpsGeom &g) {
  return static_cast<size_t>(kFixedBytes) + (arrays_in_smem(g) ? union_array_bytes(g) : 0);
}

int fps_tc_grid(const FpsGeom &g) { return std::min(g.n_layers * g.n_q_heads, kMaxCtas); }

}  // namespace

size_t fps_tc_workspace_bytes(const FpsGeom &g) {
  return arrays_in_smem(g) ? 0 : static_cast<size_t>(fps_tc_grid(g)) * union_array_bytes(g);
}

bool fps_tc_supported(const FpsGeom &g) {
  return g.dtype == BKV_BF16 && g.head_dim == kDim &&
         static_cast<long long>(g.n_layers) * g.n_q_heads * std::max(g.M, g.W) < (1LL << 31) - 256;
}

bkv_status launch_fps_tc(const FpsGeom &g, const void *beacons_in, const void *window,
                         void *beacons_out, void *ws, size_t ws_bytes, cudaStream_t stream) {
  const size_t ws_need = fps_tc_workspace_bytes(g);
  if (ws_need > 0 && (ws == nullptr || ws_bytes < ws_need ||
                      (reinterpret_cast<uintptr_t>(ws) & 15u) != 0))
    return BKV_ERR_WORKSPACE;
  const int n_qheads = g.n_layers * g.n_q_heads;
  // Tensor maps over every head's beacon slots and window rows.  A map needs
  // a non-empty tensor: an absent part (no beacons, or no window) points at
  // the other one and is never read.
  const void *bsrc = g.nb_in > 0 ? beacons_in : window;
  const void *wsrc = g.W > 0 ? window : beacons_in;
  const unsigned long long brows =
      static_cast<unsigned long long>(n_qheads) * static_cast<unsigned long long>(g.nb_in > 0 ? g.M : g.W);
  const unsigned long long wrows =
      static_cast<unsigned long long>(n_qheads) * static_cast<unsigned long long>(g.W > 0 ? g.W : g.M);
  CUtensorMap bmap, wmap;
  if (!make_bf16_rows_map(&bmap, bsrc, brows, kTileRows) ||
      !make_bf16_rows_map(&wmap, wsrc, wrows, kTileRows))
    return BKV_ERR_CUDA;
  static int attr_done[64];
  const int smem = static_cast<int>(smem_bytes(g));
  if (!ensure_smem_limit(fps_tc_kernel, kSmemLimit, attr_done)) return BKV_ERR_CUDA;
  int sms = kMaxCtas, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::max(1, std::min(fps_tc_grid(g), sms));
  fps_tc_kernel<<<grid, kThreads, smem, stream>>>(
      bmap, wmap, g, static_cast<const __nv_bfloat16 *>(beacons_in),
      static_cast<const __nv_bfloat16 *>(window), static_cast<__nv_bfloat16 *>(beacons_out),
      n_qheads, ws_need > 0 ? static_cast<float *>(ws) : nullptr);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace bkv
