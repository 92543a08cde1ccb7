// score_tc.cu -- attention-based scores with max (or mean) aggregation on the
// sm_100a tensor cores (BeaconKV, Fig. 5(b)/(c); Table 2 "Max" and "Mean").
//
// For one (layer, KV head) with observation rows q_o and keys k_j (bf16,
// head_dim 128) the scores are
//     x_oj = scale * q_o . k_j,   c_o = log sum_j exp(x_oj),
//     y_j  = max_o (x_oj - c_o),  s_j = exp(y_j).
// c_o needs every key before any y_j is final, so the contraction runs twice:
//
//   pass 1 (row statistics)   D[o][j] = Q_blk . K_tile^T, M = 128 observation
//     rows, N = 256 keys.  TMEM lane = observation row, so each epilogue
//     thread owns one row and keeps a (reference, sum of exp2) pair over the
//     columns it reads -- the reference moves up only when a block's sum
//     shows a key far above it; no cross-thread reduction per element.
//   pass 2 (column max)       D[j][o] = K_tile . Q_grp^T - c_o / scale, M = 128
//     keys, N = up to 2 x 256 observation rows.  The subtraction is one more
//     K=16 step of the same MMA: every key carries a block (1, 1, 1, 0, ...)
//     and every observation row (-c_hi, -c_mid, -c_lo, 0, ...), the three
//     bf16 parts of c_o / scale.  TMEM lane = key, so each epilogue thread owns
//     one key and takes the max over its columns in registers.  The groups of
//     rows (CTAs) of a head meet in one row of order keys (order_key.cuh): an
//     unsigned max in L2, so the top-K select reads one word per key instead
//     of one per group.  The mean variant sums exp(scale * acc) over the
//     columns instead (s_j is that sum over all rows divided by their count),
//     one partial row per group.
//
// Both passes: warp 0 issues TMA loads of the key tiles (128-byte swizzle, no
// multicast) into a ring of shared-memory stages; warp 1 allocates TMEM and
// issues tcgen05.mma from one thread, committing to mbarriers; the epilogue
// warps read the f32 accumulators with tcgen05.ld.  The observation rows are
// gathered once per CTA from the recent-query and beacon tensors with plain
// 16-byte loads and written to shared memory in the same swizzled layout.
// Every wait is bounded (sm100.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "bkv_internal.h"
#include "order_key.cuh"
#include "sm100.cuh"
#include "tma_host.h"

BKV_DEFINE_STATUS_ACCESSOR(take_status_score_tc)

namespace bkv {
namespace {

using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kDim = 128;            // head_dim of the tensor-core path
constexpr int kRowBytes = kDim * 2;  // one bf16 row
constexpr int kKbBytes = 128;        // one 64-element K block of a row

// Wait-site tags recorded with a timeout.
enum { kWhereP1Prod = 101, kWhereP1Mma = 102, kWhereP1Epi = 103, kWhereP1Drain = 104,
       kWhereP2Prod = 201, kWhereP2Mma = 202, kWhereP2Epi = 203, kWhereP2Drain = 204 };

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (three-input max, sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float max32(const float (&v)[32]) {
  float r[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) r[i] = max3f(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  r[10] = fmaxf(v[30], v[31]);
  const float a = max3f(r[0], r[1], r[2]), b = max3f(r[3], r[4], r[5]);
  const float c = max3f(r[6], r[7], r[8]), e = max3f(r[9], r[10], a);
  return max3f(b, c, e);
}

// Saturating FMA: min(max(a * b + c, 0), 1) (NaN gives 0).
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^(v * kz - m) on the FMA pipe, for a pair.  One saturating FMA per element
// maps x = v * kz - m from [-126, 128] onto y = (x + 126) / 254 in [0, 1], so
// that x below the range gives about 2^-126, x above it (and m = -inf) about
// 2^128 (p(0) * 2^128, finite and just under FLT_MAX: two such terms overflow
// a sum to inf), and NaN 2^-126; then Cody-Waite reduction of x' = 254 y -
// 126 = j + f, j = rint(x') by adding 1.5 * 2^23, f in [-0.5, 0.5]; a cubic
// p(f) ~ 2^f (coefficients from a Lawson-weighted least-squares fit, max
// relative error 7.6e-5; tests/fit_exp2_poly.py); and 2^j added into p's
// exponent field, which stays in [0, 254].  `a` = kz / 254 and `b` =
// (126 - m) / 254 are the mapping's coefficients.
__device__ __forceinline__ float2 exp2_poly2(float vx, float vy, float a, float b) {
  constexpr float kBase = 12582912.0f - 126.f;  // 1.5 * 2^23 - 126, exact
  const float2 y = make_float2(fma_sat(vx, a, b), fma_sat(vy, a, b));
  const float2 t = __ffma2_rn(y, make_float2(254.f, 254.f), make_float2(kBase, kBase));
  const float2 u = __ffma2_rn(t, make_float2(-1.f, -1.f), make_float2(kBase, kBase));
  const float2 f = __ffma2_rn(y, make_float2(254.f, 254.f), u);
  float2 p = __ffma2_rn(f, make_float2(0.05517051f, 0.05517051f),
                        make_float2(0.24260840f, 0.24260840f));
  p = __ffma2_rn(p, f, make_float2(0.69326091f, 0.69326091f));
  p = __ffma2_rn(p, f, make_float2(0.99992824f, 0.99992824f));
  const uint32_t ex = __float_as_uint(t.x) << 23, ey = __float_as_uint(t.y) << 23;
  return make_float2(__uint_as_float(__float_as_uint(p.x) + ex),
                     __uint_as_float(__float_as_uint(p.y) + ey));
}

// Sum of 2^(v[i] * kz - m) over one chunk of N (32 or 16) columns.  About
// 5 of every 16 pairs go through exp2_poly2 (FMA pipe), the rest through
// ex2.approx (MUFU), so that both pipes share the load (measured best of 0 to
// 8 on the 14B-shaped step).  An element with v * kz - m above 128 (or
// m = -inf) makes the sum exceed 2^126 or inf/NaN.
constexpr int kPolyPairs = 5;
template <int N>
__device__ __forceinline__ float chunk_exp_sum(const float (&v)[N], float kz, float m) {
  constexpr int kPoly = (kPolyPairs * N + 16) / 32;
  constexpr float kInv254 = 1.f / 254.f;
  const float a = kz * kInv254, b = fmaf(-m, kInv254, 126.f * kInv254);
  const float2 kz2 = make_float2(kz, kz), nm2 = make_float2(-m, -m);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < N / 2; ++p) {
    float2 e;
    if (p < kPoly) {
      e = exp2_poly2(v[2 * p], v[2 * p + 1], a, b);
    } else {
      const float2 x = __ffma2_rn(make_float2(v[2 * p], v[2 * p + 1]), kz2, nm2);
      e.x = ex2_approx(x.x);
      e.y = ex2_approx(x.y);
    }
    acc = __fadd2_rn(acc, e);
  }
  return acc.x + acc.y;
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Pointer to observation row o of KV head (layer, kvh).  The group's beacon
// rows come first (query head by query head, nb each), then its recent rows
// (R each), so that a row block holds one query head's consecutive beacons
// or recent rows; measured a little ahead of interleaving the two per query
// head.  The recent rows are read where they are: a dense [R][d] block per
// query head, or the newest R rows of a decode-side query ring
// (ScoreGeom::recent_cap / recent_start).
__device__ __forceinline__ const uint16_t *obs_row(const ScoreGeom &g, const uint16_t *recent,
                                                   const uint16_t *beacons, int layer, int kvh,
                                                   int o) {
  const int n_bcn = g.group * g.nb;
  const long long qh0 = static_cast<long long>(layer) * g.n_q_heads +
                        static_cast<long long>(kvh) * g.group;
  if (o < n_bcn) {
    const int gq = o / g.nb;
    return beacons + ((qh0 + gq) * g.M + (o - gq * g.nb)) * kDim;
  }
  const int gq = (o - n_bcn) / g.R;
  const int i = o - n_bcn - gq * g.R;
  // row (recent_start + i) mod recent_cap of the head's block (a ring or dense)
  return recent + ((qh0 + gq) * g.recent_cap + (g.recent_start + i) % g.recent_cap) * kDim;
}

// Gather observation rows [row0, row0 + nrows) into shared memory as a
// K-major operand: two K blocks of nrows x 128 B, 128-byte swizzle.  Rows at
// or past n_obs are zero.  With `dup_half`, rows nrows/2.. repeat rows 0..
// (row r holds observation row row0 + r mod nrows/2).
__device__ __forceinline__ void load_obs_rows_sw128(uint8_t *dst, int nrows, int row0,
                                                    const ScoreGeom &g, const uint16_t *recent,
                                                    const uint16_t *beacons, int layer, int kvh,
                                                    bool dup_half = false) {
  const int kb_stride = nrows * kKbBytes;
  for (int id = threadIdx.x; id < nrows * 16; id += blockDim.x) {
    const int r = id >> 4, c16 = id & 15, kb = c16 >> 3, c = c16 & 7;
    const int o = row0 + (dup_half ? r % (nrows / 2) : r);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (o < g.n_obs) v = ldg_nc_v4(obs_row(g, recent, beacons, layer, kvh, o) + c16 * 8);
    *reinterpret_cast<uint4 *>(dst + kb * kb_stride + sw128_offset(r, c)) = v;
  }
}

// ------------------------------------------------------------------ pass 1
constexpr int kP1Rows = 128;
constexpr int kP1Keys = 256;
constexpr int kP1Stages = 3;
constexpr int kP1EpiWarps = 16;  // 4 warpgroups: 2 per tile parity, 128 of 256 columns each
constexpr int kP1Threads = 128 + 32 * kP1EpiWarps;  // warp 0 TMA, warp 1 MMA, 4.. epilogue
constexpr int kP1ABytes = kP1Rows * kRowBytes;     // 32 KB
constexpr int kP1StageBytes = kP1Keys * kRowBytes; // 64 KB
constexpr int kP1SmallBytes = 2048;                // barriers, TMEM slot, exchange
constexpr int kP1SmemBytes = kP1SmallBytes + 1024 + kP1ABytes + kP1Stages * kP1StageBytes;

__global__ void __launch_bounds__(kP1Threads, 1)
    score_rowstats_kernel(const __grid_constant__ CUtensorMap kmap, const ScoreGeom g,
                          const uint16_t *__restrict__ recent,
                          const uint16_t *__restrict__ beacons, float *__restrict__ c_out) {
  extern __shared__ uint8_t smem_raw[];
  // small objects first, then the 1024-aligned operand tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw);  // 16 barriers
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + 128);
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t tile_base = (raw_base + kP1SmallBytes + 1023u) & ~1023u;
  uint8_t *sA = smem_raw + (tile_base - raw_base);
  uint8_t *sB = sA + kP1ABytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y, rb = blockIdx.x;
  const int layer = head / g.n_kv_heads, kvh = head - layer * g.n_kv_heads;
  const long long L = g.L;
  const int n_tiles = static_cast<int>((L + kP1Keys - 1) / kP1Keys);

  const uint32_t full0 = smem_u32(&bars[0]);    // [stages]
  const uint32_t empty0 = smem_u32(&bars[4]);   // [stages]
  const uint32_t tfull0 = smem_u32(&bars[8]);   // [2]
  const uint32_t tempty0 = smem_u32(&bars[10]); // [2]
  const uint32_t done = smem_u32(&bars[12]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kP1Stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, kP1EpiWarps / 2);  // one arrive per warp reading it
    }
    mbar_init(done, 1);
    fence_barrier_init();
    prefetch_tensormap(&kmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // A block with at most 64 valid rows (the ragged last block) holds them
  // twice, in TMEM lanes 0-63 and 64-127; each copy then takes half of every
  // tile's columns, so the block's exps are not spent on padding rows.
  const bool half = g.n_obs - rb * kP1Rows <= kP1Rows / 2;
  load_obs_rows_sw128(sA, kP1Rows, rb * kP1Rows, g, recent, beacons, layer, kvh, half);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer
      const int krow0 = static_cast<int>(static_cast<long long>(head) * g.cap);
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % kP1Stages;
        const uint32_t ph = (t / kP1Stages) & 1;
        if (!mbar_wait(empty0 + 8 * s, ph ^ 1, kWhereP1Prod)) break;
        mbar_arrive_expect_tx(full0 + 8 * s, kP1StageBytes);
        const uint32_t dst = smem_u32(sB + s * kP1StageBytes);
        tma_load_2d(dst, &kmap, full0 + 8 * s, 0, krow0 + t * kP1Keys);
        tma_load_2d(dst + kP1Keys * kKbBytes, &kmap, full0 + 8 * s, 64, krow0 + t * kP1Keys);
        issued = t + 1;
      }
      // wait for the loads still in flight before the CTA may exit
      for (int t = issued > kP1Stages ? issued - kP1Stages : 0; t < issued; ++t)
        mbar_wait(full0 + 8 * (t % kP1Stages), (t / kP1Stages) & 1, kWhereP1Drain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(kP1Rows, kP1Keys);
      const uint32_t a_base = smem_u32(sA);
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % kP1Stages, acc = t & 1;
        if (!mbar_wait(full0 + 8 * s, (t / kP1Stages) & 1, kWhereP1Mma)) break;
        if (!mbar_wait(tempty0 + 8 * acc, ((t >> 1) & 1) ^ 1, kWhereP1Mma)) break;
        tc_fence_after();
        const uint32_t b_base = smem_u32(sB + s * kP1StageBytes);
        const uint32_t d = tmem + acc * kP1Keys;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_k_sw128(a_base + kb * (kP1Rows * kKbBytes) + kk * 32);
            const uint64_t bd = smem_desc_k_sw128(b_base + kb * (kP1Keys * kKbBytes) + kk * 32);
            umma_f16(d, ad, bd, idesc, (kb | kk) != 0);
          }
        }
        umma_commit(empty0 + 8 * s);
        umma_commit(tfull0 + 8 * acc);
      }
      umma_commit(done);
      mbar_wait(done, 0, kWhereP1Drain);
    }
  } else if (warp >= 4) {
    // ---- epilogue: four warpgroups; warpgroups 0-1 take the even tiles
    // (accumulator 0) and 2-3 the odd ones, each 128 of the 256 columns in
    // two blocks of 64, so the two pairs read TMEM at different times and
    // each covers the other's load latency.  TMEM lane = observation row:
    // every thread keeps its row's reference m and the sum of
    // 2^(x log2 e - m) over its columns
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const float kz = g.scale * kLog2e;
    // in a half block, lanes 0-63 take the first 64-column block of this
    // warpgroup's 128 columns and lanes 64-127 (the same rows) the second
    const int b_first = half ? (quarter >> 1) : 0;
    const int b_last = half ? (quarter >> 1) : 1;
    float m = -INFINITY, ssum = 0.f;
    bool ok = true;
    for (int t = wg >> 1; t < n_tiles && ok; t += 2) {
      const int acc = t & 1;
      if (!mbar_wait_warp(tfull0 + 8 * acc, (t >> 1) & 1, kWhereP1Epi)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int b = b_first; b <= b_last; ++b) {
        const int col = (wg & 1) * 128 + b * 64;
        const uint32_t taddr =
            tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kP1Keys + col;
        const long long key_base = static_cast<long long>(t) * kP1Keys + col;
        float va[32], vb[32];
        tmem_ld_32x32b_x32(taddr, va);
        tmem_ld_32x32b_x32(taddr + 32, vb);
        tmem_ld_wait_regs(va);
        tmem_reg_fence(vb);
        if (b == b_last) {
          // the accumulator is free once this warp's last loads have landed
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
        }
        if (key_base + 64 > L) {  // the ragged end of the keys
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (key_base + i >= L) va[i] = -INFINITY;
            if (key_base + 32 + i >= L) vb[i] = -INFINITY;
          }
        }
        // the exps of the 64 columns are taken against the row's reference m
        // (not yet its running max); only when a sum exceeds 2^64 -- the
        // first columns of the row (m = -inf), or a column more than 64 above
        // m in log2 units -- does m move up to this block's max and the block
        // is summed again.  Every value summed stays below 2^64.
        float bs = chunk_exp_sum(va, kz, m) + chunk_exp_sum(vb, kz, m);
        if (!(bs <= 0x1p64f)) {
          const float m_new = fmaxf(m, fmaxf(max32(va), max32(vb)) * kz);
          ssum = m_new == -INFINITY ? 0.f : ssum * ex2_approx(m - m_new);
          m = m_new;
          bs = m == -INFINITY ? 0.f : chunk_exp_sum(va, kz, m) + chunk_exp_sum(vb, kz, m);
        }
        ssum += bs;
      }
    }
    // combine the partial sums of each row: the four warpgroups' (and, in a
    // half block, the two lanes that hold the same row); the exchange reuses
    // the key stages, free once every tile's MMAs have completed -- which the
    // warpgroup of the last tile has seen, so all wait for it
    named_barrier_sync(1, 32 * kP1EpiWarps);
    float *xchg = reinterpret_cast<float *>(sB);  // [4][128][2]
    xchg[(wg * kP1Rows + row) * 2] = m;
    xchg[(wg * kP1Rows + row) * 2 + 1] = ok ? ssum : -1.f;
    named_barrier_sync(1, 32 * kP1EpiWarps);
    const int n_lanes = half ? kP1Rows / 2 : kP1Rows;  // lanes holding distinct rows
    if (wg == 0 && row < n_lanes) {
      const int o = rb * kP1Rows + row;
      const int n_parts = half ? 8 : 4;
      float M = -INFINITY;
      bool all_ok = true;
      for (int p = 0; p < n_parts; ++p) {
        const int w = p & 3, r = row + (p >> 2) * (kP1Rows / 2);
        M = fmaxf(M, xchg[(w * kP1Rows + r) * 2]);
        all_ok &= xchg[(w * kP1Rows + r) * 2 + 1] >= 0.f;
      }
      if (all_ok && o < g.n_obs) {
        float S = 0.f;
        for (int p = 0; p < n_parts; ++p) {
          const int w = p & 3, r = row + (p >> 2) * (kP1Rows / 2);
          const float mw = xchg[(w * kP1Rows + r) * 2];
          const float sw = xchg[(w * kP1Rows + r) * 2 + 1];
          if (mw != -INFINITY) S += sw * ex2_approx(mw - M);
        }
        c_out[static_cast<size_t>(head) * g.n_obs_pad + o] = (M + log2f(S)) * kLn2;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ pass 2
// Max aggregation: two epilogue warpgroups, one per column sub-chunk of up to
// 256 observation rows.  Mean aggregation (an exp per element instead of a
// max) takes groups of at most 256 rows, so that a tile's accumulator fills
// half of TMEM and the MMA can run one tile ahead of the exps: four epilogue
// warpgroups, two on the even tiles (TMEM columns 0..255) and two on the odd
// ones (256..511), each pair splitting the columns in halves.
constexpr int kP2Keys = 128;
constexpr int kP2TileBytes = kP2Keys * kRowBytes;  // 32 KB
constexpr int kP2ExtraRowBytes = 32;              // the extra K=16 step, 32-byte swizzle

__host__ __device__ constexpr int p2_epi_warpgroups(bool mean) { return mean ? 4 : 2; }
// warp 0 TMA, warp 1 MMA, warps 4.. the epilogue warpgroups
__host__ __device__ constexpr int p2_threads(bool mean) { return 128 + 128 * p2_epi_warpgroups(mean); }
// barriers + TMEM slot, then [2][warpgroups - 1][128] partials for the combine
__host__ __device__ constexpr int p2_small_bytes(bool mean) {
  return 256 + 2 * (p2_epi_warpgroups(mean) - 1) * 128 * 4;
}
__host__ __device__ constexpr int p2_smem_bytes(int rows_pad, int stages, bool mean) {
  return p2_small_bytes(mean) + 1024 + rows_pad * kRowBytes + stages * kP2TileBytes +
         kP2Keys * kP2ExtraRowBytes + rows_pad * kP2ExtraRowBytes;
}

template <bool kMean>
__global__ void __launch_bounds__(p2_threads(kMean), 1)
    score_colmax_kernel(const __grid_constant__ CUtensorMap kmap, const ScoreGeom g,
                        const uint16_t *__restrict__ recent, const uint16_t *__restrict__ beacons,
                        const float *__restrict__ c_in, float *__restrict__ ypart, int n_chunks,
                        int chunk_tiles, int n_stages, int head0) {
  constexpr int kEpiWG = p2_epi_warpgroups(kMean);
  constexpr int kSplit = kEpiWG / 2;  // warpgroups per column sub-chunk
  extern __shared__ uint8_t smem_raw[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw);  // 16 barriers
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + 128);
  float *ybuf = reinterpret_cast<float *>(smem_raw + 256);  // partials of warpgroups 1..
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t tile_base = (raw_base + p2_small_bytes(kMean) + 1023u) & ~1023u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bid = blockIdx.x;
  const int gi = bid % g.n_groups;
  bid /= g.n_groups;
  const int ci = bid % n_chunks;
  const int head = head0 + bid / n_chunks;
  const int layer = head / g.n_kv_heads, kvh = head - layer * g.n_kv_heads;
  const long long L = g.L;
  const int n_tiles_all = static_cast<int>((L + kP2Keys - 1) / kP2Keys);
  const int t0 = ci * chunk_tiles;
  const int t1 = min(n_tiles_all, t0 + chunk_tiles);
  const int n_tiles = t1 > t0 ? t1 - t0 : 0;

  const int r0 = gi * g.rows_per_group;
  const int nrows = min(g.rows_per_group, g.n_obs - r0);
  const int rows_pad = (nrows + 15) & ~15;
  const int N0 = min(256, rows_pad);
  const int N1 = rows_pad - N0;
  const int n_sub = N1 > 0 ? 2 : 1;

  uint8_t *sQ = smem_raw + (tile_base - raw_base);
  uint8_t *sK = sQ + rows_pad * kRowBytes;
  uint8_t *sXk = sK + n_stages * kP2TileBytes;      // keys' extra step: (1, 1, 1, 0, ...)
  uint8_t *sXq = sXk + kP2Keys * kP2ExtraRowBytes;  // rows' extra step: -c_o / scale

  const uint32_t full0 = smem_u32(&bars[0]);    // [<=4]
  const uint32_t empty0 = smem_u32(&bars[4]);   // [<=4]
  const uint32_t tfull0 = smem_u32(&bars[8]);   // [2]
  const uint32_t tempty0 = smem_u32(&bars[10]); // [2]
  const uint32_t done = smem_u32(&bars[12]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < n_stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(tfull0 + 8 * u, 1);
      mbar_init(tempty0 + 8 * u, kMean ? 8 : 4);  // one arrive per warp reading it
    }
    mbar_init(done, 1);
    fence_barrier_init();
    prefetch_tensormap(&kmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  const float inv_scale = 1.0f / g.scale;
  for (int r = threadIdx.x; r < kP2Keys; r += blockDim.x) {
    const uint32_t one = 0x3F80u;  // bf16 1.0
    *reinterpret_cast<uint4 *>(sXk + sw32_offset(r, 0)) =
        make_uint4(one | (one << 16), one, 0u, 0u);
    *reinterpret_cast<uint4 *>(sXk + sw32_offset(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int r = threadIdx.x; r < rows_pad; r += blockDim.x) {
    // c / scale as hi + mid + lo in bf16 (exact splits in f32); padded rows
    // get a huge negative offset so that they never win the max
    uint32_t w0, w1;
    if (r < nrows) {
      const float c = c_in[static_cast<size_t>(head) * g.n_obs_pad + r0 + r] * inv_scale;
      const __nv_bfloat16 hi = __float2bfloat16_rn(-c);
      const float r1 = -c - __bfloat162float(hi);
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
      w0 = static_cast<uint32_t>(__bfloat16_as_ushort(hi)) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(mid)) << 16);
      w1 = static_cast<uint32_t>(__bfloat16_as_ushort(lo));
    } else {
      w0 = 0xF149u;  // bf16 -1e30
      w1 = 0u;
    }
    *reinterpret_cast<uint4 *>(sXq + sw32_offset(r, 0)) = make_uint4(w0, w1, 0u, 0u);
    *reinterpret_cast<uint4 *>(sXq + sw32_offset(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
  }
  load_obs_rows_sw128(sQ, rows_pad, r0, g, recent, beacons, layer, kvh);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const int krow0 = static_cast<int>(static_cast<long long>(head) * g.cap);
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int t = t0 + it;
        const int s = it % n_stages;
        const uint32_t ph = (it / n_stages) & 1;
        if (!mbar_wait(empty0 + 8 * s, ph ^ 1, kWhereP2Prod)) break;
        mbar_arrive_expect_tx(full0 + 8 * s, kP2TileBytes);
        const uint32_t dst = smem_u32(sK + s * kP2TileBytes);
        tma_load_2d(dst, &kmap, full0 + 8 * s, 0, krow0 + t * kP2Keys);
        tma_load_2d(dst + kP2Keys * kKbBytes, &kmap, full0 + 8 * s, 64, krow0 + t * kP2Keys);
        issued = it + 1;
      }
      for (int it = issued > n_stages ? issued - n_stages : 0; it < issued; ++it)
        mbar_wait(full0 + 8 * (it % n_stages), (it / n_stages) & 1, kWhereP2Drain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc0 = idesc_bf16_f32(kP2Keys, N0);
      const uint32_t idesc1 = idesc_bf16_f32(kP2Keys, N1 > 0 ? N1 : 16);
      const uint32_t q_base = smem_u32(sQ);
      const int q_kb_stride = rows_pad * kKbBytes;
      bool ok = true;
      for (int it = 0; it < n_tiles && ok; ++it) {
        const int s = it % n_stages;
        if (!mbar_wait(full0 + 8 * s, (it / n_stages) & 1, kWhereP2Mma)) break;
        const uint32_t a_base = smem_u32(sK + s * kP2TileBytes);
        for (int u = 0; u < n_sub; ++u) {
          // max: one accumulator per sub-chunk; mean (one sub-chunk): one per
          // tile parity
          const int buf = kMean ? (it & 1) : u;
          const uint32_t par = kMean ? (((it >> 1) & 1) ^ 1) : ((it & 1) ^ 1);
          if (!mbar_wait(tempty0 + 8 * buf, par, kWhereP2Mma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + buf * 256;
          const uint32_t b_rows = q_base + u * N0 * kKbBytes;
          const uint32_t idesc = u == 0 ? idesc0 : idesc1;
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc_k_sw128(a_base + kb * (kP2Keys * kKbBytes) + kk * 32);
              const uint64_t bd = smem_desc_k_sw128(b_rows + kb * q_kb_stride + kk * 32);
              umma_f16(d, ad, bd, idesc, (kb | kk) != 0);
            }
          }
          umma_f16(d, smem_desc_k_sw32(smem_u32(sXk)),
                   smem_desc_k_sw32(smem_u32(sXq) + u * N0 * kP2ExtraRowBytes), idesc, 1u);
          umma_commit(tfull0 + 8 * buf);
        }
        umma_commit(empty0 + 8 * s);
      }
      umma_commit(done);
      mbar_wait(done, 0, kWhereP2Drain);
    }
  } else if (kMean && warp >= 4) {
    // Warpgroup e takes the tiles of parity e >> 1 and the column half e & 1
    // of the group's rows (rows_pad <= 256, one sub-chunk); per key (TMEM
    // lane) it sums exp(scale * acc) over its columns, releases the
    // accumulator after its last TMEM load, and the two halves' sums meet in
    // shared memory.
    const int e = (warp - 4) >> 2;
    const int par = e >> 1, h = e & 1;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key within the tile
    const float kz = g.scale * kLog2e;
    float *yout = ypart + (static_cast<size_t>(gi) * g.n_heads() + head) * static_cast<size_t>(L);
    const int c0 = h * 128, c1 = min(N0, c0 + 128);
    const int n32 = c1 > c0 ? (c1 - c0) >> 5 : 0;
    const bool tail16 = c1 > c0 && ((c1 - c0) & 16) != 0;  // N0 is a multiple of 16
    bool ok = true;  // warp-uniform; after a timeout only the barriers remain
    for (int it = par; it < n_tiles; it += 2) {
      const int buf = it & 1;  // == par
      float y = 0.f;
      if (ok && !mbar_wait_warp(tfull0 + 8 * buf, (it >> 1) & 1, kWhereP2Epi)) ok = false;
      if (ok) {
        tc_fence_after();
        const uint32_t taddr =
            tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * 256 + c0;
        bool released = false;
        auto release = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
          released = true;
        };
        // two TMEM loads in flight; the accumulator is handed back as soon as
        // the last of this warp's loads has landed
        float va[32], vb[32];
        int i = 0;
        if (n32 > 0) {
          tmem_ld_32x32b_x32(taddr, va);
          tmem_ld_wait_regs(va);
          if (n32 == 1 && !tail16) release();
        }
#pragma unroll 1
        for (; i + 2 <= n32; i += 2) {
          tmem_ld_32x32b_x32(taddr + (i + 1) * 32, vb);
          y += chunk_exp_sum(va, kz, 0.f);
          tmem_ld_wait_regs(vb);
          if (i + 2 == n32 && !tail16) release();
          if (i + 2 < n32) tmem_ld_32x32b_x32(taddr + (i + 2) * 32, va);
          y += chunk_exp_sum(vb, kz, 0.f);
          if (i + 2 < n32) {
            tmem_ld_wait_regs(va);
            if (i + 3 == n32 && !tail16) release();
          }
        }
        if (i < n32) y += chunk_exp_sum(va, kz, 0.f);
        if (tail16) {
          float v[16];
          tmem_ld_32x32b_x16(taddr + n32 * 32, v);
          tmem_ld_wait_regs(v);
          release();
          y += chunk_exp_sum(v, kz, 0.f);
        }
        if (!released) release();  // a half with no columns
      }
      float *slot = ybuf + (par * 2 + ((it >> 1) & 1)) * 128;
      if (h == 1) slot[row] = y;
      named_barrier_sync(1 + par, 256);
      if (h == 0 && ok) {
        const long long j = static_cast<long long>(t0 + it) * kP2Keys + row;
        if (j < L) yout[j] = y + slot[row];
      }
    }
  } else if (!kMean && warp >= 4) {
    // Warpgroup e = u * kSplit + h reads column sub-chunk u, its 32-column
    // pieces h, h + kSplit, ...; per key (TMEM lane) it reduces
    // acc = q . k - c_o / scale over them: the max (max aggregation) or the
    // sum of exp(scale * acc) (mean).  The partials of warpgroups 1.. reach
    // warpgroup 0 through shared memory.
    const int e = (warp - 4) >> 2;
    const int u = e / kSplit, h = e - u * kSplit;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key within the tile
    const int n_active = n_sub * kSplit;  // warpgroups with columns to read
    const float kz = g.scale * kLog2e;
    // the head's merged maxima, as order keys: stored by a single group, else
    // combined by an unsigned max in L2 over a row of zeros (below every key)
    uint32_t *ykey = reinterpret_cast<uint32_t *>(ypart) + static_cast<size_t>(head) * static_cast<size_t>(L);
    if (u < n_sub) {
      const int Nu = u == 0 ? N0 : N1;
      const int n32 = Nu >> 5;
      const int n_mine = n32 > h ? (n32 - h + kSplit - 1) / kSplit : 0;
      const bool tail16 = (Nu & 16) && (n32 % kSplit) == h;  // Nu is a multiple of 16
      bool ok = true;  // warp-uniform; after a timeout only the barriers remain
      for (int it = 0; it < n_tiles; ++it) {
        float y0 = -INFINITY, y1 = y0;
        if (ok && !mbar_wait_warp(tfull0 + 8 * u, it & 1, kWhereP2Epi)) ok = false;
        if (ok) {
          tc_fence_after();
          const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + u * 256;
          auto piece = [&](int i) { return taddr + static_cast<uint32_t>((h + i * kSplit) * 32); };
          auto reduce32 = [&](const float (&v)[32]) {
            if (kMean) {
              y0 += chunk_exp_sum(v, kz, 0.f);
            } else {
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                y0 = max3f(y0, v[i], v[i + 1]);
                y1 = max3f(y1, v[i + 2], v[i + 3]);
              }
            }
          };
          // two TMEM loads in flight: piece i+1 lands while piece i is reduced
          float va[32], vb[32];
          int i = 0;
          if (n_mine > 0) {
            tmem_ld_32x32b_x32(piece(0), va);
            tmem_ld_wait_regs(va);
          }
#pragma unroll 1
          for (; i + 2 <= n_mine; i += 2) {
            tmem_ld_32x32b_x32(piece(i + 1), vb);
            reduce32(va);
            tmem_ld_wait_regs(vb);
            if (i + 2 < n_mine) tmem_ld_32x32b_x32(piece(i + 2), va);
            reduce32(vb);
            if (i + 2 < n_mine) tmem_ld_wait_regs(va);
          }
          if (i < n_mine) reduce32(va);
          if (tail16) {
            float v[16];
            tmem_ld_32x32b_x16(taddr + n32 * 32, v);
            tmem_ld_wait_regs(v);
            if (kMean) {
              y1 += chunk_exp_sum(v, kz, 0.f);
            } else {
#pragma unroll
              for (int t = 0; t < 16; t += 4) {
                y0 = max3f(y0, v[t], v[t + 1]);
                y1 = max3f(y1, v[t + 2], v[t + 3]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty0 + 8 * u);
        }
        float y = kMean ? y0 + y1 : fmaxf(y0, y1);
        if (n_active > 1) {
          float *slot = ybuf + (it & 1) * (kEpiWG - 1) * 128;
          if (e > 0) slot[(e - 1) * 128 + row] = y;
          named_barrier_sync(1, 128 * n_active);
          if (e == 0) {
            for (int f = 1; f < n_active; ++f) {
              const float t = slot[(f - 1) * 128 + row];
              y = kMean ? y + t : fmaxf(y, t);
            }
          }
        }
        if (e == 0 && ok) {
          const long long j = static_cast<long long>(t0 + it) * kP2Keys + row;
          const float v = y * g.scale;
          if (j < L) {
            if (g.n_groups == 1)
              ykey[j] = order_key(v);
            else if (!(v != v))  // a NaN group maximum is ignored, as fmaxf would
              atomicMax(ykey + j, order_key(v));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host
// Tensor map of the whole key cache as a 2-D bf16 array
// [n_layers * n_kv_heads * cap rows][128], boxes of 64 x box_rows, 128 B swizzle.
bool make_key_map(CUtensorMap *map, const void *k, const ScoreGeom &g, int box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t rows = static_cast<cuuint64_t>(g.n_heads()) * static_cast<cuuint64_t>(g.cap);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDim), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kRowBytes)};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(k), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bkv_status launch_score_rowstats_tc(const ScoreGeom &g, const void *k, const void *recent,
                                    const void *beacons, float *c, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  CUtensorMap map;
  if (!make_key_map(&map, k, g, kP1Keys)) return BKV_ERR_CUDA;
  static int attr_done[64];
  if (!ensure_smem_limit(score_rowstats_kernel, kP1SmemBytes, attr_done)) return BKV_ERR_CUDA;
  dim3 grid(g.n_obs_pad / kP1Rows, g.n_heads());
  score_rowstats_kernel<<<grid, kP1Threads, kP1SmemBytes, stream>>>(
      map, g, static_cast<const uint16_t *>(recent), static_cast<const uint16_t *>(beacons), c);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

bkv_status launch_score_colmax_tc(const ScoreGeom &g, const void *k, const void *recent,
                                  const void *beacons, const float *c, float *ypart, bool mean,
                                  cudaStream_t stream, int head0, int head_count) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  CUtensorMap map;
  if (!make_key_map(&map, k, g, kP2Keys)) return BKV_ERR_CUDA;
  int max_rows_pad = 0;
  for (int gi = 0; gi < g.n_groups; ++gi) {
    const int nrows = std::min(g.rows_per_group, g.n_obs - gi * g.rows_per_group);
    max_rows_pad = std::max(max_rows_pad, (nrows + 15) & ~15);
  }
  constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block on sm_100
  int stages = 4;
  while (stages > 2 && p2_smem_bytes(max_rows_pad, stages, mean) > kSmemLimit) --stages;
  const int smem = p2_smem_bytes(max_rows_pad, stages, mean);
  if (smem > kSmemLimit) return BKV_ERR_UNSUPPORTED;
  static int attr_done[2][64];
  if (!ensure_smem_limit(mean ? score_colmax_kernel<true> : score_colmax_kernel<false>,
                         kSmemLimit, attr_done[mean ? 1 : 0]))
    return BKV_ERR_CUDA;
  const int n_tiles = static_cast<int>((g.L + kP2Keys - 1) / kP2Keys);
  // Split the keys of a head into chunks so that the CTAs fill whole waves of
  // the SMs (one CTA per SM): the fewest chunks whose last wave is at least
  // 95% full, else the best fill found.  Each chunk reloads its observation
  // rows once, so chunks keep at least 8 tiles.
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  if (head_count < 0) head_count = g.n_heads() - head0;
  if (head0 < 0 || head_count <= 0 || head0 + head_count > g.n_heads()) return BKV_OK;
  const long long units = static_cast<long long>(head_count) * g.n_groups;
  int n_chunks = 1, chunk_tiles = n_tiles;
  double best_fill = 0.0;
  for (int nc = 1; nc <= std::max(1, n_tiles / 8) && nc <= 32; ++nc) {
    const int ct = (n_tiles + nc - 1) / nc;
    const int ncr = (n_tiles + ct - 1) / ct;
    const long long ctas = units * ncr;
    const long long waves = (ctas + sms - 1) / sms;
    const double fill = static_cast<double>(ctas) / static_cast<double>(waves * sms);
    if (fill > best_fill + 1e-9) {
      best_fill = fill;
      n_chunks = ncr;
      chunk_tiles = ct;
    }
    if (fill >= 0.95) break;
  }
  const long long grid = units * n_chunks;
  const auto *rq = static_cast<const uint16_t *>(recent);
  const auto *bq = static_cast<const uint16_t *>(beacons);
  // the max form's groups meet in one row of keys per head, zero to start
  if (!mean && g.n_groups > 1 &&
      cudaMemsetAsync(ypart + static_cast<size_t>(head0) * static_cast<size_t>(g.L), 0,
                      static_cast<size_t>(head_count) * static_cast<size_t>(g.L) * sizeof(float),
                      stream) != cudaSuccess)
    return BKV_ERR_CUDA;
  if (mean)
    score_colmax_kernel<true><<<static_cast<unsigned>(grid), p2_threads(true), smem, stream>>>(
        map, g, rq, bq, c, ypart, n_chunks, chunk_tiles, stages, head0);
  else
    score_colmax_kernel<false><<<static_cast<unsigned>(grid), p2_threads(false), smem, stream>>>(
        map, g, rq, bq, c, ypart, n_chunks, chunk_tiles, stages, head0);
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace bkv
