// fps_tc.cu -- Continual farthest-point sampling (BeaconKV, Fig. 7) of bf16
// queries with head_dim 128, with the dot products on tcgen05.
//
// The picks are exactly the greedy sequence (seed U[0]; each further pick is
// the unselected point farthest in cosine distance from the picked set, ties
// to the lowest index), found in speculative rounds.  Every point i keeps an
// upper bound u_i of its distance to the picked set and a stamp t_i: u_i is
// the exact distance to the first t_i picks (distances only fall as picks are
// added, so u_i bounds the true distance).  A round
//   1. selects the T = 128 points with the largest u, and the (T+1)-th,
//      whose u bounds every other point's true distance: from a 1024-bin
//      histogram of u over [0, 2] that is kept up to date across rounds
//      (rebuilt by each pass, moved by each round's write-back), the
//      threshold bin's keys ranked exactly; when that bin is too full, from
//      a two-level histogram built afresh, then a radix select;
//   2. stages the candidates' rows in the MMA's swizzled layout and forms, in
//      one tcgen05 commit, their Gram block (M = N = 128) and -- for
//      candidates whose stamp is behind -- their dots with the picks they
//      have not seen, so every candidate's distance becomes exact;
//   3. replays the greedy choice among the candidates with the Gram block
//      (one warp): the best remaining candidate is the true argmax while it
//      beats the bound, so it is picked; the round stops at the first one
//      that does not;
//   4. writes the candidates' new distances back (exact, stamped) and, in an
//      eager round, runs a distance pass that brings every point up to date.
// A round that certifies fewer than kPassBelow picks is followed by a pass
// (the next round starts from exact distances and certifies many); after a
// round that certifies more, only the next round's candidates are refreshed
// (a lazy round), which avoids re-streaming the union.  A pass costs about
// as much as 1.8 rounds' select, gather and MMAs; on the clustered queries of
// the 14B-shaped workload this policy takes ~8.4 rounds and ~5.8 passes per
// head, against ~13.6 and ~4.6 for staying eager only until the first round
// of 8 picks, and ~7.6 and ~6.6 for a pass after every round.  The
// threshold was measured: 20 picks ahead of 8, 12, 16, 24, 32 and 48.
//
// The distance pass streams the union [beacons; window] of a query head by
// TMA in tiles of 128 points (128-byte swizzle, no multicast) through a
// 4-stage ring (each row fetched into L2 by its epilogue thread kAhead tiles
// earlier; a fixed share of each union's tiles stays in L2 across passes,
// evict-last, and the rest streams evict-first) and forms D[128 points][N] =
// tile . picks^T (M = 128, K = 128, N = the picks the points have not seen,
// rounded up to 16) in one of four TMEM accumulators.  Two threads issue the MMAs (warp 1 the even tiles of
// the sequence, warp 2 the odd ones) so their instruction latencies overlap;
// two epilogue warpgroups (TMEM lane = point) turn the dots into cosine
// distances.  Between passes the ring's shared memory holds the round's
// candidate rows, Gram block and selection scratch.
//
// The grid is persistent: one CTA per SM takes query heads from a counter in
// the workspace as it becomes free.  The distance, inverse-norm and stamp
// arrays live in shared memory, or for a union too large for it in the
// caller's workspace (one slice per CTA).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "bkv_check.cuh"
#include "bkv_internal.h"
#include "fps_common.cuh"
#include "sm100.cuh"
#include "tma_host.h"

BKV_DEFINE_STATUS_ACCESSOR(take_status_fps_tc)

namespace bkv {
namespace {

using namespace sm100;
using namespace fpsk;

constexpr int kThreads = 384;  // warp 0 TMA, warps 1-2 MMA, warps 4..11 epilogues
constexpr int kWarps = kThreads / 32;
constexpr int kCand = 128;     // candidates per round (T)
constexpr int kDim = 128;
constexpr int kTileRows = 128;
constexpr int kStages = 4;     // even tiles use stages 0 and 2, odd tiles 1 and 3
constexpr int kTileBytes = kTileRows * kDim * 2;  // 32 KB
constexpr int kMaxPick = 128;                     // beacons per head on this path
constexpr int kPickRows = kMaxPick + 16;          // picks operand rows (N padding)
constexpr int kPBlock = kPickRows * 128;          // one 64-element K block of the picks
constexpr int kCBlock = kCand * 128;              // one 64-element K block of the candidates
// floats per Gram row: an odd stride keeps both the row-per-lane copy and
// the replay's column reads (lane = candidate) free of bank conflicts
constexpr int kGramStride = kCand + 1;
constexpr int kListMax = 512;                     // threshold-bin keys ranked directly
constexpr int kPassBelow = 20;                    // a round with fewer picks is followed by a pass
constexpr int kAhead = 12;                        // L2 prefetch distance of a pass, in tiles
constexpr int kSmallBytes = 8192;  // barriers, scalars, lists; the u histogram at 4096
// The persistent histogram of the live points' u over [0, 2] (the range of a
// cosine distance): bin = floor(u * 512), clamped to the last bin.
constexpr int kUBins = 1024;
constexpr float kUScale = 512.f;
constexpr int kFixedBytes = kSmallBytes + 1024 + kStages * kTileBytes + 2 * kPBlock;
constexpr int kSmemLimit = 232448;
// TMEM: two pass accumulators of up to 128 columns, the Gram and refresh blocks
constexpr uint32_t kTmemCols = 512;
// Pass accumulators (128 columns each): all of TMEM, since the Gram and
// refresh blocks (columns 256 ..) are idle while a pass runs.
constexpr int kAcc = 4;
constexpr uint32_t kGramCol = 256, kRefCol = 384;
// the serial phase's buffers inside the ring (idle between passes)
constexpr int kGramOff = 0;                        // [kCand][kGramStride] f32
constexpr int kSelOff = 69632;                     // whist [kWarps][256], list keys/indices
constexpr int kCopOff = 3 * kTileBytes;            // candidates [2][kCand][128 B]
static_assert(kGramOff + kCand * kGramStride * 4 <= kSelOff, "Gram block overlaps");
static_assert(kSelOff + (kWarps * 256 + 2 * kListMax) * 4 <= kCopOff, "selection scratch overlaps");
static_assert(kCopOff + 2 * kCBlock <= kStages * kTileBytes, "candidates overflow the ring");
static_assert(kPBlock % 1024 == 0, "picks K blocks must keep 1024-byte atoms");

// scal[] slots
enum {
  kSNp = 4,        // picks of the round
  kSFallback = 5,  // the threshold bin is too large: radix select instead
  kSKeyMin = 6,    // key range of the last pass (select_best reads 6 and 7)
  kSKeyMax = 7,
  kSAbove = 8,     // keys in bins above the threshold bin
  kSNeed = 9,      // keys wanted from the threshold bin
  kSBin = 10,      // the threshold bin
  kSCand = 11,     // candidate counter
  kSList = 12,     // threshold-bin list counter
  kSRef = 13,      // lowest stamp among the candidates
  kSDmax = 14,     // upper bound of every live distance (float bits)
  kAbort = 15,
  kSLive = 16,     // live keys counted by the histogram
  kSPlaced = 17,   // points placed above the threshold bin (fixed-range select)
  kSListed = 18,   // points listed from the threshold bin (fixed-range select)
  kSHead = 19,     // the next query head this CTA takes
  kScalWords = 32
};

enum { kWhereProd = 401, kWhereMma = 402, kWhereEpi = 403, kWhereDrain = 404 };

// Barriers: full[4] empty[4] tfull[4] tempty[4], the two MMA threads' drain
// barriers, the round's Gram/refresh commit.
constexpr int kBarFull = 0, kBarEmpty = 4, kBarTfull = 8, kBarTempty = 12, kBarDone = 16,
              kBarGram = 18;

struct Layout {
  uint64_t *bars;
  uint32_t *tmem_slot;
  int *scal;        // [kScalWords]
  uint32_t *hist;   // [256]
  int *cidx;        // [kCand + 1] candidates, then the bound
  float *cdist;     // [kCand + 1]
  int *pick;        // [kCand] candidate slots picked this round, in order
  float *pinv;      // [kPickRows] inverse norm of pick k (NaN past the last pick)
  uint32_t *uhist;  // [kUBins] live points per bin of u, kept up to date over a head
  uint8_t *ring;    // [kStages][kTileBytes]
  uint8_t *pop;     // picks, K-major 128-byte swizzle: [2][kPickRows][128 B]
  float *gram;      // (ring) [kCand][kGramStride]
  uint32_t *whist;  // (ring) [kWarps][256]
  uint32_t *lkey;   // (ring) [kListMax]
  int *lidx;        // (ring) [kListMax]
  uint8_t *cop;     // (ring) candidates, K-major 128-byte swizzle: [2][kCand][128 B]
  float *dist;      // [n] upper bound of the distance to the picked set; -1 = picked
  float *inv;       // [n] inverse norms
  uint8_t *stamp;   // [n] picks accounted for in dist
};

// Union point i of a query head: beacon i, or window row i - nb, which is row
// (w_start + i - nb) mod w_cap of the head's window block -- a dense [W][d]
// block, or the newest W rows of a decode-side query ring.
struct Head {
  const __nv_bfloat16 *B, *Wp;
  int nb;
  long long w_cap, w_start;
  __device__ const __nv_bfloat16 *point(int i) const {
    return i < nb ? B + static_cast<size_t>(i) * kDim
                  : Wp + static_cast<size_t>((w_start + (i - nb)) % w_cap) * kDim;
  }
};

// The window's tiles: the ring (or dense block) of a head is read in
// row-aligned tiles of 128 slots; tile t of the pass's window part is ring
// tile first + t.  A window that wraps around the end of the ring takes every
// ring tile; otherwise the tiles from the one holding its first slot to the
// one holding its last.  Each slot maps back to its window row.
struct WindowTiles {
  int first, count;
  __device__ WindowTiles(const FpsGeom &g) {
    if (g.W <= 0) {
      first = count = 0;
    } else if (g.w_start + g.W > g.w_cap) {
      first = 0;
      count = static_cast<int>((g.w_cap + kTileRows - 1) / kTileRows);
    } else {
      first = static_cast<int>(g.w_start / kTileRows);
      count = static_cast<int>((g.w_start + g.W - 1) / kTileRows) - first + 1;
    }
  }
};

// ---- loads under an L2 cache policy
// A 2-D tiled TMA load (as tma_load_2d) under an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t bar, int32_t x, int32_t y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// Policies for tma_load_2d_hint: lines kept in L2 with evict-last priority,
// or evicted first.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}
// Return the 128-byte L2 line holding `p` to normal eviction priority.
__device__ __forceinline__ void l2_demote_line(const void *p) {
  asm volatile("applypriority.global.L2::evict_normal [%0], 128;" ::"l"(
                   reinterpret_cast<uint64_t>(p) & ~static_cast<uint64_t>(127))
               : "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// The u-histogram bin of a live point's distance (-1 for a selected point,
// u = -1, or a distance that is not a number).  Monotonic in u.
__device__ __forceinline__ int ubin(float u) {
  return u >= 0.f ? min(kUBins - 1, static_cast<int>(u * kUScale)) : -1;
}

// Row r of tile j of a pass into L2 (its 256 bytes), if the row belongs
// to the head: a beacon slot below nb, or a ring slot below w_cap.  The
// pass's tiles are prefetched this way, by the epilogue thread of the row,
// kAhead tiles ahead of the tile it has just finished, so that the TMA unit
// moves only the ring's loads (an L2 prefetch by TMA costs the unit as much
// time as the load itself).
__device__ __forceinline__ void prefetch_row(const Head &h, const FpsGeom &g, int n_btiles,
                                             int w_first, int j, int r) {
  const __nv_bfloat16 *p = nullptr;
  if (j < n_btiles) {
    const int i = j * kTileRows + r;
    if (i < h.nb) p = h.B + static_cast<size_t>(i) * kDim;
  } else {
    const long long slot = static_cast<long long>(w_first + j - n_btiles) * kTileRows + r;
    if (slot < g.w_cap) p = h.Wp + static_cast<size_t>(slot) * kDim;
  }
  if (p != nullptr) {
    // a 16-byte load that promotes the whole 256-byte row into L2.  Nothing
    // reads its value, so the thread does not wait for it.  Measured a
    // little ahead of prefetch instructions and of a bulk prefetch of the
    // tile.
    [[maybe_unused]] uint32_t a, b, c, d;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                 : "l"(p));
  }
}

// Issue the TMA loads of tiles [0, n_tiles) of the pass that starts at
// sequence number `seq` (producer thread only): tiles below n_keep stay in
// L2 (evict-last), the rest stream through it (evict-first).  Returns false
// after a timeout.
__device__ bool issue_tiles(const Layout &s, const CUtensorMap *bmap, const CUtensorMap *wmap,
                            int qh, const FpsGeom &g, int n_btiles, int w_first, uint32_t seq,
                            int n_tiles, int n_keep) {
  const uint32_t full0 = smem_u32(&s.bars[kBarFull]), empty0 = smem_u32(&s.bars[kBarEmpty]);
  const uint64_t keep = l2_policy_evict_last(), stream = l2_policy_evict_first();
  auto map_of = [&](int j) { return j < n_btiles ? bmap : wmap; };
  auto row_of = [&](int j) {
    return j < n_btiles ? qh * g.M + j * kTileRows
                        : static_cast<int>(qh * g.w_cap) + (w_first + j - n_btiles) * kTileRows;
  };
  for (int j = 0; j < n_tiles; ++j) {
    const uint32_t q = seq + j, st = q % kStages;
    if (!mbar_wait(empty0 + 8 * st, ((q / kStages) & 1) ^ 1, kWhereProd)) return false;
    mbar_arrive_expect_tx(full0 + 8 * st, kTileBytes);
    const uint32_t dst = smem_u32(s.ring + st * kTileBytes);
    const CUtensorMap *map = map_of(j);
    const int y = row_of(j);
    const uint64_t policy = j < n_keep ? keep : stream;
    tma_load_2d_hint(dst, map, full0 + 8 * st, 0, y, policy);
    tma_load_2d_hint(dst + kTileRows * 128, map, full0 + 8 * st, 64, y, policy);
  }
  return true;
}

// Lower a point's distance by the picks s0 + j it has not seen: columns j of
// one 32-column chunk of D = point . picks^T (j >= lo; pinv NaN past the last
// pick, which fminf ignores).  x = 1 - dot * inv_i * inv_k, clamped later.
template <int kCols>
__device__ __forceinline__ float chunk_min(const float (&v)[32], const float *pinv, int c0,
                                           int lo, float inv_i, float mn) {
  const float2 ninv = make_float2(-inv_i, -inv_i);
#pragma unroll
  for (int k = 0; k < kCols; k += 2) {
    const float2 x = __ffma2_rn(__fmul2_rn(make_float2(v[k], v[k + 1]), ninv),
                                make_float2(pinv[c0 + k], pinv[c0 + k + 1]),
                                make_float2(1.f, 1.f));
    mn = fminf(mn, c0 + k >= lo ? x.x : INFINITY);
    mn = fminf(mn, c0 + k + 1 >= lo ? x.y : INFINITY);
  }
  return mn;
}

// One distance pass over every tile of the head: each unselected point i
// takes the picks [stamp_i, P) it has not seen (picks operand rows s0 .. P-1;
// the seed pass: the seed, stamp 0) and its stamp becomes P.  The producer
// (warp 0), the two MMA threads (warps 1 and 2) and the epilogue warpgroups
// (warps 4..11) run their own loops; `seq` is the number of tiles all passes
// so far have moved through the ring, so every role derives the same stage,
// accumulator and barrier phase for each tile.
__device__ void distance_pass(const Layout &s, const CUtensorMap *bmap, const CUtensorMap *wmap,
                              uint32_t tmem, int qh, const Head &h, const FpsGeom &g,
                              int n_btiles, int w_first, int n_tiles, uint32_t seq, int s0, int P,
                              bool first, int n_keep) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(&s.bars[kBarFull]), empty0 = smem_u32(&s.bars[kBarEmpty]);
  const uint32_t tfull0 = smem_u32(&s.bars[kBarTfull]), tempty0 = smem_u32(&s.bars[kBarTempty]);
  const int N = (P - s0 + 15) & ~15;  // 16 .. 128
  if (warp == 0) {
    if (lane == 0 &&
        !issue_tiles(s, bmap, wmap, qh, g, n_btiles, w_first, seq, n_tiles, n_keep))
      s.scal[kAbort] = 1;
  } else if (warp == 1 || warp == 2) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileRows, N);
      // descriptors of the K steps: the start-address field (address / 16,
      // 14 bits) is the only part that moves, and shared addresses stay
      // below 256 KB, so an offset is added to it directly
      const uint64_t b_desc =
          smem_desc_k_sw128(smem_u32(s.pop) + static_cast<uint32_t>(s0) * 128u);
      const uint64_t a_desc0 = smem_desc_k_sw128(smem_u32(s.ring));
      const uint32_t mine = static_cast<uint32_t>(warp - 1);  // accumulators mine, mine + 2
      for (int j = 0; j < n_tiles; ++j) {
        const uint32_t q = seq + j, st = q % kStages, a = q % kAcc;
        if ((a & 1u) != mine) continue;
        if (!mbar_wait(full0 + 8 * st, (q / kStages) & 1, kWhereMma) ||
            !mbar_wait(tempty0 + 8 * a, ((q / kAcc) & 1) ^ 1, kWhereMma)) {
          s.scal[kAbort] = 1;
          break;
        }
        tc_fence_after();
        const uint64_t a_desc = a_desc0 + ((st * kTileBytes) >> 4);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = a_desc + ((kb * (kTileRows * 128) + kk * 32) >> 4);
            const uint64_t bd = b_desc + ((kb * kPBlock + kk * 32) >> 4);
            umma_f16(tmem + a * 128, ad, bd, idesc, (kb | kk) != 0);
          }
        }
        // the stage is free once these MMAs complete (in the seed pass the
        // epilogue still reads it for the norms and releases it itself)
        if (!first) umma_commit(empty0 + 8 * st);
        umma_commit(tfull0 + 8 * a);
      }
    }
  } else if (warp >= 4) {
    // epilogue warpgroup w consumes accumulators w and w + 2, i.e. every
    // other tile
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    bool ok = true;  // warp-uniform; after a timeout the warp keeps only the barriers
    // the first kAhead tiles past the ring, split between the warpgroups like
    // the tiles themselves
    for (int j = kStages; j < min(n_tiles, kAhead); ++j)
      if (static_cast<int>((seq + j) & 1u) == wg) prefetch_row(h, g, n_btiles, w_first, j, r);
    for (int j = 0; j < n_tiles; ++j) {
      const uint32_t q = seq + j, a = q % kAcc;
      if (static_cast<int>(a & 1u) != wg) continue;
      int i;
      bool valid;
      if (j < n_btiles) {
        i = j * kTileRows + r;
        valid = i < g.nb_in;
      } else {
        // ring slot -> window row (slots past the ring's end, or outside the
        // window, are not points of this head)
        const long long slot = static_cast<long long>(w_first + j - n_btiles) * kTileRows + r;
        long long w = slot - g.w_start;
        if (w < 0) w += g.w_cap;
        valid = slot < g.w_cap && w < g.W;
        i = valid ? g.nb_in + static_cast<int>(w) : 0;
      }
      if (valid && !BKV_CHECK(i >= 0 && i < g.nb_in + g.W, 707)) valid = false;
      const uint32_t st = q % kStages;
      if (ok && !mbar_wait_warp(tfull0 + 8 * a, (q / kAcc) & 1, kWhereEpi)) {
        s.scal[kAbort] = 1;
        ok = false;
      }
      if (first) {
        // the seed pass also takes every point's inverse norm from its row of
        // the staged tile (0 for a zero vector, whose distance is then 1).
        // The tile's MMAs have completed (their commit was awaited above), so
        // once the warpgroup has read its rows the stage can be released.
        if (ok) {
          const uint8_t *row = s.ring + st * kTileBytes;
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
        if (ok && warp == 4 + 4 * wg && lane == 0) mbar_arrive(empty0 + 8 * st);
      }
      if (!ok) continue;
      tc_fence_after();
      const float di = !valid ? -1.f : first ? 2.f : s.dist[i];
      const int lo = (valid && !first) ? static_cast<int>(s.stamp[i]) - s0 : 0;
      const float inv_i = valid ? s.inv[i] : 0.f;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + a * 128;
      // the TMEM loads are warp-wide: every lane takes part, the live ones use them
      float mn = INFINITY;
      for (int c0 = 0; c0 < N; c0 += 32) {
        float v[32];
        if (c0 + 32 <= N) {
          tmem_ld_32x32b_x32(taddr + c0, v);
          tmem_ld_wait_regs(v);
          if (di >= 0.f) mn = chunk_min<32>(v, s.pinv + s0, c0, lo, inv_i, mn);
        } else {
          float h[16];
          tmem_ld_32x32b_x16(taddr + c0, h);
          tmem_ld_wait_regs(h);
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] = h[k];
          if (di >= 0.f) mn = chunk_min<16>(v, s.pinv + s0, c0, lo, inv_i, mn);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * a);
      // the range of the new keys, which the next selection starts from
      uint32_t kmn = 0xffffffffu, kmx = 0u;
      if (di >= 0.f) {  // a point not yet selected
        // min(di, clamp(x, 0, 2)) == max(min(di, x), 0) for di in [0, 2]
        const float nd = fmaxf(fminf(di, mn), 0.f);
        s.dist[i] = nd;
        s.stamp[i] = static_cast<uint8_t>(P);
        atomicAdd(&s.uhist[ubin(nd)], 1u);  // the pass rebuilds the histogram
        kmn = kmx = dist_key(nd);
      }
      kmn = __reduce_min_sync(0xffffffffu, kmn);
      kmx = __reduce_max_sync(0xffffffffu, kmx);
      if (lane == 0) {
        atomicMin(reinterpret_cast<unsigned int *>(&s.scal[kSKeyMin]), kmn);
        atomicMax(reinterpret_cast<unsigned int *>(&s.scal[kSKeyMax]), kmx);
      }
      if (j + kAhead < n_tiles) prefetch_row(h, g, n_btiles, w_first, j + kAhead, r);
    }
  }
}

// Exclusive prefix sum over the block of one value per thread (`scratch`:
// kWarps words); every thread gets its own prefix.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w < warp) before += scratch[w];
  return before + incl - v;
}

// Points of a union that the selection keeps in registers (n <= kPerThread *
// kThreads); larger unions take the radix select.
constexpr int kPerThread = 16;

// Warp 0: the bin of `hist` (256 bins, highest first) that holds the
// want-th key: its index, the keys in the bins above it, and the keys still
// wanted from it, in scal[kSBin], [kSAbove], [kSNeed]; scal[kSFallback] is set
// when that bin holds more than `list_max` keys or fewer than `want` keys
// are counted at all.
__device__ __forceinline__ void find_threshold_bin(const Layout &s, int want, int list_max) {
  const int lane = threadIdx.x & 31;
  // lane l holds bins 255-8l .. 248-8l: two 16-byte loads of its 8
  // consecutive words (no bank conflicts), highest bin first
  const uint4 lo4 = *reinterpret_cast<const uint4 *>(s.hist + 248 - 8 * lane);
  const uint4 hi4 = *reinterpret_cast<const uint4 *>(s.hist + 252 - 8 * lane);
  const uint32_t cnt[8] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) local += cnt[j];
  uint32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const uint32_t excl = incl - local;
  if (static_cast<int>(excl) < want && want <= static_cast<int>(incl)) {
    uint32_t acc = excl;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (static_cast<int>(acc + cnt[j]) >= want) {
        s.scal[kSBin] = 255 - 8 * lane - j;
        s.scal[kSAbove] = static_cast<int>(acc);
        s.scal[kSNeed] = want - static_cast<int>(acc);
        s.scal[kSFallback] = cnt[j] > static_cast<uint32_t>(list_max) ? 1 : 0;
        break;
      }
      acc += cnt[j];
    }
  }
  if (lane == 31 && static_cast<int>(incl) < want) s.scal[kSFallback] = 1;
}

// Step 1 of a round: the `want` live points with the largest u in (u desc,
// index asc) order: the first kCand in slots 0.. , the (kCand+1)-th -- the
// bound -- in slot kCand when `bounded`.  Two histogram levels: 256 bins of u
// over [0, dmax] find the bin holding the want-th key, then 256 sub-bins of
// that bin's range find the sub-bin holding it; keys above are taken and the
// keys of that sub-bin are ranked against each other.  Both bin maps are
// monotonic in u, so the order is exact.  Each thread keeps its points' u
// and bins in registers, and the points are placed by a block-wide prefix sum
// of per-thread counts (no atomic counters).  Returns false (nothing written)
// when the union is too large for that, the final sub-bin holds more than
// kListMax keys, or the live keys are fewer than counted (NaN distances): the
// caller then uses the radix select.
__device__ bool select_hist(const Layout &s, int n, int want, bool bounded, float dmax) {
  if (n > kPerThread * kThreads) return false;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float scale = dmax > 0.f ? 256.f / dmax : 0.f;
  for (int b = tid; b < 256; b += kThreads) s.hist[b] = 0u;
  if (tid == 0) s.scal[kSLive] = 0;
  __syncthreads();
  float du[kPerThread];
  int bins[kPerThread];
  int live = 0;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = tid + k * kThreads;
    du[k] = i < n ? s.dist[i] : -1.f;
    bins[k] = du[k] >= 0.f ? min(255, static_cast<int>(du[k] * scale)) : -1;
    if (bins[k] >= 0) {
      atomicAdd(&s.hist[bins[k]], 1u);
      ++live;
    }
  }
  live = __reduce_add_sync(0xffffffffu, live);
  if (lane == 0) atomicAdd(&s.scal[kSLive], live);
  __syncthreads();
  if (warp == 0) find_threshold_bin(s, want, n);
  __syncthreads();
  if (s.scal[kSFallback] || s.scal[kSLive] < want) return false;
  const int bstar = s.scal[kSBin], above1 = s.scal[kSAbove], need1 = s.scal[kSNeed];
  __syncthreads();  // the scalars are read; hist and scal are reused below
  // level 2: the threshold bin's range in 256 sub-bins
  for (int b = tid; b < 256; b += kThreads) s.hist[b] = 0u;
  __syncthreads();
  const float fb = static_cast<float>(bstar);
  int sub[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    sub[k] = bins[k] == bstar ? min(255, max(0, static_cast<int>((du[k] * scale - fb) * 256.f)))
                              : -1;
    if (sub[k] >= 0) atomicAdd(&s.hist[sub[k]], 1u);
  }
  __syncthreads();
  if (warp == 0) find_threshold_bin(s, need1, kListMax);
  __syncthreads();
  if (s.scal[kSFallback]) return false;
  const int sstar = s.scal[kSBin], above = above1 + s.scal[kSAbove], need = s.scal[kSNeed];
  // keys above the threshold (slots 0 .. above-1) and the keys of the final
  // sub-bin (listed), placed by a prefix sum of (above count << 16 | listed)
  uint32_t na = 0, nl = 0;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    na += (bins[k] > bstar || (bins[k] == bstar && sub[k] > sstar)) ? 1u : 0u;
    nl += (bins[k] == bstar && sub[k] == sstar) ? 1u : 0u;
  }
  const uint32_t pre = block_exclusive_scan((na << 16) | nl, s.whist);
  int pa = static_cast<int>(pre >> 16), pb = static_cast<int>(pre & 0xffffu);
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = tid + k * kThreads;
    if (bins[k] > bstar || (bins[k] == bstar && sub[k] > sstar)) {
      s.cidx[pa] = i;
      s.cdist[pa] = du[k];
      ++pa;
    } else if (bins[k] == bstar && sub[k] == sstar) {
      s.lkey[pb] = dist_key(du[k]);
      s.lidx[pb] = i;
      ++pb;
    }
  }
  const int listed = static_cast<int>(s.hist[sstar]);
  __syncthreads();
  // rank the sub-bin's keys (key desc, index asc): rank r < need is taken,
  // the last taken one (rank need-1) is the bound when the selection is bounded
  for (int e = tid; e < listed; e += kThreads) {
    const uint32_t ke = s.lkey[e];
    const int ie = s.lidx[e];
    int rank = 0;
    for (int f = 0; f < listed; ++f) {
      const uint32_t kf = s.lkey[f];
      rank += (kf > ke || (kf == ke && s.lidx[f] < ie)) ? 1 : 0;
    }
    if (rank < need) {
      const int slot = bounded && rank == need - 1 ? kCand : above + rank;
      s.cidx[slot] = ie;
      s.cdist[slot] = __uint_as_float(ke & 0x7fffffffu);
    }
  }
  __syncthreads();
  return true;
}

// Step 1 of a round from the persistent histogram (s.uhist, one count per
// live point in bin ubin(u)): warp 0 finds the bin holding the want-th key,
// every point above it is placed by a block-wide prefix sum, and the keys of
// that bin are ranked against each other (key desc, index asc), the
// (kCand+1)-th going to slot kCand when `bounded`.  The counts the placement
// finds must equal the histogram's; if they do not (or the threshold bin
// holds more than kListMax keys, or fewer than `want` keys are live), nothing
// is kept and the caller uses the other selects.
__device__ bool select_fixed(const Layout &s, int n, int want, bool bounded) {
  if (n > kPerThread * kThreads) return false;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    // lane l sums bins 1023 - 32l - 31 .. 1023 - 32l (each lane reads a
    // different bank at every step)
    uint32_t sum = 0;
#pragma unroll 8
    for (int k = 0; k < 32; ++k) sum += s.uhist[kUBins - 1 - 32 * lane - ((k + lane) & 31)];
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const uint32_t excl = incl - sum;
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    const uint32_t w = static_cast<uint32_t>(want);
    const uint32_t hold = __ballot_sync(0xffffffffu, excl < w && w <= incl);
    int fallback = total < w || hold == 0u ? 1 : 0;
    const int L = hold ? __ffs(hold) - 1 : 0;
    // lane k takes the k-th highest bin of lane L's run
    const uint32_t exL = __shfl_sync(0xffffffffu, excl, L);
    const uint32_t c = s.uhist[kUBins - 1 - 32 * L - lane];
    uint32_t inc2 = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, inc2, o);
      if (lane >= o) inc2 += t;
    }
    const uint32_t reach = __ballot_sync(0xffffffffu, exL + inc2 >= w);
    const int k = reach ? __ffs(reach) - 1 : 0;
    if (!reach) fallback = 1;
    const uint32_t ck = __shfl_sync(0xffffffffu, c, k);
    const uint32_t above = exL + __shfl_sync(0xffffffffu, inc2, k) - ck;
    if (lane == 0) {
      s.scal[kSBin] = kUBins - 1 - 32 * L - k;
      s.scal[kSAbove] = static_cast<int>(above);
      s.scal[kSNeed] = want - static_cast<int>(above);
      s.scal[kSFallback] = fallback || ck > static_cast<uint32_t>(kListMax) ? 1 : 0;
      s.scal[kSListed] = static_cast<int>(ck);
    }
  }
  __syncthreads();
  if (s.scal[kSFallback]) return false;
  const int bstar = s.scal[kSBin], above = s.scal[kSAbove], need = s.scal[kSNeed];
  const int in_bin = s.scal[kSListed];
  float du[kPerThread];
  int bins[kPerThread];
  uint32_t na = 0, nl = 0;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = tid + k * kThreads;
    du[k] = i < n ? s.dist[i] : -1.f;
    bins[k] = ubin(du[k]);
    na += bins[k] > bstar ? 1u : 0u;
    nl += bins[k] == bstar ? 1u : 0u;
  }
  const uint32_t mine = (na << 16) | nl;
  const uint32_t pre = block_exclusive_scan(mine, s.whist);
  if (tid == kThreads - 1) {
    s.scal[kSPlaced] = static_cast<int>((pre + mine) >> 16);
    s.scal[kSLive] = static_cast<int>((pre + mine) & 0xffffu);
  }
  int pa = static_cast<int>(pre >> 16), pb = static_cast<int>(pre & 0xffffu);
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = tid + k * kThreads;
    if (bins[k] > bstar) {
      if (pa <= kCand) {
        s.cidx[pa] = i;
        s.cdist[pa] = du[k];
      }
      ++pa;
    } else if (bins[k] == bstar) {
      if (pb < kListMax) {
        s.lkey[pb] = dist_key(du[k]);
        s.lidx[pb] = i;
      }
      ++pb;
    }
  }
  __syncthreads();
  if (s.scal[kSPlaced] != above || s.scal[kSLive] != in_bin) {
    // the histogram disagrees with the distances: report, use another select
    if (tid == 0) record_device_status(BKV_DEV_ASSERT, 406);
    __syncthreads();  // every thread has read the counts
    return false;
  }
  // rank the bin's keys (key desc, index asc): rank r < need is taken, the
  // last taken one (rank need-1) is the bound when the selection is bounded
  for (int e = tid; e < in_bin; e += kThreads) {
    const uint32_t ke = s.lkey[e];
    const int ie = s.lidx[e];
    int rank = 0;
    for (int f = 0; f < in_bin; ++f) {
      const uint32_t kf = s.lkey[f];
      rank += (kf > ke || (kf == ke && s.lidx[f] < ie)) ? 1 : 0;
    }
    if (rank < need) {
      const int slot = bounded && rank == need - 1 ? kCand : above + rank;
      s.cidx[slot] = ie;
      s.cdist[slot] = __uint_as_float(ke & 0x7fffffffu);
    }
  }
  __syncthreads();
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    fps_tc_kernel(const __grid_constant__ CUtensorMap bmap, const __grid_constant__ CUtensorMap wmap,
                  const FpsGeom g, const __nv_bfloat16 *__restrict__ beacons_in,
                  const __nv_bfloat16 *__restrict__ window, __nv_bfloat16 *__restrict__ beacons_out,
                  int n_qheads, uint8_t *__restrict__ garrays, size_t slice_bytes,
                  int *__restrict__ head_counter, float l2_keep) {
  extern __shared__ uint8_t smem_raw[];
  const int n = g.nb_in + g.W;
  const int m = g.n_pick;
  Layout s;
  s.bars = reinterpret_cast<uint64_t *>(smem_raw);
  s.tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + 192);  // bars: 24 slots
  s.scal = reinterpret_cast<int *>(smem_raw + 256);
  s.hist = reinterpret_cast<uint32_t *>(smem_raw + 384);
  s.cidx = reinterpret_cast<int *>(smem_raw + 1408);
  s.cdist = reinterpret_cast<float *>(smem_raw + 1936);
  s.pick = reinterpret_cast<int *>(smem_raw + 2464);
  s.pinv = reinterpret_cast<float *>(smem_raw + 2976);   // .. 3552
  s.uhist = reinterpret_cast<uint32_t *>(smem_raw + 4096);  // .. 8192
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t big = (raw_base + kSmallBytes + 1023u) & ~1023u;
  s.ring = smem_raw + (big - raw_base);
  s.pop = s.ring + kStages * kTileBytes;
  s.gram = reinterpret_cast<float *>(s.ring + kGramOff);
  s.whist = reinterpret_cast<uint32_t *>(s.ring + kSelOff);
  s.lkey = s.whist + kWarps * 256;
  s.lidx = reinterpret_cast<int *>(s.lkey + kListMax);
  s.cop = s.ring + kCopOff;
  // the distance, inverse-norm and stamp arrays: in shared memory, or this
  // CTA's slice of the workspace for a union too large for it
  uint8_t *arrays = garrays ? garrays + static_cast<size_t>(blockIdx.x) * slice_bytes
                            : s.pop + 2 * kPBlock;
  s.dist = reinterpret_cast<float *>(arrays);
  s.inv = s.dist + n;
  s.stamp = reinterpret_cast<uint8_t *>(s.inv + n);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_btiles = (g.nb_in + kTileRows - 1) / kTileRows;
  const WindowTiles wt(g);
  const int n_tiles = n_btiles + wt.count;
  // the passes keep the union's first n_keep tiles in L2 (l2_keep: the share
  // of each union the launch can keep, from launch_fps_tc)
  const int n_keep = min(n_tiles, static_cast<int>(l2_keep * n_tiles + 0.5f));
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&s.bars[kBarFull + i]), 1);
      mbar_init(smem_u32(&s.bars[kBarEmpty + i]), 1);  // the MMA's commit (seed pass: the epilogue)
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(smem_u32(&s.bars[kBarTfull + a]), 1);
      mbar_init(smem_u32(&s.bars[kBarTempty + a]), 4);  // one arrive per warp of its warpgroup
    }
    for (int a = 0; a < 2; ++a) mbar_init(smem_u32(&s.bars[kBarDone + a]), 1);
    mbar_init(smem_u32(&s.bars[kBarGram]), 1);  // the round's Gram/refresh MMAs
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

  // Query heads are handed out as CTAs become free: head blockIdx.x first,
  // then the next unclaimed one (a head's cost varies with its rounds and
  // passes by about +-20%, which static striding would leave to the slowest
  // CTA).
  auto next_head = [&]() {
    __syncthreads();  // the slot's previous value has been read by every thread
    if (tid == 0) s.scal[kSHead] = static_cast<int>(gridDim.x) + atomicAdd(head_counter, 1);
    __syncthreads();
    return s.scal[kSHead];
  };
  for (int qh = blockIdx.x; qh < n_qheads; qh = next_head()) {
    Head h{beacons_in + static_cast<size_t>(qh) * g.M * kDim,
           window + static_cast<size_t>(qh) * g.w_cap * kDim, g.nb_in,
           g.w_cap > 0 ? g.w_cap : 1, g.w_start};
    __nv_bfloat16 *out = beacons_out + static_cast<size_t>(qh) * g.M * kDim;
    // the seed U[0]: the first pick, row 0 of the picks operand and of the output
    for (int c16 = tid; c16 < 16; c16 += kThreads) {
      const uint4 v = *reinterpret_cast<const uint4 *>(h.point(0) + c16 * 8);
      *reinterpret_cast<uint4 *>(s.pop + (c16 >> 3) * kPBlock + sw128_offset(0, c16 & 7)) = v;
      *reinterpret_cast<uint4 *>(out + c16 * 8) = v;
    }
    if (tid == 0) {
      // its inverse norm, summed in the order the seed pass uses for every point
      float ss = 0.f;
      for (int t = 0; t < kDim; t += 8) {
        float u[8];
        load8(h.point(0) + t, u);
        for (int e = 0; e < 8; ++e) ss = fmaf(u[e], u[e], ss);
      }
      s.pinv[0] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
      s.scal[kSKeyMin] = -1;
      s.scal[kSKeyMax] = 0;
    }
    for (int k = 1 + tid; k < kPickRows; k += kThreads) s.pinv[k] = __int_as_float(0x7fc00000);
    if (m <= 1) continue;  // nothing past the seed (every thread sees the same m)
    for (int b = tid; b < kUBins; b += kThreads) s.uhist[b] = 0u;
    fence_proxy_async_smem();
    __syncthreads();
    distance_pass(s, &bmap, &wmap, tmem, qh, h, g, n_btiles, wt.first, n_tiles, seq, 0, 1, true,
                  n_keep);
    seq += n_tiles;
    __syncthreads();
    if (s.scal[kAbort]) break;
    if (tid == 0) {
      const int b = ubin(s.dist[0]);  // the seed leaves the live set
      if (b >= 0) s.uhist[b] -= 1u;
      s.dist[0] = -1.f;
    }
    __syncthreads();

    int P = 1;          // picks so far
    int E = 1;          // every unselected point's stamp is at least E
    bool eager = true;  // a pass preceded this round: every distance is exact
    float dmax = __uint_as_float(static_cast<uint32_t>(s.scal[kSKeyMax]) & 0x7fffffffu);
    while (P < m) {
      const int unsel = n - P;
      const int nc = min(kCand, unsel);
      const bool bounded = unsel > kCand;
      const int want = bounded ? kCand + 1 : nc;
      // ---- 1. candidates
      if (!select_fixed(s, n, want, bounded) && !select_hist(s, n, want, bounded, dmax)) {
        // a threshold bin too crowded to rank (or distances that are not
        // numbers): the radix select, then the bound moves to slot kCand
        select_best<kThreads>(s.dist, n, unsel, want, s.whist, s.hist, s.scal, s.cidx, s.cdist,
                              false);
        __syncthreads();
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
      }
      // ---- 2. the candidates' rows into the swizzled operand, and the
      // lowest stamp among them (candidates behind P are refreshed)
      if (tid == 0) s.scal[kSRef] = P;
      __syncthreads();
      {
        // every load of this thread's pieces is issued before the first store
        constexpr int kIters = (kCand * 16 + kThreads - 1) / kThreads;
        uint4 v[kIters];
#pragma unroll
        for (int u = 0; u < kIters; ++u) {
          const int e = tid + u * kThreads;
          if (e < nc * 16)
          {
            const int ci = s.cidx[e >> 4];
            if (BKV_CHECK(ci >= 0 && ci < n, 701))
              v[u] = __ldg(reinterpret_cast<const uint4 *>(h.point(ci) + (e & 15) * 8));
          }
        }
#pragma unroll
        for (int u = 0; u < kIters; ++u) {
          const int e = tid + u * kThreads;
          if (e < nc * 16) {
            const int a = e >> 4, c16 = e & 15;
            *reinterpret_cast<uint4 *>(s.cop + (c16 >> 3) * kCBlock + sw128_offset(a, c16 & 7)) =
                v[u];
          }
        }
        if (tid < nc) {
          const int ci = s.cidx[tid];
          const int t = BKV_CHECK(ci >= 0 && ci < n, 702) ? s.stamp[ci] : P;
          if (t < P) atomicMin(&s.scal[kSRef], t);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      const int t_lo = s.scal[kSRef];
      const bool refresh = t_lo < P;
      const int s_ref = t_lo & ~7;
      const int n_ref = (P - s_ref + 15) & ~15;
      // Gram block D[a][b] = cand_a . cand_b (M = N = 128), and the refresh
      // block D[a][j] = cand_a . pick_(s_ref + j): the same f32 sums of exact
      // bf16 products as the distance pass, with the candidate as operand A
      if (warp == 1 && lane == 0) {
        tc_fence_after();
        const uint32_t c_base = smem_u32(s.cop);
        const uint32_t idesc = idesc_bf16_f32(128, kCand);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_k_sw128(c_base + kb * kCBlock + kk * 32);
            umma_f16(tmem + kGramCol, ad, ad, idesc, (kb | kk) != 0);
          }
        }
        if (refresh) {
          const uint32_t p_base = smem_u32(s.pop) + static_cast<uint32_t>(s_ref) * 128u;
          const uint32_t ridesc = idesc_bf16_f32(128, n_ref);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc_k_sw128(c_base + kb * kCBlock + kk * 32);
              const uint64_t bd = smem_desc_k_sw128(p_base + kb * kPBlock + kk * 32);
              umma_f16(tmem + kRefCol, ad, bd, ridesc, (kb | kk) != 0);
            }
          }
        }
        umma_commit(smem_u32(&s.bars[kBarGram]));
      }
      if (warp >= 4 && (warp < 8 || refresh)) {
        // TMEM lane = candidate a; warps 4-7 copy the Gram rows to shared
        // memory, warps 8-11 refresh the candidates whose stamp is behind
        const int quarter = warp & 3;
        const int a = quarter * 32 + lane;
        if (mbar_wait_warp(smem_u32(&s.bars[kBarGram]), gram_phase & 1, kWhereEpi)) {
          tc_fence_after();
          const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
          if (warp < 8) {
            float *row = s.gram + a * kGramStride;
#pragma unroll 1
            for (int c0 = 0; c0 < kCand; c0 += 32) {
              float x[32];
              tmem_ld_32x32b_x32(lane_base + kGramCol + c0, x);
              tmem_ld_wait_regs(x);
              if (a < nc) {
#pragma unroll
                for (int b = 0; b < 32; ++b) row[c0 + b] = x[b];
              }
            }
          } else {
            int i = a < nc ? s.cidx[a] : 0;
            if (!BKV_CHECK(i >= 0 && i < n, 703)) i = 0;
            const int t = a < nc ? static_cast<int>(s.stamp[i]) : P;
            const float inv_a = a < nc ? s.inv[i] : 0.f;
            float mn = INFINITY;
            for (int c0 = 0; c0 < n_ref; c0 += 32) {
              float v[32];
              if (c0 + 32 <= n_ref) {
                tmem_ld_32x32b_x32(lane_base + kRefCol + c0, v);
                tmem_ld_wait_regs(v);
                if (t < P) mn = chunk_min<32>(v, s.pinv + s_ref, c0, t - s_ref, inv_a, mn);
              } else {
                float hv[16];
                tmem_ld_32x32b_x16(lane_base + kRefCol + c0, hv);
                tmem_ld_wait_regs(hv);
#pragma unroll
                for (int k = 0; k < 16; ++k) v[k] = hv[k];
                if (t < P) mn = chunk_min<16>(v, s.pinv + s_ref, c0, t - s_ref, inv_a, mn);
              }
            }
            if (t < P) s.cdist[a] = fmaxf(fminf(s.cdist[a], mn), 0.f);
          }
        } else {
          s.scal[kAbort] = 1;
        }
        tc_fence_before();
      }
      ++gram_phase;
      __syncthreads();
      if (s.scal[kAbort]) break;
      // ---- 3. replay the greedy choice among the candidates (warp 0, four
      // per lane: slots lane, lane+32, lane+64, lane+96).  The argmax in
      // (distance desc, index asc) order takes two warp reductions: the
      // largest distance key, then the lowest index holding it (with the
      // slot).
      if (warp == 0) {
        float c[4], iv[4];
        int ix[4];
        bool taken[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int a = lane + 32 * q;
          taken[q] = a >= nc;
          c[q] = taken[q] ? 0.f : s.cdist[a];
          ix[q] = taken[q] ? 0x7fffffff : s.cidx[a];
          if (!taken[q] && !BKV_CHECK(ix[q] >= 0 && ix[q] < n, 704)) {
            taken[q] = true;  // skipped: its index is not a point of the union
            ix[q] = 0x7fffffff;
          }
          iv[q] = taken[q] ? 0.f : s.inv[ix[q]];
        }
        const float bd = bounded ? s.cdist[kCand] : -3.f;
        const int bi = bounded ? s.cidx[kCand] : 0x7fffffff;
        int np = 0;
        while (P + np < m) {
          // distances are >= 0, so their bits order like the values; +1 keeps
          // 0 free for "taken"
          uint32_t kq[4], kmax = 0u;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            kq[q] = taken[q] ? 0u : __float_as_uint(c[q]) + 1u;
            kmax = max(kmax, kq[q]);
          }
          const uint32_t kbest = __reduce_max_sync(0xffffffffu, kmax);
          if (kbest == 0u) break;  // no candidate left
          // the lowest point index holding it, with its slot in the low 7
          // bits (the union has fewer than 2^24 points), so one reduction
          // names both the point and its candidate slot
          uint32_t mine = 0xffffffffu;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (kq[q] == kbest)
              mine = min(mine, (static_cast<uint32_t>(ix[q]) << 7) |
                                   static_cast<uint32_t>(lane + 32 * q));
          const uint32_t best = __reduce_min_sync(0xffffffffu, mine);
          const int best_i = static_cast<int>(best >> 7);
          const int best_a = static_cast<int>(best & 127u);
          const float best_d = __uint_as_float(kbest - 1u);
          if (bounded && !before(best_d, best_i, bd, bi)) break;
          const float inv_b = s.inv[best_i];
          if (lane == 0) s.pick[np] = best_a;
          ++np;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (lane + 32 * q == best_a) taken[q] = true;
            if (!taken[q]) {
              // D[a][best] has the candidate as operand A, like the pass
              const float dot = s.gram[(lane + 32 * q) * kGramStride + best_a];
              c[q] = fminf(c[q], cos_dist(make_float2(dot, 0.f), iv[q], inv_b));
            }
          }
        }
        // the candidates not picked keep exact distances to all P + np picks;
        // every other point's u is at most the bound.  The histogram of u
        // follows: a picked candidate leaves it, the others move bins.
        float dm = bounded ? bd : 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (lane + 32 * q >= nc) continue;
          const int bo = ubin(s.dist[ix[q]]);
          const int bn = taken[q] ? -1 : ubin(c[q]);
          if (bn != bo) {
            if (bo >= 0) atomicSub(&s.uhist[bo], 1u);
            if (bn >= 0) atomicAdd(&s.uhist[bn], 1u);
          }
          if (!taken[q]) {
            s.dist[ix[q]] = c[q];
            s.stamp[ix[q]] = static_cast<uint8_t>(P + np);
            dm = fmaxf(dm, c[q]);
          }
        }
        dm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(dm)));
        if (lane == 0) {
          s.scal[kSNp] = np;
          s.scal[kSDmax] = __float_as_int(dm);
        }
      }
      __syncthreads();
      const int np = s.scal[kSNp];
      if (np == 0 && eager) {
        // an eager round's best candidate is the true argmax, so only
        // distances that are not numbers (NaN input rows) can stop it: report
        // and stop instead of looping
        if (tid == 0) record_device_status(BKV_DEV_ASSERT, 405);
        stuck = true;
        break;
      }
      // ---- 4. the picks: rows P .. P+np-1 of the picks operand and of the
      // output (from the staged candidate rows), their inverse norms, and
      // their distances set to -1
      for (int e = tid; e < np * 16; e += kThreads) {
        const int k = e >> 4, c16 = e & 15, kb = c16 >> 3, c = c16 & 7;
        const int a = s.pick[k];
        if (!BKV_CHECK(a >= 0 && a < nc && P + k < kPickRows, 705)) continue;
        const uint4 v = *reinterpret_cast<const uint4 *>(s.cop + kb * kCBlock + sw128_offset(a, c));
        *reinterpret_cast<uint4 *>(s.pop + kb * kPBlock + sw128_offset(P + k, c)) = v;
        *reinterpret_cast<uint4 *>(out + static_cast<size_t>(P + k) * kDim + c16 * 8) = v;
        if (c16 == 0) {
          const int i = s.cidx[a];
          if (!BKV_CHECK(i >= 0 && i < n, 706)) continue;
          s.pinv[P + k] = s.inv[i];
          s.dist[i] = -1.f;
        }
      }
      P += np;
      dmax = __int_as_float(s.scal[kSDmax]);
      if (P >= m) {
        __syncthreads();
        break;
      }
      eager = np < kPassBelow;
      if (tid == 0) {  // the pass gathers the range of its new keys
        s.scal[kSKeyMin] = -1;
        s.scal[kSKeyMax] = 0;
      }
      if (eager)  // and rebuilds the histogram of u
        for (int b = tid; b < kUBins; b += kThreads) s.uhist[b] = 0u;
      fence_proxy_async_smem();
      __syncthreads();
      if (eager) {
        distance_pass(s, &bmap, &wmap, tmem, qh, h, g, n_btiles, wt.first, n_tiles, seq, E & ~7, P,
                      false, n_keep);
        seq += n_tiles;
        __syncthreads();
        if (s.scal[kAbort]) break;
        E = P;
        dmax = __uint_as_float(static_cast<uint32_t>(s.scal[kSKeyMax]) & 0x7fffffffu);
      }
    }
    // the kept tiles' lines return to normal priority, so that a finished
    // union does not hold L2 against the next heads or kernels (a hint only:
    // rows of a tile past the head's own are left as they are)
    for (int t = tid; t < 2 * n_keep * kTileRows; t += kThreads) {
      const int j = t / (2 * kTileRows), r = (t >> 1) % kTileRows;
      const __nv_bfloat16 *row = nullptr;
      if (j < n_btiles) {
        if (j * kTileRows + r < h.nb) row = h.B + static_cast<size_t>(j * kTileRows + r) * kDim;
      } else {
        const long long slot = static_cast<long long>(wt.first + j - n_btiles) * kTileRows + r;
        if (slot < h.w_cap) row = h.Wp + static_cast<size_t>(slot) * kDim;
      }
      if (row != nullptr) l2_demote_line(reinterpret_cast<const uint8_t *>(row) + (t & 1) * 128);
    }
    if (s.scal[kAbort] || stuck) break;
  }

  // drain: every TMA load and MMA issued by this CTA has completed before the
  // CTA exits and frees its TMEM (after a timeout, loads may be in flight)
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
// slice of the per-point arrays per CTA when they live there).
constexpr int kMaxCtas = 148;

// dist (f32), inv (f32) and stamp (u8) of one union, rounded to 16 bytes
size_t union_array_bytes(const FpsGeom &g) {
  const size_t n = static_cast<size_t>(g.nb_in) + g.W;
  return (9 * n + 15) / 16 * 16;
}

bool arrays_in_smem(const FpsGeom &g) {
  return static_cast<size_t>(kFixedBytes) + union_array_bytes(g) <= static_cast<size_t>(kSmemLimit);
}

size_t smem_bytes(const FpsGeom &g) {
  return static_cast<size_t>(kFixedBytes) + (arrays_in_smem(g) ? union_array_bytes(g) : 0);
}

int fps_tc_grid(const FpsGeom &g) { return std::min(g.n_layers * g.n_q_heads, kMaxCtas); }

// L2 held by the unions of the heads in flight: each CTA keeps its share of
// it (the first tiles of its union) across the passes and streams the rest.
// With 148 unions of 1.08 MB (128 beacons + a 4096-query window) a cyclic
// stream through L2 under the default policy keeps little between passes;
// keeping a fixed ~40% of each union (64 MB in all) measured 2.36 ms
// against 2.455 ms for the 40-layer launch, and larger shares less (0.55:
// 2.37, 0.7: 2.43, all: 2.455 ms), as the kept lines push each other out.
constexpr double kL2KeepBytes = 64.0 * (1 << 20);
float l2_keep_fraction(const FpsGeom &g, int grid) {
  const double union_bytes = (static_cast<double>(g.nb_in) + g.W) * kDim * 2;
  if (union_bytes <= 0) return 1.f;
  const double f = kL2KeepBytes / (grid * union_bytes);
  return static_cast<float>(std::min(1.0, std::max(1.0 / 64, f)));
}

}  // namespace

// The head counter (16 bytes), then, for a union too large for shared
// memory, one slice of the per-point arrays per CTA.
constexpr size_t kCounterBytes = 16;
size_t fps_tc_workspace_bytes(const FpsGeom &g) {
  return kCounterBytes +
         (arrays_in_smem(g) ? 0 : static_cast<size_t>(fps_tc_grid(g)) * union_array_bytes(g));
}

bool fps_tc_supported(const FpsGeom &g) {
  // a union of fewer than 2^24 points: the replay packs a point index and a
  // 7-bit candidate slot into one 32-bit word
  return g.dtype == BKV_BF16 && g.head_dim == kDim && g.M <= kMaxPick &&
         static_cast<long long>(g.nb_in) + g.W < (1LL << 24) &&
         static_cast<long long>(g.n_layers) * g.n_q_heads *
                 std::max<long long>(g.M, std::max<long long>(g.W, g.w_cap)) <
             (1LL << 31) - 256;
}

bkv_status launch_fps_tc(const FpsGeom &g, const void *beacons_in, const void *window,
                         void *beacons_out, void *ws, size_t ws_bytes, cudaStream_t stream) {
  if (injected_launch_failure()) return BKV_ERR_CUDA;
  const size_t ws_need = fps_tc_workspace_bytes(g);
  if (ws == nullptr || ws_bytes < ws_need || (reinterpret_cast<uintptr_t>(ws) & 15u) != 0)
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
      static_cast<unsigned long long>(n_qheads) * static_cast<unsigned long long>(g.W > 0 ? g.w_cap : g.M);
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
  int *counter = static_cast<int *>(ws);
  if (cudaMemsetAsync(counter, 0, sizeof(int), stream) != cudaSuccess) return BKV_ERR_CUDA;
  uint8_t *arrays = ws_need > kCounterBytes ? static_cast<uint8_t *>(ws) + kCounterBytes : nullptr;
  fps_tc_kernel<<<grid, kThreads, smem, stream>>>(
      bmap, wmap, g, static_cast<const __nv_bfloat16 *>(beacons_in),
      static_cast<const __nv_bfloat16 *>(window), static_cast<__nv_bfloat16 *>(beacons_out),
      n_qheads, arrays, union_array_bytes(g), counter, l2_keep_fraction(g, grid));
  return cudaGetLastError() == cudaSuccess ? BKV_OK : BKV_ERR_CUDA;
}

}  // namespace bkv
