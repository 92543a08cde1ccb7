// bkv_api.cu -- the C ABI of libbkv.so (include/bkv.h): argument checks,
// workspace carving and the order in which the kernels are enqueued.
//
// Every argument check runs on the host before anything is launched, so a
// rejected call leaves the outputs untouched.  Nothing here allocates device
// memory: scratch space comes from the caller's workspace.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>

#include "bkv_device_status.cuh"
#include "bkv_internal.h"

namespace bkv {

bool injected_launch_failure() {
  static const bool on = [] {
    const char *v = std::getenv("BKV_INJECT_LAUNCH_FAILURE");
    return v != nullptr && v[0] != '\0' && !(v[0] == '0' && v[1] == '\0');
  }();
  return on;
}

void finish_score_geom(ScoreGeom *g) {
  g->group = g->n_q_heads / g->n_kv_heads;
  g->n_obs = g->group * (g->R + g->nb);
  g->n_obs_pad = static_cast<int>(align_up(static_cast<size_t>(g->n_obs), 128));
  g->n_groups = (g->n_obs + 511) / 512;
  const int per = (g->n_obs + g->n_groups - 1) / g->n_groups;
  g->rows_per_group = static_cast<int>(align_up(static_cast<size_t>(per), 16));
}

size_t score_workspace_bytes(const ScoreGeom &g) {
  const size_t c = align_up(static_cast<size_t>(g.n_heads()) * g.n_obs_pad * sizeof(float), kAlign);
  const int groups = std::max(g.n_groups, mean_grouping(g).n_groups);
  const size_t y = align_up(static_cast<size_t>(groups) * g.n_heads() *
                                static_cast<size_t>(g.L) * sizeof(float),
                            kAlign);
  return c + y;
}

ScoreWorkspace carve_score_workspace(const ScoreGeom &g, void *ws) {
  uint8_t *p = static_cast<uint8_t *>(ws);
  ScoreWorkspace w;
  w.c = reinterpret_cast<float *>(p);
  p += align_up(static_cast<size_t>(g.n_heads()) * g.n_obs_pad * sizeof(float), kAlign);
  w.ypart = reinterpret_cast<float *>(p);
  return w;
}

namespace {

constexpr long long kMaxRows = (1LL << 31) - 1;

// A host-side NVTX range (visible to a profiler that records NVTX, a no-op
// otherwise) around the enqueueing of one phase of the step.
struct PhaseRange {
  explicit PhaseRange(const char *name) { nvtxRangePushA(name); }
  ~PhaseRange() { nvtxRangePop(); }
  PhaseRange(const PhaseRange &) = delete;
  PhaseRange &operator=(const PhaseRange &) = delete;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(int dtype) { return dtype == BKV_BF16 ? 2 : 4; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

bkv_status check_desc(const bkv_cache_desc *d) {
  if (!d) return BKV_ERR_INVALID_ARG;
  if (d->n_layers < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->head_dim < 1 ||
      d->capacity < 1)
    return BKV_ERR_INVALID_ARG;
  if (d->n_q_heads % d->n_kv_heads != 0) return BKV_ERR_INVALID_ARG;
  if (d->dtype != BKV_F32 && d->dtype != BKV_BF16) return BKV_ERR_INVALID_ARG;
  if ((static_cast<size_t>(d->head_dim) * elem_size(d->dtype)) % 16 != 0)
    return BKV_ERR_INVALID_ARG;
  if (static_cast<long long>(d->n_layers) * d->n_kv_heads * d->capacity > kMaxRows)
    return BKV_ERR_INVALID_ARG;
  return BKV_OK;
}

// The compute paths that exist: bf16 with head_dim 128 (tensor cores) and f32
// with head_dim <= 128 (CUDA cores).
bkv_status check_compute_supported(const bkv_cache_desc *d) {
  if (d->dtype == BKV_BF16) return d->head_dim == 128 ? BKV_OK : BKV_ERR_UNSUPPORTED;
  return (d->head_dim <= 128 && d->head_dim % 4 == 0) ? BKV_OK : BKV_ERR_UNSUPPORTED;
}

size_t cache_bytes(const bkv_cache_desc *d) {
  return static_cast<size_t>(d->n_layers) * d->n_kv_heads * static_cast<size_t>(d->capacity) *
         d->head_dim * elem_size(d->dtype);
}

size_t query_bytes(const bkv_cache_desc *d, long long rows) {
  return static_cast<size_t>(d->n_layers) * d->n_q_heads * static_cast<size_t>(rows) *
         d->head_dim * elem_size(d->dtype);
}

// recent_cap / recent_start: where recent row i of a query head lives (row
// (recent_start + i) mod recent_cap of its block); a dense [R][d] block is
// cap R, start 0.
ScoreGeom make_score_geom(const bkv_cache_desc *d, long long L, int R, int nb, int M,
                          float scale, long long recent_cap = -1, long long recent_start = 0) {
  ScoreGeom g{};
  g.recent_cap = recent_cap < 0 ? R : recent_cap;
  g.recent_start = recent_start;
  g.n_layers = d->n_layers;
  g.n_q_heads = d->n_q_heads;
  g.n_kv_heads = d->n_kv_heads;
  g.head_dim = d->head_dim;
  g.cap = d->capacity;
  g.L = L;
  g.R = R;
  g.nb = nb;
  g.M = M;
  g.scale = scale != 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d->head_dim));
  finish_score_geom(&g);
  if (d->dtype == BKV_F32) {  // the CUDA-core path writes one partial
    g.n_groups = 1;
    g.rows_per_group = g.n_obs;
  }
  return g;
}

bkv_status check_score_args(const bkv_cache_desc *d, const void *k, long long L, const void *recent,
                            int R, const void *beacons, int nb, int M) {
  bkv_status st = check_desc(d);
  if (st != BKV_OK) return st;
  if (!k || L < 1 || L > d->capacity || R < 0 || M < 0 || nb < 0 || nb > M || R + nb < 1)
    return BKV_ERR_INVALID_ARG;
  if (R > 0 && !recent) return BKV_ERR_INVALID_ARG;
  if (nb > 0 && !beacons) return BKV_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(recent) || !aligned16(beacons)) return BKV_ERR_INVALID_ARG;
  const long long n_obs = static_cast<long long>(d->n_q_heads / d->n_kv_heads) * (R + nb);
  if (n_obs > (1 << 24)) return BKV_ERR_INVALID_ARG;
  return check_compute_supported(d);
}

// Scoring into the workspace: c and ypart; returns the geometry used.
bkv_status run_score(const ScoreGeom &g, int dtype, const void *k, const void *recent,
                     const void *beacons, const ScoreWorkspace &w, bool mean, cudaStream_t s) {
  bkv_status st;
  if (dtype == BKV_BF16) {
    st = launch_score_rowstats_tc(g, k, recent, beacons, w.c, s);
    if (st != BKV_OK) return st;
    return launch_score_colmax_tc(mean ? mean_grouping(g) : g, k, recent, beacons, w.c, w.ypart,
                                  mean, s);
  }
  st = launch_score_rowstats_simt(g, static_cast<const float *>(k),
                                  static_cast<const float *>(recent),
                                  static_cast<const float *>(beacons), w.c, s);
  if (st != BKV_OK) return st;
  return launch_score_colmax_simt(g, static_cast<const float *>(k),
                                  static_cast<const float *>(recent),
                                  static_cast<const float *>(beacons), w.c, w.ypart, mean, s);
}

SelectInput score_select_input(const ScoreGeom &g, int dtype, const ScoreWorkspace &w,
                               bool mean) {
  SelectInput in;
  in.src = w.ypart;
  // the tensor-core max aggregation leaves its groups merged, as order keys
  in.keys = !mean && dtype == BKV_BF16 ? 1 : 0;
  in.n_parts = in.keys ? 1 : mean && dtype == BKV_BF16 ? mean_grouping(g).n_groups : g.n_groups;
  in.part_stride = static_cast<size_t>(g.n_heads()) * static_cast<size_t>(g.L);
  in.mean = mean ? 1 : 0;
  in.inv_count = 1.0f / static_cast<float>(g.n_obs);
  return in;
}

bkv_status score_entry(const bkv_cache_desc *desc, const void *k, int64_t L,
                       const void *recent_q, int32_t R, const void *beacons, int32_t n_beacons,
                       int32_t M, float scale, float *scores, void *workspace,
                       size_t workspace_bytes, void *stream, bool mean) {
  bkv_status st = check_score_args(desc, k, L, recent_q, R, beacons, n_beacons, M);
  if (st != BKV_OK) return st;
  if (!scores || !aligned16(scores) || !std::isfinite(scale) || scale < 0.f)
    return BKV_ERR_INVALID_ARG;
  const ScoreGeom g = make_score_geom(desc, L, R, n_beacons, M, scale);
  if (!workspace || !aligned16(workspace) || workspace_bytes < score_workspace_bytes(g))
    return BKV_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ScoreWorkspace w = carve_score_workspace(g, workspace);
  st = run_score(g, desc->dtype, k, recent_q, beacons, w, mean, s);
  if (st != BKV_OK) return st;
  return launch_finalize_scores(score_select_input(g, desc->dtype, w, mean), g.n_heads(), L,
                                scores, s);
}

// The aggregation, top-K and compaction of a step in head batches: batch b's
// aggregation on `s`, its top-K and compaction on `aux` after an event, so
// that they overlap the aggregation of batch b + 1 (the compaction, bound by
// HBM, shares the SMs with the tensor-bound aggregation).  `s` finally waits
// for `aux`.  Events [3] (after the last aggregation), [4] and [5] (after the
// join) are recorded through `mark`.
template <typename Mark>
bkv_status run_batched_tail(const ScoreGeom &g, bool mean, const void *k, const void *recent,
                            const void *bq, const ScoreWorkspace &w, const SelectInput &in,
                            const CompactArgs &c, int32_t *idx, float *scores_out,
                            long long keep, bool in_place, cudaStream_t s, cudaStream_t aux,
                            Mark &&mark) {
  constexpr int kBatches = 4;
  const int H = g.n_heads();
  const int nbat = std::min(kBatches, H);
  cudaEvent_t ev[kBatches + 1] = {};
  bkv_status st = BKV_OK;
  for (int b = 0; b <= nbat && st == BKV_OK; ++b)
    if (cudaEventCreateWithFlags(&ev[b], cudaEventDisableTiming) != cudaSuccess) st = BKV_ERR_CUDA;
  const ScoreGeom gg = mean ? mean_grouping(g) : g;
  const size_t row_bytes = static_cast<size_t>(c.row_bytes);
  for (int b = 0; b < nbat && st == BKV_OK; ++b) {
    const int h0 = static_cast<int>(static_cast<long long>(H) * b / nbat);
    const int h1 = static_cast<int>(static_cast<long long>(H) * (b + 1) / nbat);
    {
      PhaseRange r("bkv aggregation (head batch)");
      st = launch_score_colmax_tc(gg, k, recent, bq, w.c, w.ypart, mean, s, h0, h1 - h0);
    }
    if (st != BKV_OK) break;
    if (cudaEventRecord(ev[b], s) != cudaSuccess || cudaStreamWaitEvent(aux, ev[b], 0) != cudaSuccess) {
      st = BKV_ERR_CUDA;
      break;
    }
    PhaseRange r("bkv top-K + compaction (head batch)");
    SelectInput ib = in;
    ib.src = in.src + static_cast<size_t>(h0) * static_cast<size_t>(g.L);
    st = launch_select_topk(ib, h1 - h0, g.L, keep, idx + static_cast<size_t>(h0) * keep,
                            scores_out ? scores_out + static_cast<size_t>(h0) * g.L : nullptr,
                            nullptr, 0, aux);
    if (st != BKV_OK) break;
    CompactArgs cb = c;
    const size_t src_off = static_cast<size_t>(h0) * static_cast<size_t>(c.src_cap) * row_bytes;
    const size_t dst_off = static_cast<size_t>(h0) * static_cast<size_t>(c.dst_cap) * row_bytes;
    cb.k_src = c.k_src ? c.k_src + src_off : nullptr;
    cb.v_src = c.v_src ? c.v_src + src_off : nullptr;
    cb.k_dst = c.k_dst ? c.k_dst + dst_off : nullptr;
    cb.v_dst = c.v_dst ? c.v_dst + dst_off : nullptr;
    cb.idx = c.idx + static_cast<size_t>(h0) * static_cast<size_t>(keep);
    cb.n_heads = h1 - h0;
    st = in_place ? launch_compact_inplace(cb, aux) : launch_compact(cb, aux);
  }
  if (st == BKV_OK && !mark(3)) st = BKV_ERR_CUDA;
  // join (also after an error, so that `s` never runs ahead of work on `aux`)
  if (ev[nbat] != nullptr) {
    if (cudaEventRecord(ev[nbat], aux) != cudaSuccess ||
        cudaStreamWaitEvent(s, ev[nbat], 0) != cudaSuccess)
      st = BKV_ERR_CUDA;
  }
  for (int b = 0; b <= nbat; ++b)
    if (ev[b] != nullptr) cudaEventDestroy(ev[b]);
  if (st == BKV_OK && (!mark(4) || !mark(5))) st = BKV_ERR_CUDA;
  return st;
}

}  // namespace
}  // namespace bkv

using namespace bkv;

extern "C" {

const char *bkv_status_string(bkv_status status) {
  switch (status) {
    case BKV_OK: return "ok";
    case BKV_ERR_INVALID_ARG: return "invalid argument";
    case BKV_ERR_UNSUPPORTED: return "unsupported dtype or shape";
    case BKV_ERR_WORKSPACE: return "workspace missing or too small";
    case BKV_ERR_CUDA: return "CUDA error";
    case BKV_ERR_TIMEOUT: return "device-side wait timed out";
    case BKV_ERR_DEVICE_ASSERT: return "device-side check failed";
  }
  return "unknown status";
}

size_t bkv_workspace_size(const bkv_cache_desc *desc, int64_t L, int32_t R, int32_t M, int32_t W,
                          int64_t K) {
  if (check_desc(desc) != BKV_OK || L < 1 || R < 0 || M < 0 || W < 0 || K < 1) return 0;
  const ScoreGeom g = make_score_geom(desc, L, R, M, M, 0.f);
  size_t total = score_workspace_bytes(g);
  total += align_up(select_workspace_bytes(g.n_heads(), L), kAlign);
  const long long keep = std::min<long long>(K, L);
  total += align_up(static_cast<size_t>(g.n_heads()) * keep * sizeof(int32_t), kAlign);
  FpsGeom f{desc->n_layers, desc->n_q_heads, desc->head_dim, desc->dtype, M, M, W,
            std::min(M, M + W), W, 0};
  total += align_up(fps_workspace_bytes(f), kAlign);
  return total;
}

bkv_status bkv_score(const bkv_cache_desc *desc, const void *k, int64_t L, const void *recent_q,
                     int32_t R, const void *beacons, int32_t n_beacons, int32_t M, float scale,
                     float *scores, void *workspace, size_t workspace_bytes, void *stream) {
  return score_entry(desc, k, L, recent_q, R, beacons, n_beacons, M, scale, scores, workspace,
                     workspace_bytes, stream, false);
}

bkv_status bkv_score_mean(const bkv_cache_desc *desc, const void *k, int64_t L,
                          const void *recent_q, int32_t R, const void *beacons,
                          int32_t n_beacons, int32_t M, float scale, float *scores,
                          void *workspace, size_t workspace_bytes, void *stream) {
  return score_entry(desc, k, L, recent_q, R, beacons, n_beacons, M, scale, scores, workspace,
                     workspace_bytes, stream, true);
}

bkv_status bkv_select_topk(const float *scores, int32_t n_rows, int64_t L, int64_t K,
                           int32_t *idx, void *workspace, size_t workspace_bytes, void *stream) {
  if (!scores || !idx || n_rows < 1 || L < 1 || K < 1 || L > kMaxRows) return BKV_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx)) return BKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (K >= L) return launch_iota_rows(idx, n_rows, L, s);
  if (workspace_bytes < select_workspace_bytes(n_rows, L)) return BKV_ERR_WORKSPACE;
  SelectInput in{scores, 1, 0, 0, 1.f};
  return launch_select_topk(in, n_rows, L, K, idx, nullptr, workspace, workspace_bytes, s);
}

bkv_status bkv_compact(const bkv_cache_desc *src, const void *k_src, const void *v_src,
                       const int32_t *idx, int64_t n_keep, const bkv_cache_desc *dst, void *k_dst,
                       void *v_dst, void *stream) {
  bkv_status st = check_desc(src);
  if (st != BKV_OK) return st;
  st = check_desc(dst);
  if (st != BKV_OK) return st;
  if (src->n_layers != dst->n_layers || src->n_kv_heads != dst->n_kv_heads ||
      src->head_dim != dst->head_dim || src->dtype != dst->dtype)
    return BKV_ERR_INVALID_ARG;
  if (n_keep < 0 || n_keep > dst->capacity) return BKV_ERR_INVALID_ARG;
  if ((k_src == nullptr) != (k_dst == nullptr) || (v_src == nullptr) != (v_dst == nullptr))
    return BKV_ERR_INVALID_ARG;
  if (n_keep > 0 && !idx) return BKV_ERR_INVALID_ARG;
  if (!aligned16(k_src) || !aligned16(v_src) || !aligned16(k_dst) || !aligned16(v_dst) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u))
    return BKV_ERR_INVALID_ARG;
  const size_t sb = cache_bytes(src), db = cache_bytes(dst);
  if (overlaps(k_dst, db, k_src, sb) || overlaps(k_dst, db, v_src, sb) ||
      overlaps(v_dst, db, k_src, sb) || overlaps(v_dst, db, v_src, sb) ||
      overlaps(k_dst, db, v_dst, db))
    return BKV_ERR_INVALID_ARG;
  CompactArgs a;
  a.k_src = static_cast<const uint8_t *>(k_src);
  a.v_src = static_cast<const uint8_t *>(v_src);
  a.k_dst = static_cast<uint8_t *>(k_dst);
  a.v_dst = static_cast<uint8_t *>(v_dst);
  a.idx = idx;
  a.n_heads = src->n_layers * src->n_kv_heads;
  a.n_keep = n_keep;
  a.src_cap = src->capacity;
  a.dst_cap = dst->capacity;
  a.row_bytes = static_cast<int>(src->head_dim * elem_size(src->dtype));
  return launch_compact(a, static_cast<cudaStream_t>(stream));
}

bkv_status bkv_compact_inplace(const bkv_cache_desc *desc, void *k, void *v, const int32_t *idx,
                               int64_t n_keep, void *stream) {
  bkv_status st = check_desc(desc);
  if (st != BKV_OK) return st;
  if (!k || n_keep < 0 || n_keep > desc->capacity) return BKV_ERR_INVALID_ARG;
  if (n_keep > 0 && !idx) return BKV_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(idx) & 3u))
    return BKV_ERR_INVALID_ARG;
  if (v && overlaps(k, cache_bytes(desc), v, cache_bytes(desc))) return BKV_ERR_INVALID_ARG;
  CompactArgs a;
  a.k_src = static_cast<const uint8_t *>(k);
  a.v_src = static_cast<const uint8_t *>(v);
  a.k_dst = static_cast<uint8_t *>(k);
  a.v_dst = static_cast<uint8_t *>(v);
  a.idx = idx;
  a.n_heads = desc->n_layers * desc->n_kv_heads;
  a.n_keep = n_keep;
  a.src_cap = a.dst_cap = desc->capacity;
  a.row_bytes = static_cast<int>(desc->head_dim * elem_size(desc->dtype));
  return launch_compact_inplace(a, static_cast<cudaStream_t>(stream));
}

bkv_status bkv_update_beacons(const bkv_cache_desc *desc, const void *beacons_in,
                              int32_t n_beacons_in, int32_t M, const void *window, int32_t W,
                              void *beacons_out, int32_t *n_beacons_out, void *workspace,
                              size_t workspace_bytes, void *stream) {
  bkv_status st = check_desc(desc);
  if (st != BKV_OK) return st;
  if (M < 1 || n_beacons_in < 0 || n_beacons_in > M || W < 0 || n_beacons_in + W < 1)
    return BKV_ERR_INVALID_ARG;
  if ((n_beacons_in > 0 && !beacons_in) || (W > 0 && !window) || !beacons_out)
    return BKV_ERR_INVALID_ARG;
  if (!aligned16(beacons_in) || !aligned16(window) || !aligned16(beacons_out))
    return BKV_ERR_INVALID_ARG;
  const size_t bbytes = query_bytes(desc, M), wbytes = query_bytes(desc, W);
  if (overlaps(beacons_out, bbytes, beacons_in, bbytes) ||
      overlaps(beacons_out, bbytes, window, wbytes))
    return BKV_ERR_INVALID_ARG;
  if (desc->head_dim > 128) return BKV_ERR_UNSUPPORTED;
  FpsGeom f{desc->n_layers, desc->n_q_heads, desc->head_dim, desc->dtype, n_beacons_in, M, W,
            std::min(M, n_beacons_in + W), W, 0};
  if (!fps_supported(f)) return BKV_ERR_UNSUPPORTED;
  if (workspace_bytes < fps_workspace_bytes(f)) return BKV_ERR_WORKSPACE;
  st = launch_fps(f, beacons_in, window, beacons_out, workspace, workspace_bytes,
                  static_cast<cudaStream_t>(stream));
  if (st == BKV_OK && n_beacons_out) *n_beacons_out = f.n_pick;
  return st;
}

bkv_status bkv_compress_step(const bkv_step_args *a, int32_t *n_beacons_out, int64_t *new_len) {
  if (!a) return BKV_ERR_INVALID_ARG;
  const bkv_cache_desc *d = &a->cache;
  // the recent queries and the window: dense blocks, or the newest rows of a
  // decode-side query ring (slot of query t: t mod ring_cap)
  const bool ring = a->query_ring != nullptr;
  if (ring) {
    if (a->recent_q || a->window || a->ring_cap < 1 || a->R < 0 || a->W < 0 ||
        a->R > a->ring_cap || a->W > a->ring_cap || a->ring_pos < std::max<int64_t>(a->R, a->W) ||
        !aligned16(a->query_ring) ||
        static_cast<long long>(d->n_layers) * d->n_q_heads * a->ring_cap > kMaxRows)
      return BKV_ERR_INVALID_ARG;
  }
  const void *recent_src = ring ? a->query_ring : a->recent_q;
  const void *window_src = ring ? a->query_ring : a->window;
  const long long recent_cap = ring ? a->ring_cap : a->R;
  const long long recent_start = ring ? (a->ring_pos - a->R) % a->ring_cap : 0;
  const long long w_cap = ring ? a->ring_cap : a->W;
  const long long w_start = ring ? (a->ring_pos - a->W) % a->ring_cap : 0;
  const size_t wbytes = query_bytes(d, w_cap);
  const bool update = window_src != nullptr && a->W > 0;
  const int nb_used = update ? std::min(a->M, a->n_beacons_in + a->W) : a->n_beacons_in;
  // scoring arguments (the beacons it reads are the updated ones when W > 0)
  const void *score_beacons = update ? a->beacons_out : a->beacons_in;
  bkv_status st = check_score_args(d, a->k, a->L, a->R > 0 ? recent_src : nullptr, a->R,
                                   nb_used > 0 ? score_beacons : nullptr, nb_used, a->M);
  if (st != BKV_OK) return st;
  if (a->K < 1 || !a->v || !std::isfinite(a->scale) || a->scale < 0.f) return BKV_ERR_INVALID_ARG;
  if (a->aggregate != BKV_AGG_MAX && a->aggregate != BKV_AGG_MEAN) return BKV_ERR_INVALID_ARG;
  const bool mean = a->aggregate == BKV_AGG_MEAN;
  if (update) {
    if (a->n_beacons_in < 0 || a->n_beacons_in > a->M || !a->beacons_out ||
        (a->n_beacons_in > 0 && !a->beacons_in))
      return BKV_ERR_INVALID_ARG;
    if (!aligned16(window_src) || !aligned16(a->beacons_out)) return BKV_ERR_INVALID_ARG;
    const size_t bbytes = query_bytes(d, a->M);
    if (overlaps(a->beacons_out, bbytes, a->beacons_in, bbytes) ||
        overlaps(a->beacons_out, bbytes, window_src, wbytes) ||
        overlaps(a->beacons_out, bbytes, recent_src, query_bytes(d, recent_cap)))
      return BKV_ERR_INVALID_ARG;
  }
  st = check_desc(&a->dst_cache);
  if (st != BKV_OK) return st;
  const long long keep = std::min<long long>(a->K, a->L);
  const bkv_cache_desc *dd = &a->dst_cache;
  if (dd->n_layers != d->n_layers || dd->n_kv_heads != d->n_kv_heads ||
      dd->head_dim != d->head_dim || dd->dtype != d->dtype || dd->capacity < keep)
    return BKV_ERR_INVALID_ARG;
  if (!a->k_dst || !a->v_dst || !aligned16(a->k_dst) || !aligned16(a->v_dst) ||
      !aligned16(a->v) || !aligned16(a->scores_out) || !aligned16(a->idx_out))
    return BKV_ERR_INVALID_ARG;
  const size_t sb = cache_bytes(d), db = cache_bytes(dd);
  // in place: the destination is exactly the source cache
  const bool in_place = a->k_dst == a->k && a->v_dst == a->v && dd->capacity == d->capacity;
  if (in_place ? overlaps(a->k, sb, a->v, sb)
               : (overlaps(a->k_dst, db, a->k, sb) || overlaps(a->k_dst, db, a->v, sb) ||
                  overlaps(a->v_dst, db, a->k, sb) || overlaps(a->v_dst, db, a->v, sb) ||
                  overlaps(a->k_dst, db, a->v_dst, db)))
    return BKV_ERR_INVALID_ARG;

  if (a->aux_stream != nullptr && a->aux_stream == a->stream) return BKV_ERR_INVALID_ARG;
  const bool overlap = a->aux_stream != nullptr && d->dtype == BKV_BF16 && keep < a->L &&
                       d->n_layers * d->n_kv_heads >= 2;
  FpsGeom f{d->n_layers, d->n_q_heads, d->head_dim, d->dtype, a->n_beacons_in, a->M, a->W,
            nb_used, w_cap, w_start};
  if (update && !fps_supported(f)) return BKV_ERR_UNSUPPORTED;
  const ScoreGeom g = make_score_geom(d, a->L, a->R, nb_used, a->M, a->scale, recent_cap,
                                      recent_start);
  const bool need_scores = keep < a->L || a->scores_out != nullptr;
  // workspace: [score][select][idx][fps]
  const size_t score_b = need_scores ? score_workspace_bytes(g) : 0;
  const size_t sel_b = keep < a->L ? align_up(select_workspace_bytes(g.n_heads(), a->L), kAlign) : 0;
  const size_t idx_b =
      a->idx_out ? 0 : align_up(static_cast<size_t>(g.n_heads()) * keep * sizeof(int32_t), kAlign);
  const size_t fps_b = update ? align_up(fps_workspace_bytes(f), kAlign) : 0;
  const size_t need = score_b + sel_b + idx_b + fps_b;
  if (need > 0 && (!a->workspace || !aligned16(a->workspace) || a->workspace_bytes < need))
    return BKV_ERR_WORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(a->stream);
  uint8_t *ws = static_cast<uint8_t *>(a->workspace);
  const ScoreWorkspace w = carve_score_workspace(g, ws);
  void *sel_ws = ws + score_b;
  int32_t *idx = a->idx_out ? a->idx_out : reinterpret_cast<int32_t *>(ws + score_b + sel_b);
  void *fps_ws = ws + score_b + sel_b + idx_b;

  auto mark = [&](int i) -> bool {
    if (!a->phase_events || !a->phase_events[i]) return true;
    return cudaEventRecord(static_cast<cudaEvent_t>(a->phase_events[i]), s) == cudaSuccess;
  };
  PhaseRange step_range("bkv_compress_step");
  if (!mark(0)) return BKV_ERR_CUDA;
  if (update) {
    PhaseRange r("bkv continual FPS");
    st = launch_fps(f, a->beacons_in, window_src, a->beacons_out, fps_ws, fps_b, s);
    if (st != BKV_OK) return st;
  }
  if (!mark(1)) return BKV_ERR_CUDA;
  const void *bq = nb_used > 0 ? score_beacons : nullptr;
  if (need_scores) {
    PhaseRange r("bkv scoring");
    if (d->dtype == BKV_BF16) {
      st = launch_score_rowstats_tc(g, a->k, recent_src, bq, w.c, s);
      if (st != BKV_OK) return st;
      if (!mark(2)) return BKV_ERR_CUDA;
    } else {
      st = launch_score_rowstats_simt(g, static_cast<const float *>(a->k),
                                      static_cast<const float *>(recent_src),
                                      static_cast<const float *>(bq), w.c, s);
      if (st != BKV_OK) return st;
      if (!mark(2)) return BKV_ERR_CUDA;
      st = launch_score_colmax_simt(g, static_cast<const float *>(a->k),
                                    static_cast<const float *>(recent_src),
                                    static_cast<const float *>(bq), w.c, w.ypart, mean, s);
    }
    if (st != BKV_OK) return st;
  } else if (!mark(2)) {
    return BKV_ERR_CUDA;
  }
  const SelectInput in = score_select_input(g, d->dtype, w, mean);
  const bool copy_all = keep >= a->L;
  CompactArgs c;
  c.k_src = static_cast<const uint8_t *>(a->k);
  c.v_src = static_cast<const uint8_t *>(a->v);
  c.k_dst = static_cast<uint8_t *>(a->k_dst);
  c.v_dst = static_cast<uint8_t *>(a->v_dst);
  c.idx = copy_all ? nullptr : idx;
  c.n_heads = g.n_heads();
  c.n_keep = keep;
  c.src_cap = d->capacity;
  c.dst_cap = dd->capacity;
  c.row_bytes = static_cast<int>(d->head_dim * elem_size(d->dtype));
  if (overlap) {
    // Head batches: the aggregation of batch b on `s`; then, on the aux
    // stream, batch b's top-K and compaction, which touch only batch b's
    // heads, while `s` aggregates batch b + 1.  The compaction reads the
    // cache only after the aggregation of its own heads (the event), and
    // the row statistics of every head finished before the first batch.
    st = run_batched_tail(g, mean, a->k, recent_src, bq, w, in, c, idx, a->scores_out, keep,
                          in_place, s, static_cast<cudaStream_t>(a->aux_stream), mark);
    if (st != BKV_OK) return st;
    if (n_beacons_out) *n_beacons_out = nb_used;
    if (new_len) *new_len = keep;
    return BKV_OK;
  }
  if (need_scores && d->dtype == BKV_BF16) {
    PhaseRange r("bkv aggregation");
    st = launch_score_colmax_tc(mean ? mean_grouping(g) : g, a->k, recent_src, bq, w.c, w.ypart,
                                mean, s);
    if (st != BKV_OK) return st;
  }
  if (!mark(3)) return BKV_ERR_CUDA;
  {
    PhaseRange r("bkv top-K");
    if (!copy_all) {
      st = launch_select_topk(in, g.n_heads(), a->L, keep, idx, a->scores_out, sel_ws, sel_b, s);
      if (st != BKV_OK) return st;
    } else {
      if (a->scores_out) {
        st = launch_finalize_scores(in, g.n_heads(), a->L, a->scores_out, s);
        if (st != BKV_OK) return st;
      }
      if (a->idx_out) {
        st = launch_iota_rows(a->idx_out, g.n_heads(), keep, s);
        if (st != BKV_OK) return st;
      }
    }
  }
  if (!mark(4)) return BKV_ERR_CUDA;
  PhaseRange compact_range("bkv compaction");
  if (in_place) {
    // nothing to move when every row is kept
    st = copy_all ? BKV_OK : launch_compact_inplace(c, s);
  } else {
    st = launch_compact(c, s);
  }
  if (st != BKV_OK) return st;
  if (!mark(5)) return BKV_ERR_CUDA;
  if (n_beacons_out) *n_beacons_out = nb_used;
  if (new_len) *new_len = keep;
  return BKV_OK;
}

bkv_status bkv_read_device_status(void *stream, int32_t *where_out) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int where = 0;
  int code = take_status_score_tc(s, &where);
  if (code == 0) code = take_status_select(s, &where);
  if (code == 0) code = take_status_fps_tc(s, &where);
  if (code == 0) code = take_status_compact(s, &where);
  if (code == 0) code = take_status_fps(s, &where);
  if (code == 0) code = take_status_selftest(s, &where);
  if (code < 0) return BKV_ERR_CUDA;
  if (where_out) *where_out = code ? where : 0;
  if (code == 0) return BKV_OK;
  return code == BKV_DEV_TIMEOUT ? BKV_ERR_TIMEOUT : BKV_ERR_DEVICE_ASSERT;
}

}  // extern "C"
