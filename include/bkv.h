/*
 * bkv.h -- C ABI of libbkv.so, the B200 (sm_100a) BeaconKV compression step.
 *
 * The operations follow "BeaconKV: Key-Value Cache Compression Guided by Beacon
 * Queries for Efficient Large Reasoning Model Inference" (Kim, Kim, Shim, Choi):
 *   - Fig. 5(b): attention-based scores of every cached key, computed from the
 *     beacon queries and the recent queries (bkv_score);
 *   - Fig. 5(c) and Table 2: top-K selection after max aggregation over the
 *     queries and the query heads of each GQA group (bkv_score, bkv_select_topk);
 *   - abstract and Fig. 5(a): the unselected KV pairs are evicted (bkv_compact);
 *   - Fig. 7: beacon queries are maintained by Continual farthest-point
 *     sampling (bkv_update_beacons);
 *   - all of the above in one call (bkv_compress_step).
 * The page states the step in words only; the exact arithmetic implemented
 * here is:
 *   x[o][j] = scale * q_o . k_j   for the observation rows o of one KV head
 *             (the R recent and n_beacons beacon queries of each of its
 *             G = n_q_heads / n_kv_heads query heads) and every key j < L;
 *   s[j]    = max_o softmax_o(j) = max_o exp(x[o][j] - logsumexp_j' x[o][j']);
 *   idx     = the min(K, L) positions with the largest s (ties: lower
 *             position), in ascending order;
 *   FPS     = greedy farthest-point sampling in cosine distance
 *             1 - cos(a, b) over [beacons; window], seeded with the first row.
 *
 * Conventions for every entry point:
 *   - Memory: every pointer named "device" is device memory (or managed memory)
 *     of the current CUDA device; the caller allocates and owns it.  The
 *     library never allocates or frees device memory; scratch space is the
 *     caller's "workspace" buffer, sized with bkv_workspace_size().
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  All device work is enqueued on it and the call
 *     returns without synchronising.
 *   - Errors: argument checks run on the host before anything is launched; a
 *     failing check returns BKV_ERR_INVALID_ARG / _UNSUPPORTED / _WORKSPACE and
 *     leaves every output untouched.  A failed launch returns BKV_ERR_CUDA.
 *     No exception, abort or exit crosses this interface.  For tests of these
 *     paths, a non-empty environment variable BKV_INJECT_LAUNCH_FAILURE (not
 *     "0"), set before the library's first launch, makes every kernel launch
 *     fail with BKV_ERR_CUDA before anything is enqueued.
 *   - Layouts are dense and row-major.  A cache tensor is
 *     [n_layers][n_kv_heads][capacity][head_dim]; query tensors are
 *     [n_layers][n_q_heads][rows][head_dim] in the cache's dtype.  Every base
 *     pointer must be 16-byte aligned and head_dim * sizeof(dtype) must be a
 *     multiple of 16.
 *   - Supported: bf16 (the tensor-core path) with head_dim 128, and f32 (a
 *     SIMT path for small correctness workloads) with head_dim <= 128 and a
 *     multiple of 4.  bkv_compact copies bytes and accepts either dtype.
 *   - Accuracy: products of the stored values are summed in float32; exps use
 *     the hardware ex2 approximation or a cubic on the FMA pipe (relative
 *     error below 1e-4).  Scores agree with the float64 definition above to
 *     1e-6 + 1e-3 * |s| per key; the kept positions agree except where a
 *     score lies within that tolerance of the K-th; compaction is byte-exact;
 *     each FPS pick is within 1e-5 of the farthest cosine distance.
 */
#ifndef BKV_H_
#define BKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BKV_OK = 0,
  BKV_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, overlap */
  BKV_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype, head_dim) */
  BKV_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  BKV_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
  BKV_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up */
  BKV_ERR_DEVICE_ASSERT = 6  /* a device-side consistency check failed */
} bkv_status;

typedef enum { BKV_F32 = 0, BKV_BF16 = 1 } bkv_dtype;

/* How the per-row softmax probabilities p_oj of a KV head's observation rows
 * become one score per key (Table 2 of the BeaconKV page compares the two):
 *   BKV_AGG_MAX   s_j = max over the rows o of p_oj   (the method's choice)
 *   BKV_AGG_MEAN  s_j = mean over the rows o of p_oj  (the ablation) */
typedef enum { BKV_AGG_MAX = 0, BKV_AGG_MEAN = 1 } bkv_aggregate;

/* Geometry shared by a KV cache and the query tensors that go with it. */
typedef struct {
  int32_t n_layers;
  int32_t n_q_heads;   /* multiple of n_kv_heads (GQA group G = q / kv) */
  int32_t n_kv_heads;
  int32_t head_dim;
  int64_t capacity;    /* rows allocated per (layer, KV head) */
  int32_t dtype;       /* bkv_dtype */
} bkv_cache_desc;

/* Bytes of workspace that any entry point below needs for these sizes
 * (cache length L, R recent queries, M beacon slots, window W, budget K).
 * Returns 0 for invalid arguments.  Host only; no CUDA call. */
size_t bkv_workspace_size(const bkv_cache_desc *desc, int64_t L, int32_t R,
                          int32_t M, int32_t W, int64_t K);

/* Attention-based scores with max aggregation (Fig. 5(b)/(c), Table 2 "Max").
 *   k         device, cache keys [Ly][Hkv][capacity][d]; rows 0..L-1 are used
 *   recent_q  device, [Ly][Hq][R][d]
 *   beacons   device, [Ly][Hq][M][d]; rows 0..n_beacons-1 are used
 *   scale     logit scale; 0 means 1/sqrt(head_dim)
 *   scores    device out, f32 [Ly][Hkv][L]: s[j] = max over the KV head's
 *             G*(R+n_beacons) observation rows of that row's softmax at j
 * Requires 1 <= L <= capacity, R >= 0, 0 <= n_beacons <= M, R+n_beacons >= 1. */
bkv_status bkv_score(const bkv_cache_desc *desc, const void *k, int64_t L,
                     const void *recent_q, int32_t R, const void *beacons,
                     int32_t n_beacons, int32_t M, float scale, float *scores,
                     void *workspace, size_t workspace_bytes, void *stream);

/* The same scores with mean aggregation (Table 2 "Mean"): arguments, layout
 * and requirements as bkv_score, and
 *   scores    device out, f32 [Ly][Hkv][L]: s[j] = the mean over the KV
 *             head's G*(R+n_beacons) observation rows of that row's softmax
 *             at j (each row's softmax sums to 1 over j, so s sums to 1). */
bkv_status bkv_score_mean(const bkv_cache_desc *desc, const void *k, int64_t L,
                          const void *recent_q, int32_t R, const void *beacons,
                          int32_t n_beacons, int32_t M, float scale, float *scores,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Top-K budget selection (Fig. 5(c); Table 1 "maximum KV cache budget").
 *   scores  device, f32 [n_rows][L] (any finite values)
 *   idx     device out, int32 [n_rows][min(K, L)]: for every row the positions
 *           of the min(K, L) largest scores, ties to the lower position,
 *           listed in ascending order.
 * Requires n_rows >= 1, L >= 1, K >= 1. */
bkv_status bkv_select_topk(const float *scores, int32_t n_rows, int64_t L,
                           int64_t K, int32_t *idx, void *workspace,
                           size_t workspace_bytes, void *stream);

/* Compaction (eviction of the unselected KV pairs; abstract, Fig. 5(a)).
 * For every (layer, KV head) r and i < n_keep:
 *   k_dst[r][i][:] = k_src[r][idx[r][i]][:],  v_dst likewise (byte copies).
 *   src/dst   geometry of the source and destination caches: same layers,
 *             heads, head_dim and dtype; dst->capacity >= n_keep
 *   idx       device, int32 [Ly*Hkv][n_keep], each in [0, src->capacity); a
 *             position outside that range is not read: its destination row is
 *             left as it was and BKV_ERR_DEVICE_ASSERT is reported by
 *             bkv_read_device_status
 * The destination must not overlap the source.  Either pair (k_src, k_dst) or
 * (v_src, v_dst) may be NULL/NULL to copy only the other. */
bkv_status bkv_compact(const bkv_cache_desc *src, const void *k_src,
                       const void *v_src, const int32_t *idx, int64_t n_keep,
                       const bkv_cache_desc *dst, void *k_dst, void *v_dst,
                       void *stream);

/* Compaction in place: the same result as bkv_compact with the cache as both
 * source and destination, without a second cache (an ordered, chunked gather
 * within one buffer; the BeaconKV page evicts rows, Fig. 5(a), but says
 * nothing of buffers).  For
 * every (layer, KV head) r and i < n_keep, in increasing i:
 *   k[r][i][:] = k[r][idx[r][i]][:],  v likewise.
 *   idx  device, int32 [Ly*Hkv][n_keep]; every idx[r][i] must satisfy
 *        i <= idx[r][i] < capacity, which any ascending list of distinct
 *        positions does (bkv_select_topk's output, for one).  A row breaking
 *        this is skipped and reported as BKV_ERR_DEVICE_ASSERT by
 *        bkv_read_device_status; rows already in place are not copied.
 *   v may be NULL to compact only the keys.  Rows are at most 16 KB
 *   (BKV_ERR_UNSUPPORTED past that).
 * Requires 0 <= n_keep <= capacity. */
bkv_status bkv_compact_inplace(const bkv_cache_desc *desc, void *k, void *v,
                               const int32_t *idx, int64_t n_keep, void *stream);

/* Continual farthest-point sampling of the beacon queries (Fig. 7).
 * For every (layer, query head): the union U = [beacons_in rows
 * 0..n_beacons_in-1; window rows 0..W-1 (oldest first)] is sampled greedily in
 * cosine distance, seeded with U[0] and breaking ties to the lowest union
 * index; the min(M, n_beacons_in + W) picked rows are written, raw and in pick
 * order, to beacons_out[l][h][0..].  Slots past that count are left as they are.
 *   beacons_in  device, [Ly][Hq][M][d];  window device, [Ly][Hq][W][d]
 *   beacons_out device, [Ly][Hq][M][d]; must not overlap beacons_in or window
 *   n_beacons_out  host out (optional): min(M, n_beacons_in + W)
 *   workspace   device, 16-byte aligned, at least
 *               bkv_workspace_size(desc, 1, 0, M, W, 1) bytes: the counter that
 *               hands out query heads to the GPU's CTAs (16 bytes, reset at the
 *               start of every call on `stream`), plus the per-point distance
 *               arrays of unions too large for shared memory
 * Requires M >= 1, 0 <= n_beacons_in <= M, W >= 0, n_beacons_in + W >= 1. */
bkv_status bkv_update_beacons(const bkv_cache_desc *desc,
                              const void *beacons_in, int32_t n_beacons_in,
                              int32_t M, const void *window, int32_t W,
                              void *beacons_out, int32_t *n_beacons_out,
                              void *workspace, size_t workspace_bytes,
                              void *stream);

/* Arguments of one whole compression step. */
typedef struct {
  bkv_cache_desc cache;        /* source cache and query geometry */
  const void *k, *v;           /* device, source cache, rows 0..L-1 valid */
  int64_t L;                   /* current cache length */
  int64_t K;                   /* budget: rows kept */
  const void *recent_q;        /* device, [Ly][Hq][R][d] */
  int32_t R;
  const void *beacons_in;      /* device, [Ly][Hq][M][d] */
  int32_t n_beacons_in;
  int32_t M;
  const void *window;          /* device, [Ly][Hq][W][d]; NULL or W == 0: keep beacons */
  int32_t W;
  void *beacons_out;           /* device, [Ly][Hq][M][d]; required when W > 0 */
  float scale;                 /* 0: 1/sqrt(head_dim) */
  bkv_cache_desc dst_cache;    /* destination geometry, capacity >= min(K, L) */
  void *k_dst, *v_dst;         /* device, destination cache; k_dst == k and
                                  v_dst == v (with dst_cache == cache)
                                  compacts in place */
  float *scores_out;           /* device, optional f32 [Ly][Hkv][L] */
  int32_t *idx_out;            /* device, optional int32 [Ly][Hkv][min(K, L)] */
  void *workspace;
  size_t workspace_bytes;
  void *stream;
  /* Optional tracing: NULL, or BKV_STEP_EVENTS cudaEvent_t handles (as void*)
   * that the step records on `stream` at its phase boundaries: [0] start,
   * [1] after Continual FPS, [2] after the row statistics, [3] after the
   * aggregation, [4] after top-K, [5] after compaction.  A skipped phase
   * records its event at once. */
  void **phase_events;
  int32_t aggregate;           /* bkv_aggregate; 0 (a zeroed struct) = max */
  /* Optional decode-side query ring (Fig. 7's "newest window" as the decode
   * loop keeps it): NULL, or device [Ly][Hq][ring_cap][d] in which the decode
   * step writes its t-th query (t = 0, 1, ...) of every query head to slot
   * t mod ring_cap.  With a ring, recent_q and window must be NULL: the R
   * recent queries are the ring's newest R rows and the window its newest W
   * rows (oldest first), read in place where the ring wraps.
   * Requires W <= ring_cap, R <= ring_cap, ring_pos >= max(W, R). */
  const void *query_ring;
  int64_t ring_cap;            /* slots per query head */
  int64_t ring_pos;            /* queries written so far (the next slot is ring_pos mod ring_cap) */
  /* Optional second stream (cudaStream_t as void*, NULL: none).  With it, the
   * aggregation runs in head batches on `stream` and each batch's top-K and
   * compaction run on aux_stream while the next batch is aggregated; the step
   * still starts after the work already on `stream` and everything it does is
   * finished before anything enqueued on `stream` after it.  aux_stream must
   * not be `stream`.  Applies to bf16 steps that evict rows; with it, phase
   * event [3] marks the end of the last batch's aggregation and [4] and [5]
   * the end of the selections and compactions still running after it. */
  void *aux_stream;
} bkv_step_args;

#define BKV_STEP_EVENTS 6

/* The periodic compression step: when W > 0, Continual FPS updates the
 * beacons first (a reading: the page only shows the beacons being used for
 * scoring); then scoring with the (updated) beacons, aggregated as
 * args->aggregate says, top-K and compaction into the destination cache.
 * When K >= L every row is kept and copied.  scores_out holds bkv_score's
 * (max) or bkv_score_mean's (mean) scores; an aggregate other than the two
 * values of bkv_aggregate is BKV_ERR_INVALID_ARG.
 *   n_beacons_out  host out (optional): beacons valid after the step
 *   new_len        host out (optional): min(K, L) */
bkv_status bkv_compress_step(const bkv_step_args *args, int32_t *n_beacons_out,
                             int64_t *new_len);

/* Scoring without a caller workspace.  The paper has no counterpart: this is
 * an interface addition for callers that cannot allocate device memory where
 * they score -- for example code running inside another runtime's execute
 * callback that hands over only the tensors it asked for, or a serving loop
 * that must not allocate after start-up because a pool allocator has reserved
 * the device's memory.  Same arguments and results as bkv_score, without the
 * workspace: the scratch is one array of BKV_SCORE_NOALLOC_SCRATCH_BYTES
 * (32 MiB) compiled into libbkv.so, which every GPU that loads the library
 * holds until the process exits.
 *   - The first call on each device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress); make that first call before
 *     any stream capture.  The address is looked up again when the device's
 *     context has changed since (after a cudaDeviceReset, for one), so make
 *     the first call after a reset before any capture as well.
 *   - A problem whose scratch does not fit the array (at most
 *     bkv_workspace_size(desc, L, R, n_beacons, 0, 1) bytes are needed) is
 *     rejected with BKV_ERR_WORKSPACE before anything is launched.
 *   - Every call uses the same array and leaves its contents behind.  Calls
 *     whose kernels can overlap on the GPU (other streams, other host threads)
 *     race on it and produce wrong scores: order them on one stream or with
 *     events.  Nothing in the array needs to start at zero.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine. */
#define BKV_SCORE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
bkv_status bkv_score_noalloc(const bkv_cache_desc *desc, const void *k,
                             int64_t L, const void *recent_q, int32_t R,
                             const void *beacons, int32_t n_beacons, int32_t M,
                             float scale, float *scores, void *stream);

/* Device-side status.  Kernels never trap: a bounded wait that runs out or a
 * failed consistency check records BKV_ERR_TIMEOUT / BKV_ERR_DEVICE_ASSERT in
 * a status word of the library instead.  This call synchronises `stream`,
 * returns the first code recorded since the previous call (BKV_OK if none),
 * clears it, and stores an internal location tag in *where_out (optional). */
bkv_status bkv_read_device_status(void *stream, int32_t *where_out);

/* Diagnostic of the bounded device-side waits; the paper has no counterpart.
 * Launches one warp on `stream` that waits -- through the same bounded wait
 * routine the kernels use -- on an mbarrier that nothing ever arrives on,
 * with a wall-clock limit of limit_ns instead of the kernels' 0.5 s.  The
 * wait gives up, records BKV_ERR_TIMEOUT with location tag 901 for
 * bkv_read_device_status, and the kernel exits normally: no TMA load or MMA
 * is in flight, so nothing is left behind and later calls run as usual.
 *   limit_ns  1000 .. 100000000 (1 us .. 100 ms)
 *   outcome   device, int32, 4-byte aligned: 0 when the wait gave up, 1 if
 *             it was satisfied (it cannot be)
 * Errors: BKV_ERR_INVALID_ARG for a limit out of range or a null or
 * misaligned outcome (nothing launched); BKV_ERR_CUDA if the launch fails. */
bkv_status bkv_selftest_wait_timeout(int64_t limit_ns, int32_t *outcome, void *stream);

/* Static text for a status code. */
const char *bkv_status_string(bkv_status status);

#ifdef __cplusplus
}
#endif

#endif /* BKV_H_ */
