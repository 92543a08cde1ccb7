// bkv_internal.h -- geometry shared by the host layer and the kernels of
// libbkv.so, and the launchers each kernel file exports.  Not installed; the
// public interface is include/bkv.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "bkv.h"

namespace bkv {

constexpr size_t kAlign = 256;  // alignment of every workspace section

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// One scoring problem: all (layer, KV head) pairs of a cache, each with its
// observation set of G * (R + nb) query rows (the R recent queries and the
// first nb beacons of each of the G query heads of the group).
struct ScoreGeom {
  int n_layers, n_q_heads, n_kv_heads, head_dim, group;
  long long cap;        // rows allocated per (layer, KV head)
  long long L;          // rows scored
  int R, nb, M;         // recent rows, valid beacons, beacon slots
  // recent row i of a query head is row (recent_start + i) mod recent_cap of
  // that head's [recent_cap][d] block: a dense [R][d] block (cap R, start 0)
  // or the newest R rows of a decode-side query ring
  long long recent_cap, recent_start;
  int n_obs;            // observation rows per KV head
  int n_obs_pad;        // n_obs rounded up to the row-statistics block (128)
  int n_groups;         // observation groups of the aggregation pass
  int rows_per_group;   // rows per group, a multiple of 16, at most 512
  float scale;          // logit scale
  __host__ __device__ int n_heads() const { return n_layers * n_kv_heads; }
};

// Fill the derived fields of a ScoreGeom (n_obs, padding, groups).
void finish_score_geom(ScoreGeom *g);

// The grouping of the tensor-core mean aggregation: groups of at most 256
// observation rows (the max aggregation's are up to 512).
inline ScoreGeom mean_grouping(const ScoreGeom &g) {
  ScoreGeom m = g;
  m.n_groups = (g.n_obs + 255) / 256;
  const int per = (g.n_obs + m.n_groups - 1) / m.n_groups;
  m.rows_per_group = (per + 15) / 16 * 16;
  return m;
}

// Workspace sections of the scoring passes.
struct ScoreWorkspace {
  float *c;      // [n_heads][n_obs_pad]  row normalisers (natural log units)
  float *ypart;  // max aggregation (tensor cores): [n_heads][L] order keys of
                 // max_o (x - c), every group merged; otherwise [groups][n_heads][L]
                 // per group of rows: max of (x - c) or sum of exp(x - c) (mean);
                 // sized for the mean's (finer) grouping
};
size_t score_workspace_bytes(const ScoreGeom &g);
ScoreWorkspace carve_score_workspace(const ScoreGeom &g, void *ws);

// ---- score_tc.cu: bf16, head_dim 128, tcgen05 tensor cores
bkv_status launch_score_rowstats_tc(const ScoreGeom &g, const void *k, const void *recent,
                                    const void *beacons, float *c, cudaStream_t stream);
// heads [head0, head0 + head_count) only (head_count < 0: through the last head)
bkv_status launch_score_colmax_tc(const ScoreGeom &g, const void *k, const void *recent,
                                  const void *beacons, const float *c, float *ypart, bool mean,
                                  cudaStream_t stream, int head0 = 0, int head_count = -1);

// ---- score_simt.cu: f32, head_dim <= 128 (multiple of 4), CUDA cores
bkv_status launch_score_rowstats_simt(const ScoreGeom &g, const float *k, const float *recent,
                                      const float *beacons, float *c, cudaStream_t stream);
bkv_status launch_score_colmax_simt(const ScoreGeom &g, const float *k, const float *recent,
                                    const float *beacons, const float *c, float *ypart, bool mean,
                                    cudaStream_t stream);

// ---- select_topk.cu
// Selection input: per row r and position j, with v_p = src[p * part_stride +
// r * L + j] for p < n_parts, the key is
//   mean == 0:  max_p v_p                 (log-domain partial maxima)
//   mean != 0:  inv_count * sum_p v_p     (partial sums of probabilities)
// When s_out is given, the score is also written to s_out[r * L + j]: exp(key)
// for the max form, the key itself for the mean form.
struct SelectInput {
  const float *src;
  int n_parts;
  size_t part_stride;
  int mean;
  float inv_count;
  int keys = 0;  // src holds one part of order keys (order_key.cuh) as 32-bit words
};
size_t select_workspace_bytes(int n_rows, long long L);
bkv_status launch_select_topk(const SelectInput &in, int n_rows, long long L, long long K,
                              int32_t *idx, float *s_out, void *ws, size_t ws_bytes,
                              cudaStream_t stream);
// s[r][j] = the score of SelectInput's comment, for every row and position.
bkv_status launch_finalize_scores(const SelectInput &in, int n_rows, long long L, float *s,
                                  cudaStream_t stream);
// idx[r][i] = i for i < n.
bkv_status launch_iota_rows(int32_t *idx, int n_rows, long long n, cudaStream_t stream);

// ---- compact.cu
struct CompactArgs {
  const uint8_t *k_src, *v_src;
  uint8_t *k_dst, *v_dst;
  const int32_t *idx;        // [n_heads][n_keep]; NULL = identity
  int n_heads;
  long long n_keep;
  long long src_cap, dst_cap;  // rows per head
  int row_bytes;               // multiple of 16
};
bkv_status launch_compact(const CompactArgs &a, cudaStream_t stream);
// In place: k_dst/v_dst (== the source) with dst_cap; idx[i] >= i required.
bkv_status launch_compact_inplace(const CompactArgs &a, cudaStream_t stream);

// ---- fps.cu
struct FpsGeom {
  int n_layers, n_q_heads, head_dim, dtype;
  int nb_in, M, W;
  int n_pick;  // min(M, nb_in + W)
  // window row w of a query head is row (w_start + w) mod w_cap of that
  // head's [w_cap][d] block: a dense [W][d] block (cap W, start 0) or the
  // newest W rows of a decode-side query ring
  long long w_cap, w_start;
};
size_t fps_workspace_bytes(const FpsGeom &g);
bool fps_supported(const FpsGeom &g);
// fps_tc.cu: bf16, head_dim 128.  A union whose distance array does not fit
// in shared memory keeps it in the workspace: fps_tc_workspace_bytes (0 when
// it fits) covers one slice per CTA of the persistent grid.
bool fps_tc_supported(const FpsGeom &g);
size_t fps_tc_workspace_bytes(const FpsGeom &g);
bkv_status launch_fps_tc(const FpsGeom &g, const void *beacons_in, const void *window,
                         void *beacons_out, void *ws, size_t ws_bytes, cudaStream_t stream);
bkv_status launch_fps(const FpsGeom &g, const void *beacons_in, const void *window,
                      void *beacons_out, void *ws, size_t ws_bytes, cudaStream_t stream);

// Fault injection for the host-side error paths: when the environment
// variable BKV_INJECT_LAUNCH_FAILURE is set to a non-empty value other than
// "0" when the library first checks it, every kernel launcher returns
// BKV_ERR_CUDA instead of launching, as if the launch had failed, so that
// tests can check that the entry points report it and leave their outputs
// untouched.  Read once per process.
bool injected_launch_failure();

// Raise a kernel's dynamic shared-memory limit once per device (the attribute
// is per device context).  Returns false if the CUDA call fails.
template <typename Kernel>
bool ensure_smem_limit(Kernel kernel, int bytes, int *done_flags /* [64] */) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (__atomic_load_n(&done_flags[dev], __ATOMIC_ACQUIRE)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  __atomic_store_n(&done_flags[dev], 1, __ATOMIC_RELEASE);
  return true;
}

// ---- per-file device status accessors (bkv_device_status.cuh)
int take_status_score_tc(cudaStream_t, int *);
int take_status_select(cudaStream_t, int *);
int take_status_fps_tc(cudaStream_t, int *);
int take_status_compact(cudaStream_t, int *);
int take_status_fps(cudaStream_t, int *);
int take_status_selftest(cudaStream_t, int *);

}  // namespace bkv
