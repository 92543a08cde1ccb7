/*
 * bkv_oracle.c -- float64 CPU oracle for the BeaconKV KV-cache compression step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: it is used by the tests, by the smoke check and by the benchmark's
 * CPU-baseline leg.  It shares no code, header, table or constant with the CUDA
 * library and includes nothing from it.
 *
 * Source of the definitions: "BeaconKV: Key-Value Cache Compression Guided by
 * Beacon Queries for Efficient Large Reasoning Model Inference" (Kim, Kim, Shim,
 * Choi), abstract and Figures 5 and 7, Table 2.  The page gives the step only in
 * words:
 *   - Fig. 5(b): attention-based scores are computed from beacon queries and
 *     recent queries;
 *   - Fig. 5(c) and Table 2: top-K selection after *max* aggregation of those
 *     scores, taken over heads and queries alike;
 *   - abstract / Fig. 5(a): the unselected KV pairs are evicted;
 *   - Fig. 7: beacons are kept by Continual farthest-point sampling.
 * The attention-based score is read as softmax(q.k / sqrt(d)) over every cached
 * key, and FPS uses cosine distance, as the problem statement of this library
 * fixes.  Each function below is the plain definition, written with loops, in
 * double precision, with no blocking, fusion or reordering.
 *
 * Parity status: every function here is pinned by tests/test_oracle.py
 * (closed forms, invariants, brute force on tiny inputs, library routines).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Step 1 -- logits.  x[o][j] = scale * sum_t q[o][t] * k[j][t]               */
/* (Fig. 5(b): attention-based scores of the observation queries.)           */
/* q: [n_obs][d], k: [L][d], x: [n_obs][L], all row-major.                   */
/* ------------------------------------------------------------------------- */
void oracle_logits(int64_t n_obs, int64_t L, int64_t d, const double *q,
                   const double *k, double scale, double *x) {
  for (int64_t o = 0; o < n_obs; ++o) {
    for (int64_t j = 0; j < L; ++j) {
      double acc = 0.0;
      for (int64_t t = 0; t < d; ++t) acc += q[o * d + t] * k[j * d + t];
      x[o * L + j] = scale * acc;
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Step 2 -- softmax normaliser of each observation row over all L keys.      */
/* c[o] = m_o + log(sum_j exp(x[o][j] - m_o)),  m_o = max_j x[o][j],          */
/* so that softmax_o(j) = exp(x[o][j] - c[o]).                               */
/* ------------------------------------------------------------------------- */
void oracle_row_normalizer(int64_t n_obs, int64_t L, const double *x,
                           double *c) {
  for (int64_t o = 0; o < n_obs; ++o) {
    const double *row = x + o * L;
    double m = -INFINITY;
    for (int64_t j = 0; j < L; ++j)
      if (row[j] > m) m = row[j];
    double sum = 0.0;
    for (int64_t j = 0; j < L; ++j) sum += exp(row[j] - m);
    c[o] = m + log(sum);
  }
}

/* ------------------------------------------------------------------------- */
/* Step 3 -- max aggregation (Fig. 5(c); Table 2 "Max", over heads and        */
/* queries alike).  s[j] = max_o softmax_o(j) = max_o exp(x[o][j] - c[o]).   */
/* ------------------------------------------------------------------------- */
void oracle_max_aggregate(int64_t n_obs, int64_t L, const double *x,
                          const double *c, double *s) {
  for (int64_t j = 0; j < L; ++j) {
    double best = 0.0;
    for (int64_t o = 0; o < n_obs; ++o) {
      double p = exp(x[o * L + j] - c[o]);
      if (p > best) best = p;
    }
    s[j] = best;
  }
}

/* Table 2's ablation alternative: mean over the observation rows.           */
void oracle_mean_aggregate(int64_t n_obs, int64_t L, const double *x,
                           const double *c, double *s) {
  for (int64_t j = 0; j < L; ++j) {
    double sum = 0.0;
    for (int64_t o = 0; o < n_obs; ++o) sum += exp(x[o * L + j] - c[o]);
    s[j] = sum / (double)n_obs;
  }
}

/* ------------------------------------------------------------------------- */
/* Step 4 -- top-K budget selection (Fig. 5(c); Table 1 "maximum KV cache    */
/* budget").  Order keys by (score descending, position ascending), keep the */
/* first min(K, L), and emit the kept positions in ascending order.          */
/* ------------------------------------------------------------------------- */
typedef struct {
  double s;
  int32_t j;
} oracle_scored_pos;

static int oracle_cmp_score_desc(const void *a, const void *b) {
  const oracle_scored_pos *x = (const oracle_scored_pos *)a;
  const oracle_scored_pos *y = (const oracle_scored_pos *)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int oracle_cmp_int_asc(const void *a, const void *b) {
  int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

int64_t oracle_select_topk(int64_t L, const double *s, int64_t K,
                           int32_t *idx) {
  int64_t keep = K < L ? K : L;
  if (keep <= 0) return 0;
  oracle_scored_pos *all =
      (oracle_scored_pos *)malloc((size_t)L * sizeof(oracle_scored_pos));
  if (!all) return -1;
  for (int64_t j = 0; j < L; ++j) {
    all[j].s = s[j];
    all[j].j = (int32_t)j;
  }
  qsort(all, (size_t)L, sizeof(oracle_scored_pos), oracle_cmp_score_desc);
  for (int64_t i = 0; i < keep; ++i) idx[i] = all[i].j;
  qsort(idx, (size_t)keep, sizeof(int32_t), oracle_cmp_int_asc);
  free(all);
  return keep;
}

/* ------------------------------------------------------------------------- */
/* Step 5 -- compaction (eviction of the unselected KV pairs, Fig. 5(a)).    */
/* dst row i is a byte copy of src row idx[i].                               */
/* ------------------------------------------------------------------------- */
void oracle_compact(int64_t row_bytes, const uint8_t *src, const int32_t *idx,
                    int64_t n, uint8_t *dst) {
  for (int64_t i = 0; i < n; ++i)
    memcpy(dst + i * row_bytes, src + (int64_t)idx[i] * row_bytes,
           (size_t)row_bytes);
}

/* ------------------------------------------------------------------------- */
/* Step 6 -- Continual farthest-point sampling in cosine distance (Fig. 7).  */
/* U: [n][d] = the current beacons in stored order, then the newest window   */
/* of queries from oldest to newest.  Cosine distance                        */
/*     dist(a, b) = 1 - (u_a . u_b) / (|u_a| |u_b|), clamped to [0, 2],      */
/* and 1 when either vector has zero norm.  The seed is U[0]; each further   */
/* pick is the unselected point whose distance to the selected set is        */
/* largest, ties to the lowest index.  Writes min(M, n) indices into U, in   */
/* selection order, and returns that count.                                  */
/* ------------------------------------------------------------------------- */
static double oracle_cosine_distance(int64_t d, const double *a, double na,
                                     const double *b, double nb) {
  if (na == 0.0 || nb == 0.0) return 1.0;
  double dot = 0.0;
  for (int64_t t = 0; t < d; ++t) dot += a[t] * b[t];
  double dist = 1.0 - dot / (na * nb);
  if (dist < 0.0) dist = 0.0;
  if (dist > 2.0) dist = 2.0;
  return dist;
}

static void oracle_norms(int64_t n, int64_t d, const double *U, double *nrm) {
  for (int64_t i = 0; i < n; ++i) {
    double ss = 0.0;
    for (int64_t t = 0; t < d; ++t) ss += U[i * d + t] * U[i * d + t];
    nrm[i] = sqrt(ss);
  }
}

int64_t oracle_fps(int64_t n, int64_t d, const double *U, int64_t M,
                   int32_t *sel) {
  int64_t m = M < n ? M : n;
  if (m <= 0) return 0;
  double *nrm = (double *)malloc((size_t)n * sizeof(double));
  double *dist = (double *)malloc((size_t)n * sizeof(double));
  char *chosen = (char *)calloc((size_t)n, 1);
  if (!nrm || !dist || !chosen) {
    free(nrm); free(dist); free(chosen);
    return -1;
  }
  oracle_norms(n, d, U, nrm);
  sel[0] = 0;
  chosen[0] = 1;
  for (int64_t i = 0; i < n; ++i)
    dist[i] = oracle_cosine_distance(d, U + i * d, nrm[i], U, nrm[0]);
  for (int64_t t = 1; t < m; ++t) {
    int64_t best = -1;
    for (int64_t i = 0; i < n; ++i) {
      if (chosen[i]) continue;
      if (best < 0 || dist[i] > dist[best]) best = i;
    }
    sel[t] = (int32_t)best;
    chosen[best] = 1;
    for (int64_t i = 0; i < n; ++i) {
      double db = oracle_cosine_distance(d, U + i * d, nrm[i], U + best * d,
                                         nrm[best]);
      if (db < dist[i]) dist[i] = db;
    }
  }
  free(nrm); free(dist); free(chosen);
  return m;
}

/* Guided replay of FPS for comparing another implementation's picks when    */
/* the data has near-ties.  It runs the same algorithm as oracle_fps, but at */
/* step t it takes picks[t] instead of its own argmax, after checking that   */
/* picks[t] is unselected, that picks[0] is the seed 0, and that its         */
/* distance lies within tol of the largest distance.  Returns -1 when every  */
/* pick is acceptable, else the first step that is not; *gap receives the    */
/* largest shortfall (max distance minus the pick's distance) seen.          */
int64_t oracle_fps_replay(int64_t n, int64_t d, const double *U, int64_t m,
                          const int32_t *picks, double tol, double *gap) {
  *gap = 0.0;
  if (m <= 0) return -1;
  if (picks[0] != 0) return 0;
  double *nrm = (double *)malloc((size_t)n * sizeof(double));
  double *dist = (double *)malloc((size_t)n * sizeof(double));
  char *chosen = (char *)calloc((size_t)n, 1);
  if (!nrm || !dist || !chosen) {
    free(nrm); free(dist); free(chosen);
    return -2;
  }
  int64_t bad = -1;
  oracle_norms(n, d, U, nrm);
  chosen[0] = 1;
  for (int64_t i = 0; i < n; ++i)
    dist[i] = oracle_cosine_distance(d, U + i * d, nrm[i], U, nrm[0]);
  for (int64_t t = 1; t < m; ++t) {
    double dmax = -1.0;
    for (int64_t i = 0; i < n; ++i)
      if (!chosen[i] && dist[i] > dmax) dmax = dist[i];
    int64_t p = picks[t];
    if (p < 0 || p >= n || chosen[p]) { bad = t; break; }
    double shortfall = dmax - dist[p];
    if (shortfall > *gap) *gap = shortfall;
    if (shortfall > tol) { bad = t; break; }
    chosen[p] = 1;
    for (int64_t i = 0; i < n; ++i) {
      double dp = oracle_cosine_distance(d, U + i * d, nrm[i], U + p * d,
                                         nrm[p]);
      if (dp < dist[i]) dist[i] = dp;
    }
  }
  free(nrm); free(dist); free(chosen);
  return bad;
}
