/*
 * lf_oracle.c -- the CPU oracle for Longformer self-attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is built into its own shared library
 * (oracle/liblf_oracle.so) and is used by tests/, by __graft_entry__.smoke()
 * and by the cpu_baseline / reference arm of bench.py.  The product (the CUDA
 * library under sparse_sliding_window_b200/csrc) never links, loads or calls
 * it, and it shares no code, header, table or constant with that library.
 *
 * Plain, slow, obviously correct: every quantity is computed in double
 * precision, one attention head at a time, straight from the definitions.
 * The attention pattern of a head is MATERIALISED as an explicit n x n bit
 * matrix A (bit (i,j) set <=> query i attends key j) before any arithmetic,
 * and every later step only walks the set bits of A.
 *
 * Sources (page title, section):
 *  - "Longformer：处理长文档的Transformer模型" (segmentfault summary of the
 *    paper), sections 滑动窗口 (sliding window), 扩张滑动窗口 (dilated sliding
 *    window: gaps of size d), 全局注意力 (symmetric global attention),
 *    全局注意力的线性投影 (two projection sets Qs,Ks,Vs / Qg,Kg,Vg),
 *    实现 (only a fixed number of diagonals of QK^T), and its autoregressive
 *    language-modelling paragraph (causal, dilated windows).
 *  - "Longformer" (ultralytics glossary, de/ko), section "So funktioniert die
 *    Aufmerksamkeit bei Longformer": 256 tokens on each side of every token,
 *    the pair-count example |i-j| <= window/2 with token 0 global (a union).
 *  - "Longformer" (gittoolsai copy of the allenai README), section 使用方法 /
 *    运行模型: attention_mask codes 0 = no attention, 1 = local, 2 = global.
 *  The pages never print the attention formula.  The scaled dot-product
 *  softmax(s) with s = scale * <q, k>, scale = 1/sqrt(head_dim), is the
 *  standard reading this library fixes for both local and global scores.
 *
 * Readings where the pages leave a step open (each also listed in the design
 * notes of the repository):
 *  R1  r is the one-sided window: keys j = i + k*d with |k| <= r (window
 *      w = 2r, plus the token itself), as in the |i-j| <= window//2 example.
 *  R2  dilation d: the window keeps every d-th position (gaps of size d).
 *  R3  causal: only k <= 0.
 *  R4  positions outside [0, n) do not exist (no wrap-around).
 *  R5  a global key that is also inside a row's window is attended ONCE
 *      (union of the window set and the global set, as in the example).
 *  R6  global rows use Qg/Kg/Vg over every valid key; local rows use
 *      Qs/Ks/Vs for both their window keys and their global keys.
 *  R7  mask-0 tokens are never keys; as queries their output is 0 and their
 *      log-normaliser is -inf; their gradients are 0.
 *  R8  causal together with global tokens is not defined here (rejected).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_MEM 2
#define ORC_ERR_UNSUPPORTED 3

/* ------------------------------------------------------------------------ */
/* Pattern: the literal per-pair rule (R1..R8).                              */
/* ------------------------------------------------------------------------ */

/* Does query i attend key j?  m[] is the head's sequence mask (0/1/2). */
static int orc_rule(int n, int r, int d, int causal, const int32_t *m, int i,
                    int j) {
  (void)n;
  if (m[i] == 0 || m[j] == 0) return 0;   /* R7: 0 = no attention          */
  if (m[i] == 2) return 1;                /* global token sees every token */
  if (m[j] == 2) return 1;                /* every token sees global token */
  int dist = j - i;                       /* window, R1..R3                */
  if (dist % d != 0) return 0;
  int k = dist / d;
  if (k < -r || k > r) return 0;
  if (causal && k > 0) return 0;
  return 1;
}

static int orc_check(int n, int r, int d, int causal, const int32_t *m) {
  if (n < 0 || r < 0 || d < 1 || m == NULL) return ORC_ERR_ARG;
  for (int i = 0; i < n; i++) {
    if (m[i] < 0 || m[i] > 2) return ORC_ERR_ARG;
    if (causal && m[i] == 2) return ORC_ERR_UNSUPPORTED; /* R8 */
  }
  return ORC_OK;
}

typedef struct {
  int n;
  int words; /* 64-bit words per row */
  uint64_t *bits;
} orc_pattern;

static int orc_pattern_build(orc_pattern *A, int n, int r, int d, int causal,
                             const int32_t *m) {
  A->n = n;
  A->words = (n + 63) / 64;
  size_t total = (size_t)n * (size_t)A->words;
  A->bits = (uint64_t *)calloc(total ? total : 1, sizeof(uint64_t));
  if (!A->bits) return ORC_ERR_MEM;
#pragma omp parallel for schedule(dynamic, 16)
  for (int i = 0; i < n; i++) {
    uint64_t *row = A->bits + (size_t)i * A->words;
    for (int j = 0; j < n; j++)
      if (orc_rule(n, r, d, causal, m, i, j)) row[j >> 6] |= 1ull << (j & 63);
  }
  return ORC_OK;
}

static inline int orc_bit(const orc_pattern *A, int i, int j) {
  return (int)((A->bits[(size_t)i * A->words + (j >> 6)] >> (j & 63)) & 1ull);
}

static void orc_pattern_free(orc_pattern *A) {
  free(A->bits);
  A->bits = NULL;
}

static double orc_dot(const double *a, const double *b, int hd) {
  double s = 0.0;
  for (int c = 0; c < hd; c++) s += a[c] * b[c];
  return s;
}

/* ------------------------------------------------------------------------ */
/* Exported: pattern, counts, probabilities, forward, backward.              */
/* ------------------------------------------------------------------------ */

int lf_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Dense n x n 0/1 matrix of the pattern (out: n*n bytes, row-major). */
int lf_oracle_pattern(int n, int r, int d, int causal, const int32_t *m,
                      uint8_t *out) {
  int st = orc_check(n, r, d, causal, m);
  if (st) return st;
  orc_pattern A;
  if ((st = orc_pattern_build(&A, n, r, d, causal, m))) return st;
  for (int i = 0; i < n; i++)
    for (int j = 0; j < n; j++) out[(size_t)i * n + j] = (uint8_t)orc_bit(&A, i, j);
  orc_pattern_free(&A);
  return ORC_OK;
}

/* Number of attended (query, key) pairs of one head = popcount(A). */
int lf_oracle_count_pairs(int n, int r, int d, int causal, const int32_t *m,
                          int64_t *count) {
  int st = orc_check(n, r, d, causal, m);
  if (st) return st;
  orc_pattern A;
  if ((st = orc_pattern_build(&A, n, r, d, causal, m))) return st;
  int64_t c = 0;
  size_t total = (size_t)n * A.words;
  for (size_t w = 0; w < total; w++) c += __builtin_popcountll(A.bits[w]);
  *count = c;
  orc_pattern_free(&A);
  return ORC_OK;
}

/* Row i of the attention probabilities (p_row: n doubles; 0 where A=0). */
int lf_oracle_probs_row(int n, int hd, int r, int d, int causal, double scale,
                        const int32_t *m, const double *qs, const double *ks,
                        const double *qg, const double *kg, int i,
                        double *p_row) {
  int st = orc_check(n, r, d, causal, m);
  if (st) return st;
  if (i < 0 || i >= n || hd <= 0) return ORC_ERR_ARG;
  orc_pattern A;
  if ((st = orc_pattern_build(&A, n, r, d, causal, m))) return st;
  for (int j = 0; j < n; j++) p_row[j] = 0.0;
  const int glob = (m[i] == 2);
  const double *q = (glob ? qg : qs) + (size_t)i * hd;
  const double *k = glob ? kg : ks;
  double mx = -INFINITY;
  for (int j = 0; j < n; j++)
    if (orc_bit(&A, i, j)) {
      double s = scale * orc_dot(q, k + (size_t)j * hd, hd);
      p_row[j] = s;
      if (s > mx) mx = s;
    }
  double sum = 0.0;
  for (int j = 0; j < n; j++)
    if (orc_bit(&A, i, j)) sum += exp(p_row[j] - mx);
  for (int j = 0; j < n; j++)
    p_row[j] = orc_bit(&A, i, j) ? exp(p_row[j] - mx) / sum : 0.0;
  orc_pattern_free(&A);
  return ORC_OK;
}

/*
 * Forward of one head.  All matrices are n x hd, row-major, double.
 * o: n x hd output; lse: n log-normalisers (natural log; -inf for rows that
 * attend nothing).
 */
int lf_oracle_fwd_head(int n, int hd, int r, int d, int causal, double scale,
                       const int32_t *m, const double *qs, const double *ks,
                       const double *vs, const double *qg, const double *kg,
                       const double *vg, double *o, double *lse) {
  int st = orc_check(n, r, d, causal, m);
  if (st) return st;
  if (hd <= 0) return ORC_ERR_ARG;
  orc_pattern A;
  if ((st = orc_pattern_build(&A, n, r, d, causal, m))) return st;
#pragma omp parallel for schedule(dynamic, 8)
  for (int i = 0; i < n; i++) {
    double *oi = o + (size_t)i * hd;
    for (int c = 0; c < hd; c++) oi[c] = 0.0;
    const int glob = (m[i] == 2);
    const double *q = (glob ? qg : qs) + (size_t)i * hd;
    const double *k = glob ? kg : ks;
    const double *v = glob ? vg : vs;
    double mx = -INFINITY;
    for (int j = 0; j < n; j++)
      if (orc_bit(&A, i, j)) {
        double s = scale * orc_dot(q, k + (size_t)j * hd, hd);
        if (s > mx) mx = s;
      }
    if (mx == -INFINITY) { /* attends nothing (mask 0 row) */
      lse[i] = -INFINITY;
      continue;
    }
    double sum = 0.0;
    for (int j = 0; j < n; j++)
      if (orc_bit(&A, i, j)) {
        double e = exp(scale * orc_dot(q, k + (size_t)j * hd, hd) - mx);
        sum += e;
        const double *vj = v + (size_t)j * hd;
        for (int c = 0; c < hd; c++) oi[c] += e * vj[c];
      }
    for (int c = 0; c < hd; c++) oi[c] /= sum;
    lse[i] = mx + log(sum);
  }
  orc_pattern_free(&A);
  return ORC_OK;
}

/*
 * Backward of one head for the loss L = sum(o * dO): given dO (n x hd),
 * produce the six input gradients.  Gradients are OVERWRITTEN.
 *
 * Softmax Jacobian: with p_ij the probabilities of row i and
 * dp_ij = <dO_i, v_j>, ds_ij = p_ij * (dp_ij - sum_k p_ik dp_ik).
 * Then dq_i = scale * sum_j ds_ij k_j, dk_j = scale * sum_i ds_ij q_i,
 * dv_j = sum_i p_ij dO_i, where (q, k, v) is (Qg, Kg, Vg) for a global
 * row i and (Qs, Ks, Vs) for a local row i, and the gradient lands in the
 * matching tensor.
 *
 * Pass 1 (parallel over rows): lse_i, delta_i = sum_k p_ik dp_ik, dq_i.
 * Pass 2 (parallel over key columns j): walk column j of A, recompute
 * p_ij and ds_ij from lse_i and delta_i, accumulate dk_j and dv_j.
 */
int lf_oracle_bwd_head(int n, int hd, int r, int d, int causal, double scale,
                       const int32_t *m, const double *qs, const double *ks,
                       const double *vs, const double *qg, const double *kg,
                       const double *vg, const double *dO, double *dqs,
                       double *dks, double *dvs, double *dqg, double *dkg,
                       double *dvg) {
  int st = orc_check(n, r, d, causal, m);
  if (st) return st;
  if (hd <= 0) return ORC_ERR_ARG;
  orc_pattern A;
  if ((st = orc_pattern_build(&A, n, r, d, causal, m))) return st;
  double *lse = (double *)malloc(sizeof(double) * (size_t)(n ? n : 1));
  double *delta = (double *)malloc(sizeof(double) * (size_t)(n ? n : 1));
  if (!lse || !delta) {
    free(lse);
    free(delta);
    orc_pattern_free(&A);
    return ORC_ERR_MEM;
  }
  size_t nh = (size_t)n * hd;
  memset(dqs, 0, nh * sizeof(double));
  memset(dks, 0, nh * sizeof(double));
  memset(dvs, 0, nh * sizeof(double));
  memset(dqg, 0, nh * sizeof(double));
  memset(dkg, 0, nh * sizeof(double));
  memset(dvg, 0, nh * sizeof(double));

#pragma omp parallel for schedule(dynamic, 8)
  for (int i = 0; i < n; i++) {
    const int glob = (m[i] == 2);
    const double *q = (glob ? qg : qs) + (size_t)i * hd;
    const double *k = glob ? kg : ks;
    const double *v = glob ? vg : vs;
    const double *g = dO + (size_t)i * hd;
    double mx = -INFINITY;
    for (int j = 0; j < n; j++)
      if (orc_bit(&A, i, j)) {
        double s = scale * orc_dot(q, k + (size_t)j * hd, hd);
        if (s > mx) mx = s;
      }
    if (mx == -INFINITY) {
      lse[i] = -INFINITY;
      delta[i] = 0.0;
      continue;
    }
    double sum = 0.0;
    for (int j = 0; j < n; j++)
      if (orc_bit(&A, i, j)) sum += exp(scale * orc_dot(q, k + (size_t)j * hd, hd) - mx);
    lse[i] = mx + log(sum);
    double dl = 0.0;
    for (int j = 0; j < n; j++)
      if (orc_bit(&A, i, j)) {
        double p = exp(scale * orc_dot(q, k + (size_t)j * hd, hd) - lse[i]);
        dl += p * orc_dot(g, v + (size_t)j * hd, hd);
      }
    delta[i] = dl;
    double *dq = (glob ? dqg : dqs) + (size_t)i * hd;
    for (int j = 0; j < n; j++)
      if (orc_bit(&A, i, j)) {
        const double *kj = k + (size_t)j * hd;
        double p = exp(scale * orc_dot(q, kj, hd) - lse[i]);
        double ds = p * (orc_dot(g, v + (size_t)j * hd, hd) - dl);
        for (int c = 0; c < hd; c++) dq[c] += scale * ds * kj[c];
      }
  }

#pragma omp parallel for schedule(dynamic, 8)
  for (int j = 0; j < n; j++) {
    double *dk_s = dks + (size_t)j * hd, *dv_s = dvs + (size_t)j * hd;
    double *dk_g = dkg + (size_t)j * hd, *dv_g = dvg + (size_t)j * hd;
    for (int i = 0; i < n; i++) {
      if (!orc_bit(&A, i, j)) continue;
      const int glob = (m[i] == 2);
      const double *q = (glob ? qg : qs) + (size_t)i * hd;
      const double *kj = (glob ? kg : ks) + (size_t)j * hd;
      const double *vj = (glob ? vg : vs) + (size_t)j * hd;
      const double *g = dO + (size_t)i * hd;
      double p = exp(scale * orc_dot(q, kj, hd) - lse[i]);
      double ds = p * (orc_dot(g, vj, hd) - delta[i]);
      double *dk = glob ? dk_g : dk_s;
      double *dv = glob ? dv_g : dv_s;
      for (int c = 0; c < hd; c++) {
        dk[c] += scale * ds * q[c];
        dv[c] += p * g[c];
      }
    }
  }
  free(lse);
  free(delta);
  orc_pattern_free(&A);
  return ORC_OK;
}

/* ------------------------------------------------------------------------
 * The linear projections either side of the attention (segmentfault page,
 * section 全局注意力的线性投影: the hidden states are projected by separate
 * linear maps into Qs, Ks, Vs and Qg, Kg, Vg).  An affine map in the
 * [out_features, in_features] weight layout:
 *
 *   y[m][c] = sum_k x[m][k] * w[c][k] + b[c]        (b may be NULL)
 *
 * computed in double, one output element at a time, rows in parallel.
 * ------------------------------------------------------------------------ */
int lf_oracle_linear(int M, int N, int K, const double *x, const double *w, const double *b,
                     double *y) {
  if (M < 0 || N < 0 || K < 0 || !x || !w || !y) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int m = 0; m < M; m++) {
    const double *xr = x + (size_t)m * K;
    for (int c = 0; c < N; c++) {
      const double *wr = w + (size_t)c * K;
      double s = 0.0;
      for (int k = 0; k < K; k++) s += xr[k] * wr[k];
      y[(size_t)m * N + c] = s + (b ? b[c] : 0.0);
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------
 * Cross-attention of the LED decoder (segmentfault page, section
 * Longformer-Encoder-Decoder: the decoder attends the whole encoder output
 * with full attention).  One head: Lq decoder queries against Lk encoder
 * keys, every key whose kmask entry is nonzero (kmask may be NULL: all):
 *
 *   s_ij = scale * <q_i, k_j>,  o_i = sum_j softmax_j(s_ij) v_j,
 *   lse_i = log sum_j exp(s_ij)
 *
 * A query with no valid key gets o_i = 0 and lse_i = -inf.  Double
 * precision, queries in parallel.
 * ------------------------------------------------------------------------ */
int lf_oracle_cross_head(int Lq, int Lk, int hd, double scale, const int32_t *kmask,
                         const double *q, const double *k, const double *v, double *o,
                         double *lse) {
  if (Lq < 0 || Lk < 0 || hd < 1 || !q || !k || !v || !o || !lse) return ORC_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 8)
  for (int i = 0; i < Lq; i++) {
    const double *qi = q + (size_t)i * hd;
    double *oi = o + (size_t)i * hd;
    double mx = -INFINITY;
    for (int j = 0; j < Lk; j++) {
      if (kmask && kmask[j] == 0) continue;
      double s = scale * orc_dot(qi, k + (size_t)j * hd, hd);
      if (s > mx) mx = s;
    }
    for (int c = 0; c < hd; c++) oi[c] = 0.0;
    if (mx == -INFINITY) { /* no valid key */
      lse[i] = -INFINITY;
      continue;
    }
    double sum = 0.0;
    for (int j = 0; j < Lk; j++) {
      if (kmask && kmask[j] == 0) continue;
      double p = exp(scale * orc_dot(qi, k + (size_t)j * hd, hd) - mx);
      sum += p;
      const double *vj = v + (size_t)j * hd;
      for (int c = 0; c < hd; c++) oi[c] += p * vj[c];
    }
    for (int c = 0; c < hd; c++) oi[c] /= sum;
    lse[i] = mx + log(sum);
  }
  return ORC_OK;
}
