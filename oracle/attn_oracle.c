/*
 * attn_oracle.c -- plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code:
 * only the test suite, the smoke check and the bench's CPU-baseline leg load it.
 * It shares no source, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, written out element by element):
 *
 *   For segment b (query rows [cu_q[b], cu_q[b+1]), key rows [cu_k[b], cu_k[b+1])),
 *   query head h and its key/value head hk = floor(h / G), G = Hq / Hkv:
 *     s_ij  = scale * sum_d q_id k_jd                    for every key j of the segment
 *             (with a softcap c > 0: s_ij = c * tanh(scale * sum_d q_id k_jd / c))
 *     key j is allowed for row i  iff, with delta = s_k - s_q,
 *             (!causal || j <= i + delta)
 *          && (window_left  < 0 || j >= i + delta - window_left)
 *          && (window_right < 0 || j <= i + delta + window_right)
 *     LSE_i = log sum_{allowed j} exp(s_ij)              (natural log, scaled scores)
 *     P_ij  = exp(s_ij - LSE_i) for allowed j, else 0
 *     O_i   = sum_j P_ij v_j
 *   and, given dO:
 *     D_i   = sum_d dO_id O_id
 *     dP_ij = sum_d dO_id v_jd
 *     dS_ij = P_ij (dP_ij - D_i) * g_ij,  g_ij = 1 - (s_ij / c)^2 with a softcap
 *             (the derivative of c tanh(x / c) at x = scale q_i.k_j), else 1
 *     dQ_i  = scale * sum_j dS_ij k_j
 *     dK_j  = scale * sum_{h in group(hk)} sum_i dS_ij q_i
 *     dV_j  =         sum_{h in group(hk)} sum_i P_ij dO_i
 *
 * Sources: the flash-attention issue "[FA4/B200] return_lse=True makes D64
 * forward about 19% faster" (its repro checks the kernel against torch's
 * scaled_dot_product_attention and allocates the LSE as batch x heads x seqlen),
 * the "FA4 head_dim=256 B200 Regression Check" (Environment: the softmax scale is
 * head_dim^-0.5) and the FA4 repository guide (Core Abstractions: an online
 * softmax that tracks each row's max and sum; Other Components: several query
 * heads share one key/value head for GQA; Public API: varlen through
 * cu_seqlens).  The pages print no formulas; the ones above are the textbook
 * definition of softmax attention and of its gradient.
 *
 * Readings where the pages are silent:
 *   - GQA map: contiguous groups, hk = h / G.
 *   - causal alignment when s_q != s_k: bottom-right (j <= i + s_k - s_q).
 *   - a row with no allowed key: O_i = 0, LSE_i = -inf, and it contributes
 *     nothing to any gradient.
 *   - zero-length segments are allowed and produce nothing.
 *   - local (sliding-window) masks and the softcap: the FA4 repository guide
 *     (Public API) names window_size_left/right and softcap as parameters but
 *     states no formula; the reading above is the plainest one (the window
 *     bounds are inclusive distances from the bottom-right aligned diagonal, a
 *     negative bound means none; the cap applies to the scaled score).
 *
 * Layouts (row-major, last index fastest):
 *   q, out, dout, dq : [Tq][Hq][D]      k, v, dk, dv : [Tk][Hkv][D]
 *   lse              : [Hq][Tq]         cu_q, cu_k   : int32 [batch+1]
 *
 * Every entry point returns 0 on success and a negative number for bad
 * arguments (it never aborts).  All pointers are host memory.  Parallelism
 * is OpenMP over independent (head, row) or (kv-head, key) pairs; each output
 * element is computed by exactly one thread, so results do not depend on the
 * thread count.
 *
 * ORACLE_MUTATION (compile-time, default 0) plants one known mistake so the
 * test suite can show that its pins catch it; it is never set in the build
 * the tests trust.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif

/* ------------------------------------------------------------------ */
/* argument checks and index helpers                                   */
/* ------------------------------------------------------------------ */

static int check_args(const int32_t* cu_q, const int32_t* cu_k, int batch, int Hq,
                      int Hkv, int D) {
  if (!cu_q || !cu_k || batch < 0 || Hq < 1 || Hkv < 1 || D < 1) return -1;
  if (Hq % Hkv != 0) return -2;
  if (cu_q[0] != 0 || cu_k[0] != 0) return -3;
  for (int b = 0; b < batch; ++b)
    if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b]) return -4;
  return 0;
}

/* segment holding global query row r: largest b with cu[b] <= r < cu[b+1] */
static int segment_of(const int32_t* cu, int batch, long r) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if ((long)cu[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

static int kv_head_of(int h, int Hq, int Hkv) {
#if ORACLE_MUTATION == 4
  (void)Hq;
  return h % Hkv; /* planted: interleaved instead of contiguous groups */
#else
  return h / (Hq / Hkv);
#endif
}

typedef struct {
  int causal;
  long wl, wr;     /* window bounds, < 0 = none */
  double softcap;  /* <= 0 = none */
} mask_t;

static int key_allowed(const mask_t* mk, long i, long j, long sq, long sk) {
  const long diag = i + (sk - sq);
#if ORACLE_MUTATION == 3
  if (mk->causal && !(j < diag)) return 0; /* planted: diagonal excluded */
#else
  if (mk->causal && !(j <= diag)) return 0;
#endif
#if ORACLE_MUTATION == 8
  if (mk->wl >= 0 && !(j > diag - mk->wl)) return 0; /* planted: window edge excluded */
#else
  if (mk->wl >= 0 && !(j >= diag - mk->wl)) return 0;
#endif
  if (mk->wr >= 0 && !(j <= diag + mk->wr)) return 0;
  return 1;
}

/* the score of row q_i and key k_j (scaled, then capped if a softcap is set) */
static double score(const mask_t* mk, double scale, double qk) {
  if (mk->softcap <= 0.0) return scale * qk;
#if ORACLE_MUTATION == 10
  return mk->softcap * tanh(qk / mk->softcap); /* planted: cap of the unscaled score */
#else
  return mk->softcap * tanh(scale * qk / mk->softcap);
#endif
}

/* d score / d (scale q.k), from the (capped) score itself */
static double score_grad(const mask_t* mk, double s) {
#if ORACLE_MUTATION == 9
  (void)s;
  return 1.0; /* planted: the cap's derivative is dropped */
#else
  if (mk->softcap <= 0.0) return 1.0;
  const double t = s / mk->softcap;
  return 1.0 - t * t;
#endif
}

static double dot(const double* a, const double* b, int n) {
  double acc = 0.0;
  for (int d = 0; d < n; ++d) acc += a[d] * b[d];
  return acc;
}

/*
 * Everything the definition says about one query row: scores, LSE, P, O and
 * (when dout is given) D_i and dS.  s, p, ds are caller scratch of length s_k.
 * Returns the number of allowed keys.
 */
typedef struct {
  const double *q, *k, *v, *dout;
  int Hq, Hkv, D;
  double scale;
  mask_t mk;
} problem_t;

static int row_forward(const problem_t* pb, int h, long qrow, long i, long k0, long sq,
                       long sk, double* s, double* p, double* o, double* lse_out) {
  const int D = pb->D;
  const int hk = kv_head_of(h, pb->Hq, pb->Hkv);
  const double* qi = pb->q + ((size_t)qrow * pb->Hq + h) * D;
  int n_allowed = 0;
  double m = -INFINITY;
  for (long j = 0; j < sk; ++j) {
    if (!key_allowed(&pb->mk, i, j, sq, sk)) { s[j] = -INFINITY; continue; }
    const double* kj = pb->k + ((size_t)(k0 + j) * pb->Hkv + hk) * D;
    s[j] = score(&pb->mk, pb->scale, dot(qi, kj, D));
    if (s[j] > m) m = s[j];
    ++n_allowed;
  }
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (n_allowed == 0) {
    for (long j = 0; j < sk; ++j) p[j] = 0.0;
    *lse_out = -INFINITY;
    return 0;
  }
  double sum = 0.0;
  for (long j = 0; j < sk; ++j)
    if (s[j] != -INFINITY) sum += exp(s[j] - m);
#if ORACLE_MUTATION == 5
  const double lse = log(sum); /* planted: the max term is dropped */
#else
  const double lse = m + log(sum);
#endif
  for (long j = 0; j < sk; ++j) {
    p[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - lse);
    if (p[j] == 0.0) continue;
    const double* vj = pb->v + ((size_t)(k0 + j) * pb->Hkv + hk) * D;
    for (int d = 0; d < D; ++d) o[d] += p[j] * vj[d];
  }
  *lse_out = lse;
  return n_allowed;
}

/* D_i = <dO_i, O_i> */
static double row_delta(const problem_t* pb, int h, long qrow, const double* o) {
  const double* doi = pb->dout + ((size_t)qrow * pb->Hq + h) * pb->D;
#if ORACLE_MUTATION == 7
  (void)o;
  double acc = 0.0; /* planted: the O factor is dropped */
  for (int d = 0; d < pb->D; ++d) acc += doi[d];
  return acc;
#else
  return dot(doi, o, pb->D);
#endif
}

/* dS_ij for one row, given its scores s_ij, P_ij and D_i */
static void row_dscores(const problem_t* pb, int h, long qrow, long k0, long sk,
                        const double* s, const double* p, double delta, double* ds) {
  const int D = pb->D;
  const int hk = kv_head_of(h, pb->Hq, pb->Hkv);
  const double* doi = pb->dout + ((size_t)qrow * pb->Hq + h) * D;
  for (long j = 0; j < sk; ++j) {
    if (p[j] == 0.0) { ds[j] = 0.0; continue; }
    const double* vj = pb->v + ((size_t)(k0 + j) * pb->Hkv + hk) * D;
    const double dp = dot(doi, vj, D);
#if ORACLE_MUTATION == 2
    ds[j] = p[j] * (delta - dp); /* planted: sign flipped */
#else
    ds[j] = p[j] * (dp - delta);
#endif
    ds[j] *= score_grad(&pb->mk, s[j]);
  }
}

static void row_dq(const problem_t* pb, int h, long k0, long sk, const double* ds,
                   double* dq) {
  const int D = pb->D;
  const int hk = kv_head_of(h, pb->Hq, pb->Hkv);
  for (int d = 0; d < D; ++d) dq[d] = 0.0;
  for (long j = 0; j < sk; ++j) {
    if (ds[j] == 0.0) continue;
    const double* kj = pb->k + ((size_t)(k0 + j) * pb->Hkv + hk) * D;
    for (int d = 0; d < D; ++d) dq[d] += ds[j] * kj[d];
  }
#if ORACLE_MUTATION != 1 /* mutation 1 plants a missing scale on dQ */
  for (int d = 0; d < D; ++d) dq[d] *= pb->scale;
#endif
}

/*
 * dK_j and dV_j of one key row kr of kv head hk, summed over the query heads of
 * its group, given every query row's LSE and D_i ([Hq][Tq]):
 *   dV_j = sum_{h, i} P_ij dO_i,  dK_j = scale * sum_{h, i} dS_ij q_i,
 *   dS_ij = P_ij (dO_i . v_j - D_i) (times the softcap derivative).
 */
static void key_grads(const problem_t* pb, const int32_t* cu_q, const int32_t* cu_k, int batch,
                      long Tq, const double* lse_all, const double* delta_all, int hk, long kr,
                      double* dkj, double* dvj) {
  const int D = pb->D, Hq = pb->Hq, Hkv = pb->Hkv;
  const double scale = pb->scale;
  const int b = segment_of(cu_k, batch, kr);
  const long sq = cu_q[b + 1] - cu_q[b], sk = cu_k[b + 1] - cu_k[b];
  const long j = kr - cu_k[b];
  for (int d = 0; d < D; ++d) { dkj[d] = 0.0; dvj[d] = 0.0; }
  const double* kj = pb->k + ((size_t)kr * Hkv + hk) * D;
  const double* vj = pb->v + ((size_t)kr * Hkv + hk) * D;
  for (int h = 0; h < Hq; ++h) {
    if (kv_head_of(h, Hq, Hkv) != hk) continue;
    for (long i = 0; i < sq; ++i) {
      if (!key_allowed(&pb->mk, i, j, sq, sk)) continue;
      const long r = cu_q[b] + i;
      const double l = lse_all[(size_t)h * Tq + r];
      if (l == -INFINITY) continue;
      const double* qi = pb->q + ((size_t)r * Hq + h) * D;
      const double* doi = pb->dout + ((size_t)r * Hq + h) * D;
      const double sij = score(&pb->mk, scale, dot(qi, kj, D));
      const double pij = exp(sij - l);
#if ORACLE_MUTATION == 2
      double dsij = pij * (delta_all[(size_t)h * Tq + r] - dot(doi, vj, D));
#else
      double dsij = pij * (dot(doi, vj, D) - delta_all[(size_t)h * Tq + r]);
#endif
      dsij *= score_grad(&pb->mk, sij);
      for (int d = 0; d < D; ++d) {
#if ORACLE_MUTATION == 6
        dkj[d] += scale * dsij * doi[d]; /* planted: wrong operand */
#else
        dkj[d] += scale * dsij * qi[d];
#endif
        dvj[d] += pij * doi[d];
      }
    }
  }
}

static long max_seg_len(const int32_t* cu, int batch) {
  long m = 0;
  for (int b = 0; b < batch; ++b) {
    long len = (long)cu[b + 1] - cu[b];
    if (len > m) m = len;
  }
  return m;
}

/* ------------------------------------------------------------------ */
/* public entry points                                                 */
/* ------------------------------------------------------------------ */

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int oracle_mutation(void) { return ORACLE_MUTATION; }

/* Full forward: out [Tq][Hq][D], lse [Hq][Tq] (lse may be NULL).  window_left /
 * window_right < 0 mean no bound, softcap <= 0 means none. */
int oracle_fwd_ex(const double* q, const double* k, const double* v, const int32_t* cu_q,
                  const int32_t* cu_k, int batch, int Hq, int Hkv, int D, double scale,
                  int causal, long window_left, long window_right, double softcap,
                  double* out, double* lse) {
  int rc = check_args(cu_q, cu_k, batch, Hq, Hkv, D);
  if (rc) return rc;
  if (!q || !k || !v || !out) return -1;
  if (batch == 0) return 0;
  const problem_t pb = {q, k, v, NULL, Hq, Hkv, D, scale,
                        {causal, window_left, window_right, softcap}};
  const long Tq = cu_q[batch];
  const long msk = max_seg_len(cu_k, batch);
  const long n_units = (long)Hq * Tq;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (msk + 1));
    double* p = (double*)malloc(sizeof(double) * (msk + 1));
#pragma omp for schedule(dynamic, 8)
    for (long u = 0; u < n_units; ++u) {
      const int h = (int)(u / Tq);
      const long r = u % Tq;
      const int b = segment_of(cu_q, batch, r);
      const long sq = cu_q[b + 1] - cu_q[b], sk = cu_k[b + 1] - cu_k[b];
      double l;
      row_forward(&pb, h, r, r - cu_q[b], cu_k[b], sq, sk, s, p,
                  out + ((size_t)r * Hq + h) * D, &l);
      if (lse) lse[(size_t)h * Tq + r] = l;
    }
    free(s);
    free(p);
  }
  return 0;
}

int oracle_fwd(const double* q, const double* k, const double* v, const int32_t* cu_q,
               const int32_t* cu_k, int batch, int Hq, int Hkv, int D, double scale,
               int causal, double* out, double* lse) {
  return oracle_fwd_ex(q, k, v, cu_q, cu_k, batch, Hq, Hkv, D, scale, causal, -1, -1, 0.0,
                       out, lse);
}

/*
 * Full backward from first principles: recomputes P from the definition
 * (it takes no O or LSE from anywhere else).  dq like q, dk/dv like k.
 */
int oracle_bwd_ex(const double* q, const double* k, const double* v, const double* dout,
                  const int32_t* cu_q, const int32_t* cu_k, int batch, int Hq, int Hkv,
                  int D, double scale, int causal, long window_left, long window_right,
                  double softcap, double* dq, double* dk, double* dv) {
  int rc = check_args(cu_q, cu_k, batch, Hq, Hkv, D);
  if (rc) return rc;
  if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
  if (batch == 0) return 0;
  const problem_t pb = {q, k, v, dout, Hq, Hkv, D, scale,
                        {causal, window_left, window_right, softcap}};
  const long Tq = cu_q[batch], Tk = cu_k[batch];
  const long msk = max_seg_len(cu_k, batch);
  const int G = Hq / Hkv;
  double* lse_all = (double*)malloc(sizeof(double) * (size_t)Hq * (Tq ? Tq : 1));
  double* delta_all = (double*)malloc(sizeof(double) * (size_t)Hq * (Tq ? Tq : 1));
  if (!lse_all || !delta_all) { free(lse_all); free(delta_all); return -5; }

  /* pass 1: per query row -- LSE, O, D_i and dQ_i */
  const long n_rows = (long)Hq * Tq;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (msk + 1));
    double* p = (double*)malloc(sizeof(double) * (msk + 1));
    double* ds = (double*)malloc(sizeof(double) * (msk + 1));
    double* o = (double*)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 8)
    for (long u = 0; u < n_rows; ++u) {
      const int h = (int)(u / Tq);
      const long r = u % Tq;
      const int b = segment_of(cu_q, batch, r);
      const long sq = cu_q[b + 1] - cu_q[b], sk = cu_k[b + 1] - cu_k[b];
      double l;
      row_forward(&pb, h, r, r - cu_q[b], cu_k[b], sq, sk, s, p, o, &l);
      const double delta = row_delta(&pb, h, r, o);
      lse_all[(size_t)h * Tq + r] = l;
      delta_all[(size_t)h * Tq + r] = delta;
      row_dscores(&pb, h, r, cu_k[b], sk, s, p, delta, ds);
      row_dq(&pb, h, cu_k[b], sk, ds, dq + ((size_t)r * Hq + h) * D);
    }
    free(s); free(p); free(ds); free(o);
  }

  /* pass 2: per key row -- dK_j and dV_j summed over the query heads of the group */
  const long n_keys = (long)Hkv * Tk;
#pragma omp parallel for schedule(dynamic, 8)
  for (long u = 0; u < n_keys; ++u) {
    const int hk = (int)(u / (Tk ? Tk : 1));
    const long kr = u % Tk;
    key_grads(&pb, cu_q, cu_k, batch, Tq, lse_all, delta_all, hk, kr,
              dk + ((size_t)kr * Hkv + hk) * D, dv + ((size_t)kr * Hkv + hk) * D);
  }
  (void)G;
  free(lse_all);
  free(delta_all);
  return 0;
}

int oracle_bwd(const double* q, const double* k, const double* v, const double* dout,
               const int32_t* cu_q, const int32_t* cu_k, int batch, int Hq, int Hkv,
               int D, double scale, int causal, double* dq, double* dk, double* dv) {
  return oracle_bwd_ex(q, k, v, dout, cu_q, cu_k, batch, Hq, Hkv, D, scale, causal, -1, -1,
                       0.0, dq, dk, dv);
}

/*
 * Sampled rows: for n (head, global query row) pairs, the row's O, LSE and,
 * when dout is not NULL, its dQ.  Each row needs only its own scores, so this
 * is exact at any sequence length.  out_rows/dq_rows are [n][D].
 */
int oracle_rows_ex(const double* q, const double* k, const double* v, const double* dout,
                   const int32_t* cu_q, const int32_t* cu_k, int batch, int Hq, int Hkv,
                   int D, double scale, int causal, long window_left, long window_right,
                   double softcap, int n, const int32_t* row_head, const int64_t* row_index,
                   double* out_rows, double* lse_rows, double* dq_rows) {
  int rc = check_args(cu_q, cu_k, batch, Hq, Hkv, D);
  if (rc) return rc;
  if (!q || !k || !v || !row_head || !row_index || !out_rows || !lse_rows) return -1;
  if (dq_rows && !dout) return -1;
  if (batch == 0 || n == 0) return 0;
  const problem_t pb = {q, k, v, dout, Hq, Hkv, D, scale,
                        {causal, window_left, window_right, softcap}};
  const long Tq = cu_q[batch];
  for (int t = 0; t < n; ++t)
    if (row_head[t] < 0 || row_head[t] >= Hq || row_index[t] < 0 || row_index[t] >= Tq)
      return -6;
  const long msk = max_seg_len(cu_k, batch);
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (msk + 1));
    double* p = (double*)malloc(sizeof(double) * (msk + 1));
    double* ds = (double*)malloc(sizeof(double) * (msk + 1));
#pragma omp for schedule(dynamic, 1)
    for (int t = 0; t < n; ++t) {
      const int h = row_head[t];
      const long r = row_index[t];
      const int b = segment_of(cu_q, batch, r);
      const long sq = cu_q[b + 1] - cu_q[b], sk = cu_k[b + 1] - cu_k[b];
      double* o = out_rows + (size_t)t * D;
      row_forward(&pb, h, r, r - cu_q[b], cu_k[b], sq, sk, s, p, o, &lse_rows[t]);
      if (dq_rows) {
        const double delta = row_delta(&pb, h, r, o);
        row_dscores(&pb, h, r, cu_k[b], sk, s, p, delta, ds);
        row_dq(&pb, h, cu_k[b], sk, ds, dq_rows + (size_t)t * D);
      }
    }
    free(s); free(p); free(ds);
  }
  return 0;
}

int oracle_rows(const double* q, const double* k, const double* v, const double* dout,
                const int32_t* cu_q, const int32_t* cu_k, int batch, int Hq, int Hkv,
                int D, double scale, int causal, int n, const int32_t* row_head,
                const int64_t* row_index, double* out_rows, double* lse_rows,
                double* dq_rows) {
  return oracle_rows_ex(q, k, v, dout, cu_q, cu_k, batch, Hq, Hkv, D, scale, causal, -1, -1,
                        0.0, n, row_head, row_index, out_rows, lse_rows, dq_rows);
}

/*
 * Sampled key rows: for n (kv head, global key row) pairs, the row's dK and dV
 * summed over the query heads of the group.  A key row needs the LSE and D_i
 * of every query row that can see it, so the forward statistics of exactly
 * those (query head, row) pairs are computed first; the result is exact at
 * any length.  Under a causal mask a key near the end of a long segment is
 * seen by few rows, which keeps this cheap there; without a mask it costs the
 * segment's full forward for the group.  dk_rows/dv_rows are [n][D].
 */
int oracle_cols_ex(const double* q, const double* k, const double* v, const double* dout,
                   const int32_t* cu_q, const int32_t* cu_k, int batch, int Hq, int Hkv,
                   int D, double scale, int causal, long window_left, long window_right,
                   double softcap, int n, const int32_t* key_head, const int64_t* key_index,
                   double* dk_rows, double* dv_rows) {
  int rc = check_args(cu_q, cu_k, batch, Hq, Hkv, D);
  if (rc) return rc;
  if (!q || !k || !v || !dout || !key_head || !key_index || !dk_rows || !dv_rows) return -1;
  if (batch == 0 || n == 0) return 0;
  const problem_t pb = {q, k, v, dout, Hq, Hkv, D, scale,
                        {causal, window_left, window_right, softcap}};
  const long Tq = cu_q[batch], Tk = cu_k[batch];
  for (int t = 0; t < n; ++t)
    if (key_head[t] < 0 || key_head[t] >= Hkv || key_index[t] < 0 || key_index[t] >= Tk)
      return -6;
  /* which (query head, query row) pairs the sampled keys need: a row's LSE and
   * D_i enter key j's gradient only if key j is allowed for that row, so only
   * those rows get their forward statistics (the others stay at LSE = -inf,
   * which key_grads skips, as it skips rows with no allowed key) */
  unsigned char* need = (unsigned char*)calloc((size_t)Hq * (Tq ? Tq : 1), 1);
  double* lse_all = (double*)malloc(sizeof(double) * (size_t)Hq * (Tq ? Tq : 1));
  double* delta_all = (double*)malloc(sizeof(double) * (size_t)Hq * (Tq ? Tq : 1));
  if (!need || !lse_all || !delta_all) {
    free(need); free(lse_all); free(delta_all);
    return -5;
  }
  for (size_t u = 0; u < (size_t)Hq * Tq; ++u) { lse_all[u] = -INFINITY; delta_all[u] = 0.0; }
  for (int t = 0; t < n; ++t) {
    const int b = segment_of(cu_k, batch, (long)key_index[t]);
    const long sq = cu_q[b + 1] - cu_q[b], sk = cu_k[b + 1] - cu_k[b];
    const long j = (long)key_index[t] - cu_k[b];
    for (int h = 0; h < Hq; ++h) {
      if (kv_head_of(h, Hq, Hkv) != key_head[t]) continue;
      for (long i = 0; i < sq; ++i) {
#if ORACLE_MUTATION == 11
        /* planted: the row on the key's diagonal is left out of the selection */
        if (key_allowed(&pb.mk, i, j, sq, sk) && j != i + (sk - sq))
#else
        if (key_allowed(&pb.mk, i, j, sq, sk))
#endif
          need[(size_t)h * Tq + cu_q[b] + i] = 1;
      }
    }
  }
  const long msk = max_seg_len(cu_k, batch);
  const long n_rows = (long)Hq * Tq;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (msk + 1));
    double* p = (double*)malloc(sizeof(double) * (msk + 1));
    double* o = (double*)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 8)
    for (long u = 0; u < n_rows; ++u) {
      if (!need[u]) continue;
      const int h = (int)(u / Tq);
      const long r = u % Tq;
      const int b = segment_of(cu_q, batch, r);
      const long sq = cu_q[b + 1] - cu_q[b], sk = cu_k[b + 1] - cu_k[b];
      double l;
      row_forward(&pb, h, r, r - cu_q[b], cu_k[b], sq, sk, s, p, o, &l);
      lse_all[(size_t)h * Tq + r] = l;
      delta_all[(size_t)h * Tq + r] = row_delta(&pb, h, r, o);
    }
    free(s); free(p); free(o);
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < n; ++t)
    key_grads(&pb, cu_q, cu_k, batch, Tq, lse_all, delta_all, key_head[t], (long)key_index[t],
              dk_rows + (size_t)t * D, dv_rows + (size_t)t * D);
  free(need);
  free(lse_all);
  free(delta_all);
  return 0;
}
