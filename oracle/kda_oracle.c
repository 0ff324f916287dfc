/*
 * KDA oracle: the plain fp64 token-by-token recurrence of Kimi Delta Attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code with the CUDA kernels.
 *
 * What it computes (Kimi Linear summary, section 3 "Kimi Delta Attention"):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with the memory decayed before the delta-rule correction is applied, and
 * the output read from the updated state. S is d_k x d_v (row = key channel,
 * column = value channel). The gate arrives in log space, alpha = exp(log_alpha).
 *
 * Written out step by step for each token, exactly as the definition reads:
 *   1. forget:  S <- Diag(alpha_t) S
 *   2. erase:   S <- S - beta_t k_t (k_t^T S)
 *   3. write:   S <- S + beta_t k_t v_t^T
 *   4. read:    o_t = S^T q_t
 *
 * Every column of S evolves on its own (k, alpha and beta are shared by all
 * columns; only v_t[j] differs), so the work is split into independent tasks
 * of (sequence, head, block of value columns) and run with OpenMP. Splitting
 * columns does not change a single arithmetic operation of any column.
 *
 * Inputs are fp32 arrays (bf16 inputs are widened to fp32 by the caller, which
 * is exact); every operation here is fp64 with libm exp.
 *
 * Layouts (token-major, contiguous):
 *   q, k, log_alpha : [t_total, n_heads, dk]
 *   v               : [t_total, n_heads, dv]
 *   beta            : [t_total, n_heads]
 *   h0, hT          : [n_seqs, n_heads, dk, dv]   (h0 may be NULL: zero state)
 *   o               : [t_total, n_heads, dv]
 *   cu_seqlens      : [n_seqs + 1], sequence n owns tokens [cu[n], cu[n+1])
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARGS (-1)
#define ORACLE_ERR_NOMEM (-2)

static int run_chain(const float* q, const float* k, const float* v, const float* log_alpha,
                     const float* beta, const double* h0, int64_t bos, int64_t eos, int64_t h,
                     int64_t n_heads, int64_t dk, int64_t dv, int64_t j0, int64_t j1, double* o,
                     double* hT) {
  const int64_t nc = j1 - j0;
  double* S = (double*)malloc(sizeof(double) * (size_t)(dk * nc));
  double* u = (double*)malloc(sizeof(double) * (size_t)nc);
  double* alpha = (double*)malloc(sizeof(double) * (size_t)dk);
  if (!S || !u || !alpha) {
    free(S);
    free(u);
    free(alpha);
    return ORACLE_ERR_NOMEM;
  }
  for (int64_t c = 0; c < dk; ++c)
    for (int64_t j = 0; j < nc; ++j) S[c * nc + j] = h0 ? h0[c * dv + j0 + j] : 0.0;

  for (int64_t t = bos; t < eos; ++t) {
    const float* qt = q + (t * n_heads + h) * dk;
    const float* kt = k + (t * n_heads + h) * dk;
    const float* vt = v + (t * n_heads + h) * dv;
    const float* lat = log_alpha + (t * n_heads + h) * dk;
    const double bt = (double)beta[t * n_heads + h];

    /* 1. forget: S <- Diag(alpha_t) S */
    for (int64_t c = 0; c < dk; ++c) alpha[c] = exp((double)lat[c]);
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] *= alpha[c];

    /* 2. erase: S <- S - beta k (k^T S)   (k^T S uses the decayed state) */
    for (int64_t j = 0; j < nc; ++j) u[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double kc = (double)kt[c];
      for (int64_t j = 0; j < nc; ++j) u[j] += kc * S[c * nc + j];
    }
    for (int64_t c = 0; c < dk; ++c) {
      const double bk = bt * (double)kt[c];
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] -= bk * u[j];
    }

    /* 3. write: S <- S + beta k v^T */
    for (int64_t c = 0; c < dk; ++c) {
      const double bk = bt * (double)kt[c];
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] += bk * (double)vt[j0 + j];
    }

    /* 4. read: o_t = S^T q_t, from the updated state */
    double* ot = o + (t * n_heads + h) * dv;
    for (int64_t j = 0; j < nc; ++j) u[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double qc = (double)qt[c];
      for (int64_t j = 0; j < nc; ++j) u[j] += qc * S[c * nc + j];
    }
    for (int64_t j = 0; j < nc; ++j) ot[j0 + j] = u[j];
  }

  if (hT)
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < nc; ++j) hT[c * dv + j0 + j] = S[c * nc + j];
  free(S);
  free(u);
  free(alpha);
  return ORACLE_OK;
}

/* Returns 0 on success. col_block <= 0 means one block of all dv columns.
 * n_threads <= 0 lets OpenMP choose. */
int kda_oracle_forward(const float* q, const float* k, const float* v, const float* log_alpha,
                       const float* beta, const double* h0, const int64_t* cu_seqlens,
                       int64_t n_seqs, int64_t n_heads, int64_t dk, int64_t dv, int64_t t_total,
                       int64_t col_block, double* o, double* hT, int n_threads) {
  if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !o) return ORACLE_ERR_ARGS;
  if (n_seqs <= 0 || n_heads <= 0 || dk <= 0 || dv <= 0 || t_total < 0) return ORACLE_ERR_ARGS;
  if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != t_total) return ORACLE_ERR_ARGS;
  for (int64_t n = 0; n < n_seqs; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return ORACLE_ERR_ARGS;
  if (col_block <= 0 || col_block > dv) col_block = dv;
  const int64_t n_cb = (dv + col_block - 1) / col_block;
  const int64_t n_tasks = n_seqs * n_heads * n_cb;
  int status = ORACLE_OK;

#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t task = 0; task < n_tasks; ++task) {
    const int64_t cb = task % n_cb;
    const int64_t h = (task / n_cb) % n_heads;
    const int64_t n = task / (n_cb * n_heads);
    const int64_t j0 = cb * col_block;
    const int64_t j1 = (j0 + col_block < dv) ? j0 + col_block : dv;
    const double* h0n = h0 ? h0 + (n * n_heads + h) * dk * dv : NULL;
    double* hTn = hT ? hT + (n * n_heads + h) * dk * dv : NULL;
    int rc = run_chain(q, k, v, log_alpha, beta, h0n, cu_seqlens[n], cu_seqlens[n + 1], h, n_heads,
                       dk, dv, j0, j1, o, hTn);
    if (rc != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
      status = rc;
    }
  }
  return status;
}

/*
 * Gated DeltaNet, the scalar-gate case of the same family (Rationalist Deep-Dive,
 * section 2.3 "Gated DeltaNet: The Scalar Forget"; Kimi Linear summary, section 2.2):
 *
 *     S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t
 *
 * with one gate a_t per token and head, passed in log space (log_a [t_total,
 * n_heads]). Written out in the order this definition reads, which is not the
 * order of the KDA chain above:
 *   1. erase:  S <- S - beta_t k_t (k_t^T S)
 *   2. gate:   S <- a_t S
 *   3. write:  S <- S + beta_t k_t v_t^T
 *   4. read:   o_t = S^T q_t
 * Same layouts as kda_oracle_forward, except log_a.
 */
static int run_gdn_chain(const float* q, const float* k, const float* v, const float* log_a,
                         const float* beta, const double* h0, int64_t bos, int64_t eos, int64_t h,
                         int64_t n_heads, int64_t dk, int64_t dv, int64_t j0, int64_t j1,
                         double* o, double* hT) {
  const int64_t nc = j1 - j0;
  double* S = (double*)malloc(sizeof(double) * (size_t)(dk * nc));
  double* u = (double*)malloc(sizeof(double) * (size_t)nc);
  if (!S || !u) {
    free(S);
    free(u);
    return ORACLE_ERR_NOMEM;
  }
  for (int64_t c = 0; c < dk; ++c)
    for (int64_t j = 0; j < nc; ++j) S[c * nc + j] = h0 ? h0[c * dv + j0 + j] : 0.0;

  for (int64_t t = bos; t < eos; ++t) {
    const float* qt = q + (t * n_heads + h) * dk;
    const float* kt = k + (t * n_heads + h) * dk;
    const float* vt = v + (t * n_heads + h) * dv;
    const double at = exp((double)log_a[t * n_heads + h]);
    const double bt = (double)beta[t * n_heads + h];

    /* 1. erase: S <- S - beta k (k^T S) */
    for (int64_t j = 0; j < nc; ++j) u[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double kc = (double)kt[c];
      for (int64_t j = 0; j < nc; ++j) u[j] += kc * S[c * nc + j];
    }
    for (int64_t c = 0; c < dk; ++c) {
      const double bk = bt * (double)kt[c];
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] -= bk * u[j];
    }

    /* 2. gate: S <- a S */
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] *= at;

    /* 3. write: S <- S + beta k v^T */
    for (int64_t c = 0; c < dk; ++c) {
      const double bk = bt * (double)kt[c];
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] += bk * (double)vt[j0 + j];
    }

    /* 4. read: o_t = S^T q_t */
    double* ot = o + (t * n_heads + h) * dv;
    for (int64_t j = 0; j < nc; ++j) u[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double qc = (double)qt[c];
      for (int64_t j = 0; j < nc; ++j) u[j] += qc * S[c * nc + j];
    }
    for (int64_t j = 0; j < nc; ++j) ot[j0 + j] = u[j];
  }

  if (hT)
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < nc; ++j) hT[c * dv + j0 + j] = S[c * nc + j];
  free(S);
  free(u);
  return ORACLE_OK;
}

int gdn_oracle_forward(const float* q, const float* k, const float* v, const float* log_a,
                       const float* beta, const double* h0, const int64_t* cu_seqlens,
                       int64_t n_seqs, int64_t n_heads, int64_t dk, int64_t dv, int64_t t_total,
                       int64_t col_block, double* o, double* hT, int n_threads) {
  if (!q || !k || !v || !log_a || !beta || !cu_seqlens || !o) return ORACLE_ERR_ARGS;
  if (n_seqs <= 0 || n_heads <= 0 || dk <= 0 || dv <= 0 || t_total < 0) return ORACLE_ERR_ARGS;
  if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != t_total) return ORACLE_ERR_ARGS;
  for (int64_t n = 0; n < n_seqs; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return ORACLE_ERR_ARGS;
  if (col_block <= 0 || col_block > dv) col_block = dv;
  const int64_t n_cb = (dv + col_block - 1) / col_block;
  const int64_t n_tasks = n_seqs * n_heads * n_cb;
  int status = ORACLE_OK;

#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t task = 0; task < n_tasks; ++task) {
    const int64_t cb = task % n_cb;
    const int64_t h = (task / n_cb) % n_heads;
    const int64_t n = task / (n_cb * n_heads);
    const int64_t j0 = cb * col_block;
    const int64_t j1 = (j0 + col_block < dv) ? j0 + col_block : dv;
    const double* h0n = h0 ? h0 + (n * n_heads + h) * dk * dv : NULL;
    double* hTn = hT ? hT + (n * n_heads + h) * dk * dv : NULL;
    int rc = run_gdn_chain(q, k, v, log_a, beta, h0n, cu_seqlens[n], cu_seqlens[n + 1], h,
                           n_heads, dk, dv, j0, j1, o, hTn);
    if (rc != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
      status = rc;
    }
  }
  return status;
}

/*
 * General DPLR (diagonal plus low rank) recurrence, the comparison point the pages
 * hold KDA against (Rationalist Deep-Dive, section 3.2 "DPLR Structure"; Kimi Linear
 * summary, section 6.2 "Relation to DPLR"):
 *
 *     S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,   o_t = S_t^T q_t
 *
 * with free low-rank factors a_t, b_t (KDA ties them: a = beta k, b = k * alpha).
 * Written out in the order this definition reads:
 *   1. low-rank read:  u = b_t^T S_{t-1}           (of the state before the step)
 *   2. forget:         S <- Diag(alpha_t) S_{t-1}
 *   3. correct:        S <- S - a_t u
 *   4. write:          S <- S + k_t v_t^T
 *   5. read:           o_t = S^T q_t
 * Layouts as kda_oracle_forward; a and b are [t_total, n_heads, dk].
 */
static int run_dplr_chain(const float* q, const float* k, const float* v, const float* a,
                          const float* b, const float* log_alpha, const double* h0, int64_t bos,
                          int64_t eos, int64_t h, int64_t n_heads, int64_t dk, int64_t dv,
                          int64_t j0, int64_t j1, double* o, double* hT) {
  const int64_t nc = j1 - j0;
  double* S = (double*)malloc(sizeof(double) * (size_t)(dk * nc));
  double* u = (double*)malloc(sizeof(double) * (size_t)nc);
  if (!S || !u) {
    free(S);
    free(u);
    return ORACLE_ERR_NOMEM;
  }
  for (int64_t c = 0; c < dk; ++c)
    for (int64_t j = 0; j < nc; ++j) S[c * nc + j] = h0 ? h0[c * dv + j0 + j] : 0.0;

  for (int64_t t = bos; t < eos; ++t) {
    const int64_t base = (t * n_heads + h) * dk;
    const float* qt = q + base;
    const float* kt = k + base;
    const float* at = a + base;
    const float* bt = b + base;
    const float* lat = log_alpha + base;
    const float* vt = v + (t * n_heads + h) * dv;

    /* 1. low-rank read of the old state: u = b^T S */
    for (int64_t j = 0; j < nc; ++j) u[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double bc = (double)bt[c];
      for (int64_t j = 0; j < nc; ++j) u[j] += bc * S[c * nc + j];
    }
    /* 2. forget: S <- Diag(alpha) S */
    for (int64_t c = 0; c < dk; ++c) {
      const double al = exp((double)lat[c]);
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] *= al;
    }
    /* 3. correct: S <- S - a u^T */
    for (int64_t c = 0; c < dk; ++c) {
      const double ac = (double)at[c];
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] -= ac * u[j];
    }
    /* 4. write: S <- S + k v^T */
    for (int64_t c = 0; c < dk; ++c) {
      const double kc = (double)kt[c];
      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] += kc * (double)vt[j0 + j];
    }
    /* 5. read: o_t = S^T q_t */
    double* ot = o + (t * n_heads + h) * dv;
    for (int64_t j = 0; j < nc; ++j) u[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double qc = (double)qt[c];
      for (int64_t j = 0; j < nc; ++j) u[j] += qc * S[c * nc + j];
    }
    for (int64_t j = 0; j < nc; ++j) ot[j0 + j] = u[j];
  }

  if (hT)
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < nc; ++j) hT[c * dv + j0 + j] = S[c * nc + j];
  free(S);
  free(u);
  return ORACLE_OK;
}

int dplr_oracle_forward(const float* q, const float* k, const float* v, const float* a,
                        const float* b, const float* log_alpha, const double* h0,
                        const int64_t* cu_seqlens, int64_t n_seqs, int64_t n_heads, int64_t dk,
                        int64_t dv, int64_t t_total, int64_t col_block, double* o, double* hT,
                        int n_threads) {
  if (!q || !k || !v || !a || !b || !log_alpha || !cu_seqlens || !o) return ORACLE_ERR_ARGS;
  if (n_seqs <= 0 || n_heads <= 0 || dk <= 0 || dv <= 0 || t_total < 0) return ORACLE_ERR_ARGS;
  if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != t_total) return ORACLE_ERR_ARGS;
  for (int64_t n = 0; n < n_seqs; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return ORACLE_ERR_ARGS;
  if (col_block <= 0 || col_block > dv) col_block = dv;
  const int64_t n_cb = (dv + col_block - 1) / col_block;
  const int64_t n_tasks = n_seqs * n_heads * n_cb;
  int status = ORACLE_OK;

#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t task = 0; task < n_tasks; ++task) {
    const int64_t cb = task % n_cb;
    const int64_t h = (task / n_cb) % n_heads;
    const int64_t n = task / (n_cb * n_heads);
    const int64_t j0 = cb * col_block;
    const int64_t j1 = (j0 + col_block < dv) ? j0 + col_block : dv;
    const double* h0n = h0 ? h0 + (n * n_heads + h) * dk * dv : NULL;
    double* hTn = hT ? hT + (n * n_heads + h) * dk * dv : NULL;
    int rc = run_dplr_chain(q, k, v, a, b, log_alpha, h0n, cu_seqlens[n], cu_seqlens[n + 1], h,
                            n_heads, dk, dv, j0, j1, o, hTn);
    if (rc != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
      status = rc;
    }
  }
  return status;
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
