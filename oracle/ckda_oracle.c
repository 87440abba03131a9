/*
 * CKDA oracle: plain fp64 CPU recurrence, token by token.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (Semidirect Fourier Delta Attention, §1 eq. (1) and §2.2
 * eq. (9); Complex KDA, abstract, for the widened ranges):
 *
 *     S_t = (I - beta_t k_t k_t^T) diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t                (§3 eq. (14): readout of the
 *                                             state AFTER the update)
 *
 * with alpha_t in [-1,1]^{d_k} (channel-wise gate) and beta_t in [0,2]. The
 * product (I - b k k^T) D S' is expanded into the three in-place steps the
 * "Kimi Delta Attention: a bounded case study" lesson names (per-channel decay
 * S' = diag(a) S in §12.1; read-compare-correct in Exercise 2):
 *
 *     1. gate:    S   <- diag(alpha_t) S
 *     2. read:    p   <- S^T k_t
 *     3. correct: S   <- S + beta_t k_t (v_t - p)^T
 *     4. readout: o_t <- scale * S^T q_t
 *
 * Step 3 equals (I - b k k^T) S + b k v^T exactly in real arithmetic.
 * No blocking, no chunking, no reordering: one token at a time, fp64.
 *
 * Layouts (row-major, C order):
 *   q, k  : [total_T, H, d_k]      v, o : [total_T, H, d_v]
 *   alpha : [total_T, H, d_k]      beta : [total_T, H]
 *   state : [N, H, d_k, d_v]       (d_v contiguous)
 *   cu_seqlens : [N+1], sequence n owns tokens [cu[n], cu[n+1])
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* One recurrence step on one (sequence, head) state S[d_k][d_v], in place.
 * p is caller scratch of d_v doubles. */
static void ckda_oracle_step(double *S, double *p, const double *q,
                             const double *k, const double *v,
                             const double *alpha, double beta, double scale,
                             double *o, int32_t dk, int32_t dv) {
  int32_t r, c;
  /* 1. gate: row r of S is channel r of the key space */
  for (r = 0; r < dk; ++r) {
    const double a = alpha[r];
    double *row = S + (size_t)r * dv;
    for (c = 0; c < dv; ++c) row[c] *= a;
  }
  /* 2. read: p = S^T k */
  for (c = 0; c < dv; ++c) p[c] = 0.0;
  for (r = 0; r < dk; ++r) {
    const double kr = k[r];
    const double *row = S + (size_t)r * dv;
    for (c = 0; c < dv; ++c) p[c] += row[c] * kr;
  }
  /* 3. correct: S += beta k (v - p)^T */
  for (r = 0; r < dk; ++r) {
    const double bk = beta * k[r];
    double *row = S + (size_t)r * dv;
    for (c = 0; c < dv; ++c) row[c] += bk * (v[c] - p[c]);
  }
  /* 4. readout of the updated state: o = scale * S^T q */
  if (o) {
    for (c = 0; c < dv; ++c) p[c] = 0.0;
    for (r = 0; r < dk; ++r) {
      const double qr = q[r];
      const double *row = S + (size_t)r * dv;
      for (c = 0; c < dv; ++c) p[c] += row[c] * qr;
    }
    for (c = 0; c < dv; ++c) o[c] = scale * p[c];
  }
}

/* Forward over packed sequences. initial_state may be NULL (zero state);
 * final_state may be NULL (not written). Returns 0, or -1 on bad arguments,
 * -2 on allocation failure. nthreads <= 0 means the OpenMP default. */
int ckda_oracle_fwd(const double *q, const double *k, const double *v,
                    const double *alpha, const double *beta,
                    const double *initial_state, double *final_state,
                    double *o, const int32_t *cu_seqlens, int32_t N, int32_t H,
                    int32_t dk, int32_t dv, double scale, int32_t nthreads) {
  int64_t nh, total, work;
  int failed = 0;
  if (!q || !k || !v || !alpha || !beta || !o || !cu_seqlens) return -1;
  if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
  if (cu_seqlens[0] != 0) return -1;
  for (nh = 0; nh < N; ++nh)
    if (cu_seqlens[nh + 1] < cu_seqlens[nh]) return -1;
  total = (int64_t)N * H;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (work = 0; work < total; ++work) {
    const int32_t n = (int32_t)(work / H), h = (int32_t)(work % H);
    const size_t ssz = (size_t)dk * dv;
    double *S = (double *)malloc(ssz * sizeof(double));
    double *p = (double *)malloc((size_t)dv * sizeof(double));
    int32_t t;
    if (!S || !p) {
      free(S);
      free(p);
      failed |= 1;
      continue;
    }
    if (initial_state)
      memcpy(S, initial_state + (size_t)work * ssz, ssz * sizeof(double));
    else
      memset(S, 0, ssz * sizeof(double));
    for (t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
      const size_t th = (size_t)t * H + h;
      ckda_oracle_step(S, p, q + th * dk, k + th * dk, v + th * dv,
                       alpha + th * dk, beta[th], scale, o + th * dv, dk, dv);
    }
    if (final_state) memcpy(final_state + (size_t)work * ssz, S, ssz * sizeof(double));
    free(S);
    free(p);
  }
  return failed ? -2 : 0;
}

/* One decode step for N sequences x H heads, one token each, state updated in
 * place. Same four steps as above (the decode step is the recurrence applied
 * once). Token tensors are [N, H, d]; state is [N, H, d_k, d_v].
 * Only the (n, h) pairs listed in `pairs` (flattened n*H+h) are stepped when
 * pairs != NULL; npairs gives their count. */
int ckda_oracle_decode(const double *q, const double *k, const double *v,
                       const double *alpha, const double *beta, double *state,
                       double *o, int32_t N, int32_t H, int32_t dk, int32_t dv,
                       double scale, const int64_t *pairs, int64_t npairs,
                       int32_t nthreads) {
  int64_t i, count;
  int failed = 0;
  if (!q || !k || !v || !alpha || !beta || !state || !o) return -1;
  if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
  count = pairs ? npairs : (int64_t)N * H;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 4) reduction(| : failed)
  for (i = 0; i < count; ++i) {
    const int64_t w = pairs ? pairs[i] : i;
    double *p;
    if (w < 0 || w >= (int64_t)N * H) {
      failed |= 1;
      continue;
    }
    p = (double *)malloc((size_t)dv * sizeof(double));
    if (!p) {
      failed |= 2;
      continue;
    }
    ckda_oracle_step(state + (size_t)w * dk * dv, p, q + (size_t)w * dk,
                     k + (size_t)w * dk, v + (size_t)w * dv,
                     alpha + (size_t)w * dk, beta[w], scale,
                     o + (size_t)w * dv, dk, dv);
    free(p);
  }
  return failed ? -1 : 0;
}

int ckda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
