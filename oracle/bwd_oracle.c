/*
 * bwd_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain fp64 reverse-mode gradient of the Gated Delta Rule-2 token loop (the
 * erase reading R1 that the GPU implements).  Same rules as the forward oracle:
 * only the tests, the package smoke check and the CPU baseline leg of the
 * benchmark load it; it shares nothing with the CUDA path.
 *
 * Passage: the gradient of the recurrence that "[논문] 게이트형 DeltaNet-2"
 * (euno.news), section "방법론", and "NVIDIA AIがGated DeltaNet-2を発表"
 * (ai.warp-studio.com), section "Gated DeltaNet-2の核心", define:
 *
 *   S'_t = Diag(alpha_t) S_{t-1}
 *   r_t  = S'_t^T a_t,               a_t = b_t (.) k_t
 *   d_t  = u_t - r_t,                u_t = w_t (.) v_t
 *   S_t  = S'_t + k_t d_t^T
 *   o_t  = S_t^T q_t
 *
 * For a loss L with dL/do_t = dO_t and dL/dS_T = dST, the chain rule taken step
 * by step backwards, with G = dL/dS_t (starting from dST):
 *
 *   G      += q_t dO_t^T                        (o_t reads S_t)
 *   dq_t    = S_t dO_t
 *   dd      = G^T k_t,   dk_t = G d_t           (S_t = S'_t + k_t d_t^T)
 *   dv_t    = dd (.) w_t, dw_t = dd (.) v_t     (d_t = u_t - r_t)
 *   da      = -S'_t dd                          (r_t = S'_t^T a_t)
 *   dS'     = G - a_t dd^T
 *   dalpha_t[i] = sum_j dS'[i][j] S_{t-1}[i][j]
 *   G       = Diag(alpha_t) dS'                 (G is now dL/dS_{t-1})
 *   db_t    = da (.) k_t,  dk_t += da (.) b_t
 *
 * and dS0 = G after the first token.  Every state S_0 .. S_len of the head is
 * kept (the plain definition of reverse mode; no recomputation, no blocking).
 *
 * Layouts as in gdn2_oracle.c: dense [N, T, H, d] or packed [T_total, H, d]
 * with cu_seqlens; states [N, H, d_k, d_v].  S0 and dST may be NULL (zeros);
 * dS0 may be NULL (not returned).  Return 0, -1 on a bad argument, -2 when the
 * per-head state history cannot be allocated.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int bwd_one_head(const double *q, const double *k, const double *v, const double *alpha,
                        const double *b, const double *w, const double *S0, const double *dO,
                        const double *dST, double *dq, double *dk, double *dv, double *dalpha, double *db,
                        double *dw, double *dS0, int64_t bos, int64_t len, int H, int h, int DK, int DV,
                        int64_t state_off) {
  const size_t SS = (size_t)DK * DV;
  double *S = (double *)malloc((size_t)(len + 1) * SS * sizeof(double)); /* S_0 .. S_len */
  double *dlt = (double *)malloc((size_t)(len > 0 ? len : 1) * DV * sizeof(double));
  double *G = (double *)malloc(SS * sizeof(double));
  double *dSp = (double *)malloc(SS * sizeof(double));
  double *dd = (double *)malloc((size_t)DV * sizeof(double));
  double *da = (double *)malloc((size_t)DK * sizeof(double));
  if (!S || !dlt || !G || !dSp || !dd || !da) {
    free(S); free(dlt); free(G); free(dSp); free(dd); free(da);
    return -2;
  }
  if (S0) memcpy(S, S0 + state_off, SS * sizeof(double));
  else memset(S, 0, SS * sizeof(double));

  /* forward: keep every state and every d_t */
  for (int64_t t = 0; t < len; ++t) {
    const int64_t ik = ((bos + t) * H + h) * (int64_t)DK, iv = ((bos + t) * H + h) * (int64_t)DV;
    const double *Sprev = S + (size_t)t * SS;
    double *Snew = S + (size_t)(t + 1) * SS;
    for (int j = 0; j < DV; ++j) {
      double r = 0.0;
      for (int i = 0; i < DK; ++i) r += alpha[ik + i] * Sprev[(size_t)i * DV + j] * (b[ik + i] * k[ik + i]);
      dlt[(size_t)t * DV + j] = w[iv + j] * v[iv + j] - r;
    }
    for (int i = 0; i < DK; ++i)
      for (int j = 0; j < DV; ++j)
        Snew[(size_t)i * DV + j] = alpha[ik + i] * Sprev[(size_t)i * DV + j] + k[ik + i] * dlt[(size_t)t * DV + j];
  }

  /* backward */
  if (dST) memcpy(G, dST + state_off, SS * sizeof(double));
  else memset(G, 0, SS * sizeof(double));
  for (int64_t t = len - 1; t >= 0; --t) {
    const int64_t ik = ((bos + t) * H + h) * (int64_t)DK, iv = ((bos + t) * H + h) * (int64_t)DV;
    const double *St = S + (size_t)(t + 1) * SS, *Sprev = S + (size_t)t * SS;
    const double *d_t = dlt + (size_t)t * DV;
    for (int i = 0; i < DK; ++i)
      for (int j = 0; j < DV; ++j) G[(size_t)i * DV + j] += q[ik + i] * dO[iv + j];
    for (int i = 0; i < DK; ++i) {
      double sq = 0.0, sk = 0.0;
      for (int j = 0; j < DV; ++j) {
        sq += St[(size_t)i * DV + j] * dO[iv + j];
        sk += G[(size_t)i * DV + j] * d_t[j];
      }
      dq[ik + i] = sq;
      dk[ik + i] = sk;
    }
    for (int j = 0; j < DV; ++j) {
      double s = 0.0;
      for (int i = 0; i < DK; ++i) s += G[(size_t)i * DV + j] * k[ik + i];
      dd[j] = s;
      dv[iv + j] = s * w[iv + j];
      dw[iv + j] = s * v[iv + j];
    }
    for (int i = 0; i < DK; ++i) {
      const double a_i = b[ik + i] * k[ik + i];
      double s = 0.0, sa = 0.0;
      for (int j = 0; j < DV; ++j) {
        const double sp = alpha[ik + i] * Sprev[(size_t)i * DV + j];
        s -= sp * dd[j];
        dSp[(size_t)i * DV + j] = G[(size_t)i * DV + j] - a_i * dd[j];
        sa += dSp[(size_t)i * DV + j] * Sprev[(size_t)i * DV + j];
      }
      da[i] = s;
      dalpha[ik + i] = sa;
    }
    for (int i = 0; i < DK; ++i) {
      for (int j = 0; j < DV; ++j) G[(size_t)i * DV + j] = alpha[ik + i] * dSp[(size_t)i * DV + j];
      db[ik + i] = da[i] * k[ik + i];
      dk[ik + i] += da[i] * b[ik + i];
    }
  }
  if (dS0) memcpy(dS0 + state_off, G, SS * sizeof(double));
  free(S); free(dlt); free(G); free(dSp); free(dd); free(da);
  return 0;
}

int oracle_gdn2_recurrent_bwd(const double *q, const double *k, const double *v, const double *alpha,
                              const double *b, const double *w, const double *S0, const double *dO,
                              const double *dST, double *dq, double *dk, double *dv, double *dalpha,
                              double *db, double *dw, double *dS0, int N, int T, int H, int DK, int DV,
                              const int64_t *cu, int nthreads) {
  if (N < 0 || T < 0 || H <= 0 || DK <= 0 || DV <= 0) return -1;
  if (!q || !k || !v || !alpha || !b || !w || !dO || !dq || !dk || !dv || !dalpha || !db || !dw) return -1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int rc = 0;
#pragma omp parallel for schedule(dynamic) reduction(min : rc)
  for (int64_t nh = 0; nh < (int64_t)N * H; ++nh) {
    const int n = (int)(nh / H), h = (int)(nh % H);
    const int64_t bos = cu ? cu[n] : (int64_t)n * T, len = cu ? cu[n + 1] - cu[n] : T;
    const int64_t off = nh * (int64_t)DK * DV;
    const int r = len < 0 ? -1
                          : bwd_one_head(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0,
                                         bos, len, H, h, DK, DV, off);
    if (r < rc) rc = r;
  }
  return rc;
}
