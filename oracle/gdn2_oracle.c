/*
 * gdn2_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct fp64 CPU implementation of the Gated Delta
 * Rule-2 recurrence.  Only the tests, the package smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA path, and it never calls it.
 *
 * What it computes (per sequence n and head h, state S of shape d_k x d_v,
 * row index = key channel, column index = value channel):
 *
 *   for every token t of the sequence, in order:
 *     1. decay on the key axis first:        S <- Diag(alpha_t) S
 *     2. erase, gated per key channel:       r <- S^T (b_t (.) k_t)
 *     3. write, gated per value channel:     S <- S + k_t (w_t (.) v_t - r)^T
 *     4. readout from the edited state:      o_t <- S^T q_t
 *
 * Passages followed (pages on Gated DeltaNet-2, arXiv 2605.22791):
 *  - "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section
 *    "Gated DeltaNet-2の核心": per-channel erase gate b_t on the key axis,
 *    per-channel write gate w_t on the value axis, both sigmoid projections,
 *    decay applied before the active edit; reductions to KDA and Gated DeltaNet.
 *  - "[논문] 게이트형 DeltaNet-2" (euno.news), section "방법론", steps 1-3:
 *    read with a linear-attention query, b_t decides how much old key content
 *    is discarded, w_t how much new value is injected, KDA-style per-channel
 *    decay.
 *  - "Gated DeltaNet-2: Separando Borrado y Escritura en la Atención Lineal"
 *    (needhelp.icu), gate table in "Gated DeltaNet-2: La Solución".
 *
 * Readings taken where the pages print no equation (each is listed in the
 * design notes of the repository):
 *  - erase orientation: the erase is k_t (b_t (.) k_t)^T applied to the decayed
 *    state (ERASE_R1).  The other orientation, (b_t (.) k_t) k_t^T (ERASE_R2),
 *    is kept behind the `orientation` switch for comparison.
 *  - readout uses the state after the edit of step t (o_t = S_t^T q_t).
 *  - the write of step t is not decayed at step t.
 *  - no 1/sqrt(d_k) query scale; q and k arrive already normalised.
 *
 * Layouts (all arrays fp64, row-major, caller-owned host memory):
 *  - dense batch (cu_seqlens == NULL): q, k, alpha, b are [N, T, H, d_k];
 *    v, w, o are [N, T, H, d_v];
 *  - packed varlen (cu_seqlens != NULL, N+1 entries): the same tensors are
 *    [T_total, H, d], sequence n spans tokens cu_seqlens[n] .. cu_seqlens[n+1]-1,
 *    and T is ignored;
 *  - S0, ST: [N, H, d_k, d_v]; S0 == NULL means a zero initial state; ST may be
 *    NULL; ST may alias S0.
 * Return value: 0 on success, -1 on an invalid argument, -2 when memory for the
 * per-head working state cannot be allocated.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ERASE_R1 0 /* S_t = (I - k a^T) D S + k u^T, a = b (.) k  (adopted) */
#define ERASE_R2 1 /* S_t = (I - a k^T) D S + k u^T                       */

/* Planted mistakes, used only by the test that checks the pins catch them. */
enum {
  PLANT_NONE = 0,
  PLANT_NO_DECAY = 1,          /* step 1 skipped                         */
  PLANT_ERASE_SIGN = 2,        /* r added instead of subtracted          */
  PLANT_READ_BEFORE_EDIT = 3,  /* o_t read from the decayed, unedited S  */
  PLANT_DECAY_AFTER_EDIT = 4,  /* decay applied after the edit           */
  PLANT_NO_WRITE_GATE = 5,     /* w_t ignored                            */
  PLANT_NO_ERASE_GATE = 6,     /* b_t ignored                            */
  PLANT_READOUT_TRANSPOSED = 7,/* o_t = S q_t (needs d_k == d_v)          */
  PLANT_ERASE_UNDECAYED = 8,   /* r taken from S before the decay        */
  PLANT_GATES_SWAPPED = 9,     /* b on the value side, w on the key side (d_k == d_v) */
  PLANT_COUNT = 10
};

static void seq_span(const int64_t *cu, int n, int T, int64_t *bos, int64_t *len) {
  if (cu) { *bos = cu[n]; *len = cu[n + 1] - cu[n]; }
  else    { *bos = (int64_t)n * T; *len = T; }
}

/* One (sequence, head) pair, token by token. */
static int run_one_head(const double *q, const double *k, const double *v,
                        const double *alpha, const double *b, const double *w,
                        const double *S0, double *o, double *ST,
                        int64_t bos, int64_t len, int n, int h, int H, int dk, int dv,
                        int orientation, int plant) {
  double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
  double *r = (double *)malloc(sizeof(double) * (size_t)dv);
  double *a = (double *)malloc(sizeof(double) * (size_t)dk);
  double *u = (double *)malloc(sizeof(double) * (size_t)dv);
  double *Sold = (double *)malloc(sizeof(double) * (size_t)dk * dv);
  if (!S || !r || !a || !u || !Sold) { free(S); free(r); free(a); free(u); free(Sold); return -2; }

  const size_t sidx = ((size_t)n * H + h) * (size_t)dk * dv;
  for (size_t e = 0; e < (size_t)dk * dv; ++e) S[e] = S0 ? S0[sidx + e] : 0.0;

  for (int64_t t = 0; t < len; ++t) {
    const size_t row = (size_t)(bos + t) * H + h;
    const double *qt = q + row * dk, *kt = k + row * dk, *at = alpha + row * dk, *bt = b + row * dk;
    const double *vt = v + row * dv, *wt = w + row * dv;
    double *ot = o ? o + row * dv : NULL;

    /* gated erase probe a_t = b_t (.) k_t and gated write value u_t = w_t (.) v_t */
    for (int i = 0; i < dk; ++i) a[i] = (plant == PLANT_NO_ERASE_GATE ? 1.0 : bt[i]) * kt[i];
    for (int j = 0; j < dv; ++j) u[j] = (plant == PLANT_NO_WRITE_GATE ? 1.0 : wt[j]) * vt[j];
    if (plant == PLANT_GATES_SWAPPED) {
      for (int i = 0; i < dk; ++i) a[i] = wt[i] * kt[i];
      for (int j = 0; j < dv; ++j) u[j] = bt[j] * vt[j];
    }

    if (plant == PLANT_ERASE_UNDECAYED) memcpy(Sold, S, sizeof(double) * (size_t)dk * dv);

    /* 1. per-key-channel decay, before the edit */
    if (plant != PLANT_NO_DECAY && plant != PLANT_DECAY_AFTER_EDIT)
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= at[i];

    if (plant == PLANT_READ_BEFORE_EDIT && ot)
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qt[i];
        ot[j] = acc;
      }

    const double *Sr = (plant == PLANT_ERASE_UNDECAYED) ? Sold : S;
    if (orientation == ERASE_R1) {
      /* 2. r = S^T a  (what the key-side probe currently reads out) */
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += Sr[(size_t)i * dv + j] * a[i];
        r[j] = acc;
      }
      /* 3. S += k (u - r)^T : erase and write share the key vector k */
      const double sgn = (plant == PLANT_ERASE_SIGN) ? 1.0 : -1.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += kt[i] * (u[j] + sgn * r[j]);
    } else {
      /* R2: S <- (I - a k^T) S + k u^T, i.e. r = S^T k erased along a */
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += Sr[(size_t)i * dv + j] * kt[i];
        r[j] = acc;
      }
      const double sgn = (plant == PLANT_ERASE_SIGN) ? 1.0 : -1.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
          S[(size_t)i * dv + j] += sgn * a[i] * r[j] + kt[i] * u[j];
    }

    if (plant == PLANT_DECAY_AFTER_EDIT)
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= at[i];

    /* 4. readout o_t = S_t^T q_t */
    if (ot && plant != PLANT_READ_BEFORE_EDIT) {
      if (plant == PLANT_READOUT_TRANSPOSED) {
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dv + i] * qt[i];
          ot[j] = acc;
        }
      } else {
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qt[i];
          ot[j] = acc;
        }
      }
    }
  }

  if (ST) memcpy(ST + sidx, S, sizeof(double) * (size_t)dk * dv);
  free(S); free(r); free(a); free(u); free(Sold);
  return 0;
}

static int check_args(const double *q, const double *k, const double *v, const double *alpha,
                      const double *b, const double *w, int N, int T, int H, int dk, int dv,
                      const int64_t *cu) {
  if (!q || !k || !v || !alpha || !b || !w) return -1;
  if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
  if (!cu && T < 0) return -1;
  if (cu) for (int n = 0; n < N; ++n) if (cu[n + 1] < cu[n]) return -1;
  return 0;
}

static int recurrent_impl(const double *q, const double *k, const double *v, const double *alpha,
                          const double *b, const double *w, const double *S0, double *o,
                          double *ST, int N, int T, int H, int dk, int dv, const int64_t *cu,
                          int orientation, int plant, int nthreads) {
  if (check_args(q, k, v, alpha, b, w, N, T, H, dk, dv, cu)) return -1;
  if (orientation != ERASE_R1 && orientation != ERASE_R2) return -1;
  if ((plant == PLANT_READOUT_TRANSPOSED || plant == PLANT_GATES_SWAPPED) && dk != dv) return -1;
  int status = 0;
  const int pairs = N * H;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(min : status)
#endif
  for (int p = 0; p < pairs; ++p) {
    const int n = p / H, h = p % H;
    int64_t bos, len;
    seq_span(cu, n, T, &bos, &len);
    int s = run_one_head(q, k, v, alpha, b, w, S0, o, ST, bos, len, n, h, H, dk, dv,
                         orientation, plant);
    if (s < status) status = s;
  }
  (void)nthreads;
  return status;
}

/* The oracle: the token-by-token recurrence (reading ERASE_R1 unless asked). */
int oracle_gdn2_recurrent(const double *q, const double *k, const double *v, const double *alpha,
                          const double *b, const double *w, const double *S0, double *o,
                          double *ST, int N, int T, int H, int dk, int dv,
                          const int64_t *cu_seqlens, int orientation, int nthreads) {
  return recurrent_impl(q, k, v, alpha, b, w, S0, o, ST, N, T, H, dk, dv, cu_seqlens,
                        orientation, PLANT_NONE, nthreads);
}

/* The same loop with one deliberate mistake planted; for the pin-coverage test only. */
int oracle_gdn2_recurrent_planted(const double *q, const double *k, const double *v,
                                  const double *alpha, const double *b, const double *w,
                                  const double *S0, double *o, double *ST, int N, int T, int H,
                                  int dk, int dv, const int64_t *cu_seqlens, int plant) {
  if (plant < 0 || plant >= PLANT_COUNT) return -1;
  return recurrent_impl(q, k, v, alpha, b, w, S0, o, ST, N, T, H, dk, dv, cu_seqlens, ERASE_R1,
                        plant, 1);
}

int oracle_plant_count(void) { return PLANT_COUNT; }

/*
 * Companion: the chunkwise WY form of the same recurrence (reading ERASE_R1),
 * in fp64 with plain loops.  It follows the block formulation that the pages
 * describe ("Innovaciones Técnicas", item 1 "Algoritmo WY por Bloques", on the
 * needhelp.icu page; "주요 기여", "효율적인 구현" on the euno.news page): the
 * per-channel decay is folded into asymmetric erase factors so that a chunk of
 * C tokens becomes one unit-lower-triangular system.
 *
 * For one chunk with entering state S0 (tokens r, i = 0..C-1 inside the chunk):
 *   g_r      = sum_{s<=r} log alpha_s             (per key channel)
 *   L[r][i]  = sum_c a_rc k_ic exp(g_rc - g_ic),  i < r   (erase interaction)
 *   rhs_r    = u_r - S0^T (exp(g_r) (.) a_r)
 *   delta_r  = rhs_r - sum_{i<r} L[r][i] delta_i  (forward substitution)
 *   o_r      = S0^T (exp(g_r) (.) q_r) + sum_{i<=r} P[r][i] delta_i,
 *              P[r][i] = sum_c q_rc k_ic exp(g_rc - g_ic)
 *   S_C      = Diag(exp(g_{C-1})) S0 + sum_i Diag(exp(g_{C-1} - g_i)) k_i delta_i^T
 * delta_r is exactly u_r - (D_r S_{r-1})^T a_r of the token loop, so this is
 * an identity, not an approximation.  The last chunk of a sequence may be short.
 */
static int chunk_one_head(const double *q, const double *k, const double *v, const double *alpha,
                          const double *b, const double *w, const double *S0, double *o,
                          double *ST, int64_t bos, int64_t len, int n, int h, int H, int dk,
                          int dv, int C) {
  double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
  double *Snew = (double *)malloc(sizeof(double) * (size_t)dk * dv);
  double *g = (double *)malloc(sizeof(double) * (size_t)C * dk);
  double *L = (double *)malloc(sizeof(double) * (size_t)C * C);
  double *P = (double *)malloc(sizeof(double) * (size_t)C * C);
  double *D = (double *)malloc(sizeof(double) * (size_t)C * dv);
  if (!S || !Snew || !g || !L || !P || !D) {
    free(S); free(Snew); free(g); free(L); free(P); free(D);
    return -2;
  }
  const size_t sidx = ((size_t)n * H + h) * (size_t)dk * dv;
  for (size_t e = 0; e < (size_t)dk * dv; ++e) S[e] = S0 ? S0[sidx + e] : 0.0;

  for (int64_t c0 = 0; c0 < len; c0 += C) {
    const int Cc = (int)((len - c0) < C ? (len - c0) : C);
#define ROW(t) ((size_t)(bos + c0 + (t)) * H + h)
    /* cumulative log-decay inside the chunk */
    for (int r = 0; r < Cc; ++r)
      for (int c = 0; c < dk; ++c)
        g[(size_t)r * dk + c] = log(alpha[ROW(r) * dk + c]) + (r ? g[(size_t)(r - 1) * dk + c] : 0.0);
    /* erase-interaction (strictly lower) and query-key (inclusive lower) maps */
    for (int r = 0; r < Cc; ++r)
      for (int i = 0; i < Cc; ++i) {
        double l = 0.0, p = 0.0;
        if (i <= r)
          for (int c = 0; c < dk; ++c) {
            const double f = exp(g[(size_t)r * dk + c] - g[(size_t)i * dk + c]) * k[ROW(i) * dk + c];
            l += b[ROW(r) * dk + c] * k[ROW(r) * dk + c] * f;
            p += q[ROW(r) * dk + c] * f;
          }
        L[(size_t)r * C + i] = (i < r) ? l : 0.0;
        P[(size_t)r * C + i] = (i <= r) ? p : 0.0;
      }
    /* right-hand side, then forward substitution with the unit-lower (I + L) */
    for (int r = 0; r < Cc; ++r)
      for (int j = 0; j < dv; ++j) {
        double acc = w[ROW(r) * dv + j] * v[ROW(r) * dv + j];
        for (int c = 0; c < dk; ++c)
          acc -= exp(g[(size_t)r * dk + c]) * b[ROW(r) * dk + c] * k[ROW(r) * dk + c] * S[(size_t)c * dv + j];
        for (int i = 0; i < r; ++i) acc -= L[(size_t)r * C + i] * D[(size_t)i * dv + j];
        D[(size_t)r * dv + j] = acc;
      }
    /* outputs */
    if (o)
      for (int r = 0; r < Cc; ++r)
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int c = 0; c < dk; ++c)
            acc += exp(g[(size_t)r * dk + c]) * q[ROW(r) * dk + c] * S[(size_t)c * dv + j];
          for (int i = 0; i <= r; ++i) acc += P[(size_t)r * C + i] * D[(size_t)i * dv + j];
          o[ROW(r) * dv + j] = acc;
        }
    /* state carried to the next chunk */
    const double *gl = g + (size_t)(Cc - 1) * dk;
    for (int c = 0; c < dk; ++c)
      for (int j = 0; j < dv; ++j) {
        double acc = exp(gl[c]) * S[(size_t)c * dv + j];
        for (int i = 0; i < Cc; ++i)
          acc += exp(gl[c] - g[(size_t)i * dk + c]) * k[ROW(i) * dk + c] * D[(size_t)i * dv + j];
        Snew[(size_t)c * dv + j] = acc;
      }
    memcpy(S, Snew, sizeof(double) * (size_t)dk * dv);
#undef ROW
  }
  if (ST) memcpy(ST + sidx, S, sizeof(double) * (size_t)dk * dv);
  free(S); free(Snew); free(g); free(L); free(P); free(D);
  return 0;
}

int oracle_gdn2_chunkwise(const double *q, const double *k, const double *v, const double *alpha,
                          const double *b, const double *w, const double *S0, double *o,
                          double *ST, int N, int T, int H, int dk, int dv,
                          const int64_t *cu_seqlens, int chunk, int nthreads) {
  if (check_args(q, k, v, alpha, b, w, N, T, H, dk, dv, cu_seqlens)) return -1;
  if (chunk <= 0) return -1;
  int status = 0;
  const int pairs = N * H;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(min : status)
#endif
  for (int p = 0; p < pairs; ++p) {
    const int n = p / H, h = p % H;
    int64_t bos, len;
    seq_span(cu_seqlens, n, T, &bos, &len);
    int s = chunk_one_head(q, k, v, alpha, b, w, S0, o, ST, bos, len, n, h, H, dk, dv, chunk);
    if (s < status) status = s;
  }
  (void)nthreads;
  return status;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
