/*
 * block_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain fp64 CPU definitions of the elementwise and short-convolution work
 * around the Gated Delta Rule-2 mixer in its block.  Same rules as the
 * recurrence oracle: only the tests, the package smoke check and the CPU
 * baseline leg of the benchmark load it; it shares nothing with the CUDA path.
 *
 * Passage followed: "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com),
 * section "アーキテクチャとパフォーマンスベンチマーク": the query and key paths
 * are a linear projection, a short causal convolution, SiLU and L2
 * normalisation; the value path a projection, a short convolution and SiLU;
 * the decay, the erase gate and the write gate come from their own linear
 * branches; the recurrent output is RMS-normalised and multiplied by a SiLU
 * output gate before the output projection.  The projections themselves are
 * plain matrix products and are not part of this code: its inputs are their
 * outputs ("pre-activations").
 *
 * Readings taken where the pages give no formula (listed in the design notes):
 *  - the convolution is depthwise over the H*d channels of a path, of length K
 *    (1..4), causal, restarting at every sequence start:
 *        y_t[c] = sum_{j=0}^{K-1} W[c][K-1-j] x_{t-j}[c],  x before the start = 0
 *    (the last tap multiplies the current token);
 *  - SiLU(y) = y / (1 + e^-y); L2 normalisation over d_k per (token, head):
 *        q = s / sqrt(sum s^2 + 1e-6);
 *  - decay alpha = exp(-softplus(x)) = 1 / (1 + e^x); gates b, w = sigmoid(x);
 *  - output: y = o / sqrt(mean_j o_j^2 + 1e-5) * g[j] * SiLU(z), the RMS over the
 *    d_v values of one (token, head), g a weight of d_v entries shared by heads.
 *
 * Layouts: token tensors [tokens, H, d] (a dense batch is N*T tokens, sequence
 * n = tokens n*T .. n*T+T-1; a packed batch gives N+1 offsets cu_seqlens);
 * convolution weights [H*d, K].  fp64 everywhere.  Return 0, or -1 on a bad
 * argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

static double silu(double y) { return y / (1.0 + exp(-y)); }
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* First token of the sequence holding token t. */
static int64_t seq_start(const int64_t *cu, int N, int T, int64_t t) {
  if (!cu) return (t / T) * (int64_t)T;
  int lo = 0, hi = N;
  while (lo < hi) { /* largest n with cu[n] <= t */
    int mid = (lo + hi + 1) / 2;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return cu[lo];
}

/* One convolved, activated path: out[t][h][c] = SiLU(conv(x))[t][h][c], L2-normalised per (t, h)
 * over its d channels when `l2` is set. */
static void conv_path(const double *x, const double *W, double *out, int64_t tokens, int H, int d, int K,
                      const int64_t *cu, int N, int T, int l2) {
  for (int64_t t = 0; t < tokens; ++t) {
    const int64_t bos = seq_start(cu, N, T, t);
    for (int h = 0; h < H; ++h) {
      double ss = 0.0;
      for (int c = 0; c < d; ++c) {
        const int ch = h * d + c;
        double y = 0.0;
        for (int j = 0; j < K; ++j) {
          const int64_t s = t - j;
          if (s < bos) break;
          y += W[(int64_t)ch * K + (K - 1 - j)] * x[(s * H + h) * (int64_t)d + c];
        }
        const double a = silu(y);
        out[(t * H + h) * (int64_t)d + c] = a;
        ss += a * a;
      }
      if (l2) {
        const double inv = 1.0 / sqrt(ss + 1e-6);
        for (int c = 0; c < d; ++c) out[(t * H + h) * (int64_t)d + c] *= inv;
      }
    }
  }
}

int oracle_block_prologue(const double *xq, const double *xk, const double *xv, const double *xa,
                          const double *xb, const double *xw, const double *Wq, const double *Wk,
                          const double *Wv, double *q, double *k, double *v, double *alpha, double *b,
                          double *w, int N, int T, int H, int dk, int dv, int K, const int64_t *cu) {
  if (N < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || K < 1 || K > 4) return -1;
  const int64_t tokens = cu ? cu[N] : (int64_t)N * T;
  if (!cu && T == 0 && N > 0) return 0;
  conv_path(xq, Wq, q, tokens, H, dk, K, cu, N, T, 1);
  conv_path(xk, Wk, k, tokens, H, dk, K, cu, N, T, 1);
  conv_path(xv, Wv, v, tokens, H, dv, K, cu, N, T, 0);
  for (int64_t e = 0; e < tokens * H * (int64_t)dk; ++e) {
    alpha[e] = 1.0 / (1.0 + exp(xa[e])); /* exp(-softplus(x)) */
    b[e] = sigmoid(xb[e]);
  }
  for (int64_t e = 0; e < tokens * H * (int64_t)dv; ++e) w[e] = sigmoid(xw[e]);
  return 0;
}

int oracle_block_epilogue(const double *o, const double *z, const double *g, double *y, int64_t tokens, int H,
                          int dv) {
  if (tokens < 0 || H <= 0 || dv <= 0) return -1;
  for (int64_t r = 0; r < tokens * H; ++r) {
    double ms = 0.0;
    for (int j = 0; j < dv; ++j) ms += o[r * dv + j] * o[r * dv + j];
    const double inv = 1.0 / sqrt(ms / dv + 1e-5);
    for (int j = 0; j < dv; ++j) y[r * dv + j] = o[r * dv + j] * inv * g[j] * silu(z[r * dv + j]);
  }
  return 0;
}
