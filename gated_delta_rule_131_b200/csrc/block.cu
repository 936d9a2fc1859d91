// The elementwise and short-convolution work around the Gated Delta Rule-2 mixer in its block:
// "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section
// "アーキテクチャとパフォーマンスベンチマーク" -- q and k: short causal convolution, SiLU, L2
// normalisation; v: short convolution, SiLU; decay and gates from their own linear branches
// (alpha = exp(-softplus), b, w = sigmoid); after the mixer, RMS normalisation times a SiLU output
// gate.  The projections around them are plain matrix products and are not part of this file.
//
// All three kernels are HBM-bound streams: every input element is read once and every output
// element written once, in fp32 arithmetic.
#include <algorithm>

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int TT = 64;          // tokens per convolution tile
constexpr float L2_EPS = 1e-6f, RMS_EPS = 1e-5f;

__device__ __forceinline__ float silu(float y) { return y / (1.f + __expf(-y)); }
__device__ __forceinline__ float sigmoid(float x) { return 1.f / (1.f + __expf(-x)); }

struct ConvPath {
  const void *x;
  const float *W;  // [H * d, K]
  void *out;
  int d;
  int l2;          // normalise each (token, head) to unit L2 norm over its d channels
};
struct ConvArgs {
  ConvPath path[3];  // q, k, v
  const int32_t *cu;
  int N, T, H, K;
  long long tokens;
};

// First token of the sequence holding token t.
__device__ __forceinline__ long long seq_start(const ConvArgs &a, long long t) {
  if (!a.cu) return (t / a.T) * (long long)a.T;
  int lo = 0, hi = a.N;
  while (lo < hi) {  // largest n with cu[n] <= t
    const int mid = (lo + hi + 1) >> 1;
    if (a.cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return a.cu[lo];
}

// One CTA per (64-token tile, head, path); thread = channel, walking the tile's tokens with the
// convolution window in registers; blockDim = d of the path (64, 128 or 256).
template <typename T>
__global__ void __launch_bounds__(256) conv_silu_kernel(const ConvArgs a) {
  __shared__ long long s_bos[TT];
  __shared__ float s_out[TT][128 + 1];  // activated q or k of the tile (d_k <= 128)
  const ConvPath P = blockIdx.z == 0 ? a.path[0] : (blockIdx.z == 1 ? a.path[1] : a.path[2]);
  const int d = P.d, c = threadIdx.x;
  const bool act = c < d;  // the q/k launches use d_k threads of a block sized for d_v (whole warps)
  const int h = blockIdx.y;
  const long long t0 = (long long)blockIdx.x * TT;
  const int nt = (int)min((long long)TT, a.tokens - t0);
  for (int i = c; i < nt; i += blockDim.x) s_bos[i] = seq_start(a, t0 + i);
  __syncthreads();
  const T *x = reinterpret_cast<const T *>(P.x);
  T *out = reinterpret_cast<T *>(P.out);
  const size_t stride = (size_t)a.H * d;  // elements between consecutive tokens
  if (act) {
    const size_t col = (size_t)h * d + c;
    float wr[4];  // wr[j] multiplies x_{t-j}: the taps in reverse (the last tap is the current token)
#pragma unroll
    for (int j = 0; j < 4; ++j) wr[j] = j < a.K ? P.W[col * a.K + (a.K - 1 - j)] : 0.f;
    // window: xs[j] = x_{t-j} for j = 1..K-1 (zero before the sequence start)
    float xs[4] = {0.f, 0.f, 0.f, 0.f};
    const long long bos0 = s_bos[0];
#pragma unroll
    for (int j = 1; j < 4; ++j)
      if (j < a.K && t0 - j >= bos0) xs[j] = to_f32(x[(size_t)(t0 - j) * stride + col]);
#pragma unroll 8
    for (int i = 0; i < nt; ++i) {
      const long long t = t0 + i;
      if (i > 0 && s_bos[i] == t) xs[1] = xs[2] = xs[3] = 0.f;  // a new sequence starts at t
      const float xt = to_f32(x[(size_t)t * stride + col]);
      float y = wr[0] * xt;  // sum_j W[K-1-j] x_{t-j}, current token first (wr[j] = 0 for j >= K)
#pragma unroll
      for (int j = 1; j < 4; ++j) y = fmaf(wr[j], xs[j], y);
      const float s = silu(y);
      if (P.l2) s_out[i][c] = s;
      else out[(size_t)t * stride + col] = from_f32<T>(s);
      xs[3] = xs[2];
      xs[2] = xs[1];
      xs[1] = xt;
    }
  }
  if (!P.l2) return;  // uniform per block
  __syncthreads();
  // L2 normalisation: one warp per token, lanes over the channels
  const int warp = c >> 5, lane = c & 31, nw = d >> 5;
  if (!act) return;
  for (int i = warp; i < nt; i += nw) {
    float ss = 0.f;
    for (int e = lane; e < d; e += 32) ss = fmaf(s_out[i][e], s_out[i][e], ss);
    ss = warp_allreduce_sum(ss);
    const float inv = rsqrtf(ss + L2_EPS);
    for (int e = lane; e < d; e += 32) out[(size_t)(t0 + i) * stride + (size_t)h * d + e] = from_f32<T>(s_out[i][e] * inv);
  }
}

// alpha = exp(-softplus(x)) = 1 / (1 + e^x), b = sigmoid(x) over [tokens, H, d_k]; w = sigmoid(x)
// over [tokens, H, d_v].  One 16-byte vector per thread and step (both sizes are multiples of it).
template <typename T>
__global__ void __launch_bounds__(256) gates_kernel(const T *xa, const T *xb, const T *xw, T *alpha, T *b, T *w,
                                                    size_t nk, size_t nv) {
  constexpr int V = 16 / sizeof(T);
  const size_t stride = (size_t)gridDim.x * blockDim.x, nkv = nk / V, nvv = nv / V;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < nkv + nvv; e += stride) {
    if (e < nkv) {
      const uint4 ua = reinterpret_cast<const uint4 *>(xa)[e], ub = reinterpret_cast<const uint4 *>(xb)[e];
      const T *pa = reinterpret_cast<const T *>(&ua), *pb = reinterpret_cast<const T *>(&ub);
      uint4 ra, rb;
      T *qa = reinterpret_cast<T *>(&ra), *qb = reinterpret_cast<T *>(&rb);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        qa[i] = from_f32<T>(1.f / (1.f + __expf(to_f32(pa[i]))));
        qb[i] = from_f32<T>(sigmoid(to_f32(pb[i])));
      }
      reinterpret_cast<uint4 *>(alpha)[e] = ra;
      reinterpret_cast<uint4 *>(b)[e] = rb;
    } else {
      const size_t f = e - nkv;
      const uint4 uw = reinterpret_cast<const uint4 *>(xw)[f];
      const T *pw = reinterpret_cast<const T *>(&uw);
      uint4 rw;
      T *qw = reinterpret_cast<T *>(&rw);
#pragma unroll
      for (int i = 0; i < V; ++i) qw[i] = from_f32<T>(sigmoid(to_f32(pw[i])));
      reinterpret_cast<uint4 *>(w)[f] = rw;
    }
  }
}

// y = o / sqrt(mean_j o_j^2 + eps) * g_j * SiLU(z_j) over the d_v values of one (token, head):
// one warp per row.
template <typename T>
__global__ void __launch_bounds__(256) rms_gate_kernel(const T *o, const T *z, const float *g, T *y, long long rows,
                                                       int dv) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T *orow = o + (size_t)row * dv;
  float ov[8];
  float ss = 0.f;
  const int per = dv >> 5;  // 2, 4 or 8
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < per) {
      ov[i] = to_f32(orow[lane + 32 * i]);
      ss = fmaf(ov[i], ov[i], ss);
    }
  ss = warp_allreduce_sum(ss);
  const float inv = rsqrtf(ss / dv + RMS_EPS);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < per) {
      const int j = lane + 32 * i;
      y[(size_t)row * dv + j] = from_f32<T>(ov[i] * inv * g[j] * silu(to_f32(z[(size_t)row * dv + j])));
    }
}

template <typename T>
cudaError_t prologue_t(const BlockPrologueArgs &p, cudaStream_t stream) {
  ConvArgs a{};
  a.path[0] = ConvPath{p.xq, p.Wq, p.q, p.dk, 1};
  a.path[1] = ConvPath{p.xk, p.Wk, p.k, p.dk, 1};
  a.path[2] = ConvPath{p.xv, p.Wv, p.v, p.dv, 0};
  a.cu = p.cu;
  a.N = p.B;
  a.T = p.T;
  a.H = p.H;
  a.K = p.K;
  a.tokens = p.tokens;
  if (p.tokens > 0) {
    const dim3 grid((unsigned)((p.tokens + TT - 1) / TT), (unsigned)p.H, 3);
    note_launch();
    conv_silu_kernel<T><<<grid, std::max(p.dk, p.dv), 0, stream>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const size_t nk = (size_t)p.tokens * p.H * p.dk, nv = (size_t)p.tokens * p.H * p.dv;
    const size_t vecs = (nk + nv) / (16 / sizeof(T));
    const unsigned blocks = (unsigned)std::min<size_t>((vecs + 255) / 256, (size_t)148 * 16);
    note_launch();
    gates_kernel<T><<<blocks, 256, 0, stream>>>(static_cast<const T *>(p.xa), static_cast<const T *>(p.xb),
                                                 static_cast<const T *>(p.xw), static_cast<T *>(p.alpha),
                                                 static_cast<T *>(p.b), static_cast<T *>(p.w), nk, nv);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

template <typename T>
cudaError_t epilogue_t(const BlockEpilogueArgs &p, cudaStream_t stream) {
  const long long rows = p.tokens * p.H;
  if (rows == 0) return cudaSuccess;
  note_launch();
  rms_gate_kernel<T><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, stream>>>(
      static_cast<const T *>(p.o), static_cast<const T *>(p.z), p.g, static_cast<T *>(p.y), rows, p.dv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_prologue(const BlockPrologueArgs &p, bool bf16, cudaStream_t stream) {
  return bf16 ? prologue_t<__nv_bfloat16>(p, stream) : prologue_t<float>(p, stream);
}

cudaError_t launch_block_epilogue(const BlockEpilogueArgs &p, bool bf16, cudaStream_t stream) {
  return bf16 ? epilogue_t<__nv_bfloat16>(p, stream) : epilogue_t<float>(p, stream);
}

}  // namespace gdn2
