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

// 16-byte asynchronous copy global -> shared (L2 only), and the wait for all of this thread's copies.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float silu(float y) { return __fdividef(y, 1.f + __expf(-y)); }
__device__ __forceinline__ float sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

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

// One CTA of 256 threads per (64-token tile, head, path).  The tile's input rows (and the 3 rows
// before it) are staged in shared memory with 16-byte loads.  Thread = (channel, run of tokens): it
// keeps its channel's taps and convolution window in registers and walks its run from shared
// memory into an output tile; for q and k each token is then L2-normalised by one warp (from the
// activated values as stored), and the tile leaves with 16-byte stores.  Dynamic shared memory:
// (2 TT + 3) rows of the widest path.
template <typename T>
__global__ void __launch_bounds__(256) conv_silu_kernel(const ConvArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ int s_start[TT];  // per token of the tile: index (relative to the tile) of its sequence's first token
  const ConvPath P = blockIdx.z == 0 ? a.path[0] : (blockIdx.z == 1 ? a.path[1] : a.path[2]);
  const int d = P.d, tid = threadIdx.x;
  const int h = blockIdx.y;
  const long long t0 = (long long)blockIdx.x * TT;
  const int nt = (int)min((long long)TT, a.tokens - t0);
  const int halo = (int)min(t0, 3LL);  // staged rows before the tile
  const int nrows = nt + halo;
  T *__restrict__ tin = reinterpret_cast<T *>(dsm);       // [nrows][d], row halo + i = token t0 + i
  T *__restrict__ tout = tin + (TT + 3) * d;               // [nt][d]
  const T *x = reinterpret_cast<const T *>(P.x);
  T *out = reinterpret_cast<T *>(P.out);
  const size_t stride = (size_t)a.H * d;  // elements between consecutive tokens
  constexpr int V = 16 / sizeof(T);       // elements per 16-byte vector
  const int vrow = d / V;
  const T *xbase = x + (size_t)(t0 - halo) * stride + (size_t)h * d;
  for (int i = tid; i < nt; i += 256) s_start[i] = (int)max(seq_start(a, t0 + i) - t0, -4LL);
  for (int e = tid; e < nrows * vrow; e += 256) {  // all of the tile's loads in flight at once
    const int r = e / vrow, vc = e - r * vrow;
    cp_async16(reinterpret_cast<uint4 *>(tin) + e, reinterpret_cast<const uint4 *>(xbase + (size_t)r * stride) + vc);
  }
  cp_async_wait_all();
  __syncthreads();
  {
    const int per = (256 / d);           // threads per channel: 1, 2 or 4
    const int c = tid % d, run = TT / per, i0 = (tid / d) * run;
    const float *W = P.W + ((size_t)h * d + c) * a.K;
    float wr[4];  // wr[j] multiplies x_{t-j}: the taps in reverse (the last tap is the current token)
#pragma unroll
    for (int j = 0; j < 4; ++j) wr[j] = j < a.K ? W[a.K - 1 - j] : 0.f;
    // window xs[j] = x_{t-j}, j = 1..3, for t = t0 + i0 (zero before the sequence start)
    float xs[4] = {0.f, 0.f, 0.f, 0.f};
    const int st0 = i0 < nt ? s_start[i0] : 0;
#pragma unroll
    for (int j = 1; j < 4; ++j)
      if (i0 - j >= st0 && i0 - j + halo >= 0) xs[j] = to_f32(tin[(i0 - j + halo) * d + c]);
    const int i1 = min(i0 + run, nt);
    for (int i = i0; i < i1; ++i) {
      if (i > i0 && s_start[i] == i) xs[1] = xs[2] = xs[3] = 0.f;  // a new sequence starts here
      const float xt = to_f32(tin[(i + halo) * d + c]);
      const float y = fmaf(wr[3], xs[3], fmaf(wr[2], xs[2], fmaf(wr[1], xs[1], wr[0] * xt)));
      tout[i * d + c] = from_f32<T>(silu(y));
      xs[3] = xs[2];
      xs[2] = xs[1];
      xs[1] = xt;
    }
  }
  __syncthreads();
  if (P.l2) {  // L2 normalisation: one warp per token, lanes over the channels
    const int warp = tid >> 5, lane = tid & 31;
    for (int i = warp; i < nt; i += 8) {
      float ss = 0.f;
      for (int c = lane; c < d; c += 32) {
        const float v = to_f32(tout[i * d + c]);
        ss = fmaf(v, v, ss);
      }
      ss = warp_allreduce_sum(ss);
      const float inv = rsqrtf(ss + L2_EPS);
      for (int c = lane; c < d; c += 32) tout[i * d + c] = from_f32<T>(to_f32(tout[i * d + c]) * inv);
    }
    __syncthreads();
  }
  T *obase = out + (size_t)t0 * stride + (size_t)h * d;
  for (int e = tid; e < nt * vrow; e += 256) {
    const int r = e / vrow, vc = e - r * vrow;
    reinterpret_cast<uint4 *>(obase + (size_t)r * stride)[vc] = reinterpret_cast<const uint4 *>(tout)[e];
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
        qa[i] = from_f32<T>(__fdividef(1.f, 1.f + __expf(to_f32(pa[i]))));
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
// one warp per two rows (their loads issued together), each lane PER = d_v / 32 consecutive values
// moved as one vector.
template <typename T, int PER>
__global__ void __launch_bounds__(256) rms_gate_kernel(const T *o, const T *z, const float *g, T *y, long long rows) {
  constexpr int DV = 32 * PER, R = 2;
  struct alignas(sizeof(T) * PER) Vec { T e[PER]; };
  const long long row0 = (((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * R;
  const int lane = threadIdx.x & 31;
  Vec ov[R], zv[R];
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (row0 + r < rows) {
      const size_t base = (size_t)(row0 + r) * DV + lane * PER;
      ov[r] = *reinterpret_cast<const Vec *>(o + base);
      zv[r] = *reinterpret_cast<const Vec *>(z + base);
    }
  float gw[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) gw[i] = g[lane * PER + i];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (row0 + r >= rows) break;  // uniform per warp
    float of[PER], ss = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      of[i] = to_f32(ov[r].e[i]);
      ss = fmaf(of[i], of[i], ss);
    }
    ss = warp_allreduce_sum(ss);
    const float inv = rsqrtf(ss / DV + RMS_EPS);
    Vec yv;
#pragma unroll
    for (int i = 0; i < PER; ++i) yv.e[i] = from_f32<T>(of[i] * inv * gw[i] * silu(to_f32(zv[r].e[i])));
    *reinterpret_cast<Vec *>(y + (size_t)(row0 + r) * DV + lane * PER) = yv;
  }
}

template <typename T>
cudaError_t prologue_t(const BlockPrologueArgs &p, cudaStream_t stream) {
  const int smem = (2 * TT + 3) * std::max(p.dk, p.dv) * (int)sizeof(T);
  cudaError_t err = cudaFuncSetAttribute(conv_silu_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
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
    conv_silu_kernel<T><<<grid, 256, smem, stream>>>(a);
    err = cudaGetLastError();
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
  const unsigned blocks = (unsigned)(((rows + 1) / 2 * 32 + 255) / 256);  // one warp per two rows
  const T *o = static_cast<const T *>(p.o), *z = static_cast<const T *>(p.z);
  T *y = static_cast<T *>(p.y);
  note_launch();
  if (p.dv == 64) rms_gate_kernel<T, 2><<<blocks, 256, 0, stream>>>(o, z, p.g, y, rows);
  else if (p.dv == 128) rms_gate_kernel<T, 4><<<blocks, 256, 0, stream>>>(o, z, p.g, y, rows);
  else rms_gate_kernel<T, 8><<<blocks, 256, 0, stream>>>(o, z, p.g, y, rows);
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
