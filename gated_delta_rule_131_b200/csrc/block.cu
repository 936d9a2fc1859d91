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
#include <climits>

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int CE = 8;  // channels per lane in the convolution kernel
constexpr float L2_EPS = 1e-6f, RMS_EPS = 1e-5f;

constexpr int CS = 3;  // load batches in a convolution lane's ring (two in flight while one is used)

// 16-byte asynchronous copy global -> shared (through L2), a commit of this thread's copies issued
// so far as one group, and a wait until at most N of its groups are pending.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float silu(float y) { return __fdividef(y, 1.f + __expf(-y)); }

// SiLU of a pair, y / (1 + e^-y) with e^-y = 2^(-y log2 e), from the PTX approximate base-2
// exponential and reciprocal (large negative y: e^-y = inf, reciprocal 0, result -0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float2 silu2(float2 y) {
  constexpr float NEG_LOG2E = -1.4426950408889634f;
  const float2 m = __fmul2_rn(y, make_float2(NEG_LOG2E, NEG_LOG2E));
  const float2 den = __fadd2_rn(make_float2(ex2_approx(m.x), ex2_approx(m.y)), make_float2(1.f, 1.f));
  return __fmul2_rn(y, make_float2(rcp_approx(den.x), rcp_approx(den.y)));
}
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
  int R;             // tokens per run (a multiple of the tokens a lane loads at once)
};

// A bf16 is the top half of the fp32 of the same value, so widening is a shift or a mask (integer
// pipe, exact).
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// The CE channels of one token that a lane holds, as pairs, from / to their stored type.
__device__ __forceinline__ void unpack(const uint4 (&r)[1], float2 (&f)[CE / 2]) {
  f[0] = bf2_to_f2(r[0].x);
  f[1] = bf2_to_f2(r[0].y);
  f[2] = bf2_to_f2(r[0].z);
  f[3] = bf2_to_f2(r[0].w);
}
__device__ __forceinline__ void unpack(const uint4 (&r)[2], float2 (&f)[CE / 2]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    f[2 * i] = make_float2(__uint_as_float(r[i].x), __uint_as_float(r[i].y));
    f[2 * i + 1] = make_float2(__uint_as_float(r[i].z), __uint_as_float(r[i].w));
  }
}
__device__ __forceinline__ void pack(const float2 (&f)[CE / 2], uint4 (&r)[1]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __float22bfloat162_rn(f[i]);
    w[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  r[0] = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void pack(const float2 (&f)[CE / 2], uint4 (&r)[2]) {
#pragma unroll
  for (int i = 0; i < 2; ++i)
    r[i] = make_uint4(__float_as_uint(f[2 * i].x), __float_as_uint(f[2 * i].y), __float_as_uint(f[2 * i + 1].x),
                      __float_as_uint(f[2 * i + 1].y));
}

// Depthwise causal convolution of K <= 4 taps, SiLU, and (q, k) L2 normalisation, streamed through
// registers.  A group of G = d / CE lanes holds one (token, head) row, CE consecutive channels per
// lane, and walks a run of R consecutive tokens of one head: it loads the run's rows 16 bytes per
// lane, CU tokens at a time, keeps its taps and the three previous tokens in registers, clears
// that window where a sequence starts, and reduces the row's sum of squares with shuffles inside
// the group.  Loads go through a ring of CS batches in shared memory with asynchronous copies, so
// that two batches are in flight while one is used; each lane reads back only its own copies, so
// the block never synchronises.  Every row is read once (plus three halo rows per run) and written
// once.  grid = (blocks of the widest path, 3 paths); the host picks R so that the grid is one wave.
template <typename T>
__global__ void __launch_bounds__(256, 2) conv_silu_kernel(const ConvArgs a) {
  constexpr int NV = CE * (int)sizeof(T) / 16;  // 16-byte vectors per lane and token
  constexpr int CU = 8 / NV;                    // tokens per load batch
  extern __shared__ uint4 ring[];               // [CS][CU][NV][256 threads]
  const ConvPath P = blockIdx.y == 0 ? a.path[0] : (blockIdx.y == 1 ? a.path[1] : a.path[2]);
  const int G = P.d / CE;  // 8, 16 or 32 lanes, aligned within the warp
  const long long gid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / G;
  const long long runs = (a.tokens + a.R - 1) / a.R;
  if (gid >= runs * a.H) return;  // whole groups leave together
  const int lane = threadIdx.x & 31, gl = lane & (G - 1);
  const unsigned gmask = G == 32 ? 0xffffffffu : ((1u << G) - 1u) << (lane & ~(G - 1));
  const int h = (int)(gid % a.H);
  const long long t0 = (gid / a.H) * a.R, t1 = min(t0 + (long long)a.R, a.tokens);
  const size_t stride = (size_t)a.H * P.d;  // elements between consecutive tokens
  const T *x = static_cast<const T *>(P.x) + (size_t)h * P.d + gl * CE;
  T *out = static_cast<T *>(P.out) + (size_t)h * P.d + gl * CE;

  float2 w0[CE / 2], w1[CE / 2], w2[CE / 2], w3[CE / 2];  // w_j multiplies x_{t-j}: the taps reversed
  {
    const float *W = P.W + ((size_t)h * P.d + gl * CE) * a.K;
    const int K = a.K;
#pragma unroll
    for (int i = 0; i < CE / 2; ++i) {
      const float *c0 = W + (2 * i) * K, *c1 = c0 + K;
      w0[i] = make_float2(c0[K - 1], c1[K - 1]);
      w1[i] = K > 1 ? make_float2(c0[K - 2], c1[K - 2]) : make_float2(0.f, 0.f);
      w2[i] = K > 2 ? make_float2(c0[K - 3], c1[K - 3]) : make_float2(0.f, 0.f);
      w3[i] = K > 3 ? make_float2(c0[K - 4], c1[K - 4]) : make_float2(0.f, 0.f);
    }
  }
  // The sequence holding t0: its first token s0 and the next sequence start nb (beyond: none).
  long long s0, nb;
  int n = 0;
  if (!a.cu) {
    s0 = t0 - t0 % a.T;
    nb = s0 + a.T;
  } else {
    int lo = 0, hi = a.N - 1;
    while (lo < hi) {  // largest n < N with cu[n] <= t0
      const int mid = (lo + hi + 1) >> 1;
      if (a.cu[mid] <= t0) lo = mid; else hi = mid - 1;
    }
    n = lo;
    s0 = a.cu[n];
    nb = a.cu[n + 1];
    if (nb <= t0) nb = LLONG_MAX;
  }
  float2 x1[CE / 2], x2[CE / 2], x3[CE / 2];  // x_{t-1}, x_{t-2}, x_{t-3}; zero before the sequence
#pragma unroll
  for (int i = 0; i < CE / 2; ++i) x1[i] = x2[i] = x3[i] = make_float2(0.f, 0.f);
  {
    uint4 r[NV];
#pragma unroll
    for (int j = 1; j <= 3; ++j)
      if (t0 - j >= s0) {
#pragma unroll
        for (int v = 0; v < NV; ++v) r[v] = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)(t0 - j) * stride) + v);
        unpack(r, j == 1 ? x1 : (j == 2 ? x2 : x3));
      }
  }
  // Token indices below are relative to t0 (a run is at most 2^20 tokens).
  const T *xr = x + (size_t)t0 * stride;
  T *orow = out + (size_t)t0 * stride;
  const int ntok = (int)(t1 - t0), ist = (int)stride;
  int nbr = (int)min(nb - t0, (long long)INT_MAX);  // next sequence start, relative
  const int nbatch = (ntok + CU - 1) / CU;
  auto issue = [&](int bt) {  // copies of batch bt (tokens before t1 only), committed as one group
    const int slot = bt % CS;
#pragma unroll
    for (int u = 0; u < CU; ++u) {
      const int i = bt * CU + u;
      if (bt < nbatch && i < ntok)
#pragma unroll
        for (int v = 0; v < NV; ++v)
          cp_async16(&ring[((slot * CU + u) * NV + v) * 256 + threadIdx.x],
                     reinterpret_cast<const uint4 *>(xr + (long long)i * ist) + v);
    }
    cp_async_commit();
  };
  // One token: convolution, SiLU, (q, k) L2 normalisation, store; then the window moves on.
  auto token = [&](int i, int slot, int u) {
    float2 xt[CE / 2], y[CE / 2];
    {
      uint4 r[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) r[v] = ring[((slot * CU + u) * NV + v) * 256 + threadIdx.x];
      unpack(r, xt);
    }
    float2 ss = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < CE / 2; ++k) {
      float2 c = __fmul2_rn(w0[k], xt[k]);
      c = __ffma2_rn(w1[k], x1[k], c);
      c = __ffma2_rn(w2[k], x2[k], c);
      c = __ffma2_rn(w3[k], x3[k], c);
      y[k] = silu2(c);
      ss = __ffma2_rn(y[k], y[k], ss);
      x3[k] = x2[k];
      x2[k] = x1[k];
      x1[k] = xt[k];
    }
    if (P.l2) {
      float sum = ss.x + ss.y;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        if (o < G) sum += __shfl_xor_sync(gmask, sum, o);
      const float inv = rsqrtf(sum + L2_EPS);
#pragma unroll
      for (int k = 0; k < CE / 2; ++k) y[k] = __fmul2_rn(y[k], make_float2(inv, inv));
    }
    uint4 r[NV];
    pack(y, r);
#pragma unroll
    for (int v = 0; v < NV; ++v) reinterpret_cast<uint4 *>(orow + (long long)i * ist)[v] = r[v];
  };
#pragma unroll
  for (int bt = 0; bt < CS - 1; ++bt) issue(bt);
  for (int bt = 0; bt < nbatch; ++bt) {
    issue(bt + CS - 1);  // into the slot batch bt - 1 used
    cp_async_wait<CS - 1>();
    const int ib = bt * CU, slot = bt % CS;
    if (ib + CU <= ntok && nbr >= ib + CU) {  // a full batch inside one sequence: no checks
#pragma unroll
      for (int u = 0; u < CU; ++u) token(ib + u, slot, u);
    } else {
      for (int u = 0; u < CU; ++u) {
        const int i = ib + u;
        if (i >= ntok) break;  // uniform in the group
        if (i == nbr) {        // a new sequence starts here (uniform in the group)
#pragma unroll
          for (int k = 0; k < CE / 2; ++k) x1[k] = x2[k] = x3[k] = make_float2(0.f, 0.f);
          const long long t = t0 + i;
          if (!a.cu) {
            nb += a.T;
          } else {
            int m = n + 1;  // cu[m] == t; skip empty sequences
            while (m + 1 < a.N && a.cu[m + 1] <= t) ++m;
            n = m;
            nb = m + 1 <= a.N ? (long long)a.cu[m + 1] : LLONG_MAX;
            if (nb <= t) nb = LLONG_MAX;
          }
          nbr = (int)min(nb - t0, (long long)INT_MAX);
        }
        token(i, slot, u);
      }
    }
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

constexpr int CONV_SMEM = CS * 8 * 16 * 256;  // the ring: CS batches of 8 16-byte vectors per thread

// Resident 256-thread blocks of conv_silu_kernel<T> on the current device (per SM times SMs); sets
// the kernel's shared-memory limit on first use.
template <typename T>
cudaError_t conv_slots(int &slots) {
  static int cache[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && cache[dev] > 0) {
    slots = cache[dev];
    return cudaSuccess;
  }
  int per_sm = 0, sms = 0;
  err = cudaFuncSetAttribute(conv_silu_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, CONV_SMEM);
  if (err == cudaSuccess)
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, conv_silu_kernel<T>, 256, CONV_SMEM);
  if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return err;
  slots = std::max(1, per_sm) * std::max(1, sms);
  if (dev < 64) cache[dev] = slots;
  return cudaSuccess;
}

template <typename T>
cudaError_t prologue_t(const BlockPrologueArgs &p, cudaStream_t stream) {
  if (p.tokens <= 0) return cudaSuccess;
  constexpr int CU = 8 * 16 / (CE * (int)sizeof(T));  // tokens a lane loads at once (as in the kernel)
  int slots = 0;
  cudaError_t err = conv_slots<T>(slots);
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
  // One wave: lanes x tokens of all three paths over the resident lanes, in whole load batches.
  const long long lane_tokens = p.tokens * p.H * (long long)(2 * p.dk + p.dv) / CE;
  const long long per_lane = (lane_tokens + (long long)slots * 256 - 1) / ((long long)slots * 256);
  a.R = (int)std::min<long long>(std::max<long long>((per_lane + CU - 1) / CU * CU, CU), 1 << 20);
  const long long runs = (p.tokens + a.R - 1) / a.R;
  const long long blocks = (runs * p.H * (std::max(p.dk, p.dv) / CE) + 255) / 256;
  note_launch();
  conv_silu_kernel<T><<<dim3((unsigned)blocks, 3), 256, CONV_SMEM, stream>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t nk = (size_t)p.tokens * p.H * p.dk, nv = (size_t)p.tokens * p.H * p.dv;
  const size_t vecs = (nk + nv) / (16 / sizeof(T));
  const unsigned gblocks = (unsigned)std::min<size_t>((vecs + 255) / 256, (size_t)148 * 16);
  note_launch();
  gates_kernel<T><<<gblocks, 256, 0, stream>>>(static_cast<const T *>(p.xa), static_cast<const T *>(p.xb),
                                               static_cast<const T *>(p.xw), static_cast<T *>(p.alpha),
                                               static_cast<T *>(p.b), static_cast<T *>(p.w), nk, nv);
  return cudaGetLastError();
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
