// Backward of the Gated Delta Rule-2 recurrence (erase reading R1): gradients with respect to q,
// k, v, alpha, b, w and S0, given dL/do and dL/dS_T.  The recurrence is the one of
// "[논문] 게이트형 DeltaNet-2" (euno.news), section "방법론", and
// "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section "Gated DeltaNet-2の核心":
//
//   S'_t = Diag(alpha_t) S_{t-1},  d_t = w_t (.) v_t - S'_t^T (b_t (.) k_t),
//   S_t = S'_t + k_t d_t^T,        o_t = S_t^T q_t,
//
// and the chain rule taken backwards through it, with G = dL/dS_t:
//
//   G += q_t dO_t^T;  dq_t = S_t dO_t;  dd = G^T k_t;  dk_t = G d_t;
//   dv_t = dd (.) w_t;  dw_t = dd (.) v_t;  da = -S'_t dd;  dS' = G - a_t dd^T;
//   dalpha_t = rowsum(dS' (.) S_{t-1});  G = Diag(alpha_t) dS';  db_t = da (.) k_t;  dk_t += da (.) b_t.
//
// Every value column of the state evolves on its own (the key-side vectors are shared), so one
// CTA takes one (sequence, head, tile of NJ value columns), one thread per key row i: it holds row
// i of its tile of S and of G in registers.  Sums over the key rows (the erase read S'^T a and
// dd = G^T k) are block reductions; sums over the value columns (dq, dk, dalpha, da) are formed in
// each thread over its tile and added across tiles with fp32 reductions in L2, into a buffer that
// a second kernel converts to the output type.
//
// States are not kept for every token.  A first forward pass stores the tile's state every GK
// tokens (one group of GK / CK segments) and every d_t.  The backward pass walks the groups from
// the last: it first rebuilds the state before each CK-token segment of the group from the group's
// checkpoint and the stored d_t, into a scratch area of its own in the workspace, then walks the
// group's segments backwards, rebuilding each segment's CK states in shared memory from the
// scratch.  Every rebuild repeats the first pass's operations (S = d_t k + alpha S, rounded the
// same way), so it reproduces its states exactly, and no thread reads what another wrote.
#include <algorithm>

#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int NJ = 16;       // value columns per CTA
constexpr int CK = 4;        // tokens per segment rebuilt in shared memory (4 CTAs of 128 rows fit an SM)
constexpr int GK = 64;       // tokens per stored checkpoint
constexpr int GS = GK / CK;  // segments per checkpoint group

struct BwdParams {
  const void *q, *k, *v, *alpha, *b, *w, *dO;
  const float *S0, *dST;
  float4 *acc;       // [tokens, H, d_k] x (dq, dk, dalpha, db) fp32, summed over the tiles (zeroed)
  float4 *ck;        // checkpoints every GK tokens [slots, H, tiles, NJ / 4, d_k] float4
  float4 *scr;       // per CTA: the states before the segments of one group [CTAs, GS, NJ / 4, d_k] float4
  float *dl;         // d_t of every token [tokens, H, d_v] fp32, from the first pass
  void *dv, *dw;     // [tokens, H, d_v]
  float *dS0;        // [N, H, d_k, d_v] or nullptr
  const int32_t *cu;  // packed offsets [N+1] or nullptr
  int N, T, H, dv_;
};

template <typename T>
__device__ __forceinline__ float ld(const void *p, size_t i) {
  return to_f32(static_cast<const T *>(p)[i]);
}

// Adds four floats to 16 aligned bytes of global memory as one reduction in L2.
__device__ __forceinline__ void red_add4(float4 *p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Sum of p[0..15] over the 32 lanes of a warp, transposed: lane l ends with the sum of index l >> 1
// (lanes 2m and 2m+1 both hold index m).  16 shuffles instead of 80.
__device__ __forceinline__ float warp_reduce16(float (&p)[NJ], int lane) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const bool up = lane & 16;
    const float send = up ? p[m] : p[m + 8], keep = up ? p[m + 8] : p[m];
    p[m] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const bool up = lane & 8;
    const float send = up ? p[m] : p[m + 4], keep = up ? p[m + 4] : p[m];
    p[m] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const bool up = lane & 4;
    const float send = up ? p[m] : p[m + 2], keep = up ? p[m + 2] : p[m];
    p[m] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool up = lane & 2;
    const float send = up ? p[0] : p[1], keep = up ? p[1] : p[0];
    p[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  return p[0] + __shfl_xor_sync(0xffffffffu, p[0], 1);
}

template <typename T, int DK>
struct __align__(16) BwdSmem {
  static constexpr int NW = DK / 32;
  float4 seg[CK][NJ / 4][DK];  // the tile's state before each token of the segment, row-interleaved
  float u[CK][NJ];             // w (.) v of the segment's tokens
  float vv[CK][NJ];            // v and w of the segment's tokens (for dv, dw)
  float ww[CK][NJ];
  float dO[CK][NJ];            // dL/do of the segment's tokens
  float dl[CK][NJ];            // d_t of the segment's tokens
  float red[2][NJ][NW];        // warp partials of a block reduction, double-buffered
};

// One (sequence, head, NJ-column tile).  blockDim = DK; four blocks of 128 rows per SM.
template <typename T, int DK>
__global__ void __launch_bounds__(DK, 512 / DK) chunk_bwd_kernel(const BwdParams p) {
  using Smem = BwdSmem<T, DK>;
  constexpr int NW = Smem::NW;
  extern __shared__ __align__(16) uint8_t dsm[];
  Smem &sm = *reinterpret_cast<Smem *>(dsm);
  const int tile = blockIdx.x, h = blockIdx.y, n = blockIdx.z, i = threadIdx.x;
  const int lane = i & 31, warp = i >> 5;
  const int tiles = p.dv_ / NJ, j0 = tile * NJ, H = p.H, DV = p.dv_;
  long long bos, len;
  if (p.cu) {  // offsets clamped to [0, T_total], so that bad offsets cannot index out of bounds
    bos = min(max(p.cu[n], 0), p.T);
    len = min(max(p.cu[n + 1], (int)bos), p.T) - bos;
  } else {
    bos = (long long)n * p.T;
    len = p.T;
  }
  const int nseg = (int)((len + CK - 1) / CK);
  const long long slot0 = bos / GK + n;  // distinct slots for every group of every sequence
  auto ck_at = [&](int grp) { return p.ck + ((((slot0 + grp) * H + h) * tiles + tile) * (NJ / 4)) * DK + i; };
  const size_t cta = ((size_t)n * H + h) * tiles + tile;
  auto scr_at = [&](int m) { return p.scr + ((cta * GS + (m % GS)) * (NJ / 4)) * DK + i; };
  auto krow = [&](long long t) { return ((size_t)t * H + h) * DK + i; };
  auto vcol = [&](long long t, int j) { return ((size_t)t * H + h) * DV + j0 + j; };

  float s[NJ];
  {
    const size_t off = (((size_t)n * H + h) * DK + i) * DV + j0;
#pragma unroll
    for (int j = 0; j < NJ; ++j) s[j] = p.S0 ? p.S0[off + j] : 0.f;
  }
  // Block reduction of v over the key rows: every thread gets all NJ sums.  One barrier: the
  // partials alternate between two buffers, and a buffer is written again only after the next
  // reduction's barrier, which every reader of it has passed.
  int par = 0;
  auto red_sum = [&](int buf, int j) {  // the block's sum of index j from the warp partials
    if constexpr (NW == 4) {
      const float4 x = *reinterpret_cast<const float4 *>(sm.red[buf][j]);
      return (x.x + x.y) + (x.z + x.w);
    } else {
      const float2 x = *reinterpret_cast<const float2 *>(sm.red[buf][j]);
      return x.x + x.y;
    }
  };
  auto reduce = [&](float (&v)[NJ], float (&tot)[NJ]) {
    const float r = warp_reduce16(v, lane);
    if ((lane & 1) == 0) sm.red[par][lane >> 1][warp] = r;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < NJ; ++j) tot[j] = red_sum(par, j);
    par ^= 1;
  };
  // A segment's inputs, all loads issued together: the value-side ones into shared memory, this
  // row's alpha, k, b (and q) into registers.
  float ral[CK], rk[CK], rb[CK], rq[CK];
  auto load_seg = [&](long long t0, int nt, bool bwd) {
    for (int e = i; e < CK * NJ; e += DK) {
      const int u = e / NJ, j = e % NJ;
      float vv = 0.f, ww = 0.f, dd = 0.f, dl = 0.f;
      if (u < nt) {
        vv = ld<T>(p.v, vcol(t0 + u, j));
        ww = ld<T>(p.w, vcol(t0 + u, j));
        if (bwd) {
          dd = ld<T>(p.dO, vcol(t0 + u, j));
          dl = p.dl[vcol(t0 + u, j)];
        }
      }
      sm.u[u][j] = ww * vv;
      sm.vv[u][j] = vv;
      sm.ww[u][j] = ww;
      sm.dO[u][j] = dd;
      sm.dl[u][j] = dl;
    }
#pragma unroll
    for (int u = 0; u < CK; ++u) {
      const bool in = u < nt;
      ral[u] = in ? ld<T>(p.alpha, krow(t0 + u)) : 0.f;
      rk[u] = in ? ld<T>(p.k, krow(t0 + u)) : 0.f;
      rb[u] = in ? ld<T>(p.b, krow(t0 + u)) : 0.f;
      rq[u] = in && bwd ? ld<T>(p.q, krow(t0 + u)) : 0.f;
    }
  };

  // Pass 1: forward over the sequence, storing the state before every group and every d_t.
  for (int m = 0; m < nseg; ++m) {
    const long long t0 = bos + (long long)m * CK;
    const int nt = (int)min((long long)CK, len - (long long)m * CK);
    if (m % GS == 0) {
      float4 *c = ck_at(m / GS);
#pragma unroll
      for (int q4 = 0; q4 < NJ / 4; ++q4) c[q4 * DK] = make_float4(s[4 * q4], s[4 * q4 + 1], s[4 * q4 + 2], s[4 * q4 + 3]);
    }
    load_seg(t0, nt, false);
    __syncthreads();  // the segment's value-side inputs are in shared memory
#pragma unroll
    for (int u = 0; u < CK; ++u) {
      if (u >= nt) break;
      const float al = ral[u], kk = rk[u], ai = rb[u] * kk;
      float v[NJ], r[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        s[j] *= al;
        v[j] = ai * s[j];
      }
      reduce(v, r);
#pragma unroll
      for (int j = 0; j < NJ; ++j) s[j] = fmaf(kk, sm.u[u][j] - r[j], s[j]);
      if (i < NJ) p.dl[vcol(t0 + u, i)] = sm.u[u][i] - r[i];  // same value as used above
    }
    __syncthreads();  // before the next segment overwrites the value-side inputs
  }

  // Pass 2: backwards, one segment at a time.
  float g[NJ];
  {
    const size_t off = (((size_t)n * H + h) * DK + i) * DV + j0;
#pragma unroll
    for (int j = 0; j < NJ; ++j) g[j] = p.dST ? p.dST[off + j] : 0.f;
  }
  for (int m = nseg - 1; m >= 0; --m) {
    const long long t0 = bos + (long long)m * CK;
    const int nt = (int)min((long long)CK, len - (long long)m * CK);
    if (m == nseg - 1 || m % GS == GS - 1) {
      // entering group m / GS: the state before each of its segments, from the group's checkpoint
      // and the stored d_t, into this thread's row of the scratch
      const int m0 = m - m % GS;
      {
        const float4 *c = ck_at(m / GS);
#pragma unroll
        for (int q4 = 0; q4 < NJ / 4; ++q4) {
          const float4 x = c[q4 * DK];
          s[4 * q4] = x.x;
          s[4 * q4 + 1] = x.y;
          s[4 * q4 + 2] = x.z;
          s[4 * q4 + 3] = x.w;
        }
      }
      for (int mm = m0; mm <= m; ++mm) {
        float4 *sc = scr_at(mm);
#pragma unroll
        for (int q4 = 0; q4 < NJ / 4; ++q4) sc[q4 * DK] = make_float4(s[4 * q4], s[4 * q4 + 1], s[4 * q4 + 2], s[4 * q4 + 3]);
        if (mm == m) break;  // the state after segment m is not used
        const long long ta = bos + (long long)mm * CK;  // a full segment: only a sequence's last one can be short
#pragma unroll
        for (int u = 0; u < CK; ++u) {
          const float al = ld<T>(p.alpha, krow(ta + u)), kk = ld<T>(p.k, krow(ta + u));
          const float4 *dl4 = reinterpret_cast<const float4 *>(p.dl + vcol(ta + u, 0));
#pragma unroll
          for (int q4 = 0; q4 < NJ / 4; ++q4) {
            const float4 d = dl4[q4];
            s[4 * q4] = fmaf(kk, d.x, s[4 * q4] * al);
            s[4 * q4 + 1] = fmaf(kk, d.y, s[4 * q4 + 1] * al);
            s[4 * q4 + 2] = fmaf(kk, d.z, s[4 * q4 + 2] * al);
            s[4 * q4 + 3] = fmaf(kk, d.w, s[4 * q4 + 3] * al);
          }
        }
      }
    }
    const float4 *c = scr_at(m);
#pragma unroll
    for (int q4 = 0; q4 < NJ / 4; ++q4) {
      const float4 x = c[q4 * DK];
      s[4 * q4] = x.x;
      s[4 * q4 + 1] = x.y;
      s[4 * q4 + 2] = x.z;
      s[4 * q4 + 3] = x.w;
    }
    load_seg(t0, nt, true);
    __syncthreads();
    // rebuild the state before each token of the segment from the checkpoint and the stored d_t
    // (the same operations as the first pass, so the same values)
#pragma unroll
    for (int u = 0; u < CK; ++u) {
      if (u >= nt) break;
#pragma unroll
      for (int q4 = 0; q4 < NJ / 4; ++q4)
        sm.seg[u][q4][i] = make_float4(s[4 * q4], s[4 * q4 + 1], s[4 * q4 + 2], s[4 * q4 + 3]);
#pragma unroll
      for (int j = 0; j < NJ; ++j) s[j] = fmaf(rk[u], sm.dl[u][j], s[j] * ral[u]);
    }
    // backwards through the segment
#pragma unroll
    for (int u = CK - 1; u >= 0; --u) {
      if (u >= nt) continue;
      const long long t = t0 + u;
      const float al = ral[u], kk = rk[u], bb = rb[u], qq = rq[u], ai = bb * kk;
      float sp[NJ];
#pragma unroll
      for (int q4 = 0; q4 < NJ / 4; ++q4) {
        const float4 x = sm.seg[u][q4][i];
        sp[4 * q4] = x.x;
        sp[4 * q4 + 1] = x.y;
        sp[4 * q4 + 2] = x.z;
        sp[4 * q4 + 3] = x.w;
      }
      float dq = 0.f, dk = 0.f, v[NJ], dd[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float doj = sm.dO[u][j], dlj = sm.dl[u][j];
        g[j] = fmaf(qq, doj, g[j]);
        const float st = fmaf(kk, dlj, sp[j] * al);  // S_t, as the forward formed it
        dq = fmaf(st, doj, dq);
        dk = fmaf(g[j], dlj, dk);
        v[j] = g[j] * kk;
      }
      reduce(v, dd);
      if (i < NJ) {  // this thread's column: dv, dw (dd of column i, re-read from the partials)
        const float ddi = red_sum(par ^ 1, i);
        const size_t o = vcol(t, i);
        static_cast<T *>(p.dv)[o] = from_f32<T>(ddi * sm.ww[u][i]);
        static_cast<T *>(p.dw)[o] = from_f32<T>(ddi * sm.vv[u][i]);
      }
      float da = 0.f, dal = 0.f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float spj = sp[j] * al;
        da = fmaf(-spj, dd[j], da);
        const float dsp = fmaf(-ai, dd[j], g[j]);
        dal = fmaf(dsp, sp[j], dal);
        g[j] = al * dsp;
      }
      dk = fmaf(da, bb, dk);
      red_add4(p.acc + ((size_t)t * H + h) * DK + i, dq, dk, dal, da * kk);
    }
    __syncthreads();  // before the next segment overwrites the segment's inputs
  }
  if (p.dS0) {
    const size_t off = (((size_t)n * H + h) * DK + i) * DV + j0;
#pragma unroll
    for (int j = 0; j < NJ; ++j) p.dS0[off + j] = g[j];
  }
}

// acc [rows, d_k] x (dq, dk, dalpha, db) fp32 -> the four gradients [rows, d_k] in the output type.
template <typename T>
__global__ void __launch_bounds__(256) bwd_finish_kernel(const float4 *acc, T *dq, T *dk, T *dal, T *db, size_t n) {
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const float4 a = acc[e];
    dq[e] = from_f32<T>(a.x);
    dk[e] = from_f32<T>(a.y);
    dal[e] = from_f32<T>(a.z);
    db[e] = from_f32<T>(a.w);
  }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <typename T, int DK>
cudaError_t bwd_t(const BwdArgs &a, void *ws, cudaStream_t stream) {
  const long long tokens = a.cu ? (long long)a.T : (long long)a.B * a.T;
  BwdParams p{};
  p.q = a.q; p.k = a.k; p.v = a.v; p.alpha = a.alpha; p.b = a.b; p.w = a.w; p.dO = a.dO;
  p.S0 = a.S0; p.dST = a.dST; p.dv = a.dv; p.dw = a.dw; p.dS0 = a.dS0; p.cu = a.cu;
  p.N = a.B; p.T = a.T; p.H = a.H; p.dv_ = a.Dv;
  const size_t acc_elems = (size_t)tokens * a.H * DK;  // float4 each
  uint8_t *base = static_cast<uint8_t *>(ws);
  p.acc = reinterpret_cast<float4 *>(base);
  p.dl = reinterpret_cast<float *>(base + align256(acc_elems * sizeof(float4)));
  const long long slots = tokens / GK + a.B + 1;
  p.ck = reinterpret_cast<float4 *>(base + align256(acc_elems * sizeof(float4)) +
                                    align256((size_t)tokens * a.H * a.Dv * sizeof(float)));
  p.scr = reinterpret_cast<float4 *>(reinterpret_cast<uint8_t *>(p.ck) + align256((size_t)slots * a.H * DK * a.Dv * sizeof(float)));
  cudaError_t err = cudaMemsetAsync(p.acc, 0, acc_elems * sizeof(float4), stream);
  if (err != cudaSuccess) return err;
  const int smem = (int)sizeof(BwdSmem<T, DK>);
  err = cudaFuncSetAttribute(chunk_bwd_kernel<T, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  note_launch();
  chunk_bwd_kernel<T, DK><<<dim3(a.Dv / NJ, a.H, a.B), DK, smem, stream>>>(p);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (tokens == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)std::min<size_t>((acc_elems + 255) / 256, (size_t)148 * 16);
  note_launch();
  bwd_finish_kernel<T><<<blocks, 256, 0, stream>>>(p.acc, static_cast<T *>(a.dq), static_cast<T *>(a.dk),
                                                  static_cast<T *>(a.dalpha), static_cast<T *>(a.db), acc_elems);
  return cudaGetLastError();
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, bool packed) {
  const long long tokens = packed ? (long long)T : (long long)B * T;
  const long long slots = tokens / GK + B + 1;
  return align256((size_t)tokens * H * dk * sizeof(float4)) + align256((size_t)tokens * H * dv * sizeof(float)) +
         align256((size_t)slots * H * dk * dv * sizeof(float)) + (size_t)B * H * GS * dk * dv * sizeof(float);
}

cudaError_t launch_chunk_bwd(const BwdArgs &a, bool bf16, void *ws, cudaStream_t stream) {
  if (a.Dk == 128)
    return bf16 ? bwd_t<__nv_bfloat16, 128>(a, ws, stream) : bwd_t<float, 128>(a, ws, stream);
  return bf16 ? bwd_t<__nv_bfloat16, 64>(a, ws, stream) : bwd_t<float, 64>(a, ws, stream);
}

}  // namespace gdn2
