// Chunkwise WY forward of the Gated Delta Rule-2, plain SIMT fp32 version.
//
// This is the fp32 path (tensor-core operands would round below the fp32
// accuracy a float32 caller expects) and a simple correct path for bf16.
//
// Chunk form (one chunk of C tokens r, i = 0..C-1, entering state S, per key
// channel c; g = cumulative log2 decay inside the chunk):
//   L[r][i]  = sum_c a_rc k_ic 2^(g_rc - g_ic)        i <  r   (erase interaction)
//   P[r][i]  = sum_c q_rc k_ic 2^(g_rc - g_ic)        i <= r   (causal read)
//   Delta    = (I + L)^-1 (U - A_hat S),  A_hat_r = 2^g_r (.) a_r,  U_r = w_r (.) v_r
//   O        = Q_hat S + P Delta,          Q_hat_r = 2^g_r (.) q_r
//   S_next   = Diag(2^g_last) S + K_hat^T Delta,  K_hat_i = 2^(g_last - g_i) (.) k_i
// This is the block formulation of "Gated DeltaNet-2: Separando Borrado y
// Escritura en la Atención Lineal" (needhelp.icu), "Innovaciones Técnicas",
// item 1 (the per-channel decay is folded into asymmetric erase factors), with
// the per-token update of "NVIDIA AIがGated DeltaNet-2を発表"
// (ai.warp-studio.com), "Gated DeltaNet-2の核心".  Every decay factor here is
// formed as 2^(difference) <= 1, so no factor can overflow.
//
// Grid: one CTA per (sequence, head, NV-wide slice of the value channels); the
// value columns of S evolve independently, so slices need no communication.
#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kC = 64;     // chunk length
constexpr int kNT = 256;   // threads per CTA
constexpr int kNV = 32;    // value columns per CTA

template <int DK>
constexpr size_t simt_smem_bytes() {
  return sizeof(float) * (size_t)(4 * kC * (DK + 1) + DK * kNV + kC * kNV + kC * (kNV + 1) +
                                  2 * kC * (kC + 1) + DK);
}

template <int DK, typename Tin>
__global__ void __launch_bounds__(kNT) chunk_fwd_simt_kernel(ChunkArgs a) {
  constexpr int C = kC, NV = kNV, NVP = kNV + 1, DKP = DK + 1, CP = kC + 1;
  extern __shared__ float smem[];
  float *Kc = smem;              // [C][DKP]  k, later K_hat
  float *Ac = Kc + C * DKP;      // [C][DKP]  a = b*k, later A_hat
  float *Qc = Ac + C * DKP;      // [C][DKP]  q, later Q_hat
  float *G = Qc + C * DKP;       // [C][DKP]  log2 decay, then its running sum
  float *S = G + C * DKP;        // [DK][NV]  state slice (fp32)
  float *U = S + DK * NV;        // [C][NV]   w*v
  float *D = U + C * NV;         // [C][NVP]  right-hand side, then Delta
  float *L = D + C * NVP;        // [C][CP]
  float *P = L + C * CP;         // [C][CP]
  float *gl = P + C * CP;        // [DK]      2^(decay over the whole chunk)

  const int tiles = a.dv / NV;
  const int tile = blockIdx.x % tiles;
  const int h = (blockIdx.x / tiles) % a.H;
  const int n = blockIdx.x / (tiles * a.H);
  const int j0 = tile * NV;
  const int H = a.H, dv = a.dv;
  const int tid = threadIdx.x;
  int64_t bos;
  int len;
  seq_span(a, n, bos, len);

  const Tin *q = (const Tin *)a.q, *k = (const Tin *)a.k, *v = (const Tin *)a.v;
  const Tin *al = (const Tin *)a.alpha, *bg = (const Tin *)a.b, *wg = (const Tin *)a.w;
  Tin *o = (Tin *)a.o;
  const size_t sbase = ((size_t)n * H + h) * (size_t)DK * dv + j0;

  for (int e = tid; e < DK * NV; e += kNT) {
    const int c = e / NV, j = e % NV;
    S[e] = a.S0 ? a.S0[sbase + (size_t)c * dv + j] : 0.f;
  }

  for (int c0 = 0; c0 < len; c0 += C) {
    const int Cc = min(C, len - c0);
    __syncthreads();
    for (int e = tid; e < C * DK; e += kNT) {
      const int r = e / DK, c = e % DK;
      float kk = 0.f, aa = 0.f, qq = 0.f, gg = 0.f;
      if (r < Cc) {
        const size_t idx = ((size_t)(bos + c0 + r) * H + h) * DK + c;
        kk = to_f32(k[idx]);
        aa = to_f32(bg[idx]) * kk;
        qq = to_f32(q[idx]);
        gg = log2f(to_f32(al[idx]));
      }
      Kc[r * DKP + c] = kk;
      Ac[r * DKP + c] = aa;
      Qc[r * DKP + c] = qq;
      G[r * DKP + c] = gg;
    }
    for (int e = tid; e < C * NV; e += kNT) {
      const int r = e / NV, j = e % NV;
      float uu = 0.f;
      if (r < Cc) {
        const size_t idx = ((size_t)(bos + c0 + r) * H + h) * dv + j0 + j;
        uu = to_f32(wg[idx]) * to_f32(v[idx]);
      }
      U[e] = uu;
    }
    __syncthreads();
    if (tid < DK) {  // running log2 decay per key channel
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        acc += G[r * DKP + tid];
        G[r * DKP + tid] = acc;
      }
    }
    __syncthreads();

    {  // L and P by 4x4 register blocks of (r, i)
      const int rb = tid / 16, ib = tid % 16;
      float l[4][4], p[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) l[x][y] = p[x][y] = 0.f;
      if (ib <= rb) {
        for (int c = 0; c < DK; ++c) {
          float gr[4], ar[4], qr[4], gi[4], ki[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            gr[x] = G[(4 * rb + x) * DKP + c];
            ar[x] = Ac[(4 * rb + x) * DKP + c];
            qr[x] = Qc[(4 * rb + x) * DKP + c];
            gi[x] = G[(4 * ib + x) * DKP + c];
            ki[x] = Kc[(4 * ib + x) * DKP + c];
          }
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y)
              if (ib < rb || y <= x) {
                const float f = exp2f(gr[x] - gi[y]) * ki[y];
                l[x][y] = fmaf(ar[x], f, l[x][y]);
                p[x][y] = fmaf(qr[x], f, p[x][y]);
              }
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int r = 4 * rb + x, i = 4 * ib + y;
          L[r * CP + i] = (i < r) ? l[x][y] : 0.f;
          P[r * CP + i] = (i <= r) ? p[x][y] : 0.f;
        }
    }
    __syncthreads();

    // decay-absorbed factors (each <= 1)
    for (int e = tid; e < C * DK; e += kNT) {
      const int r = e / DK, c = e % DK;
      const float g = G[r * DKP + c], gC = G[(Cc - 1) * DKP + c];
      const float gam = exp2f(g);
      Ac[r * DKP + c] *= gam;
      Qc[r * DKP + c] *= gam;
      Kc[r * DKP + c] *= exp2f(gC - g);
    }
    if (tid < DK) gl[tid] = exp2f(G[(Cc - 1) * DKP + tid]);
    __syncthreads();

    // right-hand side U - A_hat S
    for (int e = tid; e < C * NV; e += kNT) {
      const int r = e / NV, j = e % NV;
      float acc = U[e];
      for (int c = 0; c < DK; ++c) acc = fmaf(-Ac[r * DKP + c], S[c * NV + j], acc);
      D[r * NVP + j] = acc;
    }
    __syncthreads();

    {  // forward substitution with the unit-lower (I + L); warp w owns NV/8 columns
      constexpr int CPW = NV / 8;
      const int warp = tid / 32, lane = tid % 32;
      float d0[CPW], d1[CPW];
#pragma unroll
      for (int x = 0; x < CPW; ++x) {
        d0[x] = D[lane * NVP + warp * CPW + x];
        d1[x] = D[(lane + 32) * NVP + warp * CPW + x];
      }
      for (int r = 1; r < C; ++r) {
        const float l0 = (lane < r) ? L[r * CP + lane] : 0.f;
        const float l1 = (lane + 32 < r) ? L[r * CP + lane + 32] : 0.f;
#pragma unroll
        for (int x = 0; x < CPW; ++x) {
          const float s = warp_allreduce_sum(fmaf(l0, d0[x], l1 * d1[x]));
          if (r < 32) {
            if (lane == r) d0[x] -= s;
          } else {
            if (lane == r - 32) d1[x] -= s;
          }
        }
      }
#pragma unroll
      for (int x = 0; x < CPW; ++x) {
        D[lane * NVP + warp * CPW + x] = d0[x];
        D[(lane + 32) * NVP + warp * CPW + x] = d1[x];
      }
    }
    __syncthreads();

    // outputs O = Q_hat S + P Delta
    for (int e = tid; e < C * NV; e += kNT) {
      const int r = e / NV, j = e % NV;
      if (r < Cc) {
        float acc = 0.f;
        for (int c = 0; c < DK; ++c) acc = fmaf(Qc[r * DKP + c], S[c * NV + j], acc);
        for (int i = 0; i <= r; ++i) acc = fmaf(P[r * CP + i], D[i * NVP + j], acc);
        o[((size_t)(bos + c0 + r) * H + h) * dv + j0 + j] = from_f32<Tin>(acc);
      }
    }
    __syncthreads();

    // state carried to the next chunk
    for (int e = tid; e < DK * NV; e += kNT) {
      const int c = e / NV, j = e % NV;
      float acc = gl[c] * S[e];
      for (int i = 0; i < Cc; ++i) acc = fmaf(Kc[i * DKP + c], D[i * NVP + j], acc);
      S[e] = acc;
    }
  }
  __syncthreads();
  if (a.ST)
    for (int e = tid; e < DK * NV; e += kNT) {
      const int c = e / NV, j = e % NV;
      a.ST[sbase + (size_t)c * dv + j] = S[e];
    }
}

template <int DK, typename Tin>
cudaError_t launch_simt_typed(const ChunkArgs &a, cudaStream_t stream) {
  const size_t smem = simt_smem_bytes<DK>();
  auto kern = chunk_fwd_simt_kernel<DK, Tin>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const long long blocks = (long long)a.B * a.H * (a.dv / kNV);
  if (blocks == 0) return cudaSuccess;
  note_launch();
  kern<<<(unsigned)blocks, kNT, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs &a, bool bf16, cudaStream_t stream) {
  if (a.dk == 64)
    return bf16 ? launch_simt_typed<64, __nv_bfloat16>(a, stream) : launch_simt_typed<64, float>(a, stream);
  return bf16 ? launch_simt_typed<128, __nv_bfloat16>(a, stream) : launch_simt_typed<128, float>(a, stream);
}

}  // namespace gdn2
