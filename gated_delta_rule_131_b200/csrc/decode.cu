// One recurrent Gated Delta Rule-2 step for a batch of single tokens.
//
// Per (batch entry, head), with a = b (.) k and u = w (.) v:
//   S' = Diag(alpha) S            decay on the key axis, first
//   r  = S'^T a,  p = S'^T q      two reductions over the key channels
//   d  = u - r                    gated erase + gated write, as one rank-1 delta
//   S  = S' + k d^T               written back once
//   o  = S^T q = p + (k.q) d      so the readout needs no second pass over S
// The per-token update of "NVIDIA AIがGated DeltaNet-2を発表"
// (ai.warp-studio.com), "Gated DeltaNet-2の核心", in the constant-memory
// recurrent form ("[논문] 게이트형 DeltaNet-2", euno.news, "결과 및 발견").
//
// Memory-bound: the fp32 state is streamed from HBM once and written once,
// with 128-bit loads/stores marked streaming (the state of a decode batch is
// far larger than L2 and is not re-read within the step).  Each CTA owns NCOL
// value columns of one head; a thread holds 4 adjacent columns (one float4)
// of DK / RG rows in registers.
#include "common.cuh"

namespace gdn2 {
namespace {

template <int DK, int NCOL, int NT, typename Tin>
__global__ void __launch_bounds__(NT) decode_step_kernel(DecodeArgs a) {
  constexpr int TPR = NCOL / 4;   // threads across one row slice
  constexpr int RG = NT / TPR;    // row groups
  constexpr int RPT = DK / RG;    // rows per thread
  static_assert(NT % TPR == 0 && DK % RG == 0, "tile shape");

  __shared__ float sq[DK], sk[DK], sa[DK], sal[DK];
  __shared__ float su[NCOL], sd[NCOL];
  __shared__ float red_r[RG][NCOL + 4], red_p[RG][NCOL + 4];
  __shared__ float s_kq;

  const int tiles = a.dv / NCOL;
  const int head = blockIdx.x / tiles;  // = b * H + h
  const int c0 = (blockIdx.x % tiles) * NCOL;
  const int tid = threadIdx.x;
  const int cq = tid % TPR, rg = tid / TPR;
  const int DV = a.dv;

  float *Sh = a.S + (size_t)head * DK * DV + c0 + 4 * cq;
  float4 s[RPT];
#pragma unroll
  for (int x = 0; x < RPT; ++x) s[x] = __ldcs(reinterpret_cast<const float4 *>(Sh + (size_t)(rg + x * RG) * DV));

  const Tin *q = (const Tin *)a.q + (size_t)head * DK, *k = (const Tin *)a.k + (size_t)head * DK;
  const Tin *al = (const Tin *)a.alpha + (size_t)head * DK, *bg = (const Tin *)a.b + (size_t)head * DK;
  const Tin *v = (const Tin *)a.v + (size_t)head * DV + c0, *wg = (const Tin *)a.w + (size_t)head * DV + c0;
  for (int i = tid; i < DK; i += NT) {
    const float kk = to_f32(k[i]);
    sk[i] = kk;
    sq[i] = to_f32(q[i]);
    sa[i] = to_f32(bg[i]) * kk;
    sal[i] = to_f32(al[i]);
  }
  for (int j = tid; j < NCOL; j += NT) su[j] = to_f32(wg[j]) * to_f32(v[j]);
  __syncthreads();
  if (tid < 32) {
    float acc = 0.f;
    for (int i = tid; i < DK; i += 32) acc = fmaf(sk[i], sq[i], acc);
    acc = warp_allreduce_sum(acc);
    if (tid == 0) s_kq = acc;
  }

  float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), p4 = r4;
#pragma unroll
  for (int x = 0; x < RPT; ++x) {
    const int row = rg + x * RG;
    const float g = sal[row], ai = sa[row], qi = sq[row];
    s[x].x *= g; s[x].y *= g; s[x].z *= g; s[x].w *= g;
    r4.x = fmaf(ai, s[x].x, r4.x); r4.y = fmaf(ai, s[x].y, r4.y);
    r4.z = fmaf(ai, s[x].z, r4.z); r4.w = fmaf(ai, s[x].w, r4.w);
    p4.x = fmaf(qi, s[x].x, p4.x); p4.y = fmaf(qi, s[x].y, p4.y);
    p4.z = fmaf(qi, s[x].z, p4.z); p4.w = fmaf(qi, s[x].w, p4.w);
  }
  *reinterpret_cast<float4 *>(&red_r[rg][4 * cq]) = r4;
  *reinterpret_cast<float4 *>(&red_p[rg][4 * cq]) = p4;
  __syncthreads();
  for (int j = tid; j < NCOL; j += NT) {
    float r = 0.f, p = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
      r += red_r[g][j];
      p += red_p[g][j];
    }
    const float d = su[j] - r;
    sd[j] = d;
    ((Tin *)a.o)[(size_t)head * DV + c0 + j] = from_f32<Tin>(fmaf(s_kq, d, p));
  }
  __syncthreads();
  const float4 d4 = *reinterpret_cast<const float4 *>(&sd[4 * cq]);
#pragma unroll
  for (int x = 0; x < RPT; ++x) {
    const float kk = sk[rg + x * RG];
    s[x].x = fmaf(kk, d4.x, s[x].x); s[x].y = fmaf(kk, d4.y, s[x].y);
    s[x].z = fmaf(kk, d4.z, s[x].z); s[x].w = fmaf(kk, d4.w, s[x].w);
    __stcs(reinterpret_cast<float4 *>(Sh + (size_t)(rg + x * RG) * DV), s[x]);
  }
}

template <int DK, int NCOL, int NT, typename Tin>
cudaError_t launch_decode_typed(const DecodeArgs &a, cudaStream_t stream) {
  const long long blocks = (long long)a.B * a.H * (a.dv / NCOL);
  if (blocks == 0) return cudaSuccess;
  note_launch();
  decode_step_kernel<DK, NCOL, NT, Tin><<<(unsigned)blocks, NT, 0, stream>>>(a);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_decode_dtype(const DecodeArgs &a, cudaStream_t stream) {
  // 64 value columns per CTA, 128 threads: 16 rows x 4 columns per thread at d_k = 128
  if (a.dk == 64) return launch_decode_typed<64, 64, 128, Tin>(a, stream);
  return launch_decode_typed<128, 64, 128, Tin>(a, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, bool bf16, cudaStream_t stream) {
  return bf16 ? launch_decode_dtype<__nv_bfloat16>(a, stream) : launch_decode_dtype<float>(a, stream);
}

}  // namespace gdn2
