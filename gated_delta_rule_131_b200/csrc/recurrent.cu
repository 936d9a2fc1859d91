// Token-by-token recurrent forward of the Gated Delta Rule-2 over whole sequences, for either
// reading of the erase orientation (the pages print no equation; see include/gdn2.h):
//
//   R1:  S_t = (I - k_t a_t^T) Diag(alpha_t) S_{t-1} + k_t u_t^T     (the reading gdn2_chunk_fwd computes)
//   R2:  S_t = (I - a_t k_t^T) Diag(alpha_t) S_{t-1} + k_t u_t^T
//   o_t = S_t^T q_t,   a_t = b_t (.) k_t,   u_t = w_t (.) v_t.
//
// Both follow the per-token rule of "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com),
// "Gated DeltaNet-2の核心": decay on the key axis first, the erase gated per key channel by b,
// the write gated per value channel by w.  With S' = Diag(alpha) S:
//   R1:  r = S'^T a,  S = S' + k (u - r)^T,           o = S'^T q + (k.q)(u - r)
//   R2:  r = S'^T k,  S = S' - a r^T + k u^T,         o = S'^T q - (a.q) r + (k.q) u
// so each token needs one pass over the state: two column reductions (r and p = S'^T q) and one
// rank-1 (R1) or rank-2 (R2) update, with the readout formed from the reductions.
//
// One CTA per (sequence, head, 64 value columns), 128 threads; the CTA keeps its slice of the
// state in registers for the whole sequence (a thread holds 4 adjacent columns of d_k / 8 rows)
// and streams the token vectors through double-buffered shared memory.  The loop over tokens is
// serial, so this kernel serves the exact recurrence (any orientation, any length) rather than
// throughput; gdn2_chunk_fwd is the fast path for R1.
#include "common.cuh"

namespace gdn2 {
namespace {

template <int DK, int NCOL, int NT, typename Tin, bool R2>
__global__ void __launch_bounds__(NT) recurrent_fwd_kernel(RecurrentArgs a) {
  constexpr int TPR = NCOL / 4;   // threads across one row slice
  constexpr int RG = NT / TPR;    // row groups
  constexpr int RPT = DK / RG;    // rows per thread
  static_assert(NT % TPR == 0 && DK % RG == 0 && NT >= DK && NT >= NCOL, "tile shape");

  __shared__ float sq[2][DK], sk[2][DK], sa[2][DK], sal[2][DK];
  __shared__ float su[2][NCOL];
  __shared__ float sd[NCOL], sr[NCOL];
  __shared__ float red_r[RG][NCOL + 4], red_p[RG][NCOL + 4];
  __shared__ float s_kq[2], s_aq[2];

  const int tiles = a.dv / NCOL;
  const int c0 = (blockIdx.x % tiles) * NCOL;
  const int h = (blockIdx.x / tiles) % a.H;
  const int n = blockIdx.x / (tiles * a.H);
  const int tid = threadIdx.x;
  const int cq = tid % TPR, rg = tid / TPR;
  const int DV = a.dv, H = a.H;

  int64_t bos;
  int len;
  if (a.cu) {
    bos = a.cu[n];
    len = a.cu[n + 1] - a.cu[n];
  } else {
    bos = (int64_t)n * a.T;
    len = a.T;
  }

  const size_t sidx = ((size_t)n * H + h) * DK * DV + c0 + 4 * cq;
  float4 s[RPT];
#pragma unroll
  for (int x = 0; x < RPT; ++x)
    s[x] = a.S0 ? *reinterpret_cast<const float4 *>(a.S0 + sidx + (size_t)(rg + x * RG) * DV)
                : make_float4(0.f, 0.f, 0.f, 0.f);

  // token t's vectors -> buffer t & 1; k.q (and a.q) from warp 0
  auto stage = [&](int t) {
    const int buf = t & 1;
    const size_t row = (size_t)(bos + t) * H + h;
    const Tin *q = (const Tin *)a.q + row * DK, *k = (const Tin *)a.k + row * DK;
    const Tin *al = (const Tin *)a.alpha + row * DK, *bg = (const Tin *)a.b + row * DK;
    const Tin *v = (const Tin *)a.v + row * DV + c0, *wg = (const Tin *)a.w + row * DV + c0;
    if (tid < DK) {
      const float kk = to_f32(k[tid]);
      sk[buf][tid] = kk;
      sq[buf][tid] = to_f32(q[tid]);
      sa[buf][tid] = to_f32(bg[tid]) * kk;
      sal[buf][tid] = to_f32(al[tid]);
    }
    if (tid < NCOL) su[buf][tid] = to_f32(wg[tid]) * to_f32(v[tid]);
  };
  if (len > 0) stage(0);
  __syncthreads();
  for (int t = 0; t < len; ++t) {
    const int buf = t & 1;
    if (tid < 32) {  // k.q and a.q of this token
      float kq = 0.f, aq = 0.f;
      for (int i = tid; i < DK; i += 32) {
        kq = fmaf(sk[buf][i], sq[buf][i], kq);
        aq = fmaf(sa[buf][i], sq[buf][i], aq);
      }
      kq = warp_allreduce_sum(kq);
      aq = warp_allreduce_sum(aq);
      if (tid == 0) {
        s_kq[buf] = kq;
        s_aq[buf] = aq;
      }
    }
    // decay, then the partial column sums r (probe a for R1, k for R2) and p (query)
    float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), p4 = r4;
#pragma unroll
    for (int x = 0; x < RPT; ++x) {
      const int row = rg + x * RG;
      const float g = sal[buf][row], pi = R2 ? sk[buf][row] : sa[buf][row], qi = sq[buf][row];
      s[x].x *= g; s[x].y *= g; s[x].z *= g; s[x].w *= g;
      r4.x = fmaf(pi, s[x].x, r4.x); r4.y = fmaf(pi, s[x].y, r4.y);
      r4.z = fmaf(pi, s[x].z, r4.z); r4.w = fmaf(pi, s[x].w, r4.w);
      p4.x = fmaf(qi, s[x].x, p4.x); p4.y = fmaf(qi, s[x].y, p4.y);
      p4.z = fmaf(qi, s[x].z, p4.z); p4.w = fmaf(qi, s[x].w, p4.w);
    }
    *reinterpret_cast<float4 *>(&red_r[rg][4 * cq]) = r4;
    *reinterpret_cast<float4 *>(&red_p[rg][4 * cq]) = p4;
    if (t + 1 < len) stage(t + 1);  // the other buffer: its last readers finished before the last barrier
    __syncthreads();
    if (tid < NCOL) {
      const int j = tid;
      float r = 0.f, p = 0.f;
#pragma unroll
      for (int g = 0; g < RG; ++g) {
        r += red_r[g][j];
        p += red_p[g][j];
      }
      const float u = su[buf][j];
      float o;
      if (R2) {
        sr[j] = r;
        o = fmaf(s_kq[buf], u, fmaf(-s_aq[buf], r, p));
      } else {
        const float d = u - r;
        sd[j] = d;
        o = fmaf(s_kq[buf], d, p);
      }
      ((Tin *)a.o)[((size_t)(bos + t) * H + h) * DV + c0 + j] = from_f32<Tin>(o);
    }
    __syncthreads();
    if (R2) {  // S = S' - a r^T + k u^T
      const float4 r = *reinterpret_cast<const float4 *>(&sr[4 * cq]);
      const float4 u = *reinterpret_cast<const float4 *>(&su[buf][4 * cq]);
#pragma unroll
      for (int x = 0; x < RPT; ++x) {
        const int row = rg + x * RG;
        const float ai = sa[buf][row], kk = sk[buf][row];
        s[x].x = fmaf(kk, u.x, fmaf(-ai, r.x, s[x].x)); s[x].y = fmaf(kk, u.y, fmaf(-ai, r.y, s[x].y));
        s[x].z = fmaf(kk, u.z, fmaf(-ai, r.z, s[x].z)); s[x].w = fmaf(kk, u.w, fmaf(-ai, r.w, s[x].w));
      }
    } else {  // S = S' + k (u - r)^T
      const float4 d = *reinterpret_cast<const float4 *>(&sd[4 * cq]);
#pragma unroll
      for (int x = 0; x < RPT; ++x) {
        const float kk = sk[buf][rg + x * RG];
        s[x].x = fmaf(kk, d.x, s[x].x); s[x].y = fmaf(kk, d.y, s[x].y);
        s[x].z = fmaf(kk, d.z, s[x].z); s[x].w = fmaf(kk, d.w, s[x].w);
      }
    }
    __syncthreads();  // sd / sr and this token's buffer are free again
  }
  if (a.ST) {
#pragma unroll
    for (int x = 0; x < RPT; ++x) *reinterpret_cast<float4 *>(a.ST + sidx + (size_t)(rg + x * RG) * DV) = s[x];
  }
}

template <int DK, typename Tin, bool R2>
cudaError_t launch_recurrent_typed(const RecurrentArgs &a, cudaStream_t stream) {
  constexpr int NCOL = 64, NT = 128;
  const long long blocks = (long long)a.B * a.H * (a.dv / NCOL);
  if (blocks == 0) return cudaSuccess;
  note_launch();
  recurrent_fwd_kernel<DK, NCOL, NT, Tin, R2><<<(unsigned)blocks, NT, 0, stream>>>(a);
  return cudaGetLastError();
}

template <typename Tin, bool R2>
cudaError_t launch_recurrent_dk(const RecurrentArgs &a, cudaStream_t stream) {
  return a.dk == 64 ? launch_recurrent_typed<64, Tin, R2>(a, stream) : launch_recurrent_typed<128, Tin, R2>(a, stream);
}

}  // namespace

cudaError_t launch_recurrent(const RecurrentArgs &a, bool bf16, bool r2, cudaStream_t stream) {
  if (bf16) return r2 ? launch_recurrent_dk<__nv_bfloat16, true>(a, stream) : launch_recurrent_dk<__nv_bfloat16, false>(a, stream);
  return r2 ? launch_recurrent_dk<float, true>(a, stream) : launch_recurrent_dk<float, false>(a, stream);
}

}  // namespace gdn2
