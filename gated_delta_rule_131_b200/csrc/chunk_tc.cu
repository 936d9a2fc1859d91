// Chunkwise WY forward of the Gated Delta Rule-2 on the sm_100a tensor cores
// (bf16 inputs, d_k = 128, fp32 state and accumulation).
//
// Per chunk of C = 64 tokens (r, i index tokens, c a key channel, m the
// running log-decay at token 31 of the chunk, g_r the running log-decay at r):
//   f_r       = exp(g_r - m)                       per key channel (bounded by the
//                                                  decay over 32 tokens either way)
//   A_m       = (b (.) k) (.) f,  Q_m = q (.) f,   K_m = k (.) 1/f
//   [L; P]    = [A_m; Q_m] K_m^T                   L strictly, P inclusively lower
//   T         = (I + L)^-1                         fp32 blocked forward substitution
//   Delta     = T U - T A_m (e^m S)                U = w (.) v
//   O         = Q S + P Delta = [P T] U + (Q_m - [P T] A_m) (e^m S)
//   S_next    = e^{g_C} S + e^{g_C - m} K_m^T Delta
// so one tensor-core pass per chunk forms, in TMEM,
//   D_a = [T U; P T U] + [-T A_m; Q_m - P T A_m] (e^m S) = [Delta; O].
// The decay-absorbed asymmetric erase factors follow the block formulation of
// "Gated DeltaNet-2: Separando Borrado y Escritura en la Atención Lineal"
// (needhelp.icu), "Innovaciones Técnicas", item 1; the update itself is the
// per-token rule of "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com),
// "Gated DeltaNet-2の核心" (decay first, key-side erase gate b, value-side write
// gate w, o_t = S_t^T q_t).
//
// One CTA per (sequence, head, 64 value columns); 256 threads; 2 CTAs per SM.
// Shared memory holds every operand in the 128-byte-swizzled layout that TMA
// writes and tcgen05.mma reads, so the raw q, k, b tiles are turned into the
// factor operands in place.  The state slice lives in fp32 registers (thread =
// key channel x 32 value columns); TMEM holds the MMA accumulators:
//   cols [0, 64)    L|P, then P T, then K_m^T Delta
//   cols [64, 192)  [T; P T] A_m
//   cols [192, 256) D_a = [Delta; O]
// Precondition of the factorisation: per key channel, the decay accumulated
// over any 32 consecutive tokens of a chunk stays above about e^-80 (the fp32
// range); every workload here is far inside it.
#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {

__device__ int g_device_status = 0;  // GDN2_ERR_TIMEOUT (4) when a bounded wait gave up

cudaError_t read_device_status(int *status, bool reset) {
  cudaError_t err = cudaMemcpyFromSymbol(status, g_device_status, sizeof(int));
  if (err == cudaSuccess && reset) {
    const int zero = 0;
    err = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  }
  return err;
}

namespace {

using namespace ptx;

constexpr int C = 64, DK = 128, NV = 64, NT = 256;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t XA_BLK = 16384;            // [A_m ; Q_m] 128 rows x 64 ch, two channel blocks
constexpr uint32_t KT_BLK = 8192;             // K_m 64 rows x 64 ch, two channel blocks
constexpr uint32_t OFF_XA = 0;
constexpr uint32_t OFF_KT = OFF_XA + 2 * XA_BLK;   // 32768
constexpr uint32_t OFF_AL = OFF_KT + 2 * KT_BLK;   // 49152: alpha tiles, then T (fp32 64x64)
constexpr uint32_t OFF_U = OFF_AL + 16384;         // 65536: v tile -> U
constexpr uint32_t OFF_W = OFF_U + 8192;           // 73728: w tile    } L (fp32 64x64) spans
constexpr uint32_t OFF_DL = OFF_W + 8192;          // 81920: Delta     }   both slots
constexpr uint32_t OFF_TP = OFF_DL + 8192;         // 90112: [T ; P | P T] 128 x 64, later e^m S
constexpr uint32_t OFF_SC = OFF_TP + 16384;        // 106496: decay products and per-channel scalars
constexpr uint32_t OFF_BAR = OFF_SC + 4 * 128 * 4 + 3 * 128 * 4;  // 110080
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base
constexpr uint32_t TMA_BYTES = 10 * 8192;          // q, k, b, alpha (2 boxes each), v, w
constexpr uint32_t TMEM_COLS = 256;
constexpr uint64_t WAIT_NS = 2000000000ull;        // bounded waits: 2 s

constexpr uint32_t ID_LP = idesc_bf16(128, 64, false, false);    // [A_m;Q_m] K_m^T
constexpr uint32_t ID_KM64 = idesc_bf16(128, 64, false, true);   // K-major A, MN-major B, N = 64
constexpr uint32_t ID_KM128 = idesc_bf16(128, 128, false, true); // same, N = 128
constexpr uint32_t ID_MNMN = idesc_bf16(128, 64, true, true);    // K_m^T Delta

// fp32 64x64 scratch with the column index XOR-swizzled by the row, so that a warp
// writing one column across 32 rows hits 32 different banks
__device__ __forceinline__ float &f64x64(float *base, int r, int c) { return base[r * 64 + (c ^ (r & 31))]; }

__device__ __forceinline__ uint4 ld_s128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void st_s128(uint8_t *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }

// Every thread waits; the CTA then agrees on the outcome (so control flow stays uniform).
__device__ __forceinline__ bool cta_wait(uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait_bounded(bar, parity, WAIT_NS);
  return !__syncthreads_or(!ok);
}

template <typename Tout>
__device__ __forceinline__ void store_row32(Tout *dst, const float (&v)[32]);
template <>
__device__ __forceinline__ void store_row32<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&v)[32]) {
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    uint4 u;
    u.x = f2_to_bf2(v[8 * x + 0], v[8 * x + 1]);
    u.y = f2_to_bf2(v[8 * x + 2], v[8 * x + 3]);
    u.z = f2_to_bf2(v[8 * x + 4], v[8 * x + 5]);
    u.w = f2_to_bf2(v[8 * x + 6], v[8 * x + 7]);
    reinterpret_cast<uint4 *>(dst)[x] = u;
  }
}

__global__ void __launch_bounds__(NT, 2)
    chunk_fwd_tc_kernel(const ChunkArgs a, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_al, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  float *pp = reinterpret_cast<float *>(sm + OFF_SC);  // [4][128] decay product of each 16-token quarter
  float *s_em = pp + 512;                              // e^m       (decay from chunk start to token 31)
  float *s_egcm = s_em + 128;                          // e^{g_C-m} (decay over tokens 32..end)
  float *s_egc = s_egcm + 128;                         // e^{g_C}   (decay over the whole chunk)
  const uint32_t bar_ld = sb + OFF_BAR, bar_mma = sb + OFF_BAR + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);
  float *Ls = reinterpret_cast<float *>(sm + OFF_W);
  float *Ts = reinterpret_cast<float *>(sm + OFF_AL);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, quad = warp & 3, half = warp >> 2;
  const int tiles = a.dv / NV;
  const int tile = blockIdx.x % tiles;
  const int h = (blockIdx.x / tiles) % a.H;
  const int n = blockIdx.x / (tiles * a.H);
  const int j0 = tile * NV;
  int64_t bos;
  int len;
  seq_span(a, n, bos, len);
  __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(a.o);

  if (tid == 0) {
    mbar_init(bar_ld, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_al); prefetch_tmap(&tm_v); prefetch_tmap(&tm_w);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16);  // this warp's TMEM lane quadrant

  // state slice: key channel c_me, value columns j0 + 32*half .. +31
  const int c_me = 32 * quad + lane;
  const size_t s_off = (((size_t)n * a.H + h) * DK + c_me) * (size_t)a.dv + j0 + 32 * half;
  float S[32];
  if (a.S0) {
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const float4 t = reinterpret_cast<const float4 *>(a.S0 + s_off)[x];
      S[4 * x] = t.x; S[4 * x + 1] = t.y; S[4 * x + 2] = t.z; S[4 * x + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int x = 0; x < 32; ++x) S[x] = 0.f;
  }

  uint32_t ph_ld = 0, ph_mma = 0;
  bool ok = true;
  for (int c0 = 0; c0 < len; c0 += C) {
    const int Cc = min(C, len - c0);
    const int tok0 = (int)(bos + c0);

    // ---------------------------------------------------------------- A: TMA loads of the chunk
    if (tid == 0) {
      fence_proxy_async();
      mbar_expect_tx(bar_ld, TMA_BYTES);
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        tma_load_3d(sb + OFF_XA + blk * XA_BLK, &tm_b, 64 * blk, h, tok0, bar_ld);         // b -> rows 0..63
        tma_load_3d(sb + OFF_XA + blk * XA_BLK + 8192, &tm_q, 64 * blk, h, tok0, bar_ld);  // q -> rows 64..127
        tma_load_3d(sb + OFF_KT + blk * KT_BLK, &tm_k, 64 * blk, h, tok0, bar_ld);
        tma_load_3d(sb + OFF_AL + blk * 8192, &tm_al, 64 * blk, h, tok0, bar_ld);
      }
      tma_load_3d(sb + OFF_U, &tm_v, j0, h, tok0, bar_ld);
      tma_load_3d(sb + OFF_W, &tm_w, j0, h, tok0, bar_ld);
    }
    if (!(ok = cta_wait(bar_ld, ph_ld))) break;
    ph_ld ^= 1;

    // ---------------------------------------------------------------- B: decay factors, operands
    const int cp = tid & 63, qq = tid >> 6;  // channel pair (2cp, 2cp+1), token quarter qq
    const int cb = (2 * cp) >> 6, cc = (2 * cp) & 63;
    {
      float p0 = 1.f, p1 = 1.f;
#pragma unroll 4
      for (int rr = 0; rr < 16; ++rr) {
        const int r = 16 * qq + rr;
        if (r < Cc) {
          const float2 al = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + OFF_AL + cb * 8192 + sw128(r, cc)));
          p0 *= al.x;
          p1 *= al.y;
        }
      }
      pp[qq * 128 + 2 * cp] = p0;
      pp[qq * 128 + 2 * cp + 1] = p1;
    }
    __syncthreads();
    if (tid < 128) {
      const float em = pp[tid] * pp[128 + tid], egcm = pp[256 + tid] * pp[384 + tid];
      s_em[tid] = em;
      s_egcm[tid] = egcm;
      s_egc[tid] = em * egcm;
    }
    {
      // f_r = e^{g_r - m}: tokens 0..31 walk backwards from token 31, tokens 32..63 forwards
      float2 run;
      if (qq == 0) run = make_float2(pp[128 + 2 * cp], pp[128 + 2 * cp + 1]);
      else if (qq == 3) run = make_float2(pp[256 + 2 * cp], pp[256 + 2 * cp + 1]);
      else run = make_float2(1.f, 1.f);
#pragma unroll 2
      for (int s = 0; s < 16; ++s) {
        const int r = (qq < 2) ? (16 * qq + 15 - s) : (16 * qq + s);
        const uint32_t oa = OFF_XA + cb * XA_BLK + sw128(r, cc);
        const uint32_t oq = oa + 8192;
        const uint32_t ok_ = OFF_KT + cb * KT_BLK + sw128(r, cc);
        float2 al = make_float2(1.f, 1.f);
        if (r < Cc) al = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + OFF_AL + cb * 8192 + sw128(r, cc)));
        float2 f, fi;
        if (qq < 2) {
          fi = run;
          f = make_float2(__frcp_rn(run.x), __frcp_rn(run.y));
          run.x *= al.x;
          run.y *= al.y;
        } else {
          run.x *= al.x;
          run.y *= al.y;
          f = run;
          fi = make_float2(__frcp_rn(run.x), __frcp_rn(run.y));
        }
        uint32_t wa = 0u, wq = 0u, wk = 0u;
        if (r < Cc) {
          const float2 bb = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + oa));
          const float2 qv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + oq));
          const float2 kv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + ok_));
          wa = f2_to_bf2(bb.x * kv.x * f.x, bb.y * kv.y * f.y);
          wq = f2_to_bf2(qv.x * f.x, qv.y * f.y);
          wk = f2_to_bf2(kv.x * fi.x, kv.y * fi.y);
        }
        *reinterpret_cast<uint32_t *>(sm + oa) = wa;
        *reinterpret_cast<uint32_t *>(sm + oq) = wq;
        *reinterpret_cast<uint32_t *>(sm + ok_) = wk;
      }
    }
    {  // U = w (.) v for the 64 value columns of this CTA
      const int r = tid >> 2;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int col = 16 * (tid & 3) + 8 * x;
        uint8_t *pu = sm + OFF_U + sw128(r, col);
        const uint4 vv = ld_s128(pu), ww = ld_s128(sm + OFF_W + sw128(r, col));
        uint4 uu = make_uint4(0u, 0u, 0u, 0u);
        if (r < Cc) {
          float2 a0 = bf2_to_f2(vv.x), b0 = bf2_to_f2(ww.x), a1 = bf2_to_f2(vv.y), b1 = bf2_to_f2(ww.y);
          float2 a2 = bf2_to_f2(vv.z), b2 = bf2_to_f2(ww.z), a3 = bf2_to_f2(vv.w), b3 = bf2_to_f2(ww.w);
          uu.x = f2_to_bf2(a0.x * b0.x, a0.y * b0.y);
          uu.y = f2_to_bf2(a1.x * b1.x, a1.y * b1.y);
          uu.z = f2_to_bf2(a2.x * b2.x, a2.y * b2.y);
          uu.w = f2_to_bf2(a3.x * b3.x, a3.y * b3.y);
        }
        st_s128(pu, uu);
      }
    }
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M1: [L; P] = [A_m; Q_m] K_m^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < DK / 16; ++k) {
        const uint32_t koff = (uint32_t)(k & 3) * 32u;
        const uint64_t ad = sdesc_sw128(sb + OFF_XA + (k >> 2) * XA_BLK + koff, 16, 1024);
        const uint64_t bd = sdesc_sw128(sb + OFF_KT + (k >> 2) * KT_BLK + koff, 16, 1024);
        mma_bf16(tmem + 0, ad, bd, ID_LP, k > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();

    // ---------------------------------------------------------------- C: T = (I + L)^-1
    {
      float v[32];
      tmem_ld32(tl + 0 + 32 * half, v);
      tmem_wait_ld();
      const int row = 32 * quad + lane;
      if (row < 64) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int i = 32 * half + j;
          f64x64(Ls, row, i) = (i < row) ? v[j] : 0.f;
        }
      } else {  // P (inclusive lower) -> rows 64..127 of the TP tile, bf16
        const int r = row - 64;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int col = 32 * half + 8 * x;
          float e[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) e[t] = (col + t <= r) ? v[8 * x + t] : 0.f;
          st_s128(sm + OFF_TP + sw128(row, col),
                  make_uint4(f2_to_bf2(e[0], e[1]), f2_to_bf2(e[2], e[3]), f2_to_bf2(e[4], e[5]), f2_to_bf2(e[6], e[7])));
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp < 2) {  // the four 16x16 diagonal blocks: lane = column j of block R
      const int R = 2 * warp + (lane >> 4), j = lane & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < r; ++i) acc = fmaf(-f64x64(Ls, 16 * R + r, 16 * R + i), x[i], acc);
        x[r] = acc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) f64x64(Ts, 16 * R + r, 16 * R + j) = x[r];
    }
    __syncthreads();
    for (int R = 1; R < 4; ++R) {  // block row R: T_RI = -T_RR sum_{J=I}^{R-1} L_RJ T_JI
      for (int e = tid; e < 256 * R; e += NT) {
        const int I = e >> 8, rr = (e >> 4) & 15, ci = e & 15;
        float acc = 0.f;
        for (int J = I; J < R; ++J)
#pragma unroll
          for (int k = 0; k < 16; ++k)
            acc = fmaf(f64x64(Ls, 16 * R + rr, 16 * J + k), f64x64(Ts, 16 * J + k, 16 * I + ci), acc);
        f64x64(Ls, 16 * I + rr, 16 * R + ci) = acc;  // park Y_RI in the unused upper block (I, R)
      }
      __syncthreads();
      for (int e = tid; e < 256 * R; e += NT) {
        const int I = e >> 8, rr = (e >> 4) & 15, ci = e & 15;
        float acc = 0.f;
        for (int k = 0; k <= rr; ++k)
          acc = fmaf(f64x64(Ts, 16 * R + rr, 16 * R + k), f64x64(Ls, 16 * I + k, 16 * R + ci), acc);
        f64x64(Ts, 16 * R + rr, 16 * I + ci) = -acc;
      }
      __syncthreads();
    }
    {  // T -> rows 0..63 of the TP tile, bf16, zero above the diagonal
      const int r = tid >> 2;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int col = 16 * (tid & 3) + 8 * x;
        float e[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) e[t] = (col + t <= r) ? f64x64(Ts, r, col + t) : 0.f;
        st_s128(sm + OFF_TP + sw128(r, col),
                make_uint4(f2_to_bf2(e[0], e[1]), f2_to_bf2(e[2], e[3]), f2_to_bf2(e[4], e[5]), f2_to_bf2(e[6], e[7])));
      }
    }
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M2: rows 64..127 <- P T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 0, sdesc_sw128(sb + OFF_TP + 32 * k, 16, 1024), sdesc_sw128(sb + OFF_TP + 2048 * k, 16384, 1024),
                 ID_KM64, k > 0 ? 1u : 0u);
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();
    if (quad >= 2) {
      float v[32];
      tmem_ld32(tl + 0 + 32 * half, v);
      tmem_wait_ld();
      const int row = 32 * quad + lane;
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int col = 32 * half + 8 * x;
        st_s128(sm + OFF_TP + sw128(row, col),
                make_uint4(f2_to_bf2(v[8 * x], v[8 * x + 1]), f2_to_bf2(v[8 * x + 2], v[8 * x + 3]),
                           f2_to_bf2(v[8 * x + 4], v[8 * x + 5]), f2_to_bf2(v[8 * x + 6], v[8 * x + 7])));
      }
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M3, M4: [T; P T] [A_m | U]
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 64, sdesc_sw128(sb + OFF_TP + 32 * k, 16, 1024),
                 sdesc_sw128(sb + OFF_XA + 2048 * k, XA_BLK, 1024), ID_KM128, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 192, sdesc_sw128(sb + OFF_TP + 32 * k, 16, 1024), sdesc_sw128(sb + OFF_U + 2048 * k, 8192, 1024),
                 ID_KM64, k > 0 ? 1u : 0u);
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();

    // ---------------------------------------------------------------- E: [-T A_m; Q_m - P T A_m] in place; e^m S
    {
      const int row = 32 * quad + lane;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float v[32];
        tmem_ld32(tl + 64 + 64 * half + 32 * part, v);
        tmem_wait_ld();
        uint8_t *base = sm + OFF_XA + half * XA_BLK;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int col = 32 * part + 8 * x;
          uint8_t *p = base + sw128(row, col);
          uint4 u;
          if (row < 64) {
            u = make_uint4(f2_to_bf2(-v[8 * x], -v[8 * x + 1]), f2_to_bf2(-v[8 * x + 2], -v[8 * x + 3]),
                           f2_to_bf2(-v[8 * x + 4], -v[8 * x + 5]), f2_to_bf2(-v[8 * x + 6], -v[8 * x + 7]));
          } else {
            const uint4 qm = ld_s128(p);
            const float2 q0 = bf2_to_f2(qm.x), q1 = bf2_to_f2(qm.y), q2 = bf2_to_f2(qm.z), q3 = bf2_to_f2(qm.w);
            u = make_uint4(f2_to_bf2(q0.x - v[8 * x], q0.y - v[8 * x + 1]), f2_to_bf2(q1.x - v[8 * x + 2], q1.y - v[8 * x + 3]),
                           f2_to_bf2(q2.x - v[8 * x + 4], q2.y - v[8 * x + 5]),
                           f2_to_bf2(q3.x - v[8 * x + 6], q3.y - v[8 * x + 7]));
          }
          st_s128(p, u);
        }
      }
      const float em = s_em[c_me];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int col = 32 * half + 8 * x;
        st_s128(sm + OFF_TP + sw128(c_me, col),
                make_uint4(f2_to_bf2(em * S[8 * x], em * S[8 * x + 1]), f2_to_bf2(em * S[8 * x + 2], em * S[8 * x + 3]),
                           f2_to_bf2(em * S[8 * x + 4], em * S[8 * x + 5]), f2_to_bf2(em * S[8 * x + 6], em * S[8 * x + 7])));
      }
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M5: D_a += [-T A_m; Q_m - P T A_m] (e^m S)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < DK / 16; ++k)
        mma_bf16(tmem + 192, sdesc_sw128(sb + OFF_XA + (k >> 2) * XA_BLK + (k & 3) * 32, 16, 1024),
                 sdesc_sw128(sb + OFF_TP + 2048 * k, 16384, 1024), ID_KM64, 1u);
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();

    // ---------------------------------------------------------------- F: Delta -> smem, O -> global
    {
      float v[32];
      tmem_ld32(tl + 192 + 32 * half, v);
      tmem_wait_ld();
      const int row = 32 * quad + lane;
      if (row < 64) {
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int col = 32 * half + 8 * x;
          st_s128(sm + OFF_DL + sw128(row, col),
                  make_uint4(f2_to_bf2(v[8 * x], v[8 * x + 1]), f2_to_bf2(v[8 * x + 2], v[8 * x + 3]),
                             f2_to_bf2(v[8 * x + 4], v[8 * x + 5]), f2_to_bf2(v[8 * x + 6], v[8 * x + 7])));
        }
      } else if (row - 64 < Cc) {
        __nv_bfloat16 *dst = o + ((size_t)(tok0 + row - 64) * a.H + h) * (size_t)a.dv + j0 + 32 * half;
        store_row32(dst, v);
      }
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M6: K_m^T Delta
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 0, sdesc_sw128(sb + OFF_KT + 2048 * k, KT_BLK, 1024), sdesc_sw128(sb + OFF_DL + 2048 * k, 8192, 1024),
                 ID_MNMN, k > 0 ? 1u : 0u);
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();

    // ---------------------------------------------------------------- G: state update
    {
      float v[32];
      tmem_ld32(tl + 0 + 32 * half, v);
      tmem_wait_ld();
      const float g1 = s_egc[c_me], g2 = s_egcm[c_me];
#pragma unroll
      for (int j = 0; j < 32; ++j) S[j] = fmaf(g2, v[j], g1 * S[j]);
    }
    tc_fence_before();
    __syncthreads();
  }

  if (ok && a.ST) {
#pragma unroll
    for (int x = 0; x < 8; ++x)
      reinterpret_cast<float4 *>(a.ST + s_off)[x] = make_float4(S[4 * x], S[4 * x + 1], S[4 * x + 2], S[4 * x + 3]);
  }
  if (!ok && tid == 0) atomicExch(&g_device_status, 4);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side: tensor maps
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// [tokens, H, D] bf16 tensor, box = 64 channels x 1 head x 64 tokens, 128-byte swizzle
bool make_map(CUtensorMap *m, const void *base, long long tokens, int H, int D) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)(tokens > 0 ? tokens : 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs &a, bool bf16) { return bf16 && a.dk == DK && a.dv % NV == 0; }

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream) {
  const long long tokens = a.cu ? (long long)a.T : (long long)a.B * a.T;
  const long long blocks = (long long)a.B * a.H * (a.dv / NV);
  if (blocks == 0) return cudaSuccess;
  // with no token in the batch no chunk is processed and no map can be encoded on a NULL base:
  // the SIMT kernel does the remaining work (S_T = S0)
  if (tokens == 0) return launch_chunk_simt(a, true, stream);
  CUtensorMap mq, mk, mb, mal, mv, mw;
  if (!make_map(&mq, a.q, tokens, a.H, DK) || !make_map(&mk, a.k, tokens, a.H, DK) ||
      !make_map(&mb, a.b, tokens, a.H, DK) || !make_map(&mal, a.alpha, tokens, a.H, DK) ||
      !make_map(&mv, a.v, tokens, a.H, a.dv) || !make_map(&mw, a.w, tokens, a.H, a.dv))
    return cudaErrorInvalidValue;
  cudaError_t err = cudaFuncSetAttribute(chunk_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (err != cudaSuccess) return err;
  note_launch();
  chunk_fwd_tc_kernel<<<(unsigned)blocks, NT, SMEM_BYTES, stream>>>(a, mq, mk, mb, mal, mv, mw);
  return cudaGetLastError();
}

}  // namespace gdn2
