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
//   O         = Q S + P Delta = Q_m (e^m S) + P Delta
//   S_next    = e^{g_C} S + e^{g_C - m} K_m^T Delta
// so, in TMEM, D_a = [T U; 0] + [-T A_m; Q_m] (e^m S) = [Delta; Q S], then
// D_a += [P; P] Delta leaves O in its lower half (the upper half, Delta, has
// been read out by then).
// The decay-absorbed asymmetric erase factors follow the block formulation of
// "Gated DeltaNet-2: Separando Borrado y Escritura en la Atención Lineal"
// (needhelp.icu), "Innovaciones Técnicas", item 1; the update itself is the
// per-token rule of "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com),
// "Gated DeltaNet-2の核心" (decay first, key-side erase gate b, value-side write
// gate w, o_t = S_t^T q_t).
//
// One CTA per (sequence, head, 64 value columns); 256 threads.
// Shared memory holds every operand in the 128-byte-swizzled layout that TMA
// writes and tcgen05.mma reads, so the raw q, k, b tiles are turned into the
// factor operands in place.  The state slice lives in fp32 registers (thread =
// key channel x 32 value columns); TMEM holds the MMA accumulators:
//   cols [0, 64)    L|P, then K_m^T Delta
//   cols [64, 192)  [T; 0] A_m
//   cols [192, 256) D_a = [Delta; O]
// T is formed in fp32: the four 16x16 diagonal blocks by right-looking
// substitution, then merged into 32x32 and 64x64 inverses with
// [[A,0],[C,B]]^-1 = [[A^-1,0],[-B^-1 C A^-1, B^-1]].
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

// shared-memory map (bytes from a 1024-aligned base); every MMA operand tile is 1024-aligned
constexpr uint32_t XA_BLK = 16384;                 // [A_m | -T A_m ; Q_m] 128 rows x 64 ch, two channel blocks
constexpr uint32_t KT_BLK = 8192;                  // K_m 64 rows x 64 ch, two channel blocks
constexpr uint32_t OFF_XA = 0;
constexpr uint32_t OFF_KT = OFF_XA + 2 * XA_BLK;   // 32768
constexpr uint32_t OFF_AL = OFF_KT + 2 * KT_BLK;   // 49152: alpha tiles (two blocks)
constexpr uint32_t OFF_U = OFF_AL + 16384;         // 65536: v tile -> U = w (.) v
constexpr uint32_t OFF_W = OFF_U + 8192;           // 73728: w tile
constexpr uint32_t OFF_DL = OFF_W + 8192;          // 81920: Delta, bf16 64 x 64
constexpr uint32_t OFF_TZ = OFF_DL + 8192;         // 90112: [T ; 0] bf16 128 x 64
constexpr uint32_t OFF_PP = OFF_TZ + 16384;        // 106496: [P ; P] bf16 128 x 64
constexpr uint32_t OFF_SM = OFF_PP + 16384;        // 122880: e^m S, bf16 128 x 64
constexpr int LDF = 68;                            // row stride of the fp32 64 x 64 scratch
constexpr uint32_t OFF_LS = OFF_SM + 16384;        // 139264: L (fp32), upper blocks reused as scratch
constexpr uint32_t OFF_TS = OFF_LS + 64 * LDF * 4; // 156672: T (fp32)
constexpr uint32_t OFF_SC = OFF_TS + 64 * LDF * 4; // 174080: decay products and per-channel scalars
constexpr uint32_t OFF_BAR = OFF_SC + 16 * 128 * 4 + 3 * 128 * 4;
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base
constexpr uint32_t TMA_BYTES = 10 * 8192;          // q, k, b, alpha (2 boxes each), v, w
constexpr uint32_t TMEM_COLS = 256;
constexpr uint64_t WAIT_NS = 2000000000ull;        // bounded waits: 2 s

constexpr uint32_t ID_LP = idesc_bf16(128, 64, false, false);    // [A_m;Q_m] K_m^T
constexpr uint32_t ID_KM64 = idesc_bf16(128, 64, false, true);   // K-major A, MN-major B, N = 64
constexpr uint32_t ID_KM128 = idesc_bf16(128, 128, false, true); // same, N = 128
constexpr uint32_t ID_MNMN = idesc_bf16(128, 64, true, true);    // K_m^T Delta

__device__ __forceinline__ uint4 ld_s128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void st_s128(uint8_t *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }
__device__ __forceinline__ uint4 pack8(const float *e) {
  return make_uint4(f2_to_bf2(e[0], e[1]), f2_to_bf2(e[2], e[3]), f2_to_bf2(e[4], e[5]), f2_to_bf2(e[6], e[7]));
}
__device__ __forceinline__ float fast_rcp(float x) { return __fdividef(1.f, x); }

// Every thread waits; the CTA then agrees on the outcome (so control flow stays uniform).
__device__ __forceinline__ bool cta_wait(uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait_bounded(bar, parity, WAIT_NS);
  return !__syncthreads_or(!ok);
}

__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16 *dst, const float (&v)[32]) {
#pragma unroll
  for (int x = 0; x < 4; ++x) reinterpret_cast<uint4 *>(dst)[x] = pack8(&v[8 * x]);
}

__device__ __forceinline__ void unpack8(uint4 u, float *e) {
  float2 t = bf2_to_f2(u.x); e[0] = t.x; e[1] = t.y;
  t = bf2_to_f2(u.y); e[2] = t.x; e[3] = t.y;
  t = bf2_to_f2(u.z); e[4] = t.x; e[5] = t.y;
  t = bf2_to_f2(u.w); e[6] = t.x; e[7] = t.y;
}

// Decay-absorbed operands of one token row for 8 key channels, in place:
// A_m = b k f, Q_m = q f, K_m = k fi with f = e^{g_r - m}, fi = 1/f; rows >= Cc are zeroed.
__device__ __forceinline__ void row_factors(uint8_t *sm, int r, int cb, int x8, int Cc, const float *f, const float *fi) {
  uint8_t *pa = sm + OFF_XA + cb * XA_BLK + sw128(r, 8 * x8);
  uint8_t *pq = pa + 8192;
  uint8_t *pk = sm + OFF_KT + cb * KT_BLK + sw128(r, 8 * x8);
  uint4 wa = make_uint4(0u, 0u, 0u, 0u), wq = wa, wk = wa;
  if (r < Cc) {
    float bb[8], qv[8], kv[8], ea[8], eq[8], ek[8];
    unpack8(ld_s128(pa), bb);
    unpack8(ld_s128(pq), qv);
    unpack8(ld_s128(pk), kv);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      ea[t] = bb[t] * kv[t] * f[t];
      eq[t] = qv[t] * f[t];
      ek[t] = kv[t] * fi[t];
    }
    wa = pack8(ea);
    wq = pack8(eq);
    wk = pack8(ek);
  }
  st_s128(pa, wa);
  st_s128(pq, wq);
  st_s128(pk, wk);
}

__global__ void __launch_bounds__(NT, 1)
    chunk_fwd_tc_kernel(const ChunkArgs a, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_al, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  float *pp = reinterpret_cast<float *>(sm + OFF_SC);  // [16][128] decay product of each 4-token group
  float *s_em = pp + 16 * 128;                         // e^m       (decay from chunk start to token 31)
  float *s_egcm = s_em + 128;                          // e^{g_C-m} (decay over tokens 32..end)
  float *s_egc = s_egcm + 128;                         // e^{g_C}   (decay over the whole chunk)
  const uint32_t bar_ld = sb + OFF_BAR, bar_mma = sb + OFF_BAR + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);
  float *Ls = reinterpret_cast<float *>(sm + OFF_LS);
  float *Ts = reinterpret_cast<float *>(sm + OFF_TS);

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
  // zero rows 64..127 of [T ; 0] once, and the never-written upper blocks of T
  for (int e = tid; e < 8192 / 16; e += NT) st_s128(sm + OFF_TZ + 8192 + 16 * e, make_uint4(0u, 0u, 0u, 0u));
  for (int e = tid; e < 64 * LDF; e += NT) Ts[e] = 0.f;
  fence_proxy_async();
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
    {
      // thread = 8 key channels (chunk x8 of channel block cb) x 4 tokens (group G = rows 4G..4G+3);
      // warps 0-3 hold tokens 0..31 (walk back to token 31), warps 4-7 tokens 32..63 (walk forward)
      const int ch8 = tid & 15, G = tid >> 4, cb = ch8 >> 3, x8 = ch8 & 7;
      float al[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * G + i;
        if (r < Cc) {
          unpack8(ld_s128(sm + OFF_AL + cb * 8192 + sw128(r, 8 * x8)), al[i]);
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) al[i][t] = 1.f;
        }
      }
      float gp[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) gp[t] = al[0][t] * al[1][t] * al[2][t] * al[3][t];
      float *scan = pp;  // [16 groups][128 channels]: product of alpha over each 4-token group
      *reinterpret_cast<float4 *>(&scan[G * 128 + 8 * ch8]) = make_float4(gp[0], gp[1], gp[2], gp[3]);
      *reinterpret_cast<float4 *>(&scan[G * 128 + 8 * ch8 + 4]) = make_float4(gp[4], gp[5], gp[6], gp[7]);
      __syncthreads();
      if (tid < 128) {
        float em = 1.f, egcm = 1.f;
        for (int g = 0; g < 8; ++g) em *= scan[g * 128 + tid];
        for (int g = 8; g < 16; ++g) egcm *= scan[g * 128 + tid];
        s_em[tid] = em;
        s_egcm[tid] = egcm;
        s_egc[tid] = em * egcm;
      }
      float run[8];  // product of alpha strictly between this group and token 31 (inclusive of 31)
#pragma unroll
      for (int t = 0; t < 8; ++t) run[t] = 1.f;
      if (G < 8) {
        for (int g = G + 1; g < 8; ++g) {
          const float4 p0 = *reinterpret_cast<const float4 *>(&scan[g * 128 + 8 * ch8]);
          const float4 p1 = *reinterpret_cast<const float4 *>(&scan[g * 128 + 8 * ch8 + 4]);
          run[0] *= p0.x; run[1] *= p0.y; run[2] *= p0.z; run[3] *= p0.w;
          run[4] *= p1.x; run[5] *= p1.y; run[6] *= p1.z; run[7] *= p1.w;
        }
#pragma unroll
        for (int i = 3; i >= 0; --i) {  // run = prod_{r < s <= 31} alpha_s
          float f[8], fi[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            fi[t] = run[t];
            f[t] = fast_rcp(run[t]);
            run[t] *= al[i][t];
          }
          row_factors(sm, 4 * G + i, cb, x8, Cc, f, fi);
        }
      } else {
        for (int g = 8; g < G; ++g) {
          const float4 p0 = *reinterpret_cast<const float4 *>(&scan[g * 128 + 8 * ch8]);
          const float4 p1 = *reinterpret_cast<const float4 *>(&scan[g * 128 + 8 * ch8 + 4]);
          run[0] *= p0.x; run[1] *= p0.y; run[2] *= p0.z; run[3] *= p0.w;
          run[4] *= p1.x; run[5] *= p1.y; run[6] *= p1.z; run[7] *= p1.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // run = prod_{32 <= s <= r} alpha_s
          float f[8], fi[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            run[t] *= al[i][t];
            f[t] = run[t];
            fi[t] = fast_rcp(run[t]);
          }
          row_factors(sm, 4 * G + i, cb, x8, Cc, f, fi);
        }
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
    {  // L (strict lower) -> fp32 scratch; P (inclusive lower) -> both halves of [P ; P]
      float v[32];
      tmem_ld32(tl + 0 + 32 * half, v);
      tmem_wait_ld();
      const int row = 32 * quad + lane;
      if (row < 64) {
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const int i = 32 * half + 4 * x;
          *reinterpret_cast<float4 *>(&Ls[row * LDF + i]) =
              make_float4(i < row ? v[4 * x] : 0.f, i + 1 < row ? v[4 * x + 1] : 0.f, i + 2 < row ? v[4 * x + 2] : 0.f,
                          i + 3 < row ? v[4 * x + 3] : 0.f);
        }
      } else {
        const int r = row - 64;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int col = 32 * half + 8 * x;
          float e[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) e[t] = (col + t <= r) ? v[8 * x + t] : 0.f;
          const uint4 u = pack8(e);
          st_s128(sm + OFF_PP + sw128(r, col), u);
          st_s128(sm + OFF_PP + sw128(row, col), u);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp < 2) {  // the four 16x16 diagonal blocks, right-looking; lane = column j of block R
      const int R = 2 * warp + (lane >> 4), j = lane & 15;
      const float *Lb = Ls + 16 * R * LDF + 16 * R;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
      for (int i = 0; i < 15; ++i)
#pragma unroll
        for (int r = i + 1; r < 16; ++r) x[r] = fmaf(-Lb[r * LDF + i], x[i], x[r]);
      float *Tb = Ts + 16 * R * LDF + 16 * R;
#pragma unroll
      for (int r = 0; r < 16; ++r) Tb[r * LDF + j] = x[r];
    }
    __syncthreads();
    {  // T_{R,R-1} for R = 1, 3: Y = L_{R,R-1} T_{R-1,R-1} (parked in the upper block (R-1, R) of L)
      float acc[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int R = 1 + 2 * u, r = tid >> 4, c = tid & 15;
        const float *Lr = Ls + (16 * R + r) * LDF + 16 * (R - 1);
        const float *Tc = Ts + 16 * (R - 1) * LDF + 16 * (R - 1) + c;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) s = fmaf(Lr[k], Tc[k * LDF], s);
        acc[u] = s;
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int R = 1 + 2 * u, r = tid >> 4, c = tid & 15;
        Ls[(16 * (R - 1) + r) * LDF + 16 * R + c] = acc[u];
      }
    }
    __syncthreads();
    {  // T_{R,R-1} = -T_RR Y
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int R = 1 + 2 * u, r = tid >> 4, c = tid & 15;
        const float *Tr = Ts + (16 * R + r) * LDF + 16 * R;
        const float *Yc = Ls + 16 * (R - 1) * LDF + 16 * R + c;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) s = fmaf(Tr[k], Yc[k * LDF], s);
        Ts[(16 * R + r) * LDF + 16 * (R - 1) + c] = -s;
      }
    }
    __syncthreads();
    {  // lower-left 32x32 block: Y = L[32:64, 0:32] T[0:32, 0:32] (parked in L[0:32, 32:64])
      const int r = tid >> 3, c4 = 4 * (tid & 7);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      const float *Lr = Ls + (32 + r) * LDF;
#pragma unroll 8
      for (int k = 0; k < 32; ++k) {
        const float l = Lr[k];
        const float4 t = *reinterpret_cast<const float4 *>(&Ts[k * LDF + c4]);
        acc.x = fmaf(l, t.x, acc.x); acc.y = fmaf(l, t.y, acc.y);
        acc.z = fmaf(l, t.z, acc.z); acc.w = fmaf(l, t.w, acc.w);
      }
      *reinterpret_cast<float4 *>(&Ls[r * LDF + 32 + c4]) = acc;  // disjoint from what this stage reads
    }
    __syncthreads();
    {  // T[32:64, 0:32] = -T[32:64, 32:64] Y
      const int r = tid >> 3, c4 = 4 * (tid & 7);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      const float *Tr = Ts + (32 + r) * LDF + 32;
#pragma unroll 8
      for (int k = 0; k < 32; ++k) {
        const float t = Tr[k];
        const float4 y = *reinterpret_cast<const float4 *>(&Ls[k * LDF + 32 + c4]);
        acc.x = fmaf(t, y.x, acc.x); acc.y = fmaf(t, y.y, acc.y);
        acc.z = fmaf(t, y.z, acc.z); acc.w = fmaf(t, y.w, acc.w);
      }
      *reinterpret_cast<float4 *>(&Ts[(32 + r) * LDF + c4]) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    __syncthreads();
    {  // T -> rows 0..63 of [T ; 0], bf16
      const int r = tid >> 2;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int col = 16 * (tid & 3) + 8 * x;
        const float4 t0 = *reinterpret_cast<const float4 *>(&Ts[r * LDF + col]);
        const float4 t1 = *reinterpret_cast<const float4 *>(&Ts[r * LDF + col + 4]);
        const float e[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
        st_s128(sm + OFF_TZ + sw128(r, col), pack8(e));
      }
    }
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M3, M4: [T; 0] [A_m | U]
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 64, sdesc_sw128(sb + OFF_TZ + 32 * k, 16, 1024),
                 sdesc_sw128(sb + OFF_XA + 2048 * k, XA_BLK, 1024), ID_KM128, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 192, sdesc_sw128(sb + OFF_TZ + 32 * k, 16, 1024), sdesc_sw128(sb + OFF_U + 2048 * k, 8192, 1024),
                 ID_KM64, k > 0 ? 1u : 0u);
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();

    // ---------------------------------------------------------------- E: -T A_m in place of A_m; e^m S
    {
      if (quad < 2) {
        const int row = 32 * quad + lane;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          float v[32];
          tmem_ld32(tl + 64 + 64 * half + 32 * part, v);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            float e[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) e[t] = -v[8 * x + t];
            st_s128(sm + OFF_XA + half * XA_BLK + sw128(row, 32 * part + 8 * x), pack8(e));
          }
        }
      }
      const float em = s_em[c_me];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        float e[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) e[t] = em * S[8 * x + t];
        st_s128(sm + OFF_SM + sw128(c_me, 32 * half + 8 * x), pack8(e));
      }
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M5: D_a += [-T A_m; Q_m] (e^m S)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < DK / 16; ++k)
        mma_bf16(tmem + 192, sdesc_sw128(sb + OFF_XA + (k >> 2) * XA_BLK + (k & 3) * 32, 16, 1024),
                 sdesc_sw128(sb + OFF_SM + 2048 * k, 16384, 1024), ID_KM64, 1u);
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();

    // ---------------------------------------------------------------- F: Delta -> smem
    if (quad < 2) {
      float v[32];
      tmem_ld32(tl + 192 + 32 * half, v);
      tmem_wait_ld();
      const int row = 32 * quad + lane;
#pragma unroll
      for (int x = 0; x < 4; ++x) st_s128(sm + OFF_DL + sw128(row, 32 * half + 8 * x), pack8(&v[8 * x]));
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();

    // ---------------------------------------------------------------- M6, M7: K_m^T Delta; D_a += [P; P] Delta
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 0, sdesc_sw128(sb + OFF_KT + 2048 * k, KT_BLK, 1024), sdesc_sw128(sb + OFF_DL + 2048 * k, 8192, 1024),
                 ID_MNMN, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tmem + 192, sdesc_sw128(sb + OFF_PP + 32 * k, 16, 1024), sdesc_sw128(sb + OFF_DL + 2048 * k, 8192, 1024),
                 ID_KM64, 1u);
      mma_commit(bar_mma);
    }
    if (!(ok = cta_wait(bar_mma, ph_mma))) break;
    ph_mma ^= 1;
    tc_fence_after();

    // ---------------------------------------------------------------- G: state update, O -> global
    {
      float v[32];
      tmem_ld32(tl + 0 + 32 * half, v);
      tmem_wait_ld();
      const float g1 = s_egc[c_me], g2 = s_egcm[c_me];
#pragma unroll
      for (int j = 0; j < 32; ++j) S[j] = fmaf(g2, v[j], g1 * S[j]);
      if (quad >= 2) {  // warp-uniform: tcgen05.ld is a warp-collective instruction
        const int r = 32 * quad + lane - 64;
        tmem_ld32(tl + 192 + 32 * half, v);
        tmem_wait_ld();
        if (r < Cc) store_row32_bf16(o + ((size_t)(tok0 + r) * a.H + h) * (size_t)a.dv + j0 + 32 * half, v);
      }
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
