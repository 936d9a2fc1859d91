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
// T is formed in fp32 storage: the four 16x16 diagonal blocks by right-looking
// substitution, then merged into 32x32 and 64x64 inverses with
// [[A,0],[C,B]]^-1 = [[A^-1,0],[-B^-1 C A^-1, B^-1]]; the merge products run on
// the warp-level tensor cores with tf32 operands (T is rounded to bf16 after).
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

cudaError_t device_status_word(int **ptr) {
  return cudaGetSymbolAddress(reinterpret_cast<void **>(ptr), g_device_status);
}

namespace {

using namespace ptx;

constexpr int C = 64, DK = 128, NV = 64;
constexpr int NT = 384;           // warps 0-3: state side; warps 4-11: key side
constexpr int NSTATE = 128, NKEY = 256;
constexpr int BAR_STATE = 1, BAR_KEY = 2;  // named barriers of the two warp groups

// shared-memory map (bytes from a 1024-aligned base); every MMA operand tile is 1024-aligned
constexpr uint32_t XA_BLK = 16384;                 // [A_m | -T A_m ; Q_m] 128 rows x 64 ch (one channel block)
constexpr uint32_t XA_BUF = 2 * XA_BLK;            // two channel blocks per chunk buffer
constexpr uint32_t KT_BLK = 8192;                  // K_m 64 rows x 64 ch
constexpr uint32_t KT_BUF = 2 * KT_BLK;
constexpr uint32_t OFF_XA = 0;                     // 2 chunk buffers
constexpr uint32_t OFF_KT = OFF_XA + 2 * XA_BUF;   // 65536: 2 chunk buffers
constexpr uint32_t OFF_U = OFF_KT + 2 * KT_BUF;    // 98304: 2 chunk buffers of v -> U = w (.) v
constexpr uint32_t OFF_AL = OFF_U + 2 * 8192;      // 114688: alpha tiles (two channel blocks)
constexpr uint32_t OFF_W = OFF_AL + 16384;         // 131072: w tile
constexpr uint32_t OFF_TZP = OFF_W + 8192;         // 139264: two chunk buffers of [T ; P] (128 x 64 bf16)
constexpr uint32_t OFF_SM = OFF_TZP + 32768;       // 172032: e^m S (128 x 64); its first 8 KB later holds Delta
constexpr int LDF = 68;                            // row stride of the fp32 64 x 64 scratch
constexpr uint32_t OFF_LS = OFF_SM + 16384;        // 188416: L (fp32); first 8 KB = decay-product scan
constexpr uint32_t OFF_TS = OFF_LS + 64 * LDF * 4; // 205824: T (fp32)
constexpr uint32_t OFF_SC = OFF_TS + 64 * LDF * 4; // 223232: per-channel scalars, 2 chunk buffers
constexpr uint32_t OFF_BAR = OFF_SC + 2 * 3 * 128 * 4;  // 226304
constexpr uint32_t SMEM_USED = OFF_BAR + 128;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base
constexpr uint32_t TMA_BYTES = 10 * 8192;          // q, k, b, alpha (2 boxes each), v, w
constexpr uint32_t TMA_BYTES_HALF = 6 * 8192;     // cluster pair: own channel block of q, k, b, alpha; v, w
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_LP = 0, TM_DX = 64, TM_DA = 192, TM_DU = 256, TM_DB = 320;
constexpr uint64_t WAIT_NS = 2000000000ull;        // bounded waits: 2 s

constexpr uint32_t ID_LP = idesc_bf16(128, 64, false, false);    // [A_m;Q_m] K_m^T
constexpr uint32_t ID_KM64 = idesc_bf16(128, 64, false, true);   // K-major A, MN-major B, N = 64
constexpr uint32_t ID_KM128 = idesc_bf16(128, 128, false, true); // same, N = 128
constexpr uint32_t ID_MNMN = idesc_bf16(128, 64, true, true);    // K_m^T Delta

// mbarriers (8 bytes each) at OFF_BAR
enum {
  B_FULL0 = 0, B_FULL1, B_KMMA, B_SMMA, B_READY0, B_READY1, B_KBDONE,
  B_HALF0, B_HALF1,    // cluster pair: the peer's channel half of chunk buffer 0 / 1 has landed here
  B_PFREE0, B_PFREE1,  // cluster pair: the peer's state side finished an even / odd chunk
  B_COUNT
};

__device__ __forceinline__ uint4 ld_s128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void st_s128(uint8_t *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }
__device__ __forceinline__ uint4 pack8(const float *e) {
  return make_uint4(f2_to_bf2(e[0], e[1]), f2_to_bf2(e[2], e[3]), f2_to_bf2(e[4], e[5]), f2_to_bf2(e[6], e[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float *e) {
  float2 t = bf2_to_f2(u.x); e[0] = t.x; e[1] = t.y;
  t = bf2_to_f2(u.y); e[2] = t.x; e[3] = t.y;
  t = bf2_to_f2(u.z); e[4] = t.x; e[5] = t.y;
  t = bf2_to_f2(u.w); e[6] = t.x; e[7] = t.y;
}
__device__ __forceinline__ float fast_rcp(float x) { return __fdividef(1.f, x); }

__device__ __forceinline__ void group_sync(int id, int count) {
  asm volatile("barrier.cta.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Barrier of one warp group that also ORs a predicate over its threads.
__device__ __forceinline__ bool group_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Every thread of a warp group waits (bounded); the group agrees on the outcome; `fail` lets the
// caller fold in an earlier failure of one thread.
__device__ __forceinline__ bool group_wait(int id, int count, uint32_t bar, uint32_t parity, bool fail = false) {
  const bool ok = mbar_wait_bounded(bar, parity, WAIT_NS);
  return !group_or(id, count, fail || !ok);
}

__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16 *dst, const float *v) {
#pragma unroll
  for (int x = 0; x < 4; ++x) reinterpret_cast<uint4 *>(dst)[x] = pack8(&v[8 * x]);
}

// Decay-absorbed operands of one token row for 8 key channels, from the raw bf16 values already in
// registers: A_m = b k f, Q_m = q f, K_m = k fi with f = e^{g_r - m}, fi = 1/f (zeros when !valid).
template <int CL>
__device__ __forceinline__ void row_factors(uint8_t *pa, uint8_t *pq, uint8_t *pk, uint4 rb, uint4 rq, uint4 rk,
                                            bool valid, const float *f, const float *fi, uint32_t peer_delta) {
  uint4 wa = make_uint4(0u, 0u, 0u, 0u), wq = wa, wk = wa;
  if (valid) {
    float bb[8], qv[8], kv[8], ea[8], eq[8], ek[8];
    unpack8(rb, bb);
    unpack8(rq, qv);
    unpack8(rk, kv);
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
  if (CL == 2) {  // the same bytes at the same offsets in the peer CTA of the cluster
    st_cluster_128(smem_u32(pa) + peer_delta, wa);
    st_cluster_128(smem_u32(pq) + peer_delta, wq);
    st_cluster_128(smem_u32(pk) + peer_delta, wk);
  }
}

// D (16 x 8) = A (16 x K) B (K x 8) on the warp-level tensor-core path (mma.sync, tf32 operands
// rounded from fp32, fp32 accumulate).  A points at element (0, 0) of a row-major fp32 block with
// row stride LDF, B likewise.  Fragment ownership follows the m16n8k8 tf32 layout: lane = 4 g + t
// holds D rows g and g + 8, columns 2t and 2t + 1.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
template <int K>
__device__ __forceinline__ void mma_tf32_16x8(const float *A, const float *B, int lane, float (&d)[4]) {
  const int g = lane >> 2, t = lane & 3;
  d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < K; kk += 8) {
    const uint32_t a0 = to_tf32(A[g * LDF + kk + t]), a1 = to_tf32(A[(g + 8) * LDF + kk + t]);
    const uint32_t a2 = to_tf32(A[g * LDF + kk + t + 4]), a3 = to_tf32(A[(g + 8) * LDF + kk + t + 4]);
    const uint32_t b0 = to_tf32(B[(kk + t) * LDF + g]), b1 = to_tf32(B[(kk + t + 4) * LDF + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}
// Store a 16 x 8 tile (times `scale`) into a row-major fp32 block with row stride LDF.
__device__ __forceinline__ void store_16x8(float *D, int lane, const float (&d)[4], float scale) {
  const int g = lane >> 2, t = lane & 3;
  *reinterpret_cast<float2 *>(&D[g * LDF + 2 * t]) = make_float2(scale * d[0], scale * d[1]);
  *reinterpret_cast<float2 *>(&D[(g + 8) * LDF + 2 * t]) = make_float2(scale * d[2], scale * d[3]);
}

struct Ctx {
  uint8_t *sm;
  uint32_t sb, tmem;
  uint32_t rank, peer_delta;  // cluster pair: this CTA's rank; peer shared::cluster address minus own
  int H, dv, h, j0, nchunks, len;
  int64_t bos;
};

__device__ __forceinline__ uint32_t bar_addr(const Ctx &x, int i) { return x.sb + OFF_BAR + 8 * i; }

// Issue the TMA loads of chunk `c` into chunk buffer c & 1 (one thread).  A cluster pair loads
// only its own channel block of q, k, b, alpha; the peer fills the other block.
template <int CL>
__device__ __forceinline__ void issue_chunk_loads(const Ctx &x, int c, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                                  const CUtensorMap *tm_b, const CUtensorMap *tm_al,
                                                  const CUtensorMap *tm_v, const CUtensorMap *tm_w) {
  const int b = c & 1;
  const int tok0 = (int)(x.bos + (int64_t)c * C);
  const uint32_t full = bar_addr(x, B_FULL0 + b);
  fence_proxy_async();
  mbar_expect_tx(full, CL == 2 ? TMA_BYTES_HALF : TMA_BYTES);
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    if (CL == 2 && blk != (int)x.rank) continue;
    tma_load_3d(x.sb + OFF_XA + b * XA_BUF + blk * XA_BLK, tm_b, 64 * blk, x.h, tok0, full);         // b -> rows 0..63
    tma_load_3d(x.sb + OFF_XA + b * XA_BUF + blk * XA_BLK + 8192, tm_q, 64 * blk, x.h, tok0, full);  // q -> rows 64..127
    tma_load_3d(x.sb + OFF_KT + b * KT_BUF + blk * KT_BLK, tm_k, 64 * blk, x.h, tok0, full);
    tma_load_3d(x.sb + OFF_AL + blk * 8192, tm_al, 64 * blk, x.h, tok0, full);
  }
  tma_load_3d(x.sb + OFF_U + b * 8192, tm_v, x.j0, x.h, tok0, full);
  tma_load_3d(x.sb + OFF_W, tm_w, x.j0, x.h, tok0, full);
}

// ==================================================================== key side (warps 4-11)
// For each chunk: decay factors, L|P, T, [T; 0][A_m | U]; hands the chunk to the state side.
template <int CL>
__device__ __forceinline__ bool key_side(const Ctx &x, const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_b,
                         const CUtensorMap *tm_al, const CUtensorMap *tm_v, const CUtensorMap *tm_w) {
  uint8_t *sm = x.sm;
  const int kt = threadIdx.x - NSTATE, kwarp = kt >> 5, lane = kt & 31, quad = kwarp & 3, khalf = kwarp >> 2;
  const uint32_t tl = x.tmem + ((uint32_t)(32 * quad) << 16);
  float *Ls = reinterpret_cast<float *>(sm + OFF_LS);
  float *Ts = reinterpret_cast<float *>(sm + OFF_TS);
  float *scan = Ls;  // [16 groups][128 channels] during the factor phase
  uint32_t kphase = 0;


  for (int c = 0; c < x.nchunks; ++c) {
    const int b = c & 1;
    const int Cc = min(C, x.len - c * C);
    uint8_t *xa = sm + OFF_XA + b * XA_BUF;
    uint8_t *ktile = sm + OFF_KT + b * KT_BUF;
    float *s_em = reinterpret_cast<float *>(sm + OFF_SC) + b * 384;
    float *s_egcm = s_em + 128, *s_egc = s_em + 256;

    // ------------------------------------------------------------ data of chunk c has landed
    if (!group_wait(BAR_KEY, NKEY, bar_addr(x, B_FULL0 + b), (c >> 1) & 1)) return false;

    // ------------------------------------------------------------ decay factors, operands in place
    if (CL == 1)
    {
      // thread = 8 key channels (chunk x8 of channel block cb) x 4 tokens (group G = rows 4G..4G+3);
      // groups 0-7 hold tokens 0..31 (walk back to token 31), groups 8-15 tokens 32..63 (walk forward).
      // All raw tiles this thread needs are loaded first, so their latency overlaps the barriers.
      const int ch8 = kt & 15, G = kt >> 4, cb = ch8 >> 3, x8 = ch8 & 7;
      uint4 ra[4], rb[4], rq[4], rk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t o = sw128(4 * G + i, 8 * x8);
        ra[i] = ld_s128(sm + OFF_AL + cb * 8192 + o);
        rb[i] = ld_s128(xa + cb * XA_BLK + o);
        rq[i] = ld_s128(xa + cb * XA_BLK + 8192 + o);
        rk[i] = ld_s128(ktile + cb * KT_BLK + o);
      }
      const int ur = kt >> 2;  // U = w (.) v: token row ur, value columns 16 (kt & 3) .. +15
      uint8_t *ub = sm + OFF_U + b * 8192;
      uint4 rv[2], rw[2];
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        rv[y] = ld_s128(ub + sw128(ur, 16 * (kt & 3) + 8 * y));
        rw[y] = ld_s128(sm + OFF_W + sw128(ur, 16 * (kt & 3) + 8 * y));
      }
      float gp[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) gp[t] = 1.f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (4 * G + i < Cc) {
          float al[8];
          unpack8(ra[i], al);
#pragma unroll
          for (int t = 0; t < 8; ++t) gp[t] *= al[t];
        }
      *reinterpret_cast<float4 *>(&scan[G * 128 + 8 * ch8]) = make_float4(gp[0], gp[1], gp[2], gp[3]);
      *reinterpret_cast<float4 *>(&scan[G * 128 + 8 * ch8 + 4]) = make_float4(gp[4], gp[5], gp[6], gp[7]);
      group_sync(BAR_KEY, NKEY);
      if (kt < 128) {  // per channel: products between each group and token 31, in place of the group products
        float p[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) p[g] = scan[g * 128 + kt];
        float acc = 1.f;
#pragma unroll
        for (int g = 7; g >= 0; --g) {
          scan[g * 128 + kt] = acc;  // prod over groups g+1..7
          acc *= p[g];
        }
        const float em = acc;
        acc = 1.f;
#pragma unroll
        for (int g = 8; g < 16; ++g) {
          scan[g * 128 + kt] = acc;  // prod over groups 8..g-1
          acc *= p[g];
        }
        s_em[kt] = em;
        s_egcm[kt] = acc;
        s_egc[kt] = em * acc;
      }
      group_sync(BAR_KEY, NKEY);
      float run[8];
      {
        const float4 p0 = *reinterpret_cast<const float4 *>(&scan[G * 128 + 8 * ch8]);
        const float4 p1 = *reinterpret_cast<const float4 *>(&scan[G * 128 + 8 * ch8 + 4]);
        run[0] = p0.x; run[1] = p0.y; run[2] = p0.z; run[3] = p0.w;
        run[4] = p1.x; run[5] = p1.y; run[6] = p1.z; run[7] = p1.w;
      }
      uint8_t *pa0 = xa + cb * XA_BLK, *pk0 = ktile + cb * KT_BLK;
      if (G < 8) {
#pragma unroll
        for (int i = 3; i >= 0; --i) {  // run = prod_{r < s <= 31} alpha_s
          const int r = 4 * G + i;
          float al[8], f[8], fi[8];
          unpack8(ra[i], al);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            fi[t] = run[t];
            f[t] = fast_rcp(run[t]);
            if (r < Cc) run[t] *= al[t];
          }
          const uint32_t o = sw128(r, 8 * x8);
          row_factors<1>(pa0 + o, pa0 + 8192 + o, pk0 + o, rb[i], rq[i], rk[i], r < Cc, f, fi, 0u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // run = prod_{32 <= s <= r} alpha_s
          const int r = 4 * G + i;
          float al[8], f[8], fi[8];
          unpack8(ra[i], al);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (r < Cc) run[t] *= al[t];
            f[t] = run[t];
            fi[t] = fast_rcp(run[t]);
          }
          const uint32_t o = sw128(r, 8 * x8);
          row_factors<1>(pa0 + o, pa0 + 8192 + o, pk0 + o, rb[i], rq[i], rk[i], r < Cc, f, fi, 0u);
        }
      }
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        float vv[8], ww[8], uu[8];
        unpack8(rv[y], vv);
        unpack8(rw[y], ww);
#pragma unroll
        for (int t = 0; t < 8; ++t) uu[t] = (ur < Cc) ? vv[t] * ww[t] : 0.f;
        st_s128(ub + sw128(ur, 16 * (kt & 3) + 8 * y), pack8(uu));
      }
    }
    else {
      // Cluster pair: this CTA forms only its own channel block cb (64 channels) and writes every
      // result both here and into the peer.  thread = 8 channels (chunk x8) x 2 tokens (group G =
      // rows 2G, 2G+1); groups 0-15 walk back to token 31, groups 16-31 walk forward.
      const int x8 = kt & 7, G = kt >> 3, cb = (int)x.rank;
      uint4 ra[2], rb[2], rq[2], rk[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t o = sw128(2 * G + i, 8 * x8);
        ra[i] = ld_s128(sm + OFF_AL + cb * 8192 + o);
        rb[i] = ld_s128(xa + cb * XA_BLK + o);
        rq[i] = ld_s128(xa + cb * XA_BLK + 8192 + o);
        rk[i] = ld_s128(ktile + cb * KT_BLK + o);
      }
      const int ur = kt >> 2;  // U = w (.) v: token row ur, value columns 16 (kt & 3) .. +15
      uint8_t *ub = sm + OFF_U + b * 8192;
      uint4 rv[2], rw[2];
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        rv[y] = ld_s128(ub + sw128(ur, 16 * (kt & 3) + 8 * y));
        rw[y] = ld_s128(sm + OFF_W + sw128(ur, 16 * (kt & 3) + 8 * y));
      }
      float gp[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) gp[t] = 1.f;
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (2 * G + i < Cc) {
          float al[8];
          unpack8(ra[i], al);
#pragma unroll
          for (int t = 0; t < 8; ++t) gp[t] *= al[t];
        }
      *reinterpret_cast<float4 *>(&scan[G * 64 + 8 * x8]) = make_float4(gp[0], gp[1], gp[2], gp[3]);
      *reinterpret_cast<float4 *>(&scan[G * 64 + 8 * x8 + 4]) = make_float4(gp[4], gp[5], gp[6], gp[7]);
      group_sync(BAR_KEY, NKEY);
      if (kt < 64) {  // per channel: products between each group and token 31, in place of the group products
        float p[32];
#pragma unroll
        for (int g = 0; g < 32; ++g) p[g] = scan[g * 64 + kt];
        float acc = 1.f;
#pragma unroll
        for (int g = 15; g >= 0; --g) {
          scan[g * 64 + kt] = acc;
          acc *= p[g];
        }
        const float em = acc;
        acc = 1.f;
#pragma unroll
        for (int g = 16; g < 32; ++g) {
          scan[g * 64 + kt] = acc;
          acc *= p[g];
        }
        const int ch = 64 * cb + kt;
        s_em[ch] = em;
        s_egcm[ch] = acc;
        s_egc[ch] = em * acc;
        st_cluster_f32(smem_u32(&s_em[ch]) + x.peer_delta, em);
        st_cluster_f32(smem_u32(&s_egcm[ch]) + x.peer_delta, acc);
        st_cluster_f32(smem_u32(&s_egc[ch]) + x.peer_delta, em * acc);
      }
      group_sync(BAR_KEY, NKEY);
      float run[8];
      {
        const float4 p0 = *reinterpret_cast<const float4 *>(&scan[G * 64 + 8 * x8]);
        const float4 p1 = *reinterpret_cast<const float4 *>(&scan[G * 64 + 8 * x8 + 4]);
        run[0] = p0.x; run[1] = p0.y; run[2] = p0.z; run[3] = p0.w;
        run[4] = p1.x; run[5] = p1.y; run[6] = p1.z; run[7] = p1.w;
      }
      uint8_t *pa0 = xa + cb * XA_BLK, *pk0 = ktile + cb * KT_BLK;
      if (G < 16) {
#pragma unroll
        for (int i = 1; i >= 0; --i) {  // run = prod_{r < s <= 31} alpha_s
          const int r = 2 * G + i;
          float al[8], f[8], fi[8];
          unpack8(ra[i], al);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            fi[t] = run[t];
            f[t] = fast_rcp(run[t]);
            if (r < Cc) run[t] *= al[t];
          }
          const uint32_t o = sw128(r, 8 * x8);
          row_factors<2>(pa0 + o, pa0 + 8192 + o, pk0 + o, rb[i], rq[i], rk[i], r < Cc, f, fi, x.peer_delta);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // run = prod_{32 <= s <= r} alpha_s
          const int r = 2 * G + i;
          float al[8], f[8], fi[8];
          unpack8(ra[i], al);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (r < Cc) run[t] *= al[t];
            f[t] = run[t];
            fi[t] = fast_rcp(run[t]);
          }
          const uint32_t o = sw128(r, 8 * x8);
          row_factors<2>(pa0 + o, pa0 + 8192 + o, pk0 + o, rb[i], rq[i], rk[i], r < Cc, f, fi, x.peer_delta);
        }
      }
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        float vv[8], ww[8], uu[8];
        unpack8(rv[y], vv);
        unpack8(rw[y], ww);
#pragma unroll
        for (int t = 0; t < 8; ++t) uu[t] = (ur < Cc) ? vv[t] * ww[t] : 0.f;
        st_s128(ub + sw128(ur, 16 * (kt & 3) + 8 * y), pack8(uu));
      }
      // make this thread's DSMEM writes visible to the peer's tensor-core (async) proxy; the key
      // leader publishes the whole half after the group barrier below
      fence_proxy_async_cluster();
    }
    fence_proxy_async();
    group_sync(BAR_KEY, NKEY);

    // ------------------------------------------------------------ M1: [L; P] = [A_m; Q_m] K_m^T
    // (the alpha and w tiles of chunk c are consumed: the state side may now load chunk c+1)
    bool kfail = false;
    if (kt == 0) {
      mbar_arrive(bar_addr(x, B_KBDONE));
      if (CL == 2) {
        // one release at cluster scope covers every key thread's DSMEM writes (ordered before it by
        // the group barrier)
        mbar_arrive_remote(bar_addr(x, B_HALF0 + b) + x.peer_delta);
        // the peer's channel half of this chunk
        kfail = !mbar_wait_bounded_cluster(bar_addr(x, B_HALF0 + b), (c >> 1) & 1, WAIT_NS);
        fence_proxy_async();
      }
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < DK / 16; ++k) {
        const uint32_t koff = (uint32_t)(k & 3) * 32u;
        const uint64_t ad = sdesc_sw128(x.sb + OFF_XA + b * XA_BUF + (k >> 2) * XA_BLK + koff, 16, 1024);
        const uint64_t bd = sdesc_sw128(x.sb + OFF_KT + b * KT_BUF + (k >> 2) * KT_BLK + koff, 16, 1024);
        mma_bf16(x.tmem + TM_LP, ad, bd, ID_LP, k > 0 ? 1u : 0u);
      }
      mma_commit(bar_addr(x, B_KMMA));
    }
    const bool fail = kfail;
    if (!group_wait(BAR_KEY, NKEY, bar_addr(x, B_KMMA), kphase, fail)) return false;
    kphase ^= 1;
    tc_fence_after();

    // ------------------------------------------------------------ T = (I + L)^-1
    uint8_t *tp = sm + OFF_TZP + b * 16384;  // [T ; P] of this chunk
    uint8_t *pt = tp + 8192;                 // P (64 x 64 bf16)
    {  // L (strict lower) -> fp32 scratch; P (inclusive lower) -> its bf16 tile
      float v[32];
      tmem_ld32(tl + TM_LP + 32 * khalf, v);
      tmem_wait_ld();
      const int row = 32 * quad + lane;
      if (row < 64) {
#pragma unroll
        for (int y = 0; y < 8; ++y) {
          const int i = 32 * khalf + 4 * y;
          *reinterpret_cast<float4 *>(&Ls[row * LDF + i]) =
              make_float4(i < row ? v[4 * y] : 0.f, i + 1 < row ? v[4 * y + 1] : 0.f, i + 2 < row ? v[4 * y + 2] : 0.f,
                          i + 3 < row ? v[4 * y + 3] : 0.f);
        }
      } else {
        const int r = row - 64;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int col = 32 * khalf + 8 * y;
          float e[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) e[t] = (col + t <= r) ? v[8 * y + t] : 0.f;
          st_s128(pt + sw128(r, col), pack8(e));
        }
      }
    }
    tc_fence_before();
    group_sync(BAR_KEY, NKEY);
    if (kwarp < 2) {  // the four 16x16 diagonal blocks, right-looking; lane = column j of block R
      const int R = 2 * kwarp + (lane >> 4), j = lane & 15;
      const float *Lb = Ls + 16 * R * LDF + 16 * R;
      float xv[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) xv[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
      for (int i = 0; i < 15; ++i)
#pragma unroll
        for (int r = i + 1; r < 16; ++r) xv[r] = fmaf(-Lb[r * LDF + i], xv[i], xv[r]);
      float *Tb = Ts + 16 * R * LDF + 16 * R;
#pragma unroll
      for (int r = 0; r < 16; ++r) Tb[r * LDF + j] = xv[r];
    }
    group_sync(BAR_KEY, NKEY);
    // merges on the warp-level tensor cores (tf32): 16x16 blocks, then the 32x32 block
    if (kwarp < 4) {  // Y_R = L_{R,R-1} T_{R-1,R-1}, R = 1, 3, parked in the upper block (R-1, R) of L
      const int R = (kwarp < 2) ? 1 : 3, nt = kwarp & 1;
      float d[4];
      mma_tf32_16x8<16>(Ls + 16 * R * LDF + 16 * (R - 1), Ts + 16 * (R - 1) * LDF + 16 * (R - 1) + 8 * nt, lane, d);
      store_16x8(Ls + 16 * (R - 1) * LDF + 16 * R + 8 * nt, lane, d, 1.f);
    }
    group_sync(BAR_KEY, NKEY);
    if (kwarp < 4) {  // T_{R,R-1} = -T_RR Y_R
      const int R = (kwarp < 2) ? 1 : 3, nt = kwarp & 1;
      float d[4];
      mma_tf32_16x8<16>(Ts + 16 * R * LDF + 16 * R, Ls + 16 * (R - 1) * LDF + 16 * R + 8 * nt, lane, d);
      store_16x8(Ts + 16 * R * LDF + 16 * (R - 1) + 8 * nt, lane, d, -1.f);
    }
    group_sync(BAR_KEY, NKEY);
    {  // lower-left 32x32 block: Y = L[32:64, 0:32] T[0:32, 0:32], parked in L[0:32, 32:64]
      const int mt = kwarp >> 2, nt = kwarp & 3;
      float d[4];
      mma_tf32_16x8<32>(Ls + (32 + 16 * mt) * LDF, Ts + 8 * nt, lane, d);
      store_16x8(Ls + 16 * mt * LDF + 32 + 8 * nt, lane, d, 1.f);  // disjoint from what this stage reads
    }
    group_sync(BAR_KEY, NKEY);
    {  // T[32:64, 0:32] = -T[32:64, 32:64] Y
      const int mt = kwarp >> 2, nt = kwarp & 3;
      float d[4];
      mma_tf32_16x8<32>(Ts + (32 + 16 * mt) * LDF + 32, Ls + 32 + 8 * nt, lane, d);
      store_16x8(Ts + (32 + 16 * mt) * LDF + 8 * nt, lane, d, -1.f);
    }
    group_sync(BAR_KEY, NKEY);
    {  // T -> rows 0..63 of [T ; P], bf16
      const int r = kt >> 2;
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        const int col = 16 * (kt & 3) + 8 * y;
        const float4 t0 = *reinterpret_cast<const float4 *>(&Ts[r * LDF + col]);
        const float4 t1 = *reinterpret_cast<const float4 *>(&Ts[r * LDF + col + 4]);
        const float e[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
        st_s128(tp + sw128(r, col), pack8(e));
      }
    }
    fence_proxy_async();
    group_sync(BAR_KEY, NKEY);

    // ------------------------------------------------------------ hand the chunk to the state side
    if (kt == 0) {
      mbar_arrive(bar_addr(x, B_READY0 + b));
    }
  }
  return true;
}

// ==================================================================== state side (warps 0-3)
// Holds the fp32 state slice (thread = key channel x 64 value columns) and runs the serial chain.
template <int CL>
__device__ __forceinline__ bool state_side(const Ctx &x, float (&S)[64], __nv_bfloat16 *o, const CUtensorMap *tm_q,
                                           const CUtensorMap *tm_k, const CUtensorMap *tm_b, const CUtensorMap *tm_al,
                                           const CUtensorMap *tm_v, const CUtensorMap *tm_w) {
  uint8_t *sm = x.sm;
  const int st = threadIdx.x, warp = st >> 5, lane = st & 31, quad = warp;
  const uint32_t tl = x.tmem + ((uint32_t)(32 * quad) << 16);
  const int c_me = st;  // key channel of this thread (TMEM lane of K_m^T Delta)
  uint32_t sphase = 0;
  // The state side's thread 0 is also the load producer.  Chunk c+1 goes into buffer (c+1)&1,
  // last used by chunk c-1, which this side has finished; it waits only until the key side has
  // read the single-buffered alpha and w tiles of chunk c.
  // In a cluster pair the peer also writes into buffer (c+1)&1, so chunk c+1 is loaded only after
  // the peer's state side has finished chunk c-1 too.
  if (st == 0 && x.nchunks > 0) issue_chunk_loads<CL>(x, 0, tm_q, tm_k, tm_b, tm_al, tm_v, tm_w);

  for (int c = 0; c < x.nchunks; ++c) {
    const int b = c & 1;
    const int Cc = min(C, x.len - c * C);
    const float *s_em = reinterpret_cast<const float *>(sm + OFF_SC) + b * 384;
    const int tok0 = (int)(x.bos + (int64_t)c * C);

    bool fail = false;
    if (st == 0 && CL == 2 && c >= 1) {  // tell the peer that chunk c-1 is done here
      mbar_arrive_remote(bar_addr(x, B_PFREE0 + ((c - 1) & 1)) + x.peer_delta);
    }
    if (st == 0 && c + 1 < x.nchunks) {
      if (CL == 2 && c >= 1)
        fail = !mbar_wait_bounded_cluster(bar_addr(x, B_PFREE0 + ((c - 1) & 1)), ((c - 1) >> 1) & 1, WAIT_NS);
      if (!fail) fail = !mbar_wait_bounded(bar_addr(x, B_KBDONE), c & 1, WAIT_NS);
      if (!fail) issue_chunk_loads<CL>(x, c + 1, tm_q, tm_k, tm_b, tm_al, tm_v, tm_w);
    }
    if (!group_wait(BAR_STATE, NSTATE, bar_addr(x, B_READY0 + b), (c >> 1) & 1, fail)) return false;

    // ------------------------------------------------------------ M3, M4: [T; P] [A_m | U]; e^m S -> shared
    const uint32_t tpa = x.sb + OFF_TZP + b * 16384;  // [T ; P] of this chunk
    if (st == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(x.tmem + TM_DX, sdesc_sw128(tpa + 32 * k, 16, 1024),
                 sdesc_sw128(x.sb + OFF_XA + b * XA_BUF + 2048 * k, XA_BLK, 1024), ID_KM128, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(x.tmem + TM_DU, sdesc_sw128(tpa + 32 * k, 16, 1024), sdesc_sw128(x.sb + OFF_U + b * 8192 + 2048 * k, 8192, 1024),
                 ID_KM64, k > 0 ? 1u : 0u);
      mma_commit(bar_addr(x, B_SMMA));
    }
    {  // rows 0..63 of the products are T A_m and T U (rows 64..127, P A_m and P U, are not used)
      const float em = s_em[c_me];
#pragma unroll
      for (int y = 0; y < 8; ++y) {
        float e[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) e[t] = em * S[8 * y + t];
        st_s128(sm + OFF_SM + sw128(c_me, 8 * y), pack8(e));
      }
    }
    if (!group_wait(BAR_STATE, NSTATE, bar_addr(x, B_SMMA), sphase)) return false;
    sphase ^= 1;
    tc_fence_after();
    if (quad < 2) {  // -T A_m in place of A_m (rows 0..63, both channel blocks)
      const int row = 32 * quad + lane;
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        float v[32];
        tmem_ld32(tl + TM_DX + 32 * part, v);
        tmem_wait_ld();
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          float e[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) e[t] = -v[8 * y + t];
          st_s128(sm + OFF_XA + b * XA_BUF + (part >> 1) * XA_BLK + sw128(row, 32 * (part & 1) + 8 * y), pack8(e));
        }
      }
    }
    tc_fence_before();
    fence_proxy_async();
    group_sync(BAR_STATE, NSTATE);

    // ------------------------------------------------------------ M5: D_a = [-T A_m; Q_m] (e^m S)
    if (st == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < DK / 16; ++k)
        mma_bf16(x.tmem + TM_DA,
                 sdesc_sw128(x.sb + OFF_XA + b * XA_BUF + (k >> 2) * XA_BLK + (k & 3) * 32, 16, 1024),
                 sdesc_sw128(x.sb + OFF_SM + 2048 * k, 16384, 1024), ID_KM64, k > 0 ? 1u : 0u);
      mma_commit(bar_addr(x, B_SMMA));
    }
    if (!group_wait(BAR_STATE, NSTATE, bar_addr(x, B_SMMA), sphase)) return false;
    sphase ^= 1;
    tc_fence_after();

    // ------------------------------------------------------------ Delta = T U + D_a -> shared (bf16)
    if (quad < 2) {
      const int row = 32 * quad + lane;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float v[32], u[32];
        tmem_ld32(tl + TM_DA + 32 * part, v);
        tmem_ld32(tl + TM_DU + 32 * part, u);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += u[j];
#pragma unroll
        for (int y = 0; y < 4; ++y) st_s128(sm + OFF_SM + sw128(row, 32 * part + 8 * y), pack8(&v[8 * y]));
      }
    }
    tc_fence_before();
    fence_proxy_async();
    group_sync(BAR_STATE, NSTATE);

    // ------------------------------------------------------------ M6, M7: K_m^T Delta; D_a += [*; P] Delta
    if (st == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(x.tmem + TM_DB, sdesc_sw128(x.sb + OFF_KT + b * KT_BUF + 2048 * k, KT_BLK, 1024),
                 sdesc_sw128(x.sb + OFF_SM + 2048 * k, 8192, 1024), ID_MNMN, k > 0 ? 1u : 0u);
      // A = [T ; P]: rows 64..127 add P Delta to Q S; rows 0..63 only touch the Delta half of D_a,
      // which has been read out already
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(x.tmem + TM_DA, sdesc_sw128(tpa + 32 * k, 16, 1024), sdesc_sw128(x.sb + OFF_SM + 2048 * k, 8192, 1024),
                 ID_KM64, 1u);
      mma_commit(bar_addr(x, B_SMMA));
    }
    if (!group_wait(BAR_STATE, NSTATE, bar_addr(x, B_SMMA), sphase)) return false;
    sphase ^= 1;
    tc_fence_after();

    // ------------------------------------------------------------ state update, O -> global
    {
      const float g1 = s_em[256 + c_me], g2 = s_em[128 + c_me];  // e^{g_C}, e^{g_C - m}
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float v[32];
        tmem_ld32(tl + TM_DB + 32 * part, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) S[32 * part + j] = fmaf(g2, v[j], g1 * S[32 * part + j]);
      }
      if (quad >= 2) {  // warp-uniform: tcgen05.ld is a warp-collective instruction
        const int r = 32 * quad + lane - 64;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          float v[32];
          tmem_ld32(tl + TM_DA + 32 * part, v);
          tmem_wait_ld();
          if (r < Cc) store_row32_bf16(o + ((size_t)(tok0 + r) * x.H + x.h) * (size_t)x.dv + x.j0 + 32 * part, v);
        }
      }
    }
    tc_fence_before();
    group_sync(BAR_STATE, NSTATE);
  }
  return true;
}

template <int CL>
__global__ void __launch_bounds__(NT, 1)
    chunk_fwd_tc_kernel(const ChunkArgs a, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_al, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ uint8_t smem_raw[];
  Ctx x;
  // align by pointer arithmetic on the shared array, so every derived pointer stays a shared-space pointer
  x.sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  x.sb = smem_u32(x.sm);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(x.sm + OFF_BAR + 8 * B_COUNT);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int tiles = a.dv / NV;
  const int tile = blockIdx.x % tiles;
  x.h = (blockIdx.x / tiles) % a.H;
  const int n = blockIdx.x / (tiles * a.H);
  x.j0 = tile * NV;
  x.H = a.H;
  x.dv = a.dv;
  seq_span(a, n, x.bos, x.len);
  x.nchunks = (x.len + C - 1) / C;

  x.rank = (CL == 2) ? cluster_ctarank() : 0u;
  x.peer_delta = (CL == 2) ? mapa(x.sb, x.rank ^ 1u) - x.sb : 0u;
  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(x.sb + OFF_BAR + 8 * i, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_al); prefetch_tmap(&tm_v); prefetch_tmap(&tm_w);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  // the never-written upper blocks of T
  float *Ts = reinterpret_cast<float *>(x.sm + OFF_TS);
  for (int e = tid; e < 64 * LDF; e += NT) Ts[e] = 0.f;
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *tmem_slot;
  if (CL == 2) cluster_sync();  // both CTAs' barriers are initialised before any remote arrive

  bool ok;
  if (warp < 4) {
    // state slice: key channel tid, value columns j0 .. j0+63
    const size_t s_off = (((size_t)n * a.H + x.h) * DK + tid) * (size_t)a.dv + x.j0;
    float S[64];
    if (a.S0) {
#pragma unroll
      for (int y = 0; y < 16; ++y) {
        const float4 t = reinterpret_cast<const float4 *>(a.S0 + s_off)[y];
        S[4 * y] = t.x; S[4 * y + 1] = t.y; S[4 * y + 2] = t.z; S[4 * y + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int y = 0; y < 64; ++y) S[y] = 0.f;
    }
    ok = state_side<CL>(x, S, reinterpret_cast<__nv_bfloat16 *>(a.o), &tm_q, &tm_k, &tm_b, &tm_al, &tm_v, &tm_w);
    if (ok && a.ST) {
#pragma unroll
      for (int y = 0; y < 16; ++y)
        reinterpret_cast<float4 *>(a.ST + s_off)[y] = make_float4(S[4 * y], S[4 * y + 1], S[4 * y + 2], S[4 * y + 3]);
    }
  } else {
    ok = key_side<CL>(x, &tm_q, &tm_k, &tm_b, &tm_al, &tm_v, &tm_w);
  }
  if (!ok && (tid == 0 || tid == NSTATE)) atomicExch(&g_device_status, 4);
  tc_fence_before();
  __syncthreads();
  if (CL == 2) cluster_sync();  // no CTA leaves while its peer may still write into it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(x.tmem, TMEM_COLS);
  }
}

// Self-test of the bounded-wait path: waits on an mbarrier that nothing ever arrives on, gives up
// after `limit_ns`, and records GDN2_ERR_TIMEOUT exactly like the chunk kernel does.  No fault, trap
// or endless loop is involved; the context stays usable afterwards.
__global__ void bounded_wait_probe_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_bounded(b, 0, limit_ns);
  const bool any_timeout = __syncthreads_or(!ok);
  if (any_timeout && threadIdx.x == 0) atomicExch(&g_device_status, 4);
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

cudaError_t launch_bounded_wait_probe(uint64_t limit_ns, cudaStream_t stream) {
  note_launch();
  bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(limit_ns);
  return cudaGetLastError();
}

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
  const bool pair = (a.dv / NV) % 2 == 0;  // the two value slices of a head share the factor work
  cudaError_t err = cudaFuncSetAttribute(pair ? chunk_fwd_tc_kernel<2> : chunk_fwd_tc_kernel<1>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (err != cudaSuccess) return err;
  note_launch();
  if (!pair) {
    chunk_fwd_tc_kernel<1><<<(unsigned)blocks, NT, SMEM_BYTES, stream>>>(a, mq, mk, mb, mal, mv, mw);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, chunk_fwd_tc_kernel<2>, a, mq, mk, mb, mal, mv, mw);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace gdn2
