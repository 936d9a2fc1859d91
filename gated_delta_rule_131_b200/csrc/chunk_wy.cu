// Chunkwise WY forward of the Gated Delta Rule-2 as two tensor-core kernels
// (bf16 inputs, d_k = 64 or 128, fp32 state and accumulation), split where the
// dependence on the state begins:
//
//   wy_factor_kernel   persistent, two CTAs per SM, one (chunk, head) record at a
//                      time, all chunks independently: the decay-absorbed erase
//                      factors, [L; P], T = (I + L)^-1, and from them the chunk's
//                      state transition and output maps, stored to a workspace
//                      record;
//   state_pass_kernel  one CTA per (sequence, head, 128 value columns): walks the
//                      chunks of its sequence in order and carries S in fp32.  A
//                      programmatic dependent launch: it may start on SMs the first
//                      kernel leaves, and reads each record once it is complete.
//
// Per chunk of C = 64 tokens (r, i index tokens, c a key channel, m the running
// log-decay at token 31 of the chunk, g_r the running log-decay at r):
//   f_r     = exp(g_r - m)  per key channel (bounded by the decay over 32 tokens either way)
//   A_m     = (b (.) k) (.) f,  Q_m = q (.) f,  K_m = k (.) 1/f
//   [L; P]  = [A_m; Q_m] K_m^T              L strictly, P inclusively lower triangular
//   T       = (I + L)^-1                    fp32 blocked forward substitution
//   W       = -T A_m
// With S the state entering the chunk and U = w (.) v, the WY form reads
//   Delta   = T U + W Diag(e^m) S
//   O       = Q_m Diag(e^m) S + P Delta
//   S_next  = Diag(e^{g_C}) S + Diag(e^{g_C - m}) K_m^T Delta,
// which the state pass evaluates as
//   S_next  = Diag(e^{g_C}) S + Mt S + Nt U,   O = Qt S + Pt U,   with
//   Mt = Diag(e^{g_C-m}) K_m^T W Diag(e^m)   (d_k x d_k)   Nt = Diag(e^{g_C-m}) K_m^T T   (d_k x C)
//   Qt = (Q_m + P W) Diag(e^m)               (C x d_k)     Pt = P T                       (C x C)
// so its serial chain per chunk is one tensor-core pass over S.  A record holds
// Mt, Nt, Qt, Pt (bf16) and e^{g_C} (fp32).
// The decay-absorbed asymmetric erase factors follow the block formulation of
// "Gated DeltaNet-2: Separando Borrado y Escritura en la Atención Lineal"
// (needhelp.icu), "Innovaciones Técnicas", item 1; the update itself is the
// per-token rule of "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com),
// "Gated DeltaNet-2の核心" (decay first, key-side erase gate b, value-side
// write gate w, o_t = S_t^T q_t).
//
// Every operand tile is a 64-column bf16 tile in the 128-byte-swizzled layout
// that TMA writes and tcgen05.mma reads, in shared memory and in the workspace
// alike, so records move between the kernels as whole TMA boxes.
// Precondition of the factorisation: per key channel, the decay accumulated
// over any 32 consecutive tokens of a chunk stays above about e^-80 (the fp32
// range); every workload here is far inside it.
#include <cuda.h>

#include <algorithm>
#include <climits>
#include <cstring>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {

namespace {

using namespace ptx;

constexpr int C = 64, DK = 128, NV = 64;
constexpr int LDF = 68;                      // row stride of the fp32 64 x 64 scratch
constexpr uint64_t WAIT_NS = 2000000000ull;  // bounded waits: 2 s

constexpr uint32_t XA_BLK = 16384;  // [A_m ; Q_m]: 128 rows x 64 channels (one channel block)
constexpr uint32_t KT_BLK = 8192;   // K_m: 64 rows x 64 channels

// workspace record of one (chunk, head), every tile K-major for the state pass's A operands:
// Mt 128 x 128 (two 128-row tiles), Nt 128 x 64, Qt 64 x 128 (two 64-row tiles), Pt 64 x 64, e^{g_C}
constexpr uint32_t REC_M = 32768, REC_N = 16384, REC_Q = 16384, REC_P = 8192, REC_G = 512;

constexpr uint32_t ID_LP = idesc_bf16(128, 64, false, false);    // [A_m;Q_m] K_m^T
constexpr uint32_t ID_KM64 = idesc_bf16(128, 64, false, true);   // K-major A, MN-major B, N = 64
constexpr uint32_t ID_KM128 = idesc_bf16(128, 128, false, true); // same, N = 128
constexpr uint32_t ID_MN64 = idesc_bf16(128, 64, true, true);    // MN-major A and B, N = 64
constexpr uint32_t ID_MN128 = idesc_bf16(128, 128, true, true);  // same, N = 128

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
// Approximate reciprocal (the hardware's single-instruction estimate; relative error about 2^-23).
__device__ __forceinline__ float fast_rcp(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// Two fp32 products at once (sm_100 packed fp32 pipe; each lane rounds exactly like a scalar product).
__device__ __forceinline__ void mul2(float *d, const float *a, const float *b) {
  const float2 r = __fmul2_rn(make_float2(a[0], a[1]), make_float2(b[0], b[1]));
  d[0] = r.x;
  d[1] = r.y;
}

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
// Every thread of a warp group waits (bounded; try_wait suspends the thread in hardware, so polling
// costs little); the group agrees on the outcome.
__device__ __forceinline__ bool group_wait(int id, int count, uint32_t bar, uint32_t parity, bool fail = false) {
  const bool ok = mbar_wait_bounded(bar, parity, WAIT_NS);
  return !group_or(id, count, fail || !ok);
}
// The same, polling without suspending (the state chain's wait on its products).
__device__ __forceinline__ bool group_wait_spin(int id, int count, uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait_spin_bounded(bar, parity, WAIT_NS);
  return !group_or(id, count, !ok);
}

// D (16 x 8) = A (16 x K) B (K x 8) on the warp-level tensor-core path (mma.sync, tf32 operands
// rounded from fp32, fp32 accumulate).  A points at element (0, 0) of a row-major fp32 block with
// row stride LDF, B likewise.  Lane 4 g + t holds D rows g and g + 8, columns 2t and 2t + 1.
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
// D (16 x 8) = A (16 x 32) Y (32 x 8) with Y in registers as two 16 x 8 accumulator fragments
// (y0: rows 0..15, y1: rows 16..31, the layout mma_tf32_16x8 returns); each B fragment element is
// fetched from the lane that holds it.
__device__ __forceinline__ void mma_tf32_16x8_yreg(const float *A, const float (&y0)[4], const float (&y1)[4], int lane,
                                                   float (&d)[4]) {
  const int g = lane >> 2, t = lane & 3;
  d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const float(&y)[4] = kk < 2 ? y0 : y1;
    const int hi = (kk & 1) ? 2 : 0;  // rows 8..15 of the fragment sit in elements 2, 3
    // B[8 kk + t][g] and B[8 kk + t + 4][g]: fragment row t (or t + 4), column g
    const float e0 = __shfl_sync(0xffffffffu, y[hi], 4 * t + (g >> 1));
    const float o0 = __shfl_sync(0xffffffffu, y[hi + 1], 4 * t + (g >> 1));
    const float e1 = __shfl_sync(0xffffffffu, y[hi], 4 * (t + 4) + (g >> 1));
    const float o1 = __shfl_sync(0xffffffffu, y[hi + 1], 4 * (t + 4) + (g >> 1));
    const uint32_t b0 = to_tf32((g & 1) ? o0 : e0), b1 = to_tf32((g & 1) ? o1 : e1);
    const int k0 = 8 * kk;
    const uint32_t a0 = to_tf32(A[g * LDF + k0 + t]), a1 = to_tf32(A[(g + 8) * LDF + k0 + t]);
    const uint32_t a2 = to_tf32(A[g * LDF + k0 + t + 4]), a3 = to_tf32(A[(g + 8) * LDF + k0 + t + 4]);
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

// Decay-absorbed operands of one token row for 8 key channels, from the raw bf16 values already in
// registers: A_m = b k f (rows 0..63 of the [A_m ; Q_m] block), Q_m = q f (rows 64..127), K_m = k fi,
// with f = e^{g_r - m}, fi = 1/f; zeros when the row is past the sequence.
__device__ __forceinline__ void row_factors(uint8_t *pa, uint8_t *pk, uint32_t o, uint4 rb, uint4 rq, uint4 rk,
                                            bool valid, const float *f, const float *fi) {
  uint4 wa = make_uint4(0u, 0u, 0u, 0u), wq = wa, wk = wa;
  if (valid) {
    float bb[8], qv[8], kv[8], ea[8], eq[8], ek[8];
    unpack8(rb, bb);
    unpack8(rq, qv);
    unpack8(rk, kv);
#pragma unroll
    for (int t = 0; t < 8; t += 2) {  // (b k) f, q f, k / f
      mul2(&ea[t], &bb[t], &kv[t]);
      mul2(&ea[t], &ea[t], &f[t]);
      mul2(&eq[t], &qv[t], &f[t]);
      mul2(&ek[t], &kv[t], &fi[t]);
    }
    wa = pack8(ea);
    wq = pack8(eq);
    wk = pack8(ek);
  }
  st_s128(pa + o, wa);
  st_s128(pa + 8192 + o, wq);
  st_s128(pk + o, wk);
}

// Sequence n holding global chunk `gidx`, from the chunk offsets of a packed batch (coff[n] = first
// global chunk of sequence n; empty sequences own no chunk).  Requires coff[0] <= gidx < coff[N].
__device__ __forceinline__ int seq_of_chunk(const int32_t *coff, int N, int gidx) {
  int lo = 0, hi = N;
  while (lo < hi) {  // largest n with coff[n] <= gidx
    const int mid = (lo + hi + 1) >> 1;
    if (coff[mid] <= gidx) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ==================================================================== kernel 1: WY factors
namespace wy {
constexpr int NT = 256;
// the thread that issues every bulk store and publishes the records: warp 4 idles during the
// triangular substitution, where the publish (a wait for the previous record's stores and a release)
// costs nothing; the loads and the products stay with thread 0
constexpr int ST_TID = 128;
// shared memory (two CTAs per SM); regions are reused once their first contents are dead
constexpr uint32_t OFF_XA = 0;                       // [A_m ; Q_m], two channel blocks -> Qt in rows 0..63
constexpr uint32_t OFF_KT = OFF_XA + 2 * XA_BLK;     // 32768: K_m, two channel blocks -> Mt tile 0
constexpr uint32_t OFF_TP = OFF_KT + 2 * KT_BLK;     // 49152: [T ; P] -> Nt; decay-product scan during the factors
constexpr uint32_t OFF_AL = OFF_TP + 16384;          // 65536: alpha tiles -> L (fp32) -> W (two 64-channel tiles) -> Mt tile 1
constexpr uint32_t OFF_TS = OFF_AL + 64 * LDF * 4;   // 82944: T (fp32) -> Pt
constexpr uint32_t OFF_SC = OFF_TS + 64 * LDF * 4;   // 100352: e^m, e^{g_C-m}, e^{g_C}
constexpr uint32_t OFF_BAR = OFF_SC + 3 * 128 * 4;   // 101888: FULL, MMA
constexpr uint32_t SMEM_USED = OFF_BAR + 32;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
constexpr uint32_t TMA_BYTES = 8 * 8192;             // q, k, b, alpha: two channel blocks each
constexpr uint32_t TMEM_COLS = 256;
static_assert(2 * (SMEM_BYTES + 1024) <= 232448, "two CTAs per SM");
static_assert(OFF_AL % 1024 == 0 && OFF_TS % 1024 == 0, "MMA operand tiles are 1024-aligned");
}  // namespace wy

struct WyParams {
  int *status;     // device status word: GDN2_ERR_TIMEOUT (4) when a bounded wait gave up
  int N;           // sequences
  int nc;          // chunks per sequence of a dense batch
  int nrec;        // records to walk: dense N * nc * H; packed capacity * H (those past the batch are skipped)
  int order;       // walking order: 0 record order; dense batches 1 chunk-major, last chunk first, 2 chunk-major
  int sms;         // SMs of the device
  int reserve;     // CTAs on SMs 0 .. reserve-1 stop claiming records at `stop_at` (0: none do)
  int stop_at;
  int64_t tokens;  // rows of the token tensors
  const int32_t *coff;  // packed batch: chunk offsets [N+1]; dense: nullptr
  float *g;             // workspace e^{g_C} [records][128]
  int *next;            // record counter, zero at launch: CTAs claim their records after the first in order
  int *ready;           // per record, zero at launch: 1 once its stores are complete (published only when
                        // the state pass runs alongside: `publish`; else it waits for every CTA to finish)
  int publish;
  int *done;            // factorisation CTAs that have finished (every record published), zero at launch
  int ctas;             // factorisation CTAs launched
};

// Workspace record of the i-th record in walking order.  Chunk-major walks take chunk c of every
// (sequence, head) before chunk c+1.  First chunk first suits a state pass that runs alongside the
// factorisation; last chunk first suits one that starts after it, because the records of the first
// chunks, which it reads first, are then the ones written last (most likely still in L2).
__device__ __forceinline__ int wy_record(const WyParams &p, int H, int i) {
  if (p.order == 0) return i;
  const int per_c = p.N * H;
  const int c = p.order == 1 ? p.nc - 1 - i / per_c : i / per_c, rem = i % per_c;
  return ((rem / H) * p.nc + c) * H + rem % H;
}

// Token row of the first token of record `rec` (global chunk * H + head), or -1 when the record lies
// past the chunks of a packed batch.
__device__ __forceinline__ int wy_tok0(const ChunkArgs &a, const WyParams &p, int rec, int *n_out, int *c_out) {
  const int gidx = rec / a.H;
  int n, c;
  if (p.coff) {
    if (gidx >= p.coff[p.N]) return -1;
    n = seq_of_chunk(p.coff, p.N, gidx);
    c = gidx - p.coff[n];
  } else {
    n = gidx / p.nc;
    c = gidx % p.nc;
  }
  int64_t bos;
  int len;
  seq_span(a, n, bos, len);
  *n_out = n;
  *c_out = c;
  return (int)(bos + (int64_t)c * C);
}

// Persistent (two CTAs per SM): CTA i takes record i first, then claims unclaimed records from a
// counter one record ahead (the claim's round trip overlaps a whole record), so records finish
// roughly in their walking order and no CTA is left with a long tail.  The set-up (barriers, tensor
// memory, descriptor prefetch) happens once; every record's inputs are prefetched into L2 one record
// ahead, and the stores of a record are waited for (their shared-memory sources read) only when the
// next record's loads are about to overwrite them.  The state pass may start before this kernel
// ends.  When it is to run alongside (`publish`), CTAs on the first `reserve` SMs stop claiming at
// `stop_at`, so that those SMs fall idle early and the state pass runs there while the other SMs
// factor the rest, and each record's flag is published once its stores are complete (during the
// next record's substitution, where the wait and the release cost least); the state pass waits on
// the flags.  Otherwise it waits for the count of finished CTAs, which each CTA raises once its last
// store is complete.
__global__ void __launch_bounds__(wy::NT, 2)
    wy_factor_kernel(const ChunkArgs a, const WyParams p, const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_al, const __grid_constant__ CUtensorMap tm_wm,
                     const __grid_constant__ CUtensorMap tm_wn, const __grid_constant__ CUtensorMap tm_wq,
                     const __grid_constant__ CUtensorMap tm_wp) {
  using namespace wy;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, quad = warp & 3, khalf = warp >> 2;

  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);
  const uint32_t bar_full = sb + OFF_BAR, bar_mma = sb + OFF_BAR + 8;
  float *Ls = reinterpret_cast<float *>(sm + OFF_AL);
  float *Ts = reinterpret_cast<float *>(sm + OFF_TS);
  float *scan = reinterpret_cast<float *>(sm + OFF_TP);  // [16 groups][128 channels]
  float *s_em = reinterpret_cast<float *>(sm + OFF_SC), *s_egcm = s_em + 128, *s_egc = s_em + 256;

  if (tid == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_b); prefetch_tmap(&tm_al);
    prefetch_tmap(&tm_wm); prefetch_tmap(&tm_wn); prefetch_tmap(&tm_wq); prefetch_tmap(&tm_wp);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16);
  griddep_launch_dependents();  // the state pass may be scheduled onto SMs as they fall idle
  bool ok = true;
  uint32_t nfull = 0, nmma = 0;  // completed phases of the two barriers
  // the next record, in one of two slots by iteration parity (a slot is rewritten only after every
  // thread has passed the barrier that follows its read)
  volatile int *s_next = reinterpret_cast<volatile int *>(sm + OFF_BAR + 20);
  const bool stops = p.reserve > 0 && (int)sm_id_count() == p.sms && (int)sm_id() < p.reserve;
  // thread 0: the record claimed for after the next one; thread ST_TID: the last record whose flag is
  // still to be published
  int claim = 0, prev = -1;
  if (tid == 0) claim = (int)gridDim.x + atomicAdd(p.next, 1);

  bool pre = false;  // this record's input loads were issued by the previous record's epilogue
  for (int it = blockIdx.x, nit = 0, par = 0; it < p.nrec; it = nit, par ^= 1) {
    const int rec = wy_record(p, a.H, it);
    const int h = rec % a.H;
    int n, c;
    const int tok0 = wy_tok0(a, p, rec, &n, &c);
    if (tid == 0) {
      s_next[par] = claim;
      claim = (claim >= p.nrec || (stops && claim >= p.stop_at)) ? p.nrec : (int)gridDim.x + atomicAdd(p.next, 1);
    }
    __syncthreads();
    nit = s_next[par];
    if (tok0 < 0) continue;  // past the chunks of a packed batch (uniform per CTA)
    int64_t bos;
    int len;
    seq_span(a, n, bos, len);
    const int Cc = min(C, len - c * C);

    // the next record of this CTA, whose loads this record's epilogue issues when it is a real one
    int nn = 0, ncc = 0;
    const int nrec_ = nit < p.nrec ? wy_record(p, a.H, nit) : 0;
    const int ntok = nit < p.nrec ? wy_tok0(a, p, nrec_, &nn, &ncc) : -1;
    if (tid == ST_TID) bulk_wait_read();  // the previous record's stores have read TP and TS (reused below)
    if (tid == 0) {
      if (!pre) {
        mbar_expect_tx(bar_full, TMA_BYTES);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          tma_load_3d(sb + OFF_XA + blk * XA_BLK, &tm_b, 64 * blk, h, tok0, bar_full);         // b -> rows 0..63
          tma_load_3d(sb + OFF_XA + blk * XA_BLK + 8192, &tm_q, 64 * blk, h, tok0, bar_full);  // q -> rows 64..127
          tma_load_3d(sb + OFF_KT + blk * KT_BLK, &tm_k, 64 * blk, h, tok0, bar_full);
          tma_load_3d(sb + OFF_AL + blk * 8192, &tm_al, 64 * blk, h, tok0, bar_full);
        }
      }
      // this CTA's next record into L2, so that its loads come from there
      if (ntok >= 0) {
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          tma_prefetch_3d(&tm_b, 64 * blk, nrec_ % a.H, ntok);
          tma_prefetch_3d(&tm_q, 64 * blk, nrec_ % a.H, ntok);
          tma_prefetch_3d(&tm_k, 64 * blk, nrec_ % a.H, ntok);
          tma_prefetch_3d(&tm_al, 64 * blk, nrec_ % a.H, ntok);
        }
      }
    }

    // ------------------------------------------------------------ decay factors, operands in place
    if (!mbar_wait_bounded(bar_full, nfull & 1, WAIT_NS)) ok = false;
    ++nfull;
    if (__syncthreads_or(!ok)) goto done;
    // the never-written blocks (0,1) and (2,3) of T, which the 32x32 merges read (the region held the
    // previous record's Mt tile 1, whose store has read it)
    for (int e = tid; e < 512; e += NT) {
      const int R = 2 * (e >> 8), r = (e >> 4) & 15, j = e & 15;
      Ts[(16 * R + r) * LDF + 16 * (R + 1) + j] = 0.f;
    }
    {
      // thread = 8 key channels (chunk x8 of channel block cb) x 4 tokens (group G = rows 4G..4G+3);
      // groups 0-7 hold tokens 0..31 (walk back to token 31), groups 8-15 tokens 32..63 (walk forward)
      const int ch8 = tid & 15, G = tid >> 4, cb = ch8 >> 3, x8 = ch8 & 7;
      uint4 ra[4], rb[4], rq[4], rk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t o = sw128(4 * G + i, 8 * x8);
        ra[i] = ld_s128(sm + OFF_AL + cb * 8192 + o);
        if (64 * cb >= a.dk) ra[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);  // bf16 1.0
        rb[i] = ld_s128(sm + OFF_XA + cb * XA_BLK + o);
        rq[i] = ld_s128(sm + OFF_XA + cb * XA_BLK + 8192 + o);
        rk[i] = ld_s128(sm + OFF_KT + cb * KT_BLK + o);
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
      __syncthreads();
      if (tid < 128) {  // per channel: products between each group and token 31, in place of the group products
        float pg[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) pg[g] = scan[g * 128 + tid];
        float acc = 1.f;
#pragma unroll
        for (int g = 7; g >= 0; --g) {
          scan[g * 128 + tid] = acc;  // prod over groups g+1..7
          acc *= pg[g];
        }
        const float em = acc;
        acc = 1.f;
#pragma unroll
        for (int g = 8; g < 16; ++g) {
          scan[g * 128 + tid] = acc;  // prod over groups 8..g-1
          acc *= pg[g];
        }
        s_em[tid] = em;
        s_egcm[tid] = acc;
        s_egc[tid] = em * acc;
      }
      __syncthreads();
      float run[8];
      {
        const float4 p0 = *reinterpret_cast<const float4 *>(&scan[G * 128 + 8 * ch8]);
        const float4 p1 = *reinterpret_cast<const float4 *>(&scan[G * 128 + 8 * ch8 + 4]);
        run[0] = p0.x; run[1] = p0.y; run[2] = p0.z; run[3] = p0.w;
        run[4] = p1.x; run[5] = p1.y; run[6] = p1.z; run[7] = p1.w;
      }
      uint8_t *pa0 = sm + OFF_XA + cb * XA_BLK, *pk0 = sm + OFF_KT + cb * KT_BLK;
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
          row_factors(pa0, pk0, sw128(r, 8 * x8), rb[i], rq[i], rk[i], r < Cc, f, fi);
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
          row_factors(pa0, pk0, sw128(r, 8 * x8), rb[i], rq[i], rk[i], r < Cc, f, fi);
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ M1: [L; P] = [A_m; Q_m] K_m^T (TMEM cols 0..63)
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
    if (!mbar_wait_bounded(bar_mma, nmma & 1, WAIT_NS)) ok = false;
    ++nmma;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();

    // ------------------------------------------------------------ T = (I + L)^-1
    {  // L (strict lower) -> fp32 scratch; P (inclusive lower) -> rows 64..127 of [T ; P]
      float v[32];
      tmem_ld32(tl + 32 * khalf, v);
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
          st_s128(sm + OFF_TP + 8192 + sw128(r, col), pack8(e));
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == ST_TID && p.publish && prev >= 0) {  // the previous record's stores are complete: publish it
      bulk_wait_done<0>();
      flag_publish(p.ready + prev);
      prev = -1;
    }
    if (warp < 2) {  // the four 16x16 diagonal blocks, right-looking; lane = column j of block R
      const int R = 2 * warp + (lane >> 4), j = lane & 15;
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
    __syncthreads();
    // merges on the warp-level tensor cores (tf32), with [[A,0],[C,B]]^-1 = [[A^-1,0],[-B^-1 C A^-1, B^-1]]:
    // 16x16 blocks first; a warp needs only its own column tile of Y, so a warp barrier suffices
    if (warp < 4) {
      const int R = (warp < 2) ? 1 : 3, nt = warp & 1;
      float d[4];
      // Y_R = L_{R,R-1} T_{R-1,R-1}, parked in the upper block (R-1, R) of L
      mma_tf32_16x8<16>(Ls + 16 * R * LDF + 16 * (R - 1), Ts + 16 * (R - 1) * LDF + 16 * (R - 1) + 8 * nt, lane, d);
      store_16x8(Ls + 16 * (R - 1) * LDF + 16 * R + 8 * nt, lane, d, 1.f);
      __syncwarp();
      // T_{R,R-1} = -T_RR Y_R
      mma_tf32_16x8<16>(Ts + 16 * R * LDF + 16 * R, Ls + 16 * (R - 1) * LDF + 16 * R + 8 * nt, lane, d);
      store_16x8(Ts + 16 * R * LDF + 16 * (R - 1) + 8 * nt, lane, d, -1.f);
    }
    __syncthreads();
    {  // lower-left 32x32 block: T[32:64, 0:32] = -T[32:64, 32:64] Y with Y = L[32:64, 0:32] T[0:32, 0:32];
       // warp (mt, nt) forms both row halves of Y's column tile nt itself and keeps them in registers
      const int mt = warp >> 2, nt = warp & 3;
      float y0[4], y1[4], d[4];
      mma_tf32_16x8<32>(Ls + 32 * LDF, Ts + 8 * nt, lane, y0);
      mma_tf32_16x8<32>(Ls + 48 * LDF, Ts + 8 * nt, lane, y1);
      mma_tf32_16x8_yreg(Ts + (32 + 16 * mt) * LDF + 32, y0, y1, lane, d);
      store_16x8(Ts + (32 + 16 * mt) * LDF + 8 * nt, lane, d, -1.f);
    }
    __syncthreads();
    {  // T -> rows 0..63 of [T ; P], bf16 (the upper-right 32x32 block is zero)
      const int r = tid >> 2;
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        const int col = 16 * (tid & 3) + 8 * y;
        float e[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (r >= 32 || col < 32) {
          const float4 t0 = *reinterpret_cast<const float4 *>(&Ts[r * LDF + col]);
          const float4 t1 = *reinterpret_cast<const float4 *>(&Ts[r * LDF + col + 4]);
          e[0] = t0.x; e[1] = t0.y; e[2] = t0.z; e[3] = t0.w; e[4] = t1.x; e[5] = t1.y; e[6] = t1.z; e[7] = t1.w;
        }
        st_s128(sm + OFF_TP + sw128(r, col), pack8(e));
      }
    }
    fence_proxy_async();
    __syncthreads();

    // ------------------------------------------------------------ product pass 1: [T; P] [A_m | T] and K_m^T T
    // TMEM cols 0..127: rows 0..63 T A_m; cols 128..191: rows 64..127 P T; cols 192..255: K_m^T T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t a_tp = sdesc_sw128(sb + OFF_TP + 32 * k, 16, 1024);
        const uint64_t b_t = sdesc_sw128(sb + OFF_TP + 2048 * k, 8192, 1024);  // T: rows = K, MN-major
        mma_bf16(tmem + 0, a_tp, sdesc_sw128(sb + OFF_XA + 2048 * k, XA_BLK, 1024), ID_KM128, k > 0 ? 1u : 0u);
        mma_bf16(tmem + 128, a_tp, b_t, ID_KM64, k > 0 ? 1u : 0u);
        mma_bf16(tmem + 192, sdesc_sw128(sb + OFF_KT + 2048 * k, KT_BLK, 1024), b_t, ID_MN64, k > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    if (!mbar_wait_bounded(bar_mma, nmma & 1, WAIT_NS)) ok = false;
    ++nmma;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    {
      const int row = 32 * quad + lane;
      if (quad < 2) {  // W' = -T A_m Diag(e^m) -> W tile khalf (64 tokens x 64 channels, MN-major B operand)
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          float v[32];
          tmem_ld32(tl + 64 * khalf + 32 * part, v);
          tmem_wait_ld();
          const float4 *em4 = reinterpret_cast<const float4 *>(s_em + 64 * khalf + 32 * part);
#pragma unroll
          for (int y = 0; y < 8; ++y) {  // times -e^m of each channel
            const float4 e = em4[y];
            const float ne[4] = {-e.x, -e.y, -e.z, -e.w};
            mul2(&v[4 * y], &v[4 * y], &ne[0]);
            mul2(&v[4 * y + 2], &v[4 * y + 2], &ne[2]);
          }
#pragma unroll
          for (int y = 0; y < 4; ++y)
            st_s128(sm + OFF_AL + khalf * 8192 + sw128(row, 32 * part + 8 * y), pack8(&v[8 * y]));
        }
      } else {  // Pt = P T -> rows 64..127 of the products; warp group khalf takes 32 columns.  Pt is
                // written twice, as rows 0..63 and 64..127 of pass 2's A operand, so that Pt A_m
                // lands in all 128 lanes and every warp can read its share of it
        float v[32];
        tmem_ld32(tl + 128 + 32 * khalf, v);
        tmem_wait_ld();
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const uint4 x = pack8(&v[8 * y]);
          st_s128(sm + OFF_TS + sw128(row - 64, 32 * khalf + 8 * y), x);
          st_s128(sm + OFF_TS + 8192 + sw128(row - 64, 32 * khalf + 8 * y), x);
        }
      }
      {  // Nt = Diag(e^{g_C-m}) K_m^T T, key channel `row`, tokens 32 khalf .. +31
        float v[32];
        tmem_ld32(tl + 192 + 32 * khalf, v);
        tmem_wait_ld();
        const float g2 = s_egcm[row];
        const float g2p[2] = {g2, g2};
#pragma unroll
        for (int j = 0; j < 32; j += 2) mul2(&v[j], &v[j], g2p);
#pragma unroll
        for (int y = 0; y < 4; ++y) st_s128(sm + OFF_TP + sw128(row, 32 * khalf + 8 * y), pack8(&v[8 * y]));
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == ST_TID) {  // Nt, Pt and e^{g_C} are final: store them while product pass 2 runs
      tma_store_2d(&tm_wn, 0, rec * 128, sb + OFF_TP);
      tma_store_2d(&tm_wp, 0, rec * 64, sb + OFF_TS);
      bulk_store(p.g + (size_t)rec * 128, sb + OFF_SC + 256 * 4, REC_G);
      bulk_commit();
    }

    // ------------------------------------------------------------ product pass 2: K_m^T W' and [Pt; *] A_m
    // TMEM cols 0..127: K_m^T W'; cols 128..255: Pt A_m in rows 0..63 and again in rows 64..127
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mma_bf16(tmem + 0, sdesc_sw128(sb + OFF_KT + 2048 * k, KT_BLK, 1024),
                 sdesc_sw128(sb + OFF_AL + 2048 * k, 8192, 1024), ID_MN128, k > 0 ? 1u : 0u);
        mma_bf16(tmem + 128, sdesc_sw128(sb + OFF_TS + 32 * k, 16, 1024),
                 sdesc_sw128(sb + OFF_XA + 2048 * k, XA_BLK, 1024), ID_KM128, k > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    // Nt and Pt: their stores have read the tiles before any thread passes the barrier below (the
    // epilogue writes Mt into them)
    if (tid == ST_TID) bulk_wait_read();
    if (!mbar_wait_bounded(bar_mma, nmma & 1, WAIT_NS)) ok = false;
    ++nmma;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // K_m and W' are dead now: the next record's k and alpha go into their tiles while this record's
    // epilogue runs (its q and b follow once Q_m is read and Qt has been stored)
    pre = ntok >= 0;
    if (tid == 0) {
      if (pre) {
        mbar_expect_tx(bar_full, TMA_BYTES);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          tma_load_3d(sb + OFF_KT + blk * KT_BLK, &tm_k, 64 * blk, nrec_ % a.H, ntok, bar_full);
          tma_load_3d(sb + OFF_AL + blk * 8192, &tm_al, 64 * blk, nrec_ % a.H, ntok, bar_full);
        }
      }
    }
    {
      const int row = 32 * quad + lane;
      // Mt = Diag(e^{g_C-m}) K_m^T W': row = key channel, input channels 64 khalf .. +63 -> TP / TS
      auto mt_epilogue = [&]() {
        const float g2 = s_egcm[row];
        const float g2p[2] = {g2, g2};
        uint8_t *dst = sm + (khalf ? OFF_TS : OFF_TP);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          float v[32];
          tmem_ld32(tl + 64 * khalf + 32 * part, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 2) mul2(&v[j], &v[j], g2p);
#pragma unroll
          for (int y = 0; y < 4; ++y) st_s128(dst + sw128(row, 32 * part + 8 * y), pack8(&v[8 * y]));
        }
      };
      {  // Qt = (Q_m - Pt A_m) Diag(e^m) in place of A_m: warp (quad, khalf) takes tokens
         // 32 (quad & 1) .. +31 of columns 32 (quad >> 1) .. +31 of channel block khalf (quads 2
         // and 3 read the copy of Pt A_m in lanes 64..127)
        const int trow = 32 * (quad & 1) + lane, part = quad >> 1;
        uint8_t *blk = sm + OFF_XA + khalf * XA_BLK;
        float v[32];
        tmem_ld32(tl + 128 + 64 * khalf + 32 * part, v);
        tmem_wait_ld();
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int col = 32 * part + 8 * y;
          float qm[8], e[8];
          unpack8(ld_s128(blk + 8192 + sw128(trow, col)), qm);
#pragma unroll
          for (int t = 0; t < 8; t += 2) {
            const float2 dq = __fadd2_rn(make_float2(qm[t], qm[t + 1]), make_float2(-v[8 * y + t], -v[8 * y + t + 1]));
            const float2 r = __fmul2_rn(dq, *reinterpret_cast<const float2 *>(&s_em[64 * khalf + col + t]));
            e[t] = r.x;
            e[t + 1] = r.y;
          }
          st_s128(blk + sw128(trow, col), pack8(e));
        }
        fence_proxy_async();
        __syncthreads();  // every Qt tile written, every Q_m row read
        if (tid == ST_TID) {  // Qt -> workspace; the next record's q into the dead Q_m rows
          tma_store_2d(&tm_wq, 0, rec * 64, sb + OFF_XA);
          tma_store_2d(&tm_wq, 64, rec * 64, sb + OFF_XA + XA_BLK);
          bulk_commit();
          if (pre) {
#pragma unroll
            for (int blk2 = 0; blk2 < 2; ++blk2)
              tma_load_3d(sb + OFF_XA + blk2 * XA_BLK + 8192, &tm_q, 64 * blk2, nrec_ % a.H, ntok, bar_full);
          }
        }
      }
      mt_epilogue();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ Mt -> workspace (waited for at the next record)
    if (tid == ST_TID) {
      tma_store_2d(&tm_wm, 0, rec * 128, sb + OFF_TP);
      tma_store_2d(&tm_wm, 64, rec * 128, sb + OFF_TS);
      bulk_commit();
      prev = rec;
      if (pre) {  // the next record's b into the rows Qt leaves, once its store has read them
        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
#pragma unroll
        for (int blk = 0; blk < 2; ++blk)
          tma_load_3d(sb + OFF_XA + blk * XA_BLK, &tm_b, 64 * blk, nrec_ % a.H, ntok, bar_full);
      }
    }
  }

done:
  if (tid == 0 && !ok) atomicExch(p.status, 4);
  if (tid == ST_TID) {
    bulk_wait_done<0>();
    if (p.publish && prev >= 0) flag_publish(p.ready + prev);
    counter_release_add(p.done);  // after this CTA's last store is complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ==================================================================== kernel 2: state pass
// One CTA per (sequence, head, 128 value columns).  The products run transposed, with the state as
// the A operand straight from tensor memory (value column = TMEM lane):
//   [D1^T | O^T] = U^T [Nt^T | Pt^T] + S^T [Mt^T | Qt^T]   (128 value columns x (128 keys + 64 tokens))
// as two MMAs of N = 192 per K step: one over U (K = 64 tokens) and one over S (K = 128 keys), whose
// B operands are Nt over Pt and Mt over Qt, stacked row-wise in shared memory.
// Roles:
//   warps 0-7   the state (thread = value column v, key-channel half hf: S[64 hf ..][v]): the serial
//               chain per chunk (D1 -> S update -> S^T into tensor memory), then, while the next
//               chunk's products run, O^T out of tensor memory into o (staged, one TMA store);
//   warp 8      lane 0 loads each chunk's Mt, e^{g_C} and Qt, lane 1 its v, w, Nt and Pt;
//   warp 9      lane 0 issues the products;
//   warps 10-13 form U = w (.) v in shared memory in place of v (tokens past a sequence's end zero).
// A chunk's buffers come in two parts, each double-buffered by chunk parity and released as soon
// as the product that reads it completes: {v, w, Nt, Pt} after the U product, {Mt, Qt, e^{g_C}}
// after the S product (and the state warps' read of e^{g_C}); so the loads of chunk c+2 start
// while chunk c+1 is still in flight.  Tensor memory is double-buffered per chunk parity.
namespace sp {
constexpr int VW = 128;        // value columns per CTA
constexpr int NSTATE = 256;    // warps 0-7
constexpr int W_LOAD = 8, W_MMA = 9, W_AUX = 10, NAUX = 128;
constexpr int NT = 448;
constexpr int BAR_STATE = 1, BAR_AUX = 2;
// one stage (chunk buffer); every operand tile 1024-aligned
constexpr uint32_t MQ_BLK = 24576;           // one input channel block: Mt (128 rows) over Qt (64 rows)
constexpr uint32_t S_MQ = 0;                 // two such blocks
constexpr uint32_t S_N = S_MQ + 2 * MQ_BLK;  // 49152: Nt, 128 rows, and right after it
constexpr uint32_t S_P = S_N + REC_N;        // 65536: Pt, 64 rows (together one 192-row operand)
constexpr uint32_t S_V = S_P + REC_P;        // 73728: v, two 64-column tiles of 64 tokens -> U = w (.) v in place
constexpr uint32_t S_W = S_V + 16384;        // 90112: w, likewise
constexpr uint32_t STAGE = S_W + 16384;      // 106496
constexpr uint32_t OFF_OST = 2 * STAGE;      // 212992: O staging, two 64-column tiles of 64 tokens
constexpr uint32_t OFF_G = OFF_OST + 16384;  // 229376: e^{g_C} of the two stages
constexpr uint32_t OFF_BAR = OFF_G + 2 * REC_G;  // 230400
constexpr uint32_t SMEM_USED = OFF_BAR + 256;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
constexpr uint32_t TMEM_COLS = 512;
// per buffer b = chunk parity (256 columns at 256 b): S^T (bf16 pairs) 64 cols, then D1^T 128 cols
// and O^T 64 cols side by side, so one MMA of N = 192 writes U^T [Nt^T | Pt^T] into both
constexpr uint32_t TM_AS = 0, TM_D1 = 64, TM_D2 = 192;
constexpr uint32_t ID_192 = idesc_bf16(128, 192, false, false), ID_128 = idesc_bf16(128, 128, false, false);
constexpr uint32_t ID_U192 = idesc_bf16(128, 192, true, false), ID_U128 = idesc_bf16(128, 128, true, false);
enum {
  B_FU0 = 0, B_FU1,          // v, w, Nt, Pt of the stage loaded
  B_FM0, B_FM1,              // Mt, Qt and e^{g_C} loaded
  B_UREADY0, B_UREADY1,      // U^T of the stage formed by the aux warps
  B_UFREE0, B_UFREE1,        // the U product of the stage complete: v, w, Nt, Pt free
  B_SREADY,                  // S^T of the next chunk is in tensor memory
  B_D1FULL0, B_D1FULL1,      // every product of the buffer's chunk complete: D1 and O^T (Mt, Qt free)
  B_D1FREE0, B_D1FREE1,      // D1 of the buffer and the stage's e^{g_C} read by the state warps
  B_OREAD0, B_OREAD1,        // O^T of the buffer read out by the aux warps
  B_COUNT
};
static_assert(SMEM_BYTES <= 232448, "one CTA per SM");
static_assert(8 * B_COUNT + 4 <= 256, "barriers and the tensor-memory slot fit their region");
}  // namespace sp

// How one state-pass CTA is placed and what it produces.  Mode 0 walks whole sequences.  For long
// sequences with few heads the walk is split into segments of `seg_len` chunks (two-level scan):
// mode 1 summarises every segment but the last as an affine map X -> A_j X + B_j of the entering
// state (A_j from the identity without U, B_j from zero, or from S0 for j = 0, with U); after the
// combine kernel has chained the maps into each segment's entry state, mode 2 walks every segment
// from its entry state and writes O (and S_T after the last).
struct ScanParams {
  int mode;        // 0 whole sequences, 1 segment summaries, 2 segments from their entry states
  int seg_len;     // chunks per segment (modes 1, 2)
  int nseg;        // segments per sequence (modes 1, 2; dense batches only)
  float *sum_a;    // [N][H][nseg-1][128][128]: A_j (mode 1)
  float *sum_b;    // [N][H][nseg-1][128][d_v]: B_j (mode 1)
  float *s_start;  // [N][H][nseg][128][d_v]: entry state of segment j >= 1 (mode 2)
};

// Shared-memory matrix descriptor of the tile at byte offset `off` from the one `base` describes
// (the start address is the descriptor's low field, in 16-byte units; offsets stay inside the CTA's
// shared memory, so the field never carries).
__device__ __forceinline__ uint64_t desc_at(uint64_t base, uint32_t off) { return base + (uint64_t)(off >> 4); }

__global__ void __launch_bounds__(sp::NT, 1)
    state_pass_kernel(const ChunkArgs a, const WyParams p, const ScanParams q, const __grid_constant__ CUtensorMap tm_wm,
                      const __grid_constant__ CUtensorMap tm_wn, const __grid_constant__ CUtensorMap tm_wq,
                      const __grid_constant__ CUtensorMap tm_wp, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_o) {
  using namespace sp;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 8 * B_COUNT);
  auto bar = [&](int i) { return sb + OFF_BAR + 8u * (uint32_t)i; };

  // ------------------------------------------------------------ placement
  const int tiles = (a.dv + VW - 1) / VW;
  int n, h, tile = 0, seg = 0;
  bool ident = false;  // mode 1, A_j: the state starts as the identity and U is left out
  if (q.mode == 1) {
    const int per = 1 + tiles;  // A_j, then one CTA per value tile for B_j
    const int t = blockIdx.x % per;
    seg = (blockIdx.x / per) % (q.nseg - 1);
    h = (blockIdx.x / (per * (q.nseg - 1))) % a.H;
    n = blockIdx.x / (per * (q.nseg - 1) * a.H);
    ident = t == 0;
    tile = ident ? 0 : t - 1;
    if (ident && seg == 0) {  // segment 0 starts from S0: its end state is all that is needed
      griddep_wait();
      return;
    }
  } else if (q.mode == 2) {
    tile = blockIdx.x % tiles;
    seg = (blockIdx.x / tiles) % q.nseg;
    h = (blockIdx.x / (tiles * q.nseg)) % a.H;
    n = blockIdx.x / (tiles * q.nseg * a.H);
  } else {
    tile = blockIdx.x % tiles;
    h = (blockIdx.x / tiles) % a.H;
    n = blockIdx.x / (tiles * a.H);
  }
  const int j0 = tile * VW;
  const int cols = ident ? DK : a.dv;  // column count of the state this CTA carries
  const bool use_u = !ident, use_o = q.mode != 1;
  int64_t bos;
  int len;
  seq_span(a, n, bos, len);
  const int nch = (len + C - 1) / C;
  const int cb = q.mode == 0 ? 0 : seg * q.seg_len;
  const int ce = q.mode == 0 ? nch : min(nch, cb + q.seg_len);
  const int nk = max(ce - cb, 0);  // chunks of this CTA, local index k -> chunk cb + k
  const int coff = p.coff ? p.coff[n] : n * p.nc;  // global chunk of this sequence's chunk 0
  auto chunk_len = [&](int c) { return min(C, len - c * C); };

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), 1u);
    fence_mbar_init();
    prefetch_tmap(&tm_wm); prefetch_tmap(&tm_wn); prefetch_tmap(&tm_wq); prefetch_tmap(&tm_wp);
    prefetch_tmap(&tm_v); prefetch_tmap(&tm_w); prefetch_tmap(&tm_o);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == W_LOAD) {
    // A chunk's record may be read once its flag is published, or once every factorisation CTA has
    // finished (the only signal when the factorisation publishes no flags).  The check comes before
    // the wait for the stage, so that its round trip overlaps that wait.
    bool all_done = false;
    auto record_ready = [&](int rec) -> bool {
      if (all_done) return true;
      if (p.publish) {
        if (counter_acquire(p.done) < p.ctas) return flag_wait_bounded(p.ready + rec, WAIT_NS);
      } else if (counter_acquire(p.done) < p.ctas) {
        const uint64_t t0 = globaltimer_ns();
        do {
          __nanosleep(256);
          if (globaltimer_ns() - t0 > WAIT_NS) return false;
        } while (counter_acquire(p.done) < p.ctas);
      }
      all_done = true;
      asm volatile("fence.proxy.async.global;" ::: "memory");
      return true;
    };
    if (lane == 0) {
      // ---------------------------------------------------------- Mt, Qt, e^{g_C} of each chunk
      for (int k = 0; k < nk; ++k) {
        const int s = k & 1, c = cb + k, ph2 = ((k - 2) >> 1) & 1;
        const uint32_t st = sb + s * STAGE, full = bar(B_FM0 + s);
        const int rec = (coff + c) * a.H + h;
        // the record's stores are complete; chunk k-2's buffers are free once its products are
        // complete and the state warps read e^{g_C}
        if (!record_ready(rec) || (k >= 2 && !(mbar_wait_bounded(bar(B_D1FULL0 + s), ph2, WAIT_NS) &&
                                               mbar_wait_bounded(bar(B_D1FREE0 + s), ph2, WAIT_NS)))) {
          ok = false;
          break;
        }
        mbar_expect_tx(full, REC_M + REC_G + (use_o ? REC_Q : 0));
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          tma_load_2d(st + S_MQ + blk * MQ_BLK, &tm_wm, 64 * blk, rec * 128, full);
          if (use_o) tma_load_2d(st + S_MQ + blk * MQ_BLK + 16384, &tm_wq, 64 * blk, rec * 64, full);
        }
        bulk_load(sb + OFF_G + s * REC_G, p.g + (size_t)rec * 128, REC_G, full);
        if (k + 2 < nk) {  // chunk k+2 into L2, so its later load from there is short
          const int rp = rec + 2 * a.H;
          tma_prefetch_2d(&tm_wm, 0, rp * 128);
          tma_prefetch_2d(&tm_wm, 64, rp * 128);
          if (use_o) {
            tma_prefetch_2d(&tm_wq, 0, rp * 64);
            tma_prefetch_2d(&tm_wq, 64, rp * 64);
          }
          bulk_prefetch(p.g + (size_t)rp * 128, REC_G);
        }
      }
    } else if (lane == 1 && use_u) {
      // ---------------------------------------------------------- v, w, Nt, Pt of each chunk
      const uint32_t bytes = 4 * 8192 + REC_N + (use_o ? REC_P : 0);
      for (int k = 0; k < nk; ++k) {
        const int s = k & 1, c = cb + k;
        const uint32_t st = sb + s * STAGE, full = bar(B_FU0 + s);
        const int rec = (coff + c) * a.H + h;
        const int tok0 = (int)(bos + (int64_t)c * C);
        if (!record_ready(rec) || (k >= 2 && !mbar_wait_bounded(bar(B_UFREE0 + s), ((k - 2) >> 1) & 1, WAIT_NS))) {
          ok = false;
          break;
        }
        mbar_expect_tx(full, bytes);
#pragma unroll
        for (int vb = 0; vb < 2; ++vb) {  // columns past d_v (d_v = 64) load as zeros
          tma_load_3d(st + S_V + vb * 8192, &tm_v, j0 + 64 * vb, h, tok0, full);
          tma_load_3d(st + S_W + vb * 8192, &tm_w, j0 + 64 * vb, h, tok0, full);
        }
        tma_load_2d(st + S_N, &tm_wn, 0, rec * 128, full);
        if (use_o) tma_load_2d(st + S_P, &tm_wp, 0, rec * 64, full);
        if (k + 2 < nk) {
          const int rp = rec + 2 * a.H, tp = tok0 + 2 * C;
#pragma unroll
          for (int vb = 0; vb < 2; ++vb)
            if (j0 + 64 * vb < a.dv) {
              tma_prefetch_3d(&tm_v, j0 + 64 * vb, h, tp);
              tma_prefetch_3d(&tm_w, j0 + 64 * vb, h, tp);
            }
          tma_prefetch_2d(&tm_wn, 0, rp * 128);
          if (use_o) tma_prefetch_2d(&tm_wp, 0, rp * 64);
        }
      }
    }
  } else if (warp == W_MMA) {
    // ---------------------------------------------------------- products (one thread)
    if (lane == 0) {
      const uint64_t dk_base = sdesc_sw128(sb, 16, 1024);    // K-major operand tiles
      const uint64_t dmn_base = sdesc_sw128(sb, 8192, 1024); // MN-major U (two 64-column tiles 8 KB apart)
      for (int k = 0; k < nk; ++k) {
        const int s = k & 1, b = k & 1, ph = (k >> 1) & 1;
        const uint32_t stg = s * STAGE;
        const uint32_t as = tmem + 256 * b + TM_AS, d1 = tmem + 256 * b + TM_D1;
        const uint32_t id = use_o ? ID_192 : ID_128;  // [D1 | O^T], or D1 alone
        if (use_u && !mbar_wait_bounded(bar(B_UREADY0 + s), ph, WAIT_NS)) { ok = false; break; }
        // D1 and O^T of this buffer were last read for chunk k-2
        if (k >= 2 && !(mbar_wait_bounded(bar(B_D1FREE0 + b), ph ^ 1, WAIT_NS) &&
                        (!use_o || mbar_wait_bounded(bar(B_OREAD0 + b), ph ^ 1, WAIT_NS)))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (use_u) {  // U^T Nt^T (and U^T Pt^T for the output), before the state is known
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(d1, desc_at(dmn_base, stg + S_V + 2048 * kk), desc_at(dk_base, stg + S_N + 32 * kk),
                     use_o ? ID_U192 : ID_U128, kk > 0 ? 1u : 0u);
          mma_commit(bar(B_UFREE0 + s));
        }
        if (!mbar_wait_bounded(bar(B_FM0 + s), ph, WAIT_NS) || !mbar_wait_spin_bounded(bar(B_SREADY), k & 1, WAIT_NS)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          mma_bf16_tmem_a(d1, as + 8 * kk, desc_at(dk_base, stg + S_MQ + (kk >> 2) * MQ_BLK + (kk & 3) * 32), id,
                          (use_u || kk > 0) ? 1u : 0u);
        mma_commit(bar(B_D1FULL0 + b));
      }
    }
  } else if (warp >= W_AUX) {
    // ---------------------------------------------------------- U formation and O readout (warps 10-13)
    const int atid = tid - W_AUX * 32;
    // U = w (.) v of chunk cb + k in place of v (16-byte pieces, each read and written by one thread);
    // tokens past the sequence (the tile holds the next sequence's tokens there) become zero
    auto form_u = [&](int k) -> bool {
      const int s = k & 1;
      if (!group_wait(BAR_AUX, NAUX, bar(B_FU0 + s), (k >> 1) & 1)) return false;
      const int Cc = chunk_len(cb + k);
      uint8_t *vt = sm + s * STAGE + S_V, *wt = sm + s * STAGE + S_W;
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // pieces: 64 rows x (2 tiles x 8); four loaded, then four stored
        uint4 vv[4], ww[4];
        uint32_t off[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = atid + NAUX * (4 * half + i), r = e >> 4, x = e & 15;
          off[i] = (uint32_t)(x >> 3) * 8192u + sw128(r, 8 * (x & 7));
          vv[i] = ld_s128(vt + off[i]);
          ww[i] = ld_s128(wt + off[i]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // bf16 x bf16 is exact in fp32: the packed product is the rounded one
          const int r = (atid + NAUX * (4 * half + i)) >> 4;
          uint4 u = make_uint4(0u, 0u, 0u, 0u);
          if (r < Cc) {
            u.x = bf2_mul(vv[i].x, ww[i].x);
            u.y = bf2_mul(vv[i].y, ww[i].y);
            u.z = bf2_mul(vv[i].z, ww[i].z);
            u.w = bf2_mul(vv[i].w, ww[i].w);
          }
          st_s128(vt + off[i], u);
        }
      }
      fence_proxy_async();
      group_sync(BAR_AUX, NAUX);
      if (atid == 0) mbar_arrive(bar(B_UREADY0 + s));
      return true;
    };
    for (int k = 0; use_u && k < nk; ++k)
      if (!form_u(k)) { ok = false; break; }
  } else if (warp < NSTATE / 32) {
    // ---------------------------------------------------------- state side
    const int q4 = warp & 3, hf = warp >> 2;
    const int v = 32 * q4 + lane;            // column within the tile (TMEM lane)
    const bool vin = j0 + v < cols;
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
    const size_t nh = (size_t)n * a.H + h;
    // S[64 hf + i][j0 + v] lives at base + i * cols in every [.., d_k, cols] state array (the caller's
    // S0 and S_T have d_k rows; with d_k = 64 the rows 64..127 the kernels carry stay zero)
    const bool kin = 64 * hf < a.dk;
    const size_t s_base = (nh * a.dk + 64 * hf) * (size_t)a.dv + j0 + v;
    float S[64];
    {
      const float *src = nullptr;
      size_t base = s_base, ld = (size_t)a.dv;
      if (q.mode == 2) {  // every segment, the first included, starts from its entry state (S_T may alias S0)
        src = q.s_start;
        base = ((nh * q.nseg + seg) * DK + 64 * hf) * (size_t)a.dv + j0 + v;
      } else if (!ident && seg == 0 && kin) {
        src = a.S0;
      }
#pragma unroll
      for (int i = 0; i < 64; ++i)
        S[i] = ident ? (64 * hf + i == v ? 1.f : 0.f) : ((src && vin) ? src[base + (size_t)i * ld] : 0.f);
    }
    // S^T of the chunk about to start -> tensor memory buffer b (bf16 pairs); signals the issuer
    auto put_state = [&](int b) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = f2_to_bf2(S[2 * i], S[2 * i + 1]);
      tmem_st32(tl + 256 * b + TM_AS + 32 * hf, r);
      tmem_wait_st();
    };
    // O of chunk cb + k, after the chain's work for the chunk (the state warps are otherwise idle until
    // the next chunk's products complete): thread (v, hf) takes tokens 32 hf .. +31 of column v out of
    // tensor memory and rounds them to bf16 into the staging tiles (the swizzled layout of the output
    // map).  A full chunk leaves by TMA; the last partial chunk of a sequence row by row (a box would
    // overrun into the next sequence): thread = token rr, a quarter qq of the tile's 128 columns.
    __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.o);
    const int rr = tid >> 2, qq = tid & 3;
    uint8_t *orow = sm + OFF_OST + (qq >> 1) * 8192;
    const int cq = 32 * (qq & 1);  // first column of the quarter inside its 64-column tile
    const bool qin = j0 + 32 * qq < a.dv;
    auto read_out = [&](int k) -> bool {
      const int b = k & 1, c = cb + k, Cc = chunk_len(c);
      const int tok0 = (int)(bos + (int64_t)c * C);
      uint32_t dp[16];  // O of tokens 32 hf .. +31, column v, as bf16 pairs
      {
        float d[32];
        tmem_ld32(tl + 256 * b + TM_D2 + 32 * hf, d);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) dp[j] = f2_to_bf2(d[2 * j], d[2 * j + 1]);
      }
      tc_fence_before();
      if (tid == 0) bulk_wait_read();  // the previous chunk's store has read the staging tiles
      group_sync(BAR_STATE, NSTATE);
      if (tid == 0) mbar_arrive(bar(B_OREAD0 + b));  // O^T of the buffer is in registers: free
      uint8_t *ot = sm + OFF_OST + (v >> 6) * 8192;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        *reinterpret_cast<uint16_t *>(ot + sw128(32 * hf + j, v & 63)) = (uint16_t)(dp[j >> 1] >> (16 * (j & 1)));
      fence_proxy_async();
      group_sync(BAR_STATE, NSTATE);
      if (Cc == C) {
        if (tid == 0) {
          tma_store_3d(&tm_o, j0, h, tok0, sb + OFF_OST);
          if (j0 + 64 < a.dv) tma_store_3d(&tm_o, j0 + 64, h, tok0, sb + OFF_OST + 8192);
          bulk_commit();
        }
      } else if (rr < Cc && qin) {
        uint4 *dst = reinterpret_cast<uint4 *>(out + ((size_t)(tok0 + rr) * a.H + h) * (size_t)a.dv + j0 + 32 * qq);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = ld_s128(orow + sw128(rr, cq + 8 * x));
      }
      return true;
    };
    if (nk > 0) {
      put_state(0);
      tc_fence_before();
      group_sync(BAR_STATE, NSTATE);
      if (tid == 0) mbar_arrive(bar(B_SREADY));
    }
    for (int k = 0; k < nk; ++k) {
      const int s = k & 1, b = k & 1, ph = (k >> 1) & 1;
      // ---------------------------------------------------------- S <- Diag(e^{g_C}) S + D1
      if (!group_wait_spin(BAR_STATE, NSTATE, bar(B_D1FULL0 + b), ph)) { ok = false; break; }
      tc_fence_after();
      {
        const float4 *g1 = reinterpret_cast<const float4 *>(sm + OFF_G + s * REC_G) + 16 * hf;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          float d[32];
          tmem_ld32(tl + 256 * b + TM_D1 + 64 * hf + 32 * part, d);
          tmem_wait_ld();
#pragma unroll
          for (int y = 0; y < 8; ++y) {  // S = e^{g_C} S + D1, two channels per packed FMA
            const float4 g = g1[8 * part + y];
            const int i = 32 * part + 4 * y;
            const float2 lo = __ffma2_rn(make_float2(g.x, g.y), make_float2(S[i], S[i + 1]), make_float2(d[4 * y], d[4 * y + 1]));
            const float2 hi =
                __ffma2_rn(make_float2(g.z, g.w), make_float2(S[i + 2], S[i + 3]), make_float2(d[4 * y + 2], d[4 * y + 3]));
            S[i] = lo.x; S[i + 1] = lo.y; S[i + 2] = hi.x; S[i + 3] = hi.y;
          }
        }
      }
      // the next chunk's S^T goes into the other buffer (its last reader, O^T of chunk k-1, is complete)
      if (k + 1 < nk) put_state(b ^ 1);
      tc_fence_before();
      group_sync(BAR_STATE, NSTATE);
      if (tid == 0) {
        mbar_arrive(bar(B_D1FREE0 + b));
        if (k + 1 < nk) mbar_arrive(bar(B_SREADY));
      }
      if (use_o && !read_out(k)) { ok = false; break; }
    }
    if (tid == 0) bulk_wait_read();  // the last O store has read the staging tiles
    // ---------------------------------------------------------- the state after this CTA's chunks
    if (ok && vin) {
      float *dst = nullptr;
      size_t base = s_base;
      if (q.mode == 1) {
        const size_t js = nh * (q.nseg - 1) + seg;
        dst = ident ? q.sum_a : q.sum_b;
        base = (js * DK + 64 * hf) * (size_t)cols + j0 + v;
      } else if ((q.mode == 0 || seg == q.nseg - 1) && kin) {
        dst = a.ST;
      }
      if (dst) {
#pragma unroll
        for (int i = 0; i < 64; ++i) dst[base + (size_t)i * cols] = S[i];
      }
    }
  }
  if (!ok) atomicExch(p.status, 4);
  // the factorisation kernel has ended too, so the stream sees both complete.  One converged warp
  // that has finished its own work waits: the wait parks the whole warp, and the idle lanes of the
  // loader and issuer warps would otherwise reach it while their working lanes still run.
  if (warp == 0) griddep_wait();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Two-level scan, between the two state passes: chains the segment maps into entry states,
// E_0 = S0, E_1 = B_0 and E_{j+1} = A_j E_j + B_j (fp32), one CTA per (sequence, head, 128 value
// columns).  E_0 is copied too, so the final pass never reads S0 while its last segment writes S_T.
__global__ void __launch_bounds__(256) segment_chain_kernel(const ChunkArgs a, const ScanParams q) {
  extern __shared__ float csm[];
  float *E = csm;                 // [128][128 + 4] entry state, columns of this tile
  float *At = csm + 128 * 132;    // [32][128 + 4] a slab of A_j, transposed (k rows, i columns)
  const int tiles = (a.dv + 127) / 128;
  const int tile = blockIdx.x % tiles, h = (blockIdx.x / tiles) % a.H, n = blockIdx.x / (tiles * a.H);
  const int j0 = 128 * tile, tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const size_t nh = (size_t)n * a.H + h;
  const int cols = min(128, a.dv - j0);
  for (int e = tid; e < 128 * 128; e += 256) {  // E_0 = S0 (zeros without one)
    const int i = e >> 7, v = e & 127;
    if (v < cols)
      q.s_start[((nh * q.nseg) * DK + i) * (size_t)a.dv + j0 + v] =
          (a.S0 && i < a.dk) ? a.S0[(nh * a.dk + i) * (size_t)a.dv + j0 + v] : 0.f;
  }
  // E_1 = B_0
  for (int e = tid; e < 128 * 128; e += 256) {
    const int i = e >> 7, v = e & 127;
    E[i * 132 + v] = v < cols ? q.sum_b[(nh * (q.nseg - 1) * DK + i) * (size_t)a.dv + j0 + v] : 0.f;
  }
  __syncthreads();
  for (int j = 1; j < q.nseg; ++j) {
    // E_j -> s_start[j]
    for (int e = tid; e < 128 * 128; e += 256) {
      const int i = e >> 7, v = e & 127;
      if (v < cols) q.s_start[((nh * q.nseg + j) * DK + i) * (size_t)a.dv + j0 + v] = E[i * 132 + v];
    }
    if (j == q.nseg - 1) break;
    // E_{j+1} = A_j E_j + B_j: thread (ty, tx) owns rows 8 ty .. +7, columns 8 tx .. +7
    const float *A = q.sum_a + (nh * (q.nseg - 1) + j) * DK * DK;
    const float *Bj = q.sum_b + ((nh * (q.nseg - 1) + j) * DK) * (size_t)a.dv + j0;
    float acc[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[r][c] = (8 * tx + c < cols) ? Bj[(size_t)(8 * ty + r) * a.dv + 8 * tx + c] : 0.f;
    for (int k0 = 0; k0 < DK; k0 += 32) {
      __syncthreads();
      for (int e = tid; e < 32 * 128; e += 256) {  // At[kk][i] = A[i][k0 + kk]
        const int i = e >> 5, kk = e & 31;
        At[kk * 132 + i] = A[i * DK + k0 + kk];
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < 32; ++kk) {
        float av[8], ev[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) av[r] = At[kk * 132 + 8 * ty + r];
#pragma unroll
        for (int c = 0; c < 8; ++c) ev[c] = E[(k0 + kk) * 132 + 8 * tx + c];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(av[r], ev[c], acc[r][c]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) E[(8 * ty + r) * 132 + 8 * tx + c] = acc[r][c];
    __syncthreads();
  }
}

// Chunk offsets of a packed batch: coff[0] = 0, coff[n+1] = coff[n] + ceil(len_n / 64).  One CTA.
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int32_t *cu, int N, int32_t *coff) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry = 0;
    coff[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < N; base += 1024) {
    const int n = base + tid;
    int x = n < N ? (cu[n + 1] - cu[n] + C - 1) / C : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {  // inclusive scan inside the warp
      const int y = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, d);
        if (lane >= d) w += y;
      }
      warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int incl = carry + x + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (n < N) coff[n + 1] = incl;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
}

// ------------------------------------------------------------------ host side
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void *q = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(q);
  }
  return fn;
}

// [tokens, H, D] bf16 token tensor, box = 64 channels x 1 head x 64 tokens, 128-byte swizzle
bool map_tokens(CUtensorMap *m, const void *base, long long tokens, int H, int D) {
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

// [rows, cols] bf16 workspace matrix, box = 64 columns x box_rows rows, 128-byte swizzle
bool map_matrix(CUtensorMap *m, void *base, long long rows, int cols, int box_rows) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Upper bound of the number of chunks of a batch: sum ceil(len_n / 64) <= floor((T + 63 N) / 64).
long long chunk_capacity(int B, int T, bool packed) {
  if (!packed) return (long long)B * ((T + C - 1) / C);
  return ((long long)T + (long long)(C - 1) * B) / C;
}

// SMs of the current device (148 on B200 if the query fails).
int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0)
    sms = 148;
  return sms;
}

// Segments per sequence of the two-level state scan (1: one walk per sequence).  It pays only when
// the (sequence, head, value tile) walks cannot fill the GPU: then the walk is cut into segments of
// at least 16 chunks, as many as let the summary pass run in one wave.
int scan_segments(int B, int T, int H, int dv, bool packed, int sms, int *seg_len) {
  *seg_len = 0;
  if (packed) return 1;
  const int nch = (T + C - 1) / C, tiles = (dv + 127) / 128;
  const long long walks = (long long)B * H * tiles;
  if (walks * 4 > sms) return 1;
  int nseg = 1 + (int)(sms / ((long long)B * H * (1 + tiles)));
  nseg = min(nseg, nch / 16);
  if (nseg < 2) return 1;
  const int len = (nch + nseg - 1) / nseg;
  *seg_len = len;
  return (nch + len - 1) / len;
}

// Workspace layout: Mt tiles | Nt tiles | Qt tiles | Pt tiles | e^{g_C} | two-level scan maps and entry
// states (long sequences only) | chunk offsets (packed only) | record counter (256 bytes) and one ready
// flag per record (int32), zeroed together before each call; 256-byte aligned arrays
struct WsLayout {
  long long records;
  int nseg, seg_len;
  size_t m, n, q, p, g, sa, sbm, ss, coff, cnt, total;
};
size_t up256(size_t x) { return (x + 255) / 256 * 256; }
WsLayout ws_layout(int B, int T, int H, int dv, bool packed, int sms) {
  WsLayout L{};
  L.records = chunk_capacity(B, T, packed) * H;
  L.nseg = scan_segments(B, T, H, dv, packed, sms, &L.seg_len);
  const size_t r = (size_t)L.records;
  const size_t pairs = (size_t)B * H, ns = L.nseg > 1 ? (size_t)L.nseg : 0;
  L.m = 0;
  L.n = L.m + r * REC_M;
  L.q = L.n + r * REC_N;
  L.p = L.q + r * REC_Q;
  L.g = L.p + r * REC_P;
  L.sa = up256(L.g + r * REC_G);
  L.sbm = up256(L.sa + (ns ? pairs * (ns - 1) * DK * DK * 4 : 0));
  L.ss = up256(L.sbm + (ns ? pairs * (ns - 1) * DK * dv * 4 : 0));
  L.coff = up256(L.ss + pairs * ns * DK * dv * 4);
  L.cnt = L.coff + (packed ? up256((size_t)(B + 1) * 4) : 0);
  L.total = L.cnt + up256(256 + r * 4);
  return L;
}

// Where the factorisation hands SMs to a state pass of `walks` CTAs (one per SM) before it ends.  Run
// beside the factorisation, the state pass takes about 1.9 us per chunk, and a factorisation CTA
// about 9 us per record (two per SM; measured on B200, 1.3B layer).  The CTAs on `walks` SMs stop
// claiming once `stop_at` records are claimed, chosen so that the other SMs factor the remaining
// records in about the state pass's time: the two then end together.  Returns -1 (no SM handed over)
// when the walks do not leave room.
int handover_stop(long long records, long long walks, int nc, int sms) {
  if (walks <= 0 || walks > sms - 16) return -1;
  const double rest = 2.0 * (double)(sms - walks) * (double)nc * 1.9 / 9.0;
  const long long stop = records - (long long)rest;
  return stop > 0 ? (int)stop : 0;
}

// Everything a call decides before it launches: the workspace layout, the grids, the walking order
// and the SM hand-over.
struct Plan {
  WsLayout L;
  bool wy_runs;        // a token and a record exist
  long long wy_ctas;   // persistent WY CTAs (two per SM)
  long long sp_ctas;   // CTAs of the first state-pass launch
  long long walks;     // (sequence, head, 128-column) walks
  int order, reserve, stop_at, publish;
  int launches;
};
Plan make_plan(int B, int T, int H, int dv, bool packed, int sms) {
  Plan P{};
  P.L = ws_layout(B, T, H, dv, packed, sms);
  const long long tokens = packed ? (long long)T : (long long)B * T;
  const long long tiles = (dv + sp::VW - 1) / sp::VW;
  P.wy_runs = P.L.records > 0 && tokens > 0;
  P.wy_ctas = P.wy_runs ? std::min<long long>(P.L.records, 2LL * sms) : 0;
  P.walks = (long long)B * H * tiles;
  P.order = packed ? 0 : 1;
  P.reserve = 0;
  P.stop_at = (int)P.L.records;
  P.publish = 0;
  if (!packed && P.L.nseg <= 1) {  // whole-sequence walks that leave SMs free: hand SMs over early
    const int stop = handover_stop(P.L.records, P.walks, (T + C - 1) / C, sms);
    if (stop >= 0) {
      P.order = 2;
      P.publish = 1;
      P.reserve = (int)P.walks;
      P.stop_at = stop;
    }
  }
  P.sp_ctas = P.L.nseg <= 1 ? P.walks : (long long)B * H * (P.L.nseg - 1) * (1 + tiles);
  P.launches = (packed ? 1 : 0) + (P.wy_runs ? 1 : 0) + (P.L.nseg <= 1 ? 1 : 3);
  return P;
}

}  // namespace

bool chunk_wy_supported(int B, int T, int H, int dk, int dv, bool packed, bool bf16) {
  if (!bf16 || (dk != 64 && dk != DK) || dv % NV != 0) return false;
  // TMA coordinates are int32: token rows (plus one chunk) and workspace rows (records x 128)
  const long long tokens = packed ? (long long)T : (long long)B * T;
  return tokens + C <= (long long)INT_MAX && chunk_capacity(B, T, packed) * H * 128 <= (long long)INT_MAX;
}

size_t chunk_wy_workspace_bytes(int B, int T, int H, int dv, bool packed) {
  return ws_layout(B, T, H, dv, packed, device_sms()).total;
}

ChunkWyPlan chunk_wy_plan(int B, int T, int H, int dv, bool packed, int sms) {
  const Plan P = make_plan(B, T, H, dv, packed, sms > 0 ? sms : device_sms());
  ChunkWyPlan r{};
  r.records = P.L.records;
  r.wy_ctas = P.wy_ctas;
  r.state_ctas = P.sp_ctas;
  r.segments = P.L.nseg;
  r.segment_chunks = P.L.nseg > 1 ? P.L.seg_len : 0;
  r.handover_sms = P.reserve;
  r.handover_at = P.reserve > 0 ? P.stop_at : P.L.records;
  r.order = P.order;
  r.launches = P.launches;
  r.workspace_bytes = P.L.total;
  return r;
}

cudaError_t launch_chunk_wy(const ChunkArgs &a, void *ws, cudaStream_t stream) {
  const long long tokens = a.cu ? (long long)a.T : (long long)a.B * a.T;
  const int sms = device_sms();
  const Plan P = make_plan(a.B, a.T, a.H, a.dv, a.cu != nullptr, sms);
  const WsLayout &L = P.L;
  uint8_t *base = static_cast<uint8_t *>(ws);
  WyParams p;
  cudaError_t err = device_status_word(&p.status);
  if (err != cudaSuccess) return err;
  p.N = a.B;
  p.nc = (a.T + C - 1) / C;
  p.tokens = tokens;
  p.coff = a.cu ? reinterpret_cast<const int32_t *>(base + L.coff) : nullptr;
  p.g = reinterpret_cast<float *>(base + L.g);
  p.nrec = (int)L.records;
  p.next = reinterpret_cast<int *>(base + L.cnt);
  p.ready = reinterpret_cast<int *>(base + L.cnt + 256);
  p.done = p.next + 1;
  p.ctas = (int)P.wy_ctas;
  p.publish = P.publish;
  p.sms = sms;
  p.reserve = P.reserve;
  p.stop_at = P.stop_at;
  p.order = P.order;
  const long long tiles = (a.dv + sp::VW - 1) / sp::VW;

  CUtensorMap mq, mk, mb, mal, mv, mw, mo, mm, mn, mqt, mp;
  if (tokens > 0) {
    // key-side maps have the caller's d_k channels: with d_k = 64 the second 64-channel box is
    // outside the tensor and arrives as zeros
    if (!map_tokens(&mq, a.q, tokens, a.H, a.dk) || !map_tokens(&mk, a.k, tokens, a.H, a.dk) ||
        !map_tokens(&mb, a.b, tokens, a.H, a.dk) || !map_tokens(&mal, a.alpha, tokens, a.H, a.dk) ||
        !map_tokens(&mv, a.v, tokens, a.H, a.dv) || !map_tokens(&mw, a.w, tokens, a.H, a.dv) ||
        !map_tokens(&mo, a.o, tokens, a.H, a.dv) ||
        !map_matrix(&mm, base + L.m, L.records * 128, 128, 128) ||
        !map_matrix(&mn, base + L.n, L.records * 128, 64, 128) ||
        !map_matrix(&mqt, base + L.q, L.records * 64, 128, 64) ||
        !map_matrix(&mp, base + L.p, L.records * 64, 64, 64))
      return cudaErrorInvalidValue;
  } else {
    // no token and no record: the state pass only copies S0 to S_T; its maps are never read
    memset(&mv, 0, sizeof(mv));
    mw = mo = mm = mn = mqt = mp = mv;
  }
  if (a.cu) {
    note_launch();
    chunk_offsets_kernel<<<1, 1024, 0, stream>>>(a.cu, a.B, const_cast<int32_t *>(p.coff));
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  const bool wy_runs = P.wy_runs;
  if (wy_runs) {
    if ((err = cudaMemsetAsync(p.next, 0, 256 + (size_t)L.records * 4, stream)) != cudaSuccess) return err;
    err = cudaFuncSetAttribute(wy_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wy::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    note_launch();
    wy_factor_kernel<<<(unsigned)P.wy_ctas, wy::NT, wy::SMEM_BYTES, stream>>>(a, p, mq, mk, mb, mal, mm, mn, mqt, mp);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  err = cudaFuncSetAttribute(state_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  // The state pass right after the factorisation is a programmatic dependent launch: its CTAs are
  // scheduled onto SMs as the factorisation leaves them, and it waits on each record's flag.
  auto state_pass = [&](long long grid, const ScanParams &sq, bool dependent) -> cudaError_t {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(sp::NT);
    cfg.dynamicSmemBytes = sp::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    note_launch();
    return cudaLaunchKernelEx(&cfg, state_pass_kernel, a, p, sq, mm, mn, mqt, mp, mv, mw, mo);
  };
  ScanParams q{};
  if (L.nseg <= 1)  // one walk per (sequence, head, value tile)
    return state_pass(P.sp_ctas, q, wy_runs);
  // two-level scan: segment maps, their chain into entry states, then the segments' walks
  q.seg_len = L.seg_len;
  q.nseg = L.nseg;
  q.sum_a = reinterpret_cast<float *>(base + L.sa);
  q.sum_b = reinterpret_cast<float *>(base + L.sbm);
  q.s_start = reinterpret_cast<float *>(base + L.ss);
  q.mode = 1;
  if ((err = state_pass(P.sp_ctas, q, wy_runs)) != cudaSuccess) return err;
  const int chain_smem = (128 * 132 + 32 * 132) * 4;
  err = cudaFuncSetAttribute(segment_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, chain_smem);
  if (err != cudaSuccess) return err;
  note_launch();
  segment_chain_kernel<<<(unsigned)(a.B * a.H * tiles), 256, chain_smem, stream>>>(a, q);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  q.mode = 2;
  return state_pass((long long)a.B * a.H * L.nseg * tiles, q, false);
}

}  // namespace gdn2
