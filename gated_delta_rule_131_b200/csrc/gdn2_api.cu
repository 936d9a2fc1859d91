// C ABI of the gdn2 library: argument validation, dispatch, status strings.
// See include/gdn2.h for the contract of every entry point.
#include <atomic>
#include <climits>
#include <mutex>

#include "common.cuh"
#include "gdn2.h"

namespace gdn2 {
static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace gdn2

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dk(int d) { return d == 64 || d == 128; }
bool supported_dv(int d) { return d == 64 || d == 128 || d == 256; }

// a*b*c*d fits in int64 with headroom (element counts of every tensor we index)
bool fits(long long a, long long b, long long c, long long d) {
  const long long lim = (1LL << 62);
  long long x = a;
  for (long long y : {b, c, d}) {
    if (y != 0 && x > lim / y) return false;
    x *= y;
  }
  return true;
}

// Stream-ordered pool of the chunk workspaces, one per device, owned by the library.  Its release
// threshold is unbounded, so memory freed back to it is kept for the next call instead of being
// unmapped at every synchronisation.
cudaError_t workspace_pool(cudaMemPool_t *pool) {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if ((err = cudaMemPoolCreate(&p, &props)) != cudaSuccess) return err;
    uint64_t threshold = UINT64_MAX;
    if ((err = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &threshold)) != cudaSuccess) {
      cudaMemPoolDestroy(p);
      return err;
    }
    pools[dev] = p;
  }
  *pool = pools[dev];
  return cudaSuccess;
}

// The tensor-core path with a workspace taken from the pool and returned to it on `stream`.
cudaError_t run_chunk_wy(const gdn2::ChunkArgs &a, cudaStream_t stream) {
  const size_t bytes = gdn2::chunk_wy_workspace_bytes(a.B, a.T, a.H, a.dv, a.cu != nullptr);
  void *ws = nullptr;
  cudaError_t err;
  if (bytes > 0) {
    cudaMemPool_t pool;
    if ((err = workspace_pool(&pool)) != cudaSuccess) return err;
    if ((err = cudaMallocFromPoolAsync(&ws, bytes, pool, stream)) != cudaSuccess) return err;
  }
  err = gdn2::launch_chunk_wy(a, ws, stream);
  if (ws) {
    const cudaError_t ferr = cudaFreeAsync(ws, stream);
    if (err == cudaSuccess) err = ferr;
  }
  return err;
}

// The backward with a workspace taken from the pool and returned to it on `stream`.
cudaError_t run_chunk_bwd(const gdn2::BwdArgs &a, bool bf16, cudaStream_t stream) {
  const size_t bytes = gdn2::chunk_bwd_workspace_bytes(a.B, a.T, a.H, a.Dk, a.Dv, a.cu != nullptr);
  cudaMemPool_t pool;
  void *ws = nullptr;
  cudaError_t err;
  if ((err = workspace_pool(&pool)) != cudaSuccess) return err;
  if ((err = cudaMallocFromPoolAsync(&ws, bytes, pool, stream)) != cudaSuccess) return err;
  err = gdn2::launch_chunk_bwd(a, bf16, ws, stream);
  const cudaError_t ferr = cudaFreeAsync(ws, stream);
  return err == cudaSuccess ? ferr : err;
}

// The fixed workspace of gdn2_chunk_fwd_noalloc: a file-scope device array, so that entry point
// allocates nothing.  Its device address is looked up once per device, with that device current.
constexpr size_t kNoallocBytes = (size_t)GDN2_NOALLOC_WORKSPACE_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_ws[kNoallocBytes];

cudaError_t noalloc_workspace(void **ptr) {
  static std::mutex mu;
  static void *addr[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *a = nullptr;
    if ((err = cudaGetSymbolAddress(&a, g_noalloc_ws)) != cudaSuccess) return err;
    addr[dev] = a;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

const char *gdn2_status_string(gdn2_status s) {
  switch (s) {
    case GDN2_OK: return "GDN2_OK";
    case GDN2_ERR_INVALID_ARG: return "GDN2_ERR_INVALID_ARG: null or misaligned pointer, or bad size";
    case GDN2_ERR_UNSUPPORTED: return "GDN2_ERR_UNSUPPORTED: head size, chunk size or dtype not implemented";
    case GDN2_ERR_CUDA: return "GDN2_ERR_CUDA: a CUDA launch failed";
    case GDN2_ERR_TIMEOUT: return "GDN2_ERR_TIMEOUT: a bounded device-side wait gave up";
  }
  return "GDN2 unknown status";
}

uint64_t gdn2_launch_count(void) { return gdn2::g_launches.load(std::memory_order_relaxed); }

gdn2_status gdn2_selftest_bounded_wait(int limit_us, gdn2_stream_t stream) {
  if (limit_us <= 0 || limit_us > 10000000) return GDN2_ERR_INVALID_ARG;
  const cudaError_t err = gdn2::launch_bounded_wait_probe((uint64_t)limit_us * 1000ull, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_device_status(int reset) {
  int st = 0;
  if (gdn2::read_device_status(&st, reset != 0) != cudaSuccess) return GDN2_ERR_CUDA;
  return st == 0 ? GDN2_OK : GDN2_ERR_TIMEOUT;
}

}  // extern "C"

namespace {

// Validation shared by the chunk entry points; on success fills `a` and `tc` (tensor-core path).
gdn2_status check_chunk(const void *q, const void *k, const void *v, const void *alpha, const void *b, const void *w,
                        const float *S0, void *o, float *S_T, int B, int T, int H, int d_k, int d_v, int chunk,
                        const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2::ChunkArgs *a, bool *tc) {
  if (B < 0 || T < 0 || H <= 0) return GDN2_ERR_INVALID_ARG;
  if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  // with no tokens at all the token tensors are empty and may be NULL
  const bool no_tokens = cu_seqlens ? (T == 0) : ((long long)B * T == 0);
  if (!no_tokens && (!q || !k || !v || !alpha || !b || !w || !o)) return GDN2_ERR_INVALID_ARG;
  for (const void *p : {q, k, v, alpha, b, w, (const void *)o})
    if (p && !aligned16(p)) return GDN2_ERR_INVALID_ARG;
  if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T))) return GDN2_ERR_INVALID_ARG;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN2_ERR_INVALID_ARG;
  if (!supported_dk(d_k) || !supported_dv(d_v) || chunk != 64) return GDN2_ERR_UNSUPPORTED;
  const long long tokens = cu_seqlens ? (long long)T : (long long)B * T;
  if (!fits(tokens, H, d_v > d_k ? d_v : d_k, 1) || !fits(B, H, d_k, d_v)) return GDN2_ERR_INVALID_ARG;
  if ((long long)B * H * 8 > INT_MAX) return GDN2_ERR_INVALID_ARG;
  *a = gdn2::ChunkArgs{q, k, v, alpha, b, w, S0, o, S_T, cu_seqlens, B, T, H, d_k, d_v};
  // bf16 runs on the tensor cores (unless too large for their 32-bit TMA coordinates); fp32, whose
  // accuracy bf16 operands cannot keep, runs the SIMT kernel
  *tc = gdn2::chunk_wy_supported(B, T, H, d_k, d_v, cu_seqlens != nullptr, dtype == GDN2_BF16);
  return GDN2_OK;
}

}  // namespace

extern "C" {

gdn2_status gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *alpha,
                           const void *b, const void *w, const float *S0, void *o, float *S_T,
                           int B, int T, int H, int d_k, int d_v, int chunk,
                           const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream) {
  gdn2::ChunkArgs a;
  bool tc = false;
  const gdn2_status st = check_chunk(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, d_k, d_v, chunk, cu_seqlens, dtype, &a, &tc);
  if (st != GDN2_OK || B == 0) return st;
  const cudaError_t err = tc ? run_chunk_wy(a, (cudaStream_t)stream)
                             : gdn2::launch_chunk_simt(a, dtype == GDN2_BF16, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *alpha,
                                   const void *b, const void *w, const float *S0, void *o, float *S_T,
                                   int B, int T, int H, int d_k, int d_v, int chunk,
                                   const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream) {
  gdn2::ChunkArgs a;
  bool tc = false;
  const gdn2_status st = check_chunk(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, d_k, d_v, chunk, cu_seqlens, dtype, &a, &tc);
  if (st != GDN2_OK || B == 0) return st;
  if (!tc) {  // the SIMT kernel needs no workspace
    const cudaError_t err = gdn2::launch_chunk_simt(a, dtype == GDN2_BF16, (cudaStream_t)stream);
    return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
  }
  // checked on the host before any launch or allocation: the shape must fit the fixed workspace (its size
  // depends on the current device's SM count, which chunk_wy_workspace_bytes queries)
  if (gdn2::chunk_wy_workspace_bytes(B, T, H, d_v, cu_seqlens != nullptr) > kNoallocBytes) return GDN2_ERR_UNSUPPORTED;
  // nothing in the workspace has to start at zero: the chunk offsets and every record are written
  // by this call's kernels before they are read
  void *ws = nullptr;
  cudaError_t err = noalloc_workspace(&ws);
  if (err == cudaSuccess) err = gdn2::launch_chunk_wy(a, ws, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_chunk_bwd(const void *q, const void *k, const void *v, const void *alpha, const void *b,
                           const void *w, const float *S0, const void *dO, const float *dS_T, void *dq, void *dk,
                           void *dv, void *dalpha, void *db, void *dw, float *dS0, int B, int T, int H, int d_k,
                           int d_v, const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream) {
  if (B < 0 || T < 0 || H <= 0) return GDN2_ERR_INVALID_ARG;
  if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  if (!supported_dk(d_k) || !supported_dv(d_v)) return GDN2_ERR_UNSUPPORTED;
  const long long tokens = cu_seqlens ? (long long)T : (long long)B * T;
  if (!fits(tokens, H, 4 * (d_v > d_k ? d_v : d_k), 1) || !fits(B, H, d_k, d_v)) return GDN2_ERR_INVALID_ARG;
  if (!fits(tokens / 8 + B + 1, H, d_k, d_v) || (long long)B * H > INT_MAX / 64) return GDN2_ERR_INVALID_ARG;
  if (tokens > 0)
    for (const void *p : {q, k, v, alpha, b, w, dO, (const void *)dq, (const void *)dk, (const void *)dv,
                          (const void *)dalpha, (const void *)db, (const void *)dw})
      if (!p || !aligned16(p)) return GDN2_ERR_INVALID_ARG;
  for (const void *p : {(const void *)S0, (const void *)dS_T, (const void *)dS0})
    if (p && !aligned16(p)) return GDN2_ERR_INVALID_ARG;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN2_ERR_INVALID_ARG;
  if (B == 0) return GDN2_OK;
  const gdn2::BwdArgs a{q, k, v, alpha, b, w, dO, S0, dS_T, dq, dk, dv, dalpha, db, dw, dS0, cu_seqlens,
                        B, T, H, d_k, d_v};
  const cudaError_t err = run_chunk_bwd(a, dtype == GDN2_BF16, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_recurrent_fwd(const void *q, const void *k, const void *v, const void *alpha, const void *b,
                               const void *w, const float *S0, void *o, float *S_T, int B, int T, int H, int d_k,
                               int d_v, const int32_t *cu_seqlens, gdn2_erase erase, gdn2_dtype dtype,
                               gdn2_stream_t stream) {
  if (erase != GDN2_ERASE_R1 && erase != GDN2_ERASE_R2) return GDN2_ERR_INVALID_ARG;
  gdn2::ChunkArgs c;
  bool tc = false;
  // the same arguments, layouts and checks as gdn2_chunk_fwd (chunk length 64 stands in: it is unused)
  const gdn2_status st = check_chunk(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, d_k, d_v, 64, cu_seqlens, dtype, &c, &tc);
  if (st != GDN2_OK || B == 0) return st;
  const gdn2::RecurrentArgs a{q, k, v, alpha, b, w, S0, o, S_T, cu_seqlens, B, T, H, d_k, d_v};
  const cudaError_t err = gdn2::launch_recurrent(a, dtype == GDN2_BF16, erase == GDN2_ERASE_R2, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

size_t gdn2_chunk_bwd_workspace_bytes(int B, int T, int H, int d_k, int d_v, int packed) {
  if (B <= 0 || T < 0 || H <= 0 || !supported_dk(d_k) || !supported_dv(d_v)) return 0;
  return gdn2::chunk_bwd_workspace_bytes(B, T, H, d_k, d_v, packed != 0);
}

gdn2_status gdn2_chunk_fwd_plan(int B, int T, int H, int d_k, int d_v, int chunk, int packed, gdn2_dtype dtype,
                                int sms, gdn2_chunk_plan *plan) {
  if (!plan || B < 0 || T < 0 || H <= 0 || sms < 0) return GDN2_ERR_INVALID_ARG;
  if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  if (!supported_dk(d_k) || !supported_dv(d_v) || chunk != 64) return GDN2_ERR_UNSUPPORTED;
  if (!gdn2::chunk_wy_supported(B, T, H, d_k, d_v, packed != 0, dtype == GDN2_BF16)) return GDN2_ERR_UNSUPPORTED;
  const gdn2::ChunkWyPlan r = gdn2::chunk_wy_plan(B, T, H, d_v, packed != 0, sms);
  plan->records = r.records;
  plan->wy_ctas = r.wy_ctas;
  plan->state_ctas = r.state_ctas;
  plan->segments = r.segments;
  plan->segment_chunks = r.segment_chunks;
  plan->handover_sms = r.handover_sms;
  plan->handover_at = r.handover_at;
  plan->order = r.order;
  plan->launches = r.launches;
  plan->workspace_bytes = r.workspace_bytes;
  return GDN2_OK;
}

size_t gdn2_chunk_fwd_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk, int packed,
                                      gdn2_dtype dtype) {
  if (B <= 0 || T < 0 || H <= 0 || chunk != 64 || !supported_dk(d_k) || !supported_dv(d_v)) return 0;
  if (dtype != GDN2_F32 && dtype != GDN2_BF16) return 0;
  if (!gdn2::chunk_wy_supported(B, T, H, d_k, d_v, packed != 0, dtype == GDN2_BF16)) return 0;
  return gdn2::chunk_wy_workspace_bytes(B, T, H, d_v, packed != 0);
}

gdn2_status gdn2_block_prologue(const void *x_q, const void *x_k, const void *x_v, const void *x_alpha,
                                const void *x_b, const void *x_w, const float *conv_q, const float *conv_k,
                                const float *conv_v, void *q, void *k, void *v, void *alpha, void *b, void *w,
                                int B, int T, int H, int d_k, int d_v, int conv_len, const int32_t *cu_seqlens,
                                gdn2_dtype dtype, gdn2_stream_t stream) {
  if (B < 0 || T < 0 || H <= 0) return GDN2_ERR_INVALID_ARG;
  if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  if (!supported_dk(d_k) || !supported_dv(d_v) || conv_len < 1 || conv_len > 4) return GDN2_ERR_UNSUPPORTED;
  const long long tokens = cu_seqlens ? (long long)T : (long long)B * T;
  if (!fits(tokens, H, d_v > d_k ? d_v : d_k, 1)) return GDN2_ERR_INVALID_ARG;
  if (!conv_q || !conv_k || !conv_v) return GDN2_ERR_INVALID_ARG;
  for (const float *p : {conv_q, conv_k, conv_v})
    if (reinterpret_cast<uintptr_t>(p) & 3u) return GDN2_ERR_INVALID_ARG;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN2_ERR_INVALID_ARG;
  if (tokens > 0) {
    for (const void *p : {x_q, x_k, x_v, x_alpha, x_b, x_w, (const void *)q, (const void *)k, (const void *)v,
                          (const void *)alpha, (const void *)b, (const void *)w})
      if (!p || !aligned16(p)) return GDN2_ERR_INVALID_ARG;
  }
  if (B == 0 || tokens == 0) return GDN2_OK;
  gdn2::BlockPrologueArgs a{x_q, x_k, x_v, x_alpha, x_b, x_w, conv_q, conv_k, conv_v, q, k, v, alpha, b, w,
                            cu_seqlens, B, T, H, d_k, d_v, conv_len, tokens};
  const cudaError_t err = gdn2::launch_block_prologue(a, dtype == GDN2_BF16, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_block_epilogue(const void *o, const void *gate, const float *norm_weight, void *y, long long tokens,
                                int H, int d_v, gdn2_dtype dtype, gdn2_stream_t stream) {
  if (tokens < 0 || H <= 0) return GDN2_ERR_INVALID_ARG;
  if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  if (!supported_dv(d_v)) return GDN2_ERR_UNSUPPORTED;
  if (!fits(tokens, H, d_v, 1)) return GDN2_ERR_INVALID_ARG;
  if (!norm_weight || (reinterpret_cast<uintptr_t>(norm_weight) & 3u)) return GDN2_ERR_INVALID_ARG;
  if (tokens > 0)
    for (const void *p : {o, gate, (const void *)y})
      if (!p || !aligned16(p)) return GDN2_ERR_INVALID_ARG;
  if (tokens == 0) return GDN2_OK;
  gdn2::BlockEpilogueArgs a{o, gate, norm_weight, y, tokens, H, d_v};
  const cudaError_t err = gdn2::launch_block_epilogue(a, dtype == GDN2_BF16, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_decode_step(const void *q, const void *k, const void *v, const void *alpha,
                             const void *b, const void *w, float *S, void *o, int B, int H,
                             int d_k, int d_v, gdn2_dtype dtype, gdn2_stream_t stream) {
  if (B < 0 || H <= 0) return GDN2_ERR_INVALID_ARG;
  if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  if (!q || !k || !v || !alpha || !b || !w || !S || !o) return GDN2_ERR_INVALID_ARG;
  for (const void *p : {q, k, v, alpha, b, w, (const void *)S, (const void *)o})
    if (!aligned16(p)) return GDN2_ERR_INVALID_ARG;
  if (!supported_dk(d_k) || !supported_dv(d_v)) return GDN2_ERR_UNSUPPORTED;
  if (!fits(B, H, d_k, d_v) || (long long)B * H * 4 > INT_MAX) return GDN2_ERR_INVALID_ARG;
  if (B == 0) return GDN2_OK;

  gdn2::DecodeArgs a{q, k, v, alpha, b, w, S, o, B, H, d_k, d_v};
  const cudaError_t err = gdn2::launch_decode(a, dtype == GDN2_BF16, (cudaStream_t)stream);
  return err == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

}  // extern "C"
