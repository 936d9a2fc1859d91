// C ABI of the gdn2 library: argument validation, dispatch, status strings.
// See include/gdn2.h for the contract of every entry point.
#include <atomic>
#include <climits>

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

gdn2_status gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *alpha,
                           const void *b, const void *w, const float *S0, void *o, float *S_T,
                           int B, int T, int H, int d_k, int d_v, int chunk,
                           const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream) {
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
  if (B == 0) return GDN2_OK;

  gdn2::ChunkArgs a{q, k, v, alpha, b, w, S0, o, S_T, cu_seqlens, B, T, H, d_k, d_v};
  const bool bf16 = dtype == GDN2_BF16;
  // bf16 with d_k = 128 runs on the tensor cores; fp32 (whose accuracy bf16 operands cannot
  // keep) and d_k = 64 run the SIMT kernel
  const cudaError_t err = gdn2::chunk_tc_supported(a, bf16) ? gdn2::launch_chunk_tc(a, (cudaStream_t)stream)
                                                            : gdn2::launch_chunk_simt(a, bf16, (cudaStream_t)stream);
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
