/*
 * gdn2.h -- C ABI of the Gated Delta Rule-2 kernels for NVIDIA B200 (sm_100a).
 *
 * The operation (for one sequence and one head; state S is d_k x d_v, row =
 * key channel, column = value channel; a_t = b_t (.) k_t, u_t = w_t (.) v_t):
 *
 *     S_t = Diag(alpha_t) S_{t-1}                         decay on the key axis, first
 *         + k_t ( u_t - (Diag(alpha_t) S_{t-1})^T a_t )^T erase gated per key channel by b_t,
 *                                                         write gated per value channel by w_t
 *     o_t = S_t^T q_t                                     readout of the edited state
 *
 * Defined by the pages on "Gated DeltaNet-2: Decoupling Erase and Write in
 * Linear Attention" (arXiv 2605.22791):
 *   - "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section
 *     "Gated DeltaNet-2の核心": b_t per key channel, w_t per value channel,
 *     both sigmoid projections, decay before the active edit; KDA is the case
 *     b_t = w_t = one scalar, Gated DeltaNet additionally a scalar decay;
 *   - "[논문] 게이트형 DeltaNet-2" (euno.news), section "방법론", steps 1-4:
 *     linear-attention read, the two gates, KDA-style per-channel decay,
 *     chunkwise WY update for parallel training;
 *   - "Gated DeltaNet-2: Separando Borrado y Escritura en la Atención Lineal"
 *     (needhelp.icu), "Innovaciones Técnicas", item 1: the chunkwise algorithm
 *     folds the per-channel decay into asymmetric erase factors.
 * The pages print no equation; the erase is read as k_t (b_t (.) k_t)^T, the
 * readout as S_t^T q_t with no 1/sqrt(d_k) scale.
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, densely packed row-major.  The library keeps no per-call state
 *     between calls.  gdn2_chunk_fwd on its tensor-core path (bf16, d_k = 128)
 *     takes a workspace of gdn2_chunk_fwd_workspace_bytes() bytes from a
 *     stream-ordered memory pool that the library creates once per device, and
 *     gives it back on `stream` after its kernels; the pool keeps memory given
 *     back to it for later calls until the process exits.  gdn2_chunk_bwd takes
 *     its workspace from the same pool.  No other call allocates device memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise.  A validation failure returns before any
 *     launch and writes nothing.  A launch failure returns GDN2_ERR_CUDA.  No
 *     C++ exception crosses this interface.
 *   - q, k, v, alpha, b, w and o share one element type `dtype` (fp32 or bf16);
 *     states are always fp32.  alpha holds decay values in (0, 1] (the log is
 *     never taken by the caller); b and w hold gate values (already sigmoid-ed);
 *     q and k are used as given (the token mixer normalises them before).
 *   - Supported head sizes: d_k in {64, 128}, d_v in {64, 128, 256}; anything
 *     else returns GDN2_ERR_UNSUPPORTED.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN2_API __attribute__((visibility("default")))
#else
#define GDN2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN2_OK = 0,
  GDN2_ERR_INVALID_ARG = 1, /* null / misaligned pointer, negative or overflowing size */
  GDN2_ERR_UNSUPPORTED = 2, /* valid but not implemented: head size, chunk size, dtype */
  GDN2_ERR_CUDA = 3,        /* a CUDA launch or attribute call failed                 */
  GDN2_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (see gdn2_device_status) */
} gdn2_status;

typedef enum { GDN2_F32 = 0, GDN2_BF16 = 1 } gdn2_dtype;

/* Same type as cudaStream_t, declared here so the header needs no CUDA include. */
typedef struct CUstream_st *gdn2_stream_t;

/*
 * gdn2_chunk_fwd -- chunkwise parallel forward (prefill / training forward).
 *
 * Computes o_t for every token and the final state of every sequence, using
 * the chunkwise WY form: inside a chunk of `chunk` tokens the per-channel decay
 * is folded into the erase factors and the chunk's erase interactions form one
 * unit-lower-triangular system; the state is carried across chunks in fp32.
 * The result equals the token-by-token recurrence up to rounding.
 *
 * Layout, dense batch (cu_seqlens == NULL): B sequences of T tokens each;
 *   q, k, alpha, b : [B, T, H, d_k]     v, w, o : [B, T, H, d_v]
 * Layout, packed varlen (cu_seqlens != NULL): B sequences packed end to end,
 *   T = total tokens = cu_seqlens[B]; cu_seqlens is a DEVICE int32 array of
 *   B+1 non-decreasing offsets starting at 0 (not read on the host; a
 *   violation of this precondition is undefined);
 *   q, k, alpha, b : [T, H, d_k]        v, w, o : [T, H, d_v]
 * States: S0, S_T : [B, H, d_k, d_v] fp32 (d_v contiguous).
 *   S0 == NULL means a zero initial state; S_T == NULL skips the final state;
 *   S_T may alias S0 (the state is read before it is overwritten).
 * chunk: 64 (the only supported chunk length).
 * T == 0 (or an empty sequence) is valid: its S_T equals its S0; when the
 * batch holds no token at all, the token pointers (q .. w, o) may be NULL.
 * bf16 (d_k = 64 or 128, d_v = 64, 128 or 256) runs two tensor-core kernels over a workspace: the
 * first forms the chunk's WY factors (T = (I + L)^-1, W = -T A, and the decay-
 * absorbed q and k) for every chunk at once, the second carries the state
 * through each sequence's chunks in order (d_k = 64 is carried as 128 key
 * channels whose upper half stays zero, d_v = 64 as a 128-column tile whose
 * upper half stays zero); fp32 runs one SIMT kernel without a workspace (bf16
 * tensor-core operands cannot keep the fp32 tolerance), as do bf16 shapes too
 * large for the kernels' 32-bit TMA coordinates.
 * Returns GDN2_OK, or an error status with nothing launched; GDN2_ERR_CUDA
 * also when the workspace cannot be allocated.
 */
GDN2_API gdn2_status gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *alpha,
                           const void *b, const void *w, const float *S0, void *o, float *S_T,
                           int B, int T, int H, int d_k, int d_v, int chunk,
                           const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_chunk_fwd_noalloc -- gdn2_chunk_fwd without any device allocation.
 *
 * It has no counterpart in the pages.  Same arguments, layouts, results and validation as
 * gdn2_chunk_fwd.  It serves callers that cannot call cudaMalloc or a stream-ordered allocator
 * once they run: a serving process that reserves all of its device memory at start-up and must not
 * grow it, or a host program that embeds this library under a memory manager of its own that owns
 * every allocation on the device.  Instead of the pooled workspace it uses one fixed device array
 * of GDN2_NOALLOC_WORKSPACE_BYTES bytes compiled into the library; every GPU that loads the library
 * holds that array until the process exits.
 *   - Set-up: the first call on a device, with that device current, looks the array's device
 *     address up (cudaGetSymbolAddress) and keeps it; make that first call before any stream
 *     capture.  Later calls on the device reuse the address.
 *   - Limit: a tensor-core call (bf16) whose workspace, gdn2_chunk_fwd_workspace_bytes()
 *     for this shape on the current device, exceeds the array returns GDN2_ERR_UNSUPPORTED before
 *     any launch or allocation.  That size depends on the device's SM count (the number of segments
 *     of the two-level state scan), so a shape near the limit may fit on one device and not on
 *     another.  Calls that run the SIMT kernel need no workspace and are not limited.
 *   - Sharing: every call uses the same array, which keeps what the previous call left in it; the
 *     kernels write every word they read first, so nothing from an earlier call leaks into a
 *     result.  Calls that overlap in time on one device (different streams, or different host
 *     threads) race on the array and must not be issued; calls on one stream are ordered and safe.
 */
#define GDN2_NOALLOC_WORKSPACE_BYTES (64u << 20) /* 64 MiB */
GDN2_API gdn2_status gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *alpha,
                                   const void *b, const void *w, const float *S0, void *o, float *S_T,
                                   int B, int T, int H, int d_k, int d_v, int chunk,
                                   const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_chunk_fwd_workspace_bytes -- device bytes gdn2_chunk_fwd takes from its pool for a call
 * of this shape (packed != 0: a packed batch with cu_seqlens, B sequences, T tokens in total).
 * 0 when the call runs without a workspace or the shape is not supported.  Host only.
 */
GDN2_API size_t gdn2_chunk_fwd_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk, int packed,
                                               gdn2_dtype dtype);

/*
 * gdn2_chunk_plan / gdn2_chunk_fwd_plan -- what a tensor-core gdn2_chunk_fwd call of this shape
 * decides before it launches, for a device of `sms` SMs (0: the current device, which is then
 * queried; no other CUDA call is made and nothing is launched or allocated).  It has no
 * counterpart in the pages: it describes how this library schedules the chunkwise form.
 *   records          (chunk, head) records the WY kernel writes (a packed batch: its chunk
 *                    capacity, sum over sequences of ceil(len / 64) at most, times H)
 *   wy_ctas          persistent WY-kernel CTAs (two per SM, at most one per record)
 *   state_ctas       CTAs of the first state-pass launch
 *   segments         segments per (sequence, head, 128-column) walk of the two-level scan, 1 for
 *                    whole-sequence walks; segment_chunks their length in chunks (0 when 1)
 *   handover_sms     SMs whose WY CTAs stop claiming records early so that the state pass runs
 *                    there alongside the rest of the factorisation (0: none)
 *   handover_at      records claimed before they stop (records when handover_sms is 0)
 *   order            the WY kernel's walking order: 0 record order (packed batches), 1 chunk-major
 *                    with the last chunk first, 2 chunk-major with the first chunk first
 *   launches         kernel launches of the call
 *   workspace_bytes  as gdn2_chunk_fwd_workspace_bytes() for that SM count
 * Returns GDN2_OK; GDN2_ERR_INVALID_ARG for a NULL plan or a negative size; GDN2_ERR_UNSUPPORTED
 * when the shape does not take the tensor-core path (fp32, or sizes outside it).
 */
typedef struct gdn2_chunk_plan {
  long long records, wy_ctas, state_ctas;
  int segments, segment_chunks, handover_sms;
  long long handover_at;
  int order, launches;
  size_t workspace_bytes;
} gdn2_chunk_plan;
GDN2_API gdn2_status gdn2_chunk_fwd_plan(int B, int T, int H, int d_k, int d_v, int chunk, int packed,
                                         gdn2_dtype dtype, int sms, gdn2_chunk_plan *plan);

/*
 * gdn2_recurrent_fwd -- the token-by-token recurrence over whole sequences, in either reading of
 * the erase orientation.
 *
 * The pages state the erase in words only: b_t gates the erase per key channel ("NVIDIA AIが
 * Gated DeltaNet-2を発表", ai.warp-studio.com, "Gated DeltaNet-2の核心"; "[논문] 게이트형 DeltaNet-2",
 * euno.news, "방법론", step 2), which leaves open on which side of the rank-1 erase the gate sits:
 *   GDN2_ERASE_R1:  S_t = (I - k_t (b_t (.) k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t (.) v_t)^T
 *                   (the reading every other call of this library computes)
 *   GDN2_ERASE_R2:  S_t = (I - (b_t (.) k_t) k_t^T) Diag(alpha_t) S_{t-1} + k_t (w_t (.) v_t)^T
 * and o_t = S_t^T q_t in both.  Both reduce to KDA when b_t = w_t = one scalar and to Gated
 * DeltaNet when alpha_t is a scalar as well.
 *
 * Arguments, layouts (dense or packed with cu_seqlens), aliasing, supported head sizes and errors
 * are those of gdn2_chunk_fwd (without `chunk`); erase is GDN2_ERASE_R1 or GDN2_ERASE_R2, anything
 * else is GDN2_ERR_INVALID_ARG.  fp32 arithmetic and state; o is rounded to dtype once.  It walks
 * the tokens of each sequence in order in one kernel (one CTA per sequence, head and 64 value
 * columns), so it costs time linear in the longest sequence; it allocates nothing.
 */
typedef enum { GDN2_ERASE_R1 = 0, GDN2_ERASE_R2 = 1 } gdn2_erase;
GDN2_API gdn2_status gdn2_recurrent_fwd(const void *q, const void *k, const void *v, const void *alpha,
                                        const void *b, const void *w, const float *S0, void *o, float *S_T,
                                        int B, int T, int H, int d_k, int d_v, const int32_t *cu_seqlens,
                                        gdn2_erase erase, gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_chunk_bwd -- gradients of a loss L through gdn2_chunk_fwd (erase reading R1).
 *
 * Passage: the recurrence of "[논문] 게이트형 DeltaNet-2" (euno.news), section "방법론",
 * and "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section
 * "Gated DeltaNet-2の核心"; the pages name a gate-aware backward of the chunked
 * form as a contribution but print no formula, so this is the chain rule taken
 * backwards through the token loop that gdn2_chunk_fwd computes:
 *     G += q_t dO_t^T,  dq_t = S_t dO_t,  dd = G^T k_t,  dk_t = G d_t + da (.) b_t,
 *     dv_t = dd (.) w_t,  dw_t = dd (.) v_t,  da = -(Diag(alpha_t) S_{t-1}) dd,
 *     db_t = da (.) k_t,  dS' = G - (b_t (.) k_t) dd^T,
 *     dalpha_t = rowsum(dS' (.) S_{t-1}),  G <- Diag(alpha_t) dS',
 * with G = dL/dS_t starting from dL/dS_T, d_t = w_t (.) v_t - (Diag(alpha_t) S_{t-1})^T (b_t (.) k_t),
 * and dS0 = G after the first token.
 *
 *   q, k, v, alpha, b, w, S0, B, T, H, d_k, d_v, cu_seqlens, dtype: as for gdn2_chunk_fwd (the same
 *           forward inputs; S0 may be NULL = zeros).
 *   dO      [.., H, d_v] in dtype: dL/do (layout of o).
 *   dS_T    [B, H, d_k, d_v] fp32: dL/dS_T, or NULL (zero).
 *   dq, dk, dalpha, db   [.., H, d_k] in dtype (out), dv, dw [.., H, d_v] in dtype (out).
 *   dS0     [B, H, d_k, d_v] fp32 (out), or NULL (not returned).  dS0 may alias dS_T.
 * Arithmetic is fp32; the gradients are rounded to dtype once.  dq, dk, dalpha and db are sums
 * over 16-column tiles of the state formed with fp32 reductions in L2, so their last bits may
 * differ from run to run; dv, dw and dS0 are reproducible.  The call takes a workspace of
 * gdn2_chunk_bwd_workspace_bytes() bytes from the library's pool (a gradient accumulator, the
 * per-token d_t, state checkpoints every 64 tokens and a per-(sequence, head) scratch of 16 states)
 * and gives it back on `stream`.  Errors as for gdn2_chunk_fwd.
 */
GDN2_API gdn2_status gdn2_chunk_bwd(const void *q, const void *k, const void *v, const void *alpha,
                                    const void *b, const void *w, const float *S0, const void *dO,
                                    const float *dS_T, void *dq, void *dk, void *dv, void *dalpha, void *db,
                                    void *dw, float *dS0, int B, int T, int H, int d_k, int d_v,
                                    const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_chunk_bwd_workspace_bytes -- device bytes gdn2_chunk_bwd takes from its pool for a call of
 * this shape (packed != 0: B sequences, T tokens in total); 0 for an unsupported shape.  Host only.
 */
GDN2_API size_t gdn2_chunk_bwd_workspace_bytes(int B, int T, int H, int d_k, int d_v, int packed);

/*
 * gdn2_decode_step -- one recurrent step for a batch of single tokens.
 *
 * For every (batch entry, head): S <- the edited state after one token; o <- S^T q.
 * The state is read once and written once (memory-bound).
 *   q, k, alpha, b : [B, H, d_k]     v, w, o : [B, H, d_v]
 *   S              : [B, H, d_k, d_v] fp32, updated in place.
 * o must not overlap S or the inputs.
 */
GDN2_API gdn2_status gdn2_decode_step(const void *q, const void *k, const void *v, const void *alpha,
                             const void *b, const void *w, float *S, void *o, int B, int H,
                             int d_k, int d_v, gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_block_prologue -- the mixer's inputs from the block's projections.
 *
 * "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section
 * "アーキテクチャとパフォーマンスベンチマーク": the query and key paths apply a short causal
 * convolution, SiLU and L2 normalisation to their projection, the value path a short convolution
 * and SiLU; the decay and both gates come from their own linear branches.  The projections
 * (matrix products) are the caller's; this call takes their outputs:
 *   x_q, x_k, x_alpha, x_b : [tokens, H, d_k]     x_v, x_w : [tokens, H, d_v]   (dtype)
 *   conv_q, conv_k : [H * d_k, conv_len] fp32     conv_v : [H * d_v, conv_len] fp32
 * and writes, in the layouts gdn2_chunk_fwd reads:
 *   q = L2norm(SiLU(conv_q * x_q)), k likewise (over d_k per token and head, eps 1e-6 under the
 *   root), v = SiLU(conv_v * x_v), alpha = exp(-softplus(x_alpha)), b = sigmoid(x_b),
 *   w = sigmoid(x_w).
 * The convolution is depthwise and causal, y_t = sum_j conv[c][conv_len-1-j] x_{t-j}[c] (the last
 * tap multiplies the current token), and restarts at every sequence start: dense batches are B
 * sequences of T tokens; packed batches (cu_seqlens != NULL, device int32 [B+1]) have T tokens in
 * total.  conv_len: 1 to 4.  d_k in {64, 128}, d_v in {64, 128, 256}.  Token tensors 16-byte
 * aligned, weights 4-byte aligned; outputs must not overlap the inputs.  fp32 arithmetic.
 * Asynchronous on `stream`; validation errors return before any launch.
 */
GDN2_API gdn2_status gdn2_block_prologue(const void *x_q, const void *x_k, const void *x_v, const void *x_alpha,
                                         const void *x_b, const void *x_w, const float *conv_q, const float *conv_k,
                                         const float *conv_v, void *q, void *k, void *v, void *alpha, void *b,
                                         void *w, int B, int T, int H, int d_k, int d_v, int conv_len,
                                         const int32_t *cu_seqlens, gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_block_epilogue -- the output gate after the mixer (same page and section): the recurrent
 * output is RMS-normalised and multiplied by a SiLU output gate (before the output projection,
 * the caller's).  For every token and head, over its d_v values:
 *   y = o / sqrt(mean(o^2) + 1e-5) * norm_weight * SiLU(gate)
 *   o, gate, y : [tokens, H, d_v] (dtype, 16-byte aligned)   norm_weight : [d_v] fp32
 * y may alias o.  d_v in {64, 128, 256}.  fp32 arithmetic.  Asynchronous on `stream`.
 */
GDN2_API gdn2_status gdn2_block_epilogue(const void *o, const void *gate, const float *norm_weight, void *y,
                                         long long tokens, int H, int d_v, gdn2_dtype dtype, gdn2_stream_t stream);

/* Human-readable name of a status; never NULL. */
GDN2_API const char *gdn2_status_string(gdn2_status status);

/*
 * gdn2_device_status -- the sticky device-side status of the tensor-core kernels.
 * Their waits on asynchronous copies and tensor-core completions are bounded
 * (2 s); a wait that gives up makes the kernel skip the rest of its work, free
 * its tensor memory and record GDN2_ERR_TIMEOUT here.  Synchronises with the
 * device (it copies one int).  reset != 0 clears the word after reading it.
 * Returns GDN2_OK, GDN2_ERR_TIMEOUT, or GDN2_ERR_CUDA if the copy failed.
 */
GDN2_API gdn2_status gdn2_device_status(int reset);

/*
 * gdn2_selftest_bounded_wait -- exercises the failure path of the bounded device-side waits.
 * Launches one CTA that waits on a barrier nothing arrives on; after `limit_us` microseconds
 * (1 .. 10,000,000) the wait gives up and records GDN2_ERR_TIMEOUT in the status word that
 * gdn2_device_status() reads -- the same path the tensor-core kernels take.  Nothing faults and
 * the context stays usable.  Asynchronous on `stream`.  Returns GDN2_OK, GDN2_ERR_INVALID_ARG
 * for a limit out of range, or GDN2_ERR_CUDA if the launch failed.
 */
GDN2_API gdn2_status gdn2_selftest_bounded_wait(int limit_us, gdn2_stream_t stream);

/* Number of kernel launches this library has issued in this process (all calls, all threads). */
GDN2_API uint64_t gdn2_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
