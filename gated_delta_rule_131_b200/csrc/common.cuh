// Shared device helpers of the gdn2 CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn2 {

// Arguments of one gdn2_chunk_fwd call, already validated by the API layer.
struct ChunkArgs {
  const void *q, *k, *v, *alpha, *b, *w;
  const float *S0;
  void *o;
  float *ST;
  const int32_t *cu;  // device offsets [B+1] or nullptr
  int B, T, H, dk, dv;
};

// Arguments of one gdn2_recurrent_fwd call (validated by the API layer); layouts as ChunkArgs.
struct RecurrentArgs {
  const void *q, *k, *v, *alpha, *b, *w;
  const float *S0;
  void *o;
  float *ST;
  const int32_t *cu;  // device offsets [B+1] or nullptr
  int B, T, H, dk, dv;
};

// Arguments of one gdn2_decode_step call.
struct DecodeArgs {
  const void *q, *k, *v, *alpha, *b, *w;
  float *S;
  void *o;
  int B, H, dk, dv;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_allreduce_sum(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// Token span of sequence n: dense batches use n*T .. n*T+T-1, packed ones cu[n] .. cu[n+1]-1.
__device__ __forceinline__ void seq_span(const ChunkArgs &a, int n, int64_t &bos, int &len) {
  if (a.cu) {
    bos = a.cu[n];
    len = a.cu[n + 1] - a.cu[n];
  } else {
    bos = (int64_t)n * a.T;
    len = a.T;
  }
}

// Arguments of the block prologue / epilogue around the mixer (validated by the API layer).
struct BlockPrologueArgs {
  const void *xq, *xk, *xv, *xa, *xb, *xw;  // pre-activations, [tokens, H, d]
  const float *Wq, *Wk, *Wv;                // short causal convolution weights, [H * d, K]
  void *q, *k, *v, *alpha, *b, *w;          // outputs, [tokens, H, d]
  const int32_t *cu;                        // packed batch offsets [B+1] or nullptr
  int B, T, H, dk, dv, K;
  long long tokens;
};
struct BlockEpilogueArgs {
  const void *o, *z;  // mixer output and output-gate pre-activation, [tokens, H, d_v]
  const float *g;     // RMS-normalisation weight [d_v]
  void *y;
  long long tokens;
  int H, dv;
};

// Arguments of one gdn2_chunk_bwd call (validated by the API layer).
struct BwdArgs {
  const void *q, *k, *v, *alpha, *b, *w, *dO;  // forward inputs and dL/do, [tokens, H, d]
  const float *S0, *dST;                       // [B, H, d_k, d_v] or nullptr (zeros)
  void *dq, *dk, *dv, *dalpha, *db, *dw;        // gradients, layouts of their inputs
  float *dS0;                                  // [B, H, d_k, d_v] or nullptr
  const int32_t *cu;                           // packed offsets [B+1] or nullptr
  int B, T, H, Dk, Dv;
};

// Host side: every kernel launch of the library is counted here.
void note_launch();

// Launchers (return the CUDA error of the launch).
cudaError_t launch_chunk_simt(const ChunkArgs &a, bool bf16, cudaStream_t stream);
// Two-kernel tensor-core path (WY factors of all chunks, then the state pass) over a workspace of
// chunk_wy_workspace_bytes(...) bytes, 256-byte aligned, that it fully writes before reading.
// The workspace depends only on the batch shape (B sequences, T tokens each or in total, H heads, d_v).
bool chunk_wy_supported(int B, int T, int H, int dk, int dv, bool packed, bool bf16);
size_t chunk_wy_workspace_bytes(int B, int T, int H, int dv, bool packed);
// The launch plan of that path for a device of `sms` SMs (0: the current device); host only.
struct ChunkWyPlan {
  long long records, wy_ctas, state_ctas;
  int segments, segment_chunks, handover_sms;
  long long handover_at;
  int order, launches;
  size_t workspace_bytes;
};
ChunkWyPlan chunk_wy_plan(int B, int T, int H, int dv, bool packed, int sms);
// Backward of the recurrence over a workspace of chunk_bwd_workspace_bytes(...) bytes, 256-byte
// aligned (a gradient accumulator it clears, and state checkpoints it writes before reading).
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, bool packed);
cudaError_t launch_chunk_bwd(const BwdArgs &a, bool bf16, void *ws, cudaStream_t stream);
cudaError_t launch_chunk_wy(const ChunkArgs &a, void *workspace, cudaStream_t stream);
cudaError_t launch_bounded_wait_probe(uint64_t limit_ns, cudaStream_t stream);
// Reads (and optionally clears) the device-side status word that bounded waits set.
cudaError_t read_device_status(int *status, bool reset);
// Device address of that word, for kernels compiled in other files.
cudaError_t device_status_word(int **ptr);
cudaError_t launch_decode(const DecodeArgs &a, bool bf16, cudaStream_t stream);
// Token-loop forward over whole sequences; r2 selects the second erase orientation.
cudaError_t launch_recurrent(const RecurrentArgs &a, bool bf16, bool r2, cudaStream_t stream);
cudaError_t launch_block_prologue(const BlockPrologueArgs &p, bool bf16, cudaStream_t stream);
cudaError_t launch_block_epilogue(const BlockEpilogueArgs &p, bool bf16, cudaStream_t stream);

}  // namespace gdn2
