// Device-side status word of the tensor-core kernels and the self-test of their bounded waits.
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

// Waits on an mbarrier that nothing ever arrives on, gives up after `limit_ns`, and records
// GDN2_ERR_TIMEOUT exactly like the chunk kernels do.  No fault, trap or endless loop is involved;
// the context stays usable afterwards.
__global__ void bounded_wait_probe_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = ptx::smem_u32(&bar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(b, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = ptx::mbar_wait_bounded(b, 0, limit_ns);
  const bool any_timeout = __syncthreads_or(!ok);
  if (any_timeout && threadIdx.x == 0) atomicExch(&g_device_status, 4);
}

}  // namespace

cudaError_t launch_bounded_wait_probe(uint64_t limit_ns, cudaStream_t stream) {
  note_launch();
  bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(limit_ns);
  return cudaGetLastError();
}

}  // namespace gdn2
