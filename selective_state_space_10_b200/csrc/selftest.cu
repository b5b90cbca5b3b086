// selftest.cu -- a self-test of the bounded device-side waits the tensor-core prefill
// kernels use (sm100::mbar_wait): one CTA waits on an mbarrier that, when `expire` is
// set, nothing ever arrives on.  The wait gives up after `limit_ns` of %globaltimer,
// sets the workspace's error word exactly as a prefill kernel would, and the kernel
// returns; the host then reads the word back with ssd_prefill_device_status.  No trap,
// no fault, no endless loop: the context stays usable.
#include "common.cuh"
#include "sm100.cuh"
#include "ssd.h"

namespace ssd {
namespace {

__global__ void __launch_bounds__(64) k_wait_selftest(int *err, uint64_t limit_ns, int expire) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 32 && !expire) sm100::mbar_arrive(&bar);  // the producer that, when expiring, never comes
  if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
  __syncthreads();
}

}  // namespace
}  // namespace ssd

extern "C" SSD_API ssd_status ssd_wait_selftest(void *workspace, size_t workspace_bytes, uint64_t limit_ns, int expire,
                                                ssd_stream_t stream) {
  if (workspace == nullptr || workspace_bytes < sizeof(int) || (reinterpret_cast<uintptr_t>(workspace) % 16) != 0)
    return SSD_ERR_INVALID_ARG;
  if (limit_ns == 0 || limit_ns > 100000000ull) return SSD_ERR_INVALID_ARG;  // at most 100 ms
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return SSD_ERR_CUDA;
  ssd::k_wait_selftest<<<1, 64, 0, st>>>(static_cast<int *>(workspace), limit_ns, expire ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
