// noalloc.cu -- ssd_prefill_noalloc: the chunked prefill with its scratch taken from a
// fixed array compiled into the library, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand out device memory of their own: plugins
// running inside a host process whose device allocator belongs to the host framework,
// and serving loops that forbid any allocation once they have started.  They call this
// entry point instead of ssd_prefill; it computes exactly the same thing, with the
// prefill's workspace placed in g_noalloc_scratch below.
//
// The array lives in this translation unit's module, so a process holds its
// kNoAllocScratchBytes on a device only once it has used this entry point there, and
// then until it exits.  Host code cannot pass the array's name to a kernel (on the host
// it is only a stand-in for the device symbol), so the device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, and cached.
#include <atomic>
#include <mutex>

#include "api_internal.h"
#include "ssd.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_ptr[kMaxDevices];
std::mutex g_setup_mutex;

// Device address of the scratch array on the current device (set-up on first use).
ssd_status scratch_on_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SSD_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SSD_ERR_UNSUPPORTED;
  void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SSD_ERR_CUDA;
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return SSD_OK;
}

}  // namespace

extern "C" {

size_t ssd_prefill_noalloc_max_workspace(void) { return kNoAllocScratchBytes; }

ssd_status ssd_prefill_noalloc(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt, const float *A,
                               const void *B, const void *C, const float *D, int chunk, float *y, float *final_state,
                               ssd_stream_t stream) {
  // Invalid arguments give a workspace size of 0; the shared prefill path then reports
  // them exactly as ssd_prefill does, before any CUDA call.
  const size_t need = ssd_prefill_workspace_size(dims, dtype, chunk);
  if (need > kNoAllocScratchBytes) return SSD_ERR_WORKSPACE;
  if (need == 0)
    return ssd::prefill_into_workspace(dims, dtype, x, dt, A, B, C, D, chunk, y, final_state, nullptr, 0, stream);
  void *ws = nullptr;
  const ssd_status s = scratch_on_current_device(&ws);
  if (s != SSD_OK) return s;
  // Only the error word at the start of the workspace must start at zero; the prefill
  // clears it on the stream itself, and every other byte it reads it first writes.
  return ssd::prefill_into_workspace(dims, dtype, x, dt, A, B, C, D, chunk, y, final_state, ws,
                                     kNoAllocScratchBytes, stream);
}

}  // extern "C"
