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
// cudaGetSymbolAddress.  The module, and with it the array's address, belongs to a CUDA
// context: the look-up is done once per context (keyed by the context's unique id, which
// the driver never reuses), so a context created after cudaDeviceReset, or another
// context the caller made current on the same device, gets its own look-up instead of a
// stale address.
#include <cuda.h>

#include <mutex>

#include "api_internal.h"
#include "ssd.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct ScratchTable {
  std::mutex mu;
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
  bool resolved = false;
  static constexpr int kEntries = 64;
  unsigned long long id[kEntries] = {};
  void *ptr[kEntries] = {};
  int used = 0, next = 0;
};
ScratchTable g_table;

template <typename Fn>
Fn driver_entry(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Unique id of the context current on this thread (the runtime's primary context of the
// current device unless the caller bound another); 0 if none could be found.
unsigned long long current_context_id() {
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_table.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (g_table.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array in the current context (looked up on first use).
ssd_status scratch_in_current_context(void **out) {
  std::lock_guard<std::mutex> lock(g_table.mu);
  if (!g_table.resolved) {
    g_table.get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
    g_table.get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
    g_table.resolved = true;
  }
  if (!g_table.get_current || !g_table.get_id) return SSD_ERR_CUDA;
  unsigned long long id = current_context_id();
  void *p = nullptr;
  if (id == 0) {
    // No context bound to this thread yet: the runtime binds its primary context of the
    // current device on its first call, which this look-up is.
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SSD_ERR_CUDA;
    if ((id = current_context_id()) == 0) return SSD_ERR_CUDA;
  }
  for (int i = 0; i < g_table.used; ++i)
    if (g_table.id[i] == id) {
      *out = g_table.ptr[i];
      return SSD_OK;
    }
  if (p == nullptr && (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)) return SSD_ERR_CUDA;
  const int slot = g_table.used < ScratchTable::kEntries ? g_table.used++ : (g_table.next++ % ScratchTable::kEntries);
  g_table.id[slot] = id;
  g_table.ptr[slot] = p;
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
  const ssd_status s = scratch_in_current_context(&ws);
  if (s != SSD_OK) return s;
  // Only the error word at the start of the workspace must start at zero; the prefill
  // clears it on the stream itself, and every other byte it reads it first writes.
  return ssd::prefill_into_workspace(dims, dtype, x, dt, A, B, C, D, chunk, y, final_state, ws,
                                     kNoAllocScratchBytes, stream);
}

ssd_status ssd_prefill_noalloc_device_status(ssd_stream_t stream) {
  void *ws = nullptr;
  const ssd_status s = scratch_in_current_context(&ws);
  if (s != SSD_OK) return s;
  return ssd_prefill_device_status(ws, kNoAllocScratchBytes, stream);
}

}  // extern "C"
