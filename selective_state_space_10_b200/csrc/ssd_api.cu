// ssd_api.cu -- the C ABI of libssd (include/ssd.h): host-side validation, workspace
// layout and kernel dispatch.  Every entry point validates all arguments before it
// enqueues anything; validation makes no CUDA call, so it behaves the same on a host
// without a GPU.
#include <stdint.h>
#include <string.h>

#include "ssd.h"
#include "kernels.h"

namespace {

using ssd::Dims;

constexpr int kVersion = 100;  // 0.1.0
constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

bool supported_dstate(int64_t n) { return n == 16 || n == 32 || n == 64 || n == 128 || n == 256; }

// Shape checks shared by both calls.  Returns SSD_OK and fills `d` on success.
ssd_status check_dims(const ssd_dims *dims, ssd_dtype dtype, bool prefill, Dims *d) {
  if (!dims) return SSD_ERR_INVALID_ARG;
  if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  const int64_t lim = (int64_t)1 << 30;
  if (dims->batch < 0 || dims->batch > lim) return SSD_ERR_INVALID_ARG;
  if (prefill && (dims->seqlen < 0 || dims->seqlen > lim)) return SSD_ERR_INVALID_ARG;
  if (dims->nheads < 1 || dims->nheads > 65535) return SSD_ERR_INVALID_ARG;
  if (dims->ngroups < 1 || dims->nheads % dims->ngroups != 0) return SSD_ERR_INVALID_ARG;
  if (dims->headdim < 1 || dims->headdim > 256) return SSD_ERR_INVALID_ARG;
  if (dims->dstate < 1) return SSD_ERR_INVALID_ARG;
  if (!supported_dstate(dims->dstate)) return SSD_ERR_UNSUPPORTED;
  // Element counts must stay far from 64-bit overflow and grid limits.
  const int64_t L = prefill ? dims->seqlen : 1;
  const double xs = (double)dims->batch * (double)L * (double)dims->nheads * (double)dims->headdim;
  const double ss = (double)dims->batch * (double)dims->nheads * (double)dims->headdim * (double)dims->dstate;
  if (xs > 4e12 || ss > 4e12) return SSD_ERR_INVALID_ARG;
  if ((double)dims->batch * (double)dims->nheads > 2147483647.0) return SSD_ERR_INVALID_ARG;
  d->b = (int)dims->batch;
  d->L = prefill ? (int)dims->seqlen : 1;
  d->H = (int)dims->nheads;
  d->P = (int)dims->headdim;
  d->N = (int)dims->dstate;
  d->G = (int)dims->ngroups;
  d->hpg = d->H / d->G;
  return SSD_OK;
}

// Every non-empty array must be non-NULL and aligned.
bool check_ptr(const void *p, int64_t elems, size_t align) {
  if (elems == 0) return true;
  return p != nullptr && aligned(p, align);
}

enum class Path { kNone, kSimt, kTensorCore };

// Workspace layout of one prefill.  Offset 0 always holds a 256-byte region whose first
// int is the device-side error word (non-zero after a bounded wait expired).
struct PrefillPlan {
  Path path = Path::kNone;
  int nc = 0;             // chunks per sequence
  size_t cum_off = 0;     // SIMT: float [b][H][nc][Q] in-chunk cumulative decay
  size_t states_off = 0;  // both: float [b][nc][H][P][N] chunk states (SIMT: replaced by h_prev)
  size_t tab_off = 0;     // tensor cores: float [b][H][nc][4 + 2Q] decay table (D, chunk decay, c2, dt)
  size_t cdecay_off = 0;  // tensor cores: float [b][H][nc] total decay of each chunk
  size_t hprev_off = 0;   // tensor cores: bf16 [b][nc][H][P][N] state entering each chunk
  size_t bytes = 0;
  int launches = 0;
};

PrefillPlan plan_prefill(const Dims &d, ssd_dtype dtype, int Q) {
  PrefillPlan pl;
  pl.nc = (int)(((int64_t)d.L + Q - 1) / Q);
  if (d.b == 0 || d.L == 0) return pl;
  const size_t nstate = (size_t)d.b * pl.nc * d.H * (size_t)d.P * d.N;
  if (dtype == SSD_BF16 && ssd::tc_prefill_supported(d, Q)) {
    pl.path = Path::kTensorCore;
    pl.states_off = kAlign;
    pl.cdecay_off = pl.states_off + align_up(nstate * sizeof(float));
    pl.hprev_off = pl.cdecay_off + align_up((size_t)d.b * d.H * pl.nc * sizeof(float));
    pl.tab_off = pl.hprev_off + align_up(nstate * sizeof(__nv_bfloat16));
    pl.bytes = pl.tab_off + align_up(ssd::tc_prefill_table_floats(d, Q, pl.nc) * sizeof(float));
    pl.launches = 3;
  } else {
    pl.path = Path::kSimt;
    pl.cum_off = kAlign;
    pl.states_off = pl.cum_off + align_up((size_t)d.b * d.H * pl.nc * Q * sizeof(float));
    pl.bytes = pl.states_off + align_up(nstate * sizeof(float));
    pl.launches = 4;
  }
  return pl;
}

ssd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA; }

// Records events[i] before kernel i (and events[k] after the last) when events != NULL.
struct Marker {
  cudaEvent_t const *ev;
  cudaStream_t st;
  int i = 0;
  cudaError_t mark() { return ev ? cudaEventRecord(ev[i++], st) : cudaSuccess; }
};

template <typename T>
ssd_status run_prefill(const Dims &d, int Q, const PrefillPlan &pl, const T *x, const float *dt,
                       const float *A, const T *B, const T *C, const float *D, const float *init, float *y,
                       float *final_state, float *cstates, char *ws, cudaStream_t st, cudaEvent_t const *ev) {
  float *cum = reinterpret_cast<float *>(ws + pl.cum_off);
  float *states = reinterpret_cast<float *>(ws + pl.states_off);
  Marker m{ev, st};
  cudaError_t e = m.mark();
  if (e == cudaSuccess) e = ssd::launch_dA_cumsum(dt, A, cum, d, Q, pl.nc, st);
  if (e == cudaSuccess) e = m.mark();
  if (e == cudaSuccess) e = ssd::launch_chunk_state_simt<T>(x, dt, B, cum, states, d, Q, pl.nc, st);
  if (e == cudaSuccess) e = m.mark();
  if (e == cudaSuccess) e = ssd::launch_state_passing(states, cum, init, final_state, cstates, d, Q, pl.nc, st);
  if (e == cudaSuccess) e = m.mark();
  if (e == cudaSuccess) e = ssd::launch_chunk_scan_simt<T>(x, dt, B, C, D, cum, states, y, d, Q, pl.nc, st);
  if (e == cudaSuccess) e = m.mark();
  return cuda_status(e);
}

const char *const kSimtKernelNames[] = {"dA_cumsum", "chunk_state_simt", "state_passing", "chunk_scan_simt"};
const char *const kTcKernelNames[] = {"chunk_state_tc", "state_passing_bf16", "chunk_scan_tc"};

}  // namespace

extern "C" {

const char *ssd_status_string(ssd_status s) {
  switch (s) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape outside the supported set";
    case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA launch or runtime error";
    case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: bounded device wait expired";
  }
  return "unknown ssd_status";
}

int ssd_version(void) { return kVersion; }

size_t ssd_prefill_workspace_size(const ssd_dims *dims, ssd_dtype dtype, int chunk) {
  Dims d;
  if (check_dims(dims, dtype, true, &d) != SSD_OK) return 0;
  if (!is_pow2(chunk) || chunk > 256) return 0;
  return plan_prefill(d, dtype, chunk).bytes;
}

int ssd_prefill_kernel_launches(const ssd_dims *dims, ssd_dtype dtype, int chunk) {
  Dims d;
  if (check_dims(dims, dtype, true, &d) != SSD_OK) return -1;
  if (!is_pow2(chunk) || chunk > 256) return -1;
  return plan_prefill(d, dtype, chunk).launches;
}

static ssd_status prefill_impl(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                               const float *A, const void *B, const void *C, const float *D, int chunk,
                               const float *init, float *y, float *final_state, float *cstates, void *workspace,
                               size_t workspace_bytes, ssd_stream_t stream, void *const *events, int num_events,
                               bool timed) {
  Dims d;
  ssd_status s = check_dims(dims, dtype, true, &d);
  if (s != SSD_OK) return s;
  if (!is_pow2(chunk) || chunk > 256) return SSD_ERR_INVALID_ARG;
  const int64_t ntok = (int64_t)d.b * d.L;
  const int64_t nx = ntok * d.H * d.P, nbc = ntok * d.G * d.N, nst = (int64_t)d.b * d.H * d.P * d.N;
  if (!check_ptr(x, nx, 16) || !check_ptr(B, nbc, 16) || !check_ptr(C, nbc, 16) || !check_ptr(y, nx, 16) ||
      !check_ptr(dt, ntok * d.H, 4) || !check_ptr(final_state, nst, 16))
    return SSD_ERR_INVALID_ARG;
  // optional arrays: NULL means "none"; when given they must be aligned
  const int64_t ncs = (int64_t)d.b * ((d.L + chunk - 1) / chunk) * d.H * d.P * d.N;
  if ((init != nullptr && !check_ptr(init, nst, 16)) || (cstates != nullptr && !check_ptr(cstates, ncs, 16)))
    return SSD_ERR_INVALID_ARG;
  const bool any_heads = d.b > 0 && d.L > 0;
  if (!check_ptr(A, any_heads ? d.H : 0, 4) || !check_ptr(D, any_heads ? d.H : 0, 4)) return SSD_ERR_INVALID_ARG;
  const PrefillPlan pl = plan_prefill(d, dtype, chunk);
  if (timed) {
    if (events == nullptr || num_events < pl.launches + 1) return SSD_ERR_INVALID_ARG;
    for (int i = 0; i < pl.launches + 1; ++i)
      if (events[i] == nullptr) return SSD_ERR_INVALID_ARG;
  }
  if (pl.bytes > 0 && (workspace == nullptr || !aligned(workspace, 16) || workspace_bytes < pl.bytes))
    return SSD_ERR_WORKSPACE;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d.b == 0) return SSD_OK;
  if (d.L == 0) {  // no tokens: the final state is the initial one
    if (init == nullptr) return cuda_status(cudaMemsetAsync(final_state, 0, (size_t)nst * sizeof(float), st));
    if (init == final_state) return SSD_OK;
    return cuda_status(cudaMemcpyAsync(final_state, init, (size_t)nst * sizeof(float), cudaMemcpyDeviceToDevice, st));
  }
  char *ws = static_cast<char *>(workspace);
  cudaEvent_t const *ev = timed ? reinterpret_cast<cudaEvent_t const *>(events) : nullptr;
  // The device error word starts at zero: the tensor-core path's first kernel clears it
  // itself; the CUDA-core path (which has no bounded waits) clears it here.
  if (pl.path == Path::kTensorCore)
    return cuda_status(ssd::launch_tc_prefill(
        static_cast<const __nv_bfloat16 *>(x), dt, A, static_cast<const __nv_bfloat16 *>(B),
        static_cast<const __nv_bfloat16 *>(C), D, init, y, final_state, cstates, reinterpret_cast<float *>(ws + pl.tab_off),
        reinterpret_cast<float *>(ws + pl.states_off),
        reinterpret_cast<float *>(ws + pl.cdecay_off), reinterpret_cast<__nv_bfloat16 *>(ws + pl.hprev_off),
        reinterpret_cast<int *>(ws), d, chunk, pl.nc, st, ev));
  if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return SSD_ERR_CUDA;
  if (dtype == SSD_F32)
    return run_prefill<float>(d, chunk, pl, static_cast<const float *>(x), dt, A, static_cast<const float *>(B),
                              static_cast<const float *>(C), D, init, y, final_state, cstates, ws, st, ev);
  return run_prefill<__nv_bfloat16>(d, chunk, pl, static_cast<const __nv_bfloat16 *>(x), dt, A,
                                    static_cast<const __nv_bfloat16 *>(B), static_cast<const __nv_bfloat16 *>(C), D,
                                    init, y, final_state, cstates, ws, st, ev);
}

ssd_status ssd_prefill(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt, const float *A,
                       const void *B, const void *C, const float *D, int chunk, float *y, float *final_state,
                       void *workspace, size_t workspace_bytes, ssd_stream_t stream) {
  return prefill_impl(dims, dtype, x, dt, A, B, C, D, chunk, nullptr, y, final_state, nullptr, workspace,
                      workspace_bytes, stream, nullptr, 0, false);
}

ssd_status ssd_prefill_ex(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt, const float *A,
                          const void *B, const void *C, const float *D, int chunk, const float *initial_state,
                          float *y, float *final_state, float *chunk_states, void *workspace, size_t workspace_bytes,
                          ssd_stream_t stream) {
  return prefill_impl(dims, dtype, x, dt, A, B, C, D, chunk, initial_state, y, final_state, chunk_states, workspace,
                      workspace_bytes, stream, nullptr, 0, false);
}

ssd_status ssd_prefill_timed(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt, const float *A,
                             const void *B, const void *C, const float *D, int chunk, float *y, float *final_state,
                             void *workspace, size_t workspace_bytes, ssd_stream_t stream, void *const *events,
                             int num_events) {
  return prefill_impl(dims, dtype, x, dt, A, B, C, D, chunk, nullptr, y, final_state, nullptr, workspace,
                      workspace_bytes, stream, events, num_events, true);
}

namespace {
// Offsets in ssd_prefill_host's device buffer: the input copies, the outputs, then the
// prefill workspace, each 256-byte aligned.
struct HostPlan {
  int64_t nx, ndt, nbc, ny, nst;  // element counts
  size_t esz;
  size_t x, dt, A, B, C, D, y, fs, ws, ws_bytes, bytes;
};
bool plan_host(const ssd_dims *dims, ssd_dtype dtype, int chunk, HostPlan *hp) {
  Dims d;
  if (check_dims(dims, dtype, true, &d) != SSD_OK || !is_pow2(chunk) || chunk > 256) return false;
  const int64_t ntok = (int64_t)d.b * d.L;
  hp->esz = dtype == SSD_F32 ? 4 : 2;
  hp->nx = ntok * d.H * d.P;
  hp->ndt = ntok * d.H;
  hp->nbc = ntok * d.G * d.N;
  hp->ny = hp->nx;
  hp->nst = (int64_t)d.b * d.H * d.P * d.N;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  hp->x = take((size_t)hp->nx * hp->esz);
  hp->dt = take((size_t)hp->ndt * 4);
  hp->A = take((size_t)d.H * 4);
  hp->B = take((size_t)hp->nbc * hp->esz);
  hp->C = take((size_t)hp->nbc * hp->esz);
  hp->D = take((size_t)d.H * 4);
  hp->y = take((size_t)hp->ny * 4);
  hp->fs = take((size_t)hp->nst * 4);
  hp->ws_bytes = plan_prefill(d, dtype, chunk).bytes;
  hp->ws = take(hp->ws_bytes);
  hp->bytes = off;
  return true;
}
}  // namespace

size_t ssd_prefill_host_buffer_size(const ssd_dims *dims, ssd_dtype dtype, int chunk) {
  HostPlan hp;
  return plan_host(dims, dtype, chunk, &hp) ? hp.bytes : 0;
}

ssd_status ssd_prefill_host(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt, const float *A,
                            const void *B, const void *C, const float *D, int chunk, float *y, float *final_state,
                            void *device_buffer, size_t device_buffer_bytes, ssd_stream_t stream) {
  Dims d;
  ssd_status s = check_dims(dims, dtype, true, &d);
  if (s != SSD_OK) return s;
  if (!is_pow2(chunk) || chunk > 256) return SSD_ERR_INVALID_ARG;
  HostPlan hp;
  if (!plan_host(dims, dtype, chunk, &hp)) return SSD_ERR_INVALID_ARG;
  // host arrays: non-NULL when non-empty, no alignment needed
  if ((hp.nx > 0 && (x == nullptr || y == nullptr)) || (hp.ndt > 0 && dt == nullptr) ||
      (hp.nbc > 0 && (B == nullptr || C == nullptr)) || (hp.nst > 0 && final_state == nullptr) ||
      (d.b > 0 && (A == nullptr || D == nullptr)))
    return SSD_ERR_INVALID_ARG;
  if (d.b == 0) return SSD_OK;  // nothing to compute or copy
  if (device_buffer == nullptr || !aligned(device_buffer, 16) || device_buffer_bytes < hp.bytes)
    return SSD_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *dev = static_cast<uint8_t *>(device_buffer);
  auto h2d = [&](size_t off, const void *src, size_t bytes) {
    return bytes == 0 ? cudaSuccess : cudaMemcpyAsync(dev + off, src, bytes, cudaMemcpyHostToDevice, st);
  };
  cudaError_t e = h2d(hp.x, x, (size_t)hp.nx * hp.esz);
  if (e == cudaSuccess) e = h2d(hp.dt, dt, (size_t)hp.ndt * 4);
  if (e == cudaSuccess) e = h2d(hp.A, A, d.b > 0 ? (size_t)d.H * 4 : 0);
  if (e == cudaSuccess) e = h2d(hp.B, B, (size_t)hp.nbc * hp.esz);
  if (e == cudaSuccess) e = h2d(hp.C, C, (size_t)hp.nbc * hp.esz);
  if (e == cudaSuccess) e = h2d(hp.D, D, d.b > 0 ? (size_t)d.H * 4 : 0);
  if (e != cudaSuccess) return cuda_status(e);
  s = ssd_prefill(dims, dtype, dev + hp.x, reinterpret_cast<const float *>(dev + hp.dt),
                  reinterpret_cast<const float *>(dev + hp.A), dev + hp.B, dev + hp.C,
                  reinterpret_cast<const float *>(dev + hp.D), chunk, reinterpret_cast<float *>(dev + hp.y),
                  reinterpret_cast<float *>(dev + hp.fs), dev + hp.ws, hp.ws_bytes, stream);
  if (s != SSD_OK) return s;
  if (hp.ny > 0) e = cudaMemcpyAsync(y, dev + hp.y, (size_t)hp.ny * 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess && hp.nst > 0)
    e = cudaMemcpyAsync(final_state, dev + hp.fs, (size_t)hp.nst * 4, cudaMemcpyDeviceToHost, st);
  return cuda_status(e);
}

const char *ssd_prefill_kernel_name(const ssd_dims *dims, ssd_dtype dtype, int chunk, int i) {
  Dims d;
  if (check_dims(dims, dtype, true, &d) != SSD_OK || !is_pow2(chunk) || chunk > 256) return nullptr;
  const PrefillPlan pl = plan_prefill(d, dtype, chunk);
  if (i < 0 || i >= pl.launches) return nullptr;
  return pl.path == Path::kTensorCore ? kTcKernelNames[i] : kSimtKernelNames[i];
}

ssd_status ssd_prefill_device_status(const void *workspace, size_t workspace_bytes, ssd_stream_t stream) {
  if (workspace == nullptr || workspace_bytes < sizeof(int) || !aligned(workspace, 16)) return SSD_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SSD_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
  return word == 0 ? SSD_OK : SSD_ERR_TIMEOUT;
}

ssd_status ssd_decode_step(const ssd_dims *dims, ssd_dtype dtype, float *state, const void *x, const float *dt,
                           const float *A, const void *B, const void *C, const float *D, float *y,
                           ssd_stream_t stream) {
  Dims d;
  ssd_status s = check_dims(dims, dtype, false, &d);
  if (s != SSD_OK) return s;
  const int64_t nx = (int64_t)d.b * d.H * d.P, nbc = (int64_t)d.b * d.G * d.N;
  const int64_t nst = (int64_t)d.b * d.H * d.P * d.N;
  const int64_t nh = d.b > 0 ? d.H : 0;
  if (!check_ptr(state, nst, 16) || !check_ptr(x, nx, 16) || !check_ptr(B, nbc, 16) || !check_ptr(C, nbc, 16) ||
      !check_ptr(y, nx, 16) || !check_ptr(dt, (int64_t)d.b * d.H, 4) || !check_ptr(A, nh, 4) || !check_ptr(D, nh, 4))
    return SSD_ERR_INVALID_ARG;
  if (d.b == 0) return SSD_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SSD_F32)
    return cuda_status(ssd::launch_decode_step<float>(state, static_cast<const float *>(x), dt, A,
                                                      static_cast<const float *>(B), static_cast<const float *>(C),
                                                      D, y, d, st));
  return cuda_status(ssd::launch_decode_step<__nv_bfloat16>(
      state, static_cast<const __nv_bfloat16 *>(x), dt, A, static_cast<const __nv_bfloat16 *>(B),
      static_cast<const __nv_bfloat16 *>(C), D, y, d, st));
}

ssd_status ssd_frontend(const ssd_dims *dims, ssd_dtype dtype, const void *xbc, const float *conv_w,
                        const float *conv_b, const float *conv_state_in, float *conv_state_out, const float *dt_raw,
                        const float *dt_bias, void *x, void *B, void *C, float *dt, ssd_stream_t stream) {
  Dims d;
  ssd_status s = check_dims(dims, dtype, true, &d);
  if (s != SSD_OK) return s;
  const int64_t ntok = (int64_t)d.b * d.L, ch = (int64_t)d.H * d.P + 2 * (int64_t)d.G * d.N;
  const int64_t nx = ntok * d.H * d.P, nbc = ntok * d.G * d.N, any = ntok > 0 ? 1 : 0;
  const size_t esz = dtype == SSD_F32 ? 4 : 2;
  if (!check_ptr(xbc, ntok * ch, esz) || !check_ptr(conv_w, any * ch * 4, 16) || !check_ptr(x, nx, 16) ||
      !check_ptr(B, nbc, 16) || !check_ptr(C, nbc, 16) || !check_ptr(dt_raw, ntok * d.H, 4) ||
      !check_ptr(dt_bias, any * d.H, 4) || !check_ptr(dt, ntok * d.H, 4))
    return SSD_ERR_INVALID_ARG;
  if (d.b > 65535 || (ch + 255) / 256 > 65535) return SSD_ERR_INVALID_ARG;  // launch grid limits
  const int64_t nstate = (int64_t)d.b * 3 * ch;
  if ((conv_b != nullptr && !check_ptr(conv_b, ch, 4)) || (conv_state_in != nullptr && !check_ptr(conv_state_in, nstate, 4)) ||
      (conv_state_out != nullptr && !check_ptr(conv_state_out, nstate, 4)))
    return SSD_ERR_INVALID_ARG;
  if (d.b == 0) return SSD_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d.L == 0) {  // no tokens: the conv state carries over unchanged
    if (conv_state_out == nullptr || conv_state_out == conv_state_in) return SSD_OK;
    if (conv_state_in == nullptr) return cuda_status(cudaMemsetAsync(conv_state_out, 0, (size_t)nstate * 4, st));
    return cuda_status(cudaMemcpyAsync(conv_state_out, conv_state_in, (size_t)nstate * 4, cudaMemcpyDeviceToDevice, st));
  }
  if (dtype == SSD_F32)
    return cuda_status(ssd::launch_frontend<float>(static_cast<const float *>(xbc), conv_w, conv_b, conv_state_in,
                                                   conv_state_out, dt_raw, dt_bias, static_cast<float *>(x),
                                                   static_cast<float *>(B), static_cast<float *>(C), dt, d, st));
  return cuda_status(ssd::launch_frontend<__nv_bfloat16>(
      static_cast<const __nv_bfloat16 *>(xbc), conv_w, conv_b, conv_state_in, conv_state_out, dt_raw, dt_bias,
      static_cast<__nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(B), static_cast<__nv_bfloat16 *>(C), dt, d, st));
}

ssd_status ssd_decode_window_step(const ssd_dims *dims, ssd_dtype dtype, int window, int pos, const float *state,
                                  void *win_x, float *win_dt, void *win_B, const void *x, const float *dt,
                                  const float *A, const void *B, const void *C, const float *D, float *y,
                                  ssd_stream_t stream) {
  Dims d;
  ssd_status s = check_dims(dims, dtype, false, &d);
  if (s != SSD_OK) return s;
  if (window < 1 || window > 16 || pos < 0 || pos >= window) return SSD_ERR_INVALID_ARG;
  const int64_t nx = (int64_t)d.b * d.H * d.P, nbc = (int64_t)d.b * d.G * d.N;
  const int64_t nst = (int64_t)d.b * d.H * d.P * d.N, nh = d.b > 0 ? d.H : 0;
  if (!check_ptr(state, nst, 16) || !check_ptr(x, nx, 16) || !check_ptr(B, nbc, 16) || !check_ptr(C, nbc, 16) ||
      !check_ptr(y, nx, 16) || !check_ptr(dt, (int64_t)d.b * d.H, 4) || !check_ptr(A, nh, 4) ||
      !check_ptr(D, nh, 4) || !check_ptr(win_x, nx * window, 16) || !check_ptr(win_dt, (int64_t)d.b * d.H * window, 4) ||
      !check_ptr(win_B, nbc * window, 16))
    return SSD_ERR_INVALID_ARG;
  if (d.b == 0) return SSD_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SSD_F32)
    return cuda_status(ssd::launch_decode_window_step<float>(
        state, static_cast<float *>(win_x), win_dt, static_cast<float *>(win_B), window, pos,
        static_cast<const float *>(x), dt, A, static_cast<const float *>(B), static_cast<const float *>(C), D, y, d,
        st));
  return cuda_status(ssd::launch_decode_window_step<__nv_bfloat16>(
      state, static_cast<__nv_bfloat16 *>(win_x), win_dt, static_cast<__nv_bfloat16 *>(win_B), window, pos,
      static_cast<const __nv_bfloat16 *>(x), dt, A, static_cast<const __nv_bfloat16 *>(B),
      static_cast<const __nv_bfloat16 *>(C), D, y, d, st));
}

ssd_status ssd_decode_window_flush(const ssd_dims *dims, ssd_dtype dtype, int window, int count, float *state,
                                   const void *win_x, const float *win_dt, const void *win_B, const float *A,
                                   ssd_stream_t stream) {
  Dims d;
  ssd_status s = check_dims(dims, dtype, false, &d);
  if (s != SSD_OK) return s;
  if (window < 1 || window > 16 || count < 0 || count > window) return SSD_ERR_INVALID_ARG;
  const int64_t nx = (int64_t)d.b * d.H * d.P, nbc = (int64_t)d.b * d.G * d.N;
  const int64_t nst = (int64_t)d.b * d.H * d.P * d.N, nh = d.b > 0 ? d.H : 0;
  if (!check_ptr(state, nst, 16) || !check_ptr(A, nh, 4) || !check_ptr(win_x, nx * window, 16) ||
      !check_ptr(win_dt, (int64_t)d.b * d.H * window, 4) || !check_ptr(win_B, nbc * window, 16))
    return SSD_ERR_INVALID_ARG;
  if (d.b == 0 || count == 0) return SSD_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SSD_F32)
    return cuda_status(ssd::launch_decode_window_flush<float>(state, static_cast<const float *>(win_x), win_dt,
                                                              static_cast<const float *>(win_B), window, count, A,
                                                              d, st));
  return cuda_status(ssd::launch_decode_window_flush<__nv_bfloat16>(
      state, static_cast<const __nv_bfloat16 *>(win_x), win_dt, static_cast<const __nv_bfloat16 *>(win_B), window,
      count, A, d, st));
}

}  // extern "C"

namespace ssd {

// Internal entry for other translation units of the library: ssd_prefill with a given
// workspace (same validation, computation and errors).
ssd_status prefill_into_workspace(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                                  const float *A, const void *B, const void *C, const float *D, int chunk,
                                  float *y, float *final_state, void *workspace, size_t workspace_bytes,
                                  ssd_stream_t stream) {
  return prefill_impl(dims, dtype, x, dt, A, B, C, D, chunk, nullptr, y, final_state, nullptr, workspace,
                      workspace_bytes, stream, nullptr, 0, false);
}

}  // namespace ssd
