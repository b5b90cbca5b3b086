// frontend.cu -- the steps of the Mamba-2 block right before the SSD layer ("Engineering
// Hybrid State-Space Models" section 3, the block diagram: a width-4 1-D convolution and
// SiLU; Delta = Softplus(Linear(x) + bias); the session's convState of the last dConv-1
// inputs per channel), fused into one pass over the projected inputs:
//
//   u = xbc [b, L, H*P + 2*G*N]   (the x, B and C channels, in that order)
//   a[t, c] = silu( sum_k w[c, k] u[t - 3 + k, c] + bias[c] )   (inputs before the first
//             token from the conv state, or zero)
//   x = a[:, :, :HP], B = a[:, :, HP:HP+GN], C = a[:, :, HP+GN:]   (the SSD layouts)
//   dt[t, h] = softplus(dt_raw[t, h] + dt_bias[h])
//
// k_frontend: one thread per (4 channels, 8-token run) -- grid (token runs, channel tiles,
// batch rows); consecutive threads take consecutive channel groups, so every vector load
// and store of a warp is one contiguous run of the token's row, and all of a thread's
// inputs are loaded before the first use.  fp32 arithmetic; outputs in the call's dtype
// (round to nearest even for bf16).  The CTAs of the first channel tile
// also form dt for their tokens.  k_frontend_state then writes the new conv state (the
// last three inputs), after every read of the old one, so the state may be updated in
// place.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace ssd {

// tokens per thread: the staged tile of 3 + tokens rows x 256 V channels stays within 48 KB
template <typename T> constexpr int fe_tokens() { return sizeof(T) == 2 ? 16 : 8; }

// cp.async of 4, 8 or 16 bytes global -> shared (both addresses aligned to the size)
template <int BYTES>
__device__ __forceinline__ void cp_async(void *dst, const void *src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(d), "l"(src), "n"(BYTES) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// v * sigmoid(v) with the fast reciprocal (about 1 ulp; 0 once exp(-v) overflows): the
// fp32 outputs.  For bf16 outputs one special-function op instead of two:
// v * sigmoid(v) = (v / 2) (1 + tanh(v / 2)), with the hardware tanh (relative error about
// 2^-10.7, under half the output's own rounding of 2^-9).
__device__ __forceinline__ float silu_f(float v) { return v * __fdividef(1.f, 1.f + __expf(-v)); }
__device__ __forceinline__ float silu_tanh(float v) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * v));
  return 0.5f * v * (1.f + t);
}
template <typename T> __device__ __forceinline__ float silu_out(float v) {
  return sizeof(T) == 2 ? silu_tanh(v) : silu_f(v);
}
__device__ __forceinline__ float softplus_f(float z) { return z > 20.f ? z : log1pf(__expf(z)); }
__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// V consecutive channels of one token: loads and stores of V elements at once (V = 4:
// 8 bytes of bf16 or 16 bytes of fp32), V = 1 the scalar fallback.
template <typename T, int V> struct Vec;
template <> struct Vec<float, 1> {
  static __device__ __forceinline__ void load(const float *p, float (&v)[1]) { v[0] = *p; }
  static __device__ __forceinline__ void store(float *p, const float (&v)[1]) { *p = v[0]; }
};
template <> struct Vec<__nv_bfloat16, 1> {
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[1]) { v[0] = __bfloat162float(*p); }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[1]) { *p = __float2bfloat16_rn(v[0]); }
};
template <> struct Vec<float, 4> {
  static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4 *>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  static __device__ __forceinline__ void store(float *p, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct Vec<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    v[0] = __uint_as_float(q.x << 16); v[1] = __uint_as_float(q.x & 0xffff0000u);
    v[2] = __uint_as_float(q.y << 16); v[3] = __uint_as_float(q.y & 0xffff0000u);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 q;
    q.x = *reinterpret_cast<const uint32_t *>(&a);
    q.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = q;
  }
};

// One thread per (V channels, fe_tokens<T>()-token run): grid (token runs, channel tiles of
// 256 * V, batch rows).  V = 4 needs H * P to be a multiple of 4 (then no group of four
// straddles the x | B | C boundaries, and every vector access is aligned).
template <typename T, int V>
__global__ void __launch_bounds__(256, 4)
k_frontend(const T *__restrict__ xbc, const float *__restrict__ w, const float *__restrict__ bias,
           const float *__restrict__ state_in, const float *dt_raw, const float *__restrict__ dt_bias,
           T *__restrict__ x, T *__restrict__ B, T *__restrict__ C, float *dt, Dims d) {
  const int HP = d.H * d.P, GN = d.G * d.N, CH = HP + 2 * GN;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * V;
  constexpr int kFeTokens = fe_tokens<T>();
  const int t0 = blockIdx.x * kFeTokens, bi = blockIdx.z;
  const int t1 = min(t0 + kFeTokens, d.L);
  // Stage this CTA's inputs -- rows t0-3 .. t1-1 of its 256 * V channels -- in shared
  // memory with asynchronous copies (nothing held in registers while they fly): with 4
  // channels a thread, one bulk copy per row, the rows spread over the eight warps (a
  // thread completes about one bulk copy per half microsecond), each warp arriving on the
  // mbarrier with its own byte count; otherwise a cp.async per thread and row.  Rows before
  // the sequence come from the conv state or are zero.
  __shared__ __align__(16) T tile[3 + kFeTokens][256 * V];
  __shared__ uint64_t rows_full;
  const int tl = threadIdx.x * V;  // this thread's first channel within the tile
  const bool active = c < CH;
  const int cbase = blockIdx.y * 256 * V, nch = min(256 * V, CH - cbase);
  const bool bulk = V == 4 && (nch * (int)sizeof(T)) % 16 == 0 && ((size_t)CH * sizeof(T)) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(xbc) % 16 == 0;
  const T *uc = xbc + (size_t)bi * d.L * CH + c;
  const int nwarps = blockDim.x >> 5, warp = threadIdx.x >> 5;
  if (bulk) {
    if (threadIdx.x == 0) {
      sm100::mbar_init(&rows_full, nwarps);
      sm100::mbar_fence_init();
    }
    __syncthreads();  // the barrier is initialised before any thread arrives on it
    if ((threadIdx.x & 31) == 0) {
      uint32_t bytes = 0;
      for (int j = warp; j < 3 + kFeTokens; j += nwarps) {
        const int t = t0 - 3 + j;
        if (t >= 0 && t < t1) bytes += (uint32_t)nch * sizeof(T);
      }
      sm100::mbar_arrive_expect_tx(&rows_full, bytes);
      for (int j = warp; j < 3 + kFeTokens; j += nwarps) {
        const int t = t0 - 3 + j;
        if (t >= 0 && t < t1)
          sm100::bulk_load(&tile[j][0], xbc + ((size_t)bi * d.L + t) * CH + cbase, (uint32_t)nch * sizeof(T),
                           &rows_full);
      }
    }
  } else if (active) {
#pragma unroll
    for (int j = 0; j < 3 + kFeTokens; ++j) {
      const int t = t0 - 3 + j;
      if (t >= 0 && t < t1) {
        if constexpr (sizeof(T) * V >= 4)
          cp_async<sizeof(T) * V>(&tile[j][tl], uc + (size_t)t * CH);
        else
          tile[j][tl] = uc[(size_t)t * CH];  // the scalar bf16 fallback (2 bytes)
      }
    }
  }
  if (active)
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int t = t0 - 3 + j;
      if (t < 0)
#pragma unroll
        for (int q = 0; q < V; ++q)
          tile[j][tl + q] = from_f32<T>(state_in ? state_in[((size_t)bi * 3 + (3 + t)) * CH + c + q] : 0.f);
    }
  if (blockIdx.y == 0) {  // dt for this run of tokens (all loads issued before any use)
    for (int h = threadIdx.x; h < d.H; h += blockDim.x) {
      const float bh = dt_bias[h];
      float z[kFeTokens];
#pragma unroll
      for (int j = 0; j < kFeTokens; ++j)
        z[j] = (t0 + j < t1) ? dt_raw[((size_t)bi * d.L + t0 + j) * d.H + h] : 0.f;
#pragma unroll
      for (int j = 0; j < kFeTokens; ++j)
        if (t0 + j < t1) dt[((size_t)bi * d.L + t0 + j) * d.H + h] = softplus_f(z[j] + bh);
    }
  }
  // the filters while the copies fly
  float4 wc[V];
  float bc[V];
#pragma unroll
  for (int q = 0; q < V; ++q) {
    wc[q] = active ? *reinterpret_cast<const float4 *>(w + (size_t)(c + q) * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    bc[q] = (active && bias) ? bias[c + q] : 0.f;
  }
  // the copies have landed (bounded wait: after 2 s the CTA gives up, its outputs undefined)
  const bool landed = bulk ? sm100::mbar_wait_drain(&rows_full, 0) : (cp_async_wait_all(), true);
  __syncthreads();
  if (!active || !landed) return;
  T *dst;
  size_t stride;
  if (c < HP) {
    dst = x + (size_t)bi * d.L * HP + c;
    stride = HP;
  } else if (c < HP + GN) {
    dst = B + (size_t)bi * d.L * GN + (c - HP);
    stride = GN;
  } else {
    dst = C + (size_t)bi * d.L * GN + (c - HP - GN);
    stride = GN;
  }
  // each token from its four input rows in shared memory (a rolling window of rows)
  float r0[V], r1[V], r2[V];
  Vec<T, V>::load(&tile[0][tl], r0);
  Vec<T, V>::load(&tile[1][tl], r1);
  Vec<T, V>::load(&tile[2][tl], r2);
#pragma unroll
  for (int j = 0; j < kFeTokens; ++j) {
    if (t0 + j < t1) {
      float r3[V], o[V];
      Vec<T, V>::load(&tile[3 + j][tl], r3);
#pragma unroll
      for (int q = 0; q < V; ++q) {
        o[q] = silu_out<T>(fmaf(wc[q].x, r0[q], fmaf(wc[q].y, r1[q], fmaf(wc[q].z, r2[q], fmaf(wc[q].w, r3[q], bc[q])))));
        r0[q] = r1[q];
        r1[q] = r2[q];
        r2[q] = r3[q];
      }
      Vec<T, V>::store(dst + (size_t)(t0 + j) * stride, o);
    }
  }
}

// The streaming form, for 4 channels a thread when every row of a tile is a whole number
// of 16-byte units: one CTA per (range of tokens, channel tile of 1024, batch row), sized
// to about three CTAs per SM.  The range is walked in runs of R tokens through kFeBufs
// shared-memory buffers, each filled by one bulk copy per row on its own mbarrier, so that
// the next runs are in flight while one is computed; the last three inputs of a run stay
// in registers as the first taps of the next, so only the range's first three rows are
// read twice.  dt is formed for the range by every tile, each for its share of the heads.
constexpr int kFeBufs = 2;
template <typename T> constexpr int fe_run() { return sizeof(T) == 2 ? 16 : 8; }  // rows of 2 or 4 KB
template <typename T> constexpr size_t fe_stream_smem() { return (size_t)kFeBufs * fe_run<T>() * 1024 * sizeof(T); }

template <typename T>
__global__ void __launch_bounds__(256, 3)
k_frontend_stream(const T *__restrict__ xbc, const float *__restrict__ w, const float *__restrict__ bias,
                  const float *__restrict__ state_in, const float *dt_raw, const float *__restrict__ dt_bias,
                  T *__restrict__ x, T *__restrict__ B, T *__restrict__ C, float *dt, Dims d, int range) {
  constexpr int V = 4, R = fe_run<T>();
  extern __shared__ __align__(16) uint8_t fe_smem[];
  T(*buf)[R][256 * V] = reinterpret_cast<T(*)[R][256 * V]>(fe_smem);
  __shared__ uint64_t full[kFeBufs];
  const int HP = d.H * d.P, GN = d.G * d.N, CH = HP + 2 * GN;
  const int cbase = blockIdx.y * 256 * V, nch = min(256 * V, CH - cbase);
  const int c = cbase + threadIdx.x * V;
  const int T0 = blockIdx.x * range, bi = blockIdx.z;
  const int T1 = min(T0 + range, d.L);
  const int tl = threadIdx.x * V;
  const bool active = c < CH;
  const int nruns = (T1 - T0 + R - 1) / R;
  const T *rows = xbc + (size_t)bi * d.L * CH + cbase;  // row t of this tile at rows + t * CH
  // run i into buffer i % kFeBufs: one bulk copy per row, the rows spread over the eight
  // warps (lane 0 of each), each arriving on the buffer's barrier with its own byte count
  const int nwarps = blockDim.x >> 5, warp = threadIdx.x >> 5;
  auto issue = [&](int i) {
    const int ta = T0 + i * R, nr = min(R, T1 - ta);
    uint64_t *bar = &full[i % kFeBufs];
    uint32_t bytes = 0;
    for (int j = warp; j < nr; j += nwarps) bytes += (uint32_t)nch * sizeof(T);
    sm100::mbar_arrive_expect_tx(bar, bytes);
    for (int j = warp; j < nr; j += nwarps)
      sm100::bulk_load(&buf[i % kFeBufs][j][0], rows + (size_t)(ta + j) * CH, (uint32_t)nch * sizeof(T), bar);
  };
  if (threadIdx.x == 0) {
    for (int b = 0; b < kFeBufs; ++b) sm100::mbar_init(&full[b], nwarps);
    sm100::mbar_fence_init();
  }
  __syncthreads();  // the barriers are initialised before any warp arrives on them
  if ((threadIdx.x & 31) == 0)
    for (int i = 0; i < kFeBufs && i < nruns; ++i) issue(i);
  {  // dt for this range of tokens and this tile's share of the heads
    const int per = (d.H + gridDim.y - 1) / gridDim.y, hlo = blockIdx.y * per, nhs = min(per, d.H - hlo);
    const int count = nhs > 0 ? (T1 - T0) * nhs : 0;
    for (int i = threadIdx.x; i < count; i += blockDim.x) {
      const int t = T0 + i / nhs, h = hlo + i % nhs;
      const size_t at = ((size_t)bi * d.L + t) * d.H + h;
      dt[at] = softplus_f(dt_raw[at] + dt_bias[h]);
    }
  }
  // the three inputs before the range: earlier tokens, the conv state, or zero
  float win[3][V];
  float4 wc[V];
  float bc[V];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int t = T0 - 3 + j;
#pragma unroll
    for (int q = 0; q < V; ++q) win[j][q] = 0.f;
    if (active) {
      if (t >= 0)
        Vec<T, V>::load(xbc + ((size_t)bi * d.L + t) * CH + c, win[j]);
      else if (state_in)
#pragma unroll
        for (int q = 0; q < V; ++q) win[j][q] = state_in[((size_t)bi * 3 + (3 + t)) * CH + c + q];
    }
  }
#pragma unroll
  for (int q = 0; q < V; ++q) {
    wc[q] = active ? *reinterpret_cast<const float4 *>(w + (size_t)(c + q) * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    bc[q] = (active && bias) ? bias[c + q] : 0.f;
  }
  T *dst = nullptr;
  size_t stride = 0;
  if (c < HP) {
    dst = x + (size_t)bi * d.L * HP + c;
    stride = HP;
  } else if (c < HP + GN) {
    dst = B + (size_t)bi * d.L * GN + (c - HP);
    stride = GN;
  } else {
    dst = C + (size_t)bi * d.L * GN + (c - HP - GN);
    stride = GN;
  }
  bool ok = true;
  int waited = 0;  // runs whose copies this thread has seen land
  for (int i = 0; i < nruns; ++i) {
    // bounded wait (1 s): on expiry the CTA stops; its remaining outputs are undefined
    ok = ok && sm100::mbar_wait_drain(&full[i % kFeBufs], (uint32_t)((i / kFeBufs) & 1));
    if (ok) waited = i + 1;
    const int ta = T0 + i * R;
    if (ok && active) {
#pragma unroll
      for (int j = 0; j < R; ++j) {
        if (ta + j < T1) {
          float r3[V], o[V];
          Vec<T, V>::load(&buf[i % kFeBufs][j][tl], r3);
#pragma unroll
          for (int q = 0; q < V; ++q) {
            o[q] = silu_out<T>(fmaf(wc[q].x, win[0][q], fmaf(wc[q].y, win[1][q], fmaf(wc[q].z, win[2][q], fmaf(wc[q].w, r3[q], bc[q])))));
            win[0][q] = win[1][q];
            win[1][q] = win[2][q];
            win[2][q] = r3[q];
          }
          Vec<T, V>::store(dst + (size_t)(ta + j) * stride, o);
        }
      }
    }
    __syncthreads();  // every thread has read buffer i % kFeBufs
    if ((threadIdx.x & 31) == 0 && ok && i + kFeBufs < nruns) issue(i + kFeBufs);
  }
  if (!ok && threadIdx.x == 0) {  // let this CTA's own copies land before it exits
    const int issued = min(nruns, waited + kFeBufs);
    for (int i = waited; i < issued; ++i) sm100::mbar_wait_drain(&full[i % kFeBufs], (uint32_t)((i / kFeBufs) & 1));
  }
}

// new_state[j, c] = input at token L - 3 + j (j = 0..2), from this call's tokens or, when
// L < 3, from the old state; each thread reads all it needs before it writes.
template <typename T>
__global__ void __launch_bounds__(256)
k_frontend_state(const T *__restrict__ xbc, const float *state_in, float *state_out, Dims d) {
  const int CH = d.H * d.P + 2 * d.G * d.N;
  const int c = blockIdx.x * blockDim.x + threadIdx.x, bi = blockIdx.y;
  if (c >= CH) return;
  float v[3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int t = d.L - 3 + j;
    v[j] = t >= 0 ? to_f32(xbc[((size_t)bi * d.L + t) * CH + c])
                  : (state_in ? state_in[((size_t)bi * 3 + (3 + t)) * CH + c] : 0.f);
  }
#pragma unroll
  for (int j = 0; j < 3; ++j) state_out[((size_t)bi * 3 + j) * CH + c] = v[j];
}

template <typename T>
cudaError_t launch_frontend(const T *xbc, const float *w, const float *bias, const float *state_in,
                            float *state_out, const float *dt_raw, const float *dt_bias, T *x, T *B, T *C, float *dt,
                            const Dims &d, cudaStream_t st) {
  const int CH = d.H * d.P + 2 * d.G * d.N;
  // token runs on x (up to 2^31 - 1), channel tiles on y and batch rows on z (the host
  // checks both stay within 65535)
  const unsigned runs = (unsigned)((d.L + fe_tokens<T>() - 1) / fe_tokens<T>());
  cudaError_t e;
  // the streaming kernel: ranges of tokens sized for about three CTAs per SM over the
  // channel tiles and batch rows, each a multiple of the run length; worth it once a range
  // holds enough runs to keep its copies ahead (measured: 19 runs gain 5 %, 4 runs lose 7 %
  // against one tile per CTA)
  static const int sms = [] {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
  }();
  const int tiles = (CH + 1023) / 1024, R = fe_run<T>();
  const long want = std::max(1L, (3L * sms + (long)tiles * d.b - 1) / ((long)tiles * d.b));
  int range = (int)std::min<long>(d.L, (d.L + want - 1) / want);
  range = (range + R - 1) / R * R;
  if ((d.H * d.P) % 4 == 0 && ((size_t)CH * sizeof(T)) % 16 == 0 && reinterpret_cast<uintptr_t>(xbc) % 16 == 0 &&
      range >= 8 * R) {
    const unsigned nranges = (unsigned)((d.L + range - 1) / range);
    e = cudaFuncSetAttribute(k_frontend_stream<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fe_stream_smem<T>());
    if (e != cudaSuccess) return e;
    k_frontend_stream<T><<<dim3(nranges, (unsigned)tiles, (unsigned)d.b), 256, fe_stream_smem<T>(), st>>>(
        xbc, w, bias, state_in, dt_raw, dt_bias, x, B, C, dt, d, range);
  } else if ((d.H * d.P) % 4 == 0) {
    k_frontend<T, 4><<<dim3(runs, (unsigned)((CH / 4 + 255) / 256), (unsigned)d.b), 256, 0, st>>>(
        xbc, w, bias, state_in, dt_raw, dt_bias, x, B, C, dt, d);
  } else {
    k_frontend<T, 1><<<dim3(runs, (unsigned)((CH + 255) / 256), (unsigned)d.b), 256, 0, st>>>(
        xbc, w, bias, state_in, dt_raw, dt_bias, x, B, C, dt, d);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || state_out == nullptr) return e;
  k_frontend_state<T><<<dim3((unsigned)((CH + 255) / 256), (unsigned)d.b), 256, 0, st>>>(xbc, state_in, state_out, d);
  return cudaGetLastError();
}

template cudaError_t launch_frontend<float>(const float *, const float *, const float *, const float *, float *,
                                            const float *, const float *, float *, float *, float *, float *,
                                            const Dims &, cudaStream_t);
template cudaError_t launch_frontend<__nv_bfloat16>(const __nv_bfloat16 *, const float *, const float *, const float *,
                                                    float *, const float *, const float *, __nv_bfloat16 *,
                                                    __nv_bfloat16 *, __nv_bfloat16 *, float *, const Dims &,
                                                    cudaStream_t);

}  // namespace ssd
