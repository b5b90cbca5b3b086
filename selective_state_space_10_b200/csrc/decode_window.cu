// decode_window.cu -- windowed cached decode: the state is read every step but written
// only once per window of W buffered tokens (ReplaySSM, as summarised in "SketchSSM:
// Write to the Full State, Read from a Compact Sketch", abstract and Table 4: read D,
// write D/W per state head per decode step, against read D + write D for the standard
// step).
//
// With h0 the committed state and tokens s = 0 .. pos of the current window (s = pos the
// new one), cum_s = sum_{i <= s} dt_i A_h:
//
//   y_pos[p] = exp(cum_pos) sum_n C[n] h0[p,n]
//            + sum_{s <= pos} exp(cum_pos - cum_s) dt_s (C . B_s) x_s[p] + D_h x_pos[p]
//
// which is the recurrence of "Engineering Hybrid State-Space Models" section 2 unrolled
// over the window (the same sum the chunked form uses inside a chunk).  The flush folds
// the window into the state:
//
//   h0[p,n] <- exp(cum_last) h0[p,n] + sum_s exp(cum_last - cum_s) dt_s x_s[p] B_s[n].
//
// Both kernels: one CTA of 256 threads per (batch row, head); state rows are covered as
// in the single-step decode kernel (LPR lanes per row with float4 accesses, all loads of
// a pass in flight before any arithmetic).  The step issues its state loads first and
// forms the window's terms while they fly; the flush stages the window's tokens in shared
// memory, already weighted by their decay coefficients.  Window lengths up to 16.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

constexpr int kWinMax = 16;
constexpr int kPMax = 256;

// The window's decay scan, by the 32 lanes of one warp (lane s holds dt_s, 0 past the
// window's n tokens): dec[s] = exp(cum_last - cum_s) dt_s for s < n and
// dec[kWinMax] = exp(cum_last), cum_s = sum_{i <= s} dt_i A_h.
__device__ __forceinline__ void window_decays(int n, float Ah, float dts, float *dec) {
  const int lane = threadIdx.x & 31;
  float cum = dts * Ah;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, cum, o);
    if (lane >= o) cum += u;
  }
  const float last = __shfl_sync(0xffffffffu, cum, (n - 1) & 31);
  if (lane < n) dec[lane] = expf(last - cum) * dts;
  if (lane == 0) dec[kWinMax] = expf(last);
}

template <typename T, int N>
__global__ void __launch_bounds__(256, 4)
k_decode_window_step(const float *__restrict__ state, T *__restrict__ win_x, float *__restrict__ win_dt,
                     T *__restrict__ win_B, int W, int pos, const T *__restrict__ x, const float *__restrict__ dt,
                     const float *__restrict__ A, const T *__restrict__ B, const T *__restrict__ C,
                     const float *__restrict__ D, float *__restrict__ y, Dims d) {
  constexpr int NV = N / 4;
  constexpr int LPR = NV < 32 ? NV : 32;
  constexpr int VPL = NV / LPR;
  constexpr int RPW = 32 / LPR;
  constexpr int ROWS = 8 * RPW;
  constexpr int UNR = (8 / (RPW * VPL)) > 0 ? 8 / (RPW * VPL) : 1;
  __shared__ float dec[kWinMax + 1];    // exp(cum_pos - cum_s) dt_s; [kWinMax]: exp(cum_pos)
  __shared__ float qs[kWinMax];         // C . B_s
  __shared__ float wsum[kPMax];         // the window's sum, this token included

  const int bh = blockIdx.x;
  const int bi = bh / d.H, h = bh - bi * d.H;
  const int g = h / d.hpg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, l = lane % LPR;
  const int n = pos + 1;  // tokens of the window including this one
  const float Ah = A[h];
  const float dtv = dt[bh];
  const size_t wtok = (size_t)bi * W;  // first window slot of this batch row
  const T *Cg = C + ((size_t)bi * d.G + g) * N;
  const float4 *st = reinterpret_cast<const float4 *>(state) + (size_t)bh * d.P * NV;

  // The first pass of the state (the whole of it for P <= 8 * ROWS) and C are loaded
  // before the window bookkeeping, so that the step's HBM traffic is in flight while the
  // window terms are formed.
  float4 cv[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) cv[v] = load4(Cg + (size_t)(v * LPR + l) * 4);
  float4 hv[UNR][VPL];
#pragma unroll
  for (int u = 0; u < UNR; ++u) {
    const int row = u * ROWS + warp * RPW + sub;
    if (row < d.P) {
#pragma unroll
      for (int v = 0; v < VPL; ++v) hv[u][v] = __ldcs(st + (size_t)row * NV + v * LPR + l);
    }
  }

  // Every global load of the window bookkeeping is issued here, before any of it is
  // used: the window's dt (warp 0), the B_s rows of the C . B_s dots (warp w: tokens w
  // and w + 8) and the window's x values.  For the window sum, four threads share a channel
  // (thread 4p' + j of a block of 64 channels holds x_s for s = j, j + 4, j + 8, j + 12)
  // and add their partial sums with two shuffles, so no thread walks the whole window.
  float dts = 0.f;
  if (warp == 0 && lane < n) dts = lane < pos ? win_dt[(wtok + lane) * d.H + h] : dtv;
  float q[2] = {0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int s = warp + 8 * j;
    if (s < n) {
      const T *Bs = (s < pos) ? win_B + ((wtok + s) * d.G + g) * N : B + ((size_t)bi * d.G + g) * N;
#pragma unroll
      for (int k = lane * 4; k < N; k += 128) {
        const float4 c4 = load4(Cg + k), b4 = load4(Bs + k);
        q[j] = fmaf(c4.x, b4.x, fmaf(c4.y, b4.y, fmaf(c4.z, b4.z, fmaf(c4.w, b4.w, q[j]))));
      }
    }
  }
  const T *wxh = win_x + (wtok * d.H + h) * (size_t)d.P;  // slot s of this head at s * H * P
  const T *xh = x + (size_t)bh * d.P;
  const int pj = threadIdx.x >> 2, jw = threadIdx.x & 3;   // channel within a block of 64, window phase
  float xw[kWinMax / 4];
#pragma unroll
  for (int i = 0; i < kWinMax / 4; ++i) {  // the first block of channels, loaded up front
    const int s = jw + 4 * i;
    xw[i] = (pj < d.P && s < pos) ? to_f32(wxh[(size_t)s * d.H * d.P + pj]) : 0.f;
  }
  if (warp == 0) window_decays(n, Ah, dts, dec);  // dec[s] = exp(cum_pos - cum_s) dt_s, dec[kWinMax] = exp(cum_pos)
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float qq = warp_sum(q[j], 32);
    if (lane == 0 && warp + 8 * j < n) qs[warp + 8 * j] = qq;
  }
  __syncthreads();
  // wsum[p] = sum_{s <= pos} dec_s (C . B_s) x_s[p]
  for (int pb = 0; pb < d.P; pb += 64) {
    const int p = pb + pj;
    if (pb > 0) {  // later blocks (P > 64)
#pragma unroll
      for (int i = 0; i < kWinMax / 4; ++i) {
        const int s = jw + 4 * i;
        xw[i] = (p < d.P && s < pos) ? to_f32(wxh[(size_t)s * d.H * d.P + p]) : 0.f;
      }
    }
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < kWinMax / 4; ++i) {
      const int s = jw + 4 * i;
      if (s < pos) part = fmaf(dec[s] * qs[s], xw[i], part);
    }
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if (jw == 0 && p < d.P) wsum[p] = fmaf(dec[pos] * qs[pos], to_f32(xh[p]), part);
  }
  __syncthreads();

  // this token joins the window (slot pos); B once per group, by its first head
  T *slot_x = win_x + ((wtok + pos) * d.H + h) * (size_t)d.P;
  for (int p = threadIdx.x; p < d.P; p += blockDim.x) slot_x[p] = xh[p];
  if (threadIdx.x == 0) win_dt[(wtok + pos) * d.H + h] = dtv;
  if (h % d.hpg == 0)
    for (int k = threadIdx.x; k < N; k += blockDim.x)
      win_B[((wtok + pos) * d.G + g) * N + k] = B[((size_t)bi * d.G + g) * N + k];

  float *yh = y + (size_t)bh * d.P;
  const float Dh = D[h], tot = dec[kWinMax];
  for (int r0 = 0; r0 < d.P; r0 += ROWS * UNR) {
    if (r0 > 0) {  // later passes (P > 8 * ROWS)
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int row = r0 + u * ROWS + warp * RPW + sub;
        if (row < d.P) {
#pragma unroll
          for (int v = 0; v < VPL; ++v) hv[u][v] = __ldcs(st + (size_t)row * NV + v * LPR + l);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int row = r0 + u * ROWS + warp * RPW + sub;
      float acc = 0.f;
      if (row < d.P) {
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          acc = fmaf(cv[v].x, hv[u][v].x, acc);
          acc = fmaf(cv[v].y, hv[u][v].y, acc);
          acc = fmaf(cv[v].z, hv[u][v].z, acc);
          acc = fmaf(cv[v].w, hv[u][v].w, acc);
        }
      }
      acc = warp_sum(acc, LPR);
      if (l == 0 && row < d.P) yh[row] = fmaf(tot, acc, wsum[row]) + Dh * to_f32(xh[row]);
    }
  }
}

template <typename T, int N>
__global__ void __launch_bounds__(256, 4)
k_decode_window_flush(float *__restrict__ state, const T *__restrict__ win_x, const float *__restrict__ win_dt,
                      const T *__restrict__ win_B, int W, int count, const float *__restrict__ A, Dims d) {
  constexpr int NV = N / 4;
  constexpr int LPR = NV < 32 ? NV : 32;
  constexpr int VPL = NV / LPR;
  constexpr int RPW = 32 / LPR;
  constexpr int ROWS = 8 * RPW;
  constexpr int UNR = (8 / (RPW * VPL)) > 0 ? 8 / (RPW * VPL) : 1;
  __shared__ float dec[kWinMax + 1];                   // exp(cum_last - cum_s) dt_s; [kWinMax]: exp(cum_last)
  __shared__ float wx[kWinMax][kPMax];                 // dec_s x_s[p]
  __shared__ __align__(16) float wb[kWinMax][N];       // B_s[n]

  const int bh = blockIdx.x;
  const int bi = bh / d.H, h = bh - bi * d.H;
  const int g = h / d.hpg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, l = lane % LPR;
  const size_t wtok = (size_t)bi * W;
  float4 *st = reinterpret_cast<float4 *>(state) + (size_t)bh * d.P * NV;
  float4 hv[UNR][VPL];  // the first pass of the state, loaded before the window bookkeeping
#pragma unroll
  for (int u = 0; u < UNR; ++u) {
    const int row = u * ROWS + warp * RPW + sub;
    if (row < d.P) {
#pragma unroll
      for (int v = 0; v < VPL; ++v) hv[u][v] = __ldcs(st + (size_t)row * NV + v * LPR + l);
    }
  }
  // the window's data: the first kFlushStage values of x and of B per thread are loaded
  // together before any use, the rest (larger windows, P or N) by the loops below
  const float dts = (warp == 0 && lane < count) ? win_dt[(wtok + lane) * d.H + h] : 0.f;
  const T *wxh = win_x + (wtok * d.H + h) * (size_t)d.P;  // slot s of this head at s * H * P
  const T *wbg = win_B + (wtok * d.G + g) * (size_t)N;    // slot s of this group at s * G * N
  const int nx = count * d.P, nb = count * N;
  constexpr int kFlushStage = 4;  // values of x and of B each thread loads up front
  float xr[kFlushStage], br[kFlushStage];
#pragma unroll
  for (int j = 0; j < kFlushStage; ++j) {
    const int i = threadIdx.x + 256 * j;
    xr[j] = 0.f;
    br[j] = 0.f;
    if (i < nx) {
      const int s = i / d.P;
      xr[j] = to_f32(wxh[(size_t)s * d.H * d.P + (i - s * d.P)]);
    }
    if (i < nb) {
      const int s = i / N;
      br[j] = to_f32(wbg[(size_t)s * d.G * N + (i - s * N)]);
    }
  }
  if (warp == 0) window_decays(count, A[h], dts, dec);
  __syncthreads();
  const float tot = dec[kWinMax];
#pragma unroll
  for (int j = 0; j < kFlushStage; ++j) {
    const int i = threadIdx.x + 256 * j;
    if (i < nx) {
      const int s = i / d.P;
      wx[s][i - s * d.P] = dec[s] * xr[j];
    }
    if (i < nb) {
      const int s = i / N;
      wb[s][i - s * N] = br[j];
    }
  }
  for (int i = threadIdx.x + 256 * kFlushStage; i < nx; i += blockDim.x) {
    const int s = i / d.P;
    wx[s][i - s * d.P] = dec[s] * to_f32(wxh[(size_t)s * d.H * d.P + (i - s * d.P)]);
  }
#pragma unroll 4
  for (int i = threadIdx.x + 256 * kFlushStage; i < nb; i += blockDim.x) {
    const int s = i / N;
    wb[s][i - s * N] = to_f32(wbg[(size_t)s * d.G * N + (i - s * N)]);
  }
  __syncthreads();

  for (int r0 = 0; r0 < d.P; r0 += ROWS * UNR) {
    if (r0 > 0) {
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int row = r0 + u * ROWS + warp * RPW + sub;
        if (row < d.P) {
#pragma unroll
          for (int v = 0; v < VPL; ++v) hv[u][v] = __ldcs(st + (size_t)row * NV + v * LPR + l);
        }
      }
    }
    // token-outer: each B_s chunk is read from shared memory once and used for all of
    // this thread's rows of the pass
#pragma unroll
    for (int u = 0; u < UNR; ++u)
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        hv[u][v].x *= tot;
        hv[u][v].y *= tot;
        hv[u][v].z *= tot;
        hv[u][v].w *= tot;
      }
    for (int s = 0; s < count; ++s) {
      float4 b4[VPL];
#pragma unroll
      for (int v = 0; v < VPL; ++v) b4[v] = *reinterpret_cast<const float4 *>(&wb[s][(v * LPR + l) * 4]);
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int row = r0 + u * ROWS + warp * RPW + sub;
        const float cx = row < d.P ? wx[s][row] : 0.f;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          hv[u][v].x = fmaf(cx, b4[v].x, hv[u][v].x);
          hv[u][v].y = fmaf(cx, b4[v].y, hv[u][v].y);
          hv[u][v].z = fmaf(cx, b4[v].z, hv[u][v].z);
          hv[u][v].w = fmaf(cx, b4[v].w, hv[u][v].w);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int row = r0 + u * ROWS + warp * RPW + sub;
      if (row >= d.P) continue;
#pragma unroll
      for (int v = 0; v < VPL; ++v) __stcs(st + (size_t)row * NV + v * LPR + l, hv[u][v]);
    }
  }
}

template <typename T>
cudaError_t launch_decode_window_step(const float *state, T *win_x, float *win_dt, T *win_B, int W, int pos,
                                      const T *x, const float *dt, const float *A, const T *B, const T *C,
                                      const float *D, float *y, const Dims &d, cudaStream_t st) {
  const dim3 grid((unsigned)((size_t)d.b * d.H));
#define SSD_WSTEP(NN)                                                                                              \
  k_decode_window_step<T, NN><<<grid, 256, 0, st>>>(state, win_x, win_dt, win_B, W, pos, x, dt, A, B, C, D, y, \
                                                       d)
  switch (d.N) {
    case 16: SSD_WSTEP(16); break;
    case 32: SSD_WSTEP(32); break;
    case 64: SSD_WSTEP(64); break;
    case 128: SSD_WSTEP(128); break;
    case 256: SSD_WSTEP(256); break;
    default: return cudaErrorInvalidValue;
  }
#undef SSD_WSTEP
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_decode_window_flush(float *state, const T *win_x, const float *win_dt, const T *win_B, int W,
                                       int count, const float *A, const Dims &d, cudaStream_t st) {
  const dim3 grid((unsigned)((size_t)d.b * d.H));
  switch (d.N) {
    case 16: k_decode_window_flush<T, 16><<<grid, 256, 0, st>>>(state, win_x, win_dt, win_B, W, count, A, d); break;
    case 32: k_decode_window_flush<T, 32><<<grid, 256, 0, st>>>(state, win_x, win_dt, win_B, W, count, A, d); break;
    case 64: k_decode_window_flush<T, 64><<<grid, 256, 0, st>>>(state, win_x, win_dt, win_B, W, count, A, d); break;
    case 128: k_decode_window_flush<T, 128><<<grid, 256, 0, st>>>(state, win_x, win_dt, win_B, W, count, A, d); break;
    case 256: k_decode_window_flush<T, 256><<<grid, 256, 0, st>>>(state, win_x, win_dt, win_B, W, count, A, d); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template cudaError_t launch_decode_window_step<float>(const float *, float *, float *, float *, int, int,
                                                      const float *, const float *, const float *, const float *,
                                                      const float *, const float *, float *, const Dims &,
                                                      cudaStream_t);
template cudaError_t launch_decode_window_step<__nv_bfloat16>(const float *, __nv_bfloat16 *, float *,
                                                              __nv_bfloat16 *, int, int, const __nv_bfloat16 *,
                                                              const float *, const float *, const __nv_bfloat16 *,
                                                              const __nv_bfloat16 *, const float *, float *,
                                                              const Dims &, cudaStream_t);
template cudaError_t launch_decode_window_flush<float>(float *, const float *, const float *, const float *, int, int,
                                                       const float *, const Dims &, cudaStream_t);
template cudaError_t launch_decode_window_flush<__nv_bfloat16>(float *, const __nv_bfloat16 *, const float *,
                                                               const __nv_bfloat16 *, int, int, const float *,
                                                               const Dims &, cudaStream_t);

}  // namespace ssd
