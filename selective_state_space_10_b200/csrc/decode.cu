// decode.cu -- one cached single-token decode step, in place on the fp32 state.
//
//   a = exp(dt A_h);  h[p,n] <- a h[p,n] + dt x[p] B[n];  y[p] = sum_n C[n] h[p,n] + D_h x[p]
//
// The recurrent mode of the layer ("Mamba and Selective State Space Models" section 3;
// "Compiler-First State Space Duality ..." abstract: O(1) per step).  The step is bound
// by HBM: each head's P x N fp32 state is read once and written once (the "Standard"
// traffic of 2 x state bytes per head per step in "SketchSSM: Write to the Full State,
// Read from a Compact Sketch", Table 4) and everything else is a few KB.
//
// One CTA of 256 threads per (batch row, head).  A row of the state (N fp32) is covered
// by LPR lanes with float4 accesses; every thread issues all of its state loads before
// any arithmetic (UNR rows x VPL vectors in flight), then writes back with streaming
// stores.  The y reduction over n is a shuffle across the LPR lanes of a row.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

template <typename T, int N>
__global__ void __launch_bounds__(256)
k_decode_step(float *__restrict__ state, const T *__restrict__ x, const float *__restrict__ dt,
              const float *__restrict__ A, const T *__restrict__ B, const T *__restrict__ C,
              const float *__restrict__ D, float *__restrict__ y, Dims d) {
  constexpr int NV = N / 4;                 // float4 per state row
  constexpr int LPR = NV < 32 ? NV : 32;    // lanes per row
  constexpr int VPL = NV / LPR;             // float4 per lane per row
  constexpr int RPW = 32 / LPR;             // rows per warp per pass
  constexpr int ROWS = 8 * RPW;             // rows per CTA per pass (8 warps)
  constexpr int UNR = (8 / (RPW * VPL)) > 0 ? 8 / (RPW * VPL) : 1;  // passes in flight

  const int bh = blockIdx.x;
  const int bi = bh / d.H, h = bh - bi * d.H;
  const int g = h / d.hpg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, l = lane % LPR;

  const float dtv = dt[bh];
  const float a = expf(dtv * A[h]);
  const float Dh = D[h];
  float4 bv[VPL], cv[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const size_t off = ((size_t)bi * d.G + g) * N + (size_t)(v * LPR + l) * 4;
    bv[v] = load4(B + off);
    cv[v] = load4(C + off);
  }
  float4 *st = reinterpret_cast<float4 *>(state) + (size_t)bh * d.P * NV;
  const T *xh = x + (size_t)bh * d.P;
  float *yh = y + (size_t)bh * d.P;

  for (int r0 = 0; r0 < d.P; r0 += ROWS * UNR) {
    float4 hv[UNR][VPL];
    float xv[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int row = r0 + u * ROWS + warp * RPW + sub;
      xv[u] = 0.f;
      if (row < d.P) {
        xv[u] = to_f32(xh[row]);
#pragma unroll
        for (int v = 0; v < VPL; ++v) hv[u][v] = __ldcs(st + (size_t)row * NV + v * LPR + l);
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int row = r0 + u * ROWS + warp * RPW + sub;
      float acc = 0.f;
      if (row < d.P) {
        const float dx = dtv * xv[u];
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          float4 hn;
          hn.x = fmaf(a, hv[u][v].x, dx * bv[v].x);
          hn.y = fmaf(a, hv[u][v].y, dx * bv[v].y);
          hn.z = fmaf(a, hv[u][v].z, dx * bv[v].z);
          hn.w = fmaf(a, hv[u][v].w, dx * bv[v].w);
          acc = fmaf(cv[v].x, hn.x, acc);
          acc = fmaf(cv[v].y, hn.y, acc);
          acc = fmaf(cv[v].z, hn.z, acc);
          acc = fmaf(cv[v].w, hn.w, acc);
          __stcs(st + (size_t)row * NV + v * LPR + l, hn);
        }
      }
      acc = warp_sum(acc, LPR);
      if (l == 0 && row < d.P) yh[row] = acc + Dh * xv[u];
    }
  }
}

template <typename T>
cudaError_t launch_decode_step(float *state, const T *x, const float *dt, const float *A, const T *B,
                               const T *C, const float *D, float *y, const Dims &d, cudaStream_t st) {
  const dim3 grid((unsigned)((size_t)d.b * d.H));
  switch (d.N) {
    case 16: k_decode_step<T, 16><<<grid, 256, 0, st>>>(state, x, dt, A, B, C, D, y, d); break;
    case 32: k_decode_step<T, 32><<<grid, 256, 0, st>>>(state, x, dt, A, B, C, D, y, d); break;
    case 64: k_decode_step<T, 64><<<grid, 256, 0, st>>>(state, x, dt, A, B, C, D, y, d); break;
    case 128: k_decode_step<T, 128><<<grid, 256, 0, st>>>(state, x, dt, A, B, C, D, y, d); break;
    case 256: k_decode_step<T, 256><<<grid, 256, 0, st>>>(state, x, dt, A, B, C, D, y, d); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template cudaError_t launch_decode_step<float>(float *, const float *, const float *, const float *,
                                               const float *, const float *, const float *, float *,
                                               const Dims &, cudaStream_t);
template cudaError_t launch_decode_step<__nv_bfloat16>(float *, const __nv_bfloat16 *, const float *,
                                                       const float *, const __nv_bfloat16 *,
                                                       const __nv_bfloat16 *, const float *, float *,
                                                       const Dims &, cudaStream_t);

}  // namespace ssd
