// prefill_simt.cu -- chunked SSD prefill on CUDA cores (fp32 arithmetic).
//
// This is the whole prefill for fp32 inputs (whose 1e-4 RMS error bound rules out bf16
// or TF32 tensor cores) and for shapes outside the tensor-core kernels' set.  Four
// kernels, following the chunked form of "Engineering Hybrid State-Space Models"
// section 2 (chunks of Q tokens, Y = (M o C B^T) X inside a chunk):
//   (a) k_dA_cumsum       cum[t] = sum_{s<=t in chunk} dt_s A_h           (log of M's products)
//   (b) k_chunk_state     S_c[p,n] = sum_t exp(cum_end - cum_t) dt_t x_t[p] B_t[n]
//   (c) k_state_passing   h_c = exp(cum_end,c) h_{c-1} + S_c; S_c is replaced in place
//                         by the state entering chunk c; the last h is the final state
//                         (the first-order associative recurrence of "Mamba and Selective
//                         State Space Models" section 5, run sequentially over chunks)
//   (d) k_chunk_scan      y_t = sum_{s<=t} exp(cum_t - cum_s) dt_s (C_t.B_s) x_s
//                               + exp(cum_t) C_t . h_prev + D_h x_t
// Decays are always formed from differences cum_t - cum_s with s <= t, so no factor
// exceeds 1 and nothing overflows however long the chunk.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

// ------------------------------------------------------------------------ (a)
// grid (nc * b), block 128: one warp per head at a time, scanning 32 tokens per step.
// Positions past the end of the sequence add zero, so cum[Q-1] is the decay of the
// whole (possibly partial) chunk.
__global__ void k_dA_cumsum(const float *__restrict__ dt, const float *__restrict__ A,
                            float *__restrict__ cum, Dims d, int Q, int nc) {
  const int c = blockIdx.x % nc, bi = blockIdx.x / nc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = c * Q;
  const int valid = min(Q, d.L - t0);
  for (int h = warp; h < d.H; h += blockDim.x >> 5) {
    const float Ah = A[h];
    float *out = cum + (((size_t)bi * d.H + h) * nc + c) * Q;
    float carry = 0.f;
    for (int s0 = 0; s0 < Q; s0 += 32) {
      const int t = s0 + lane;
      float v = (t < valid) ? dt[((size_t)bi * d.L + t0 + t) * d.H + h] * Ah : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      v += carry;
      if (t < Q) out[t] = v;
      carry = __shfl_sync(0xffffffffu, v, 31);
    }
  }
}

// ------------------------------------------------------------------------ (b)
// grid (b * H * nc, ceil(P/64) * ceil(N/64)), block 256 (16 x 16 threads, 4 x 4 outputs
// each): a 64 x 64 tile of S_c for one (batch, chunk, head), K = tokens of the chunk.
template <typename T>
__global__ void __launch_bounds__(256)
k_chunk_state_simt(const T *__restrict__ x, const float *__restrict__ dt, const T *__restrict__ B,
                   const float *__restrict__ cum, float *__restrict__ states, Dims d, int Q, int nc) {
  __shared__ __align__(16) float xs[32][68];  // [token][p], x scaled by its decay weight
  __shared__ __align__(16) float bs[32][68];  // [token][n]
  __shared__ float wk[32];
  const int ntn = (d.N + 63) / 64;
  const int p0 = (blockIdx.y / ntn) * 64, n0 = (blockIdx.y % ntn) * 64;
  const int c = blockIdx.x % nc, h = (blockIdx.x / nc) % d.H, bi = blockIdx.x / (nc * d.H);
  const int g = h / d.hpg;
  const int t0 = c * Q, valid = min(Q, d.L - t0);
  const float *cumc = cum + (((size_t)bi * d.H + h) * nc + c) * Q;
  const float cend = cumc[Q - 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < valid; k0 += 32) {
    if (threadIdx.x < 32) {
      const int t = k0 + threadIdx.x;
      wk[threadIdx.x] = (t < valid) ? expf(cend - cumc[t]) * dt[((size_t)bi * d.L + t0 + t) * d.H + h] : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * 64; i += 256) {
      const int k = i >> 6, col = i & 63;
      const int t = k0 + k;
      float xv = 0.f, bv = 0.f;
      if (t < valid) {
        const size_t tok = (size_t)bi * d.L + t0 + t;
        if (p0 + col < d.P) xv = to_f32(x[(tok * d.H + h) * d.P + p0 + col]) * wk[k];
        if (n0 + col < d.N) bv = to_f32(B[(tok * d.G + g) * d.N + n0 + col]);
      }
      xs[k][col] = xv;
      bs[k][col] = bv;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const float4 a = *reinterpret_cast<const float4 *>(&xs[k][ty * 4]);
      const float4 b = *reinterpret_cast<const float4 *>(&bs[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float *out = states + (((size_t)bi * nc + c) * d.H + h) * (size_t)d.P * d.N;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = p0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (p < d.P && n < d.N) out[(size_t)p * d.N + n] = acc[i][j];
    }
}

// ------------------------------------------------------------------------ (c)
// grid (b * H, ceil(P*N/4 / 256)), block 256: one float4 of the state per thread,
// sequential over chunks.  The recurrence starts from `init` (zero if NULL); with
// `cstates` non-NULL the state after every chunk is also written there.  `init` may be
// final_state: each thread reads its element before it writes it.
__global__ void __launch_bounds__(256)
k_state_passing(float *__restrict__ states, const float *__restrict__ cum, const float *init,
                float *final_state, float *__restrict__ cstates, Dims d, int Q, int nc) {
  const int PN4 = d.P * d.N / 4;
  const int e = blockIdx.y * blockDim.x + threadIdx.x;
  const int h = blockIdx.x % d.H, bi = blockIdx.x / d.H;
  if (e >= PN4) return;
  const float *cumh = cum + ((size_t)bi * d.H + h) * nc * Q;
  const size_t chunk_stride4 = (size_t)d.H * PN4;  // float4s between consecutive chunks
  float4 *sp = reinterpret_cast<float4 *>(states) + ((size_t)bi * nc * d.H + h) * PN4 + e;
  const size_t own4 = ((size_t)bi * d.H + h) * PN4 + e;  // this element in a [b][H][P][N] state
  float4 hs = init ? reinterpret_cast<const float4 *>(init)[own4] : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 *cs = cstates ? reinterpret_cast<float4 *>(cstates) + ((size_t)bi * nc * d.H + h) * PN4 + e : nullptr;
  float4 s = sp[0];
  for (int c = 0; c < nc; ++c) {
    const float4 s_next = (c + 1 < nc) ? sp[(c + 1) * chunk_stride4] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float dec = expf(cumh[(size_t)c * Q + Q - 1]);
    sp[c * chunk_stride4] = hs;  // state entering chunk c
    hs.x = fmaf(dec, hs.x, s.x);
    hs.y = fmaf(dec, hs.y, s.y);
    hs.z = fmaf(dec, hs.z, s.z);
    hs.w = fmaf(dec, hs.w, s.w);
    if (cs) cs[c * chunk_stride4] = hs;  // state after chunk c
    s = s_next;
  }
  reinterpret_cast<float4 *>(final_state)[own4] = hs;
}

// ------------------------------------------------------------------------ (d)
// grid (b * H * nc, ceil(Q/64) * ceil(P/64)), block 256 (16 x 16 threads, 4 x 4 outputs):
// outputs of 64 tokens x 64 head channels of one (batch, chunk, head).
// Dynamic shared memory: see chunk_scan_simt_smem_bytes().
template <typename T>
__global__ void __launch_bounds__(256)
k_chunk_scan_simt(const T *__restrict__ x, const float *__restrict__ dt, const T *__restrict__ B,
                  const T *__restrict__ C, const float *__restrict__ D, const float *__restrict__ cum,
                  const float *__restrict__ hprev, float *__restrict__ y, Dims d, int Q, int nc) {
  extern __shared__ __align__(16) float sm[];
  const int NS = d.N + 1;                  // padded row length of C/B tiles
  float *cs = sm;                          // [64][NS]   C rows of this token tile
  float *bsm = cs + 64 * NS;               // [32][NS]   B rows of one source tile (aliases hps)
  const int bsz = max(32 * NS, 64 * 33);
  float *hps = bsm;                        // [64][33]   h_prev[p][n-slice]
  float *wsm = bsm + bsz;                  // [64][33]   decayed scores W[t][s]
  float *xsm = wsm + 64 * 33;              // [32][68]   x[s][p]
  float *dts = xsm + 32 * 68;              // [32]
  float *cums = dts + 32;                  // [32]
  float *cumt = cums + 32;                 // [64]

  const int ntp = (d.P + 63) / 64;
  const int tt0 = (blockIdx.y / ntp) * 64, p0 = (blockIdx.y % ntp) * 64;
  const int c = blockIdx.x % nc, h = (blockIdx.x / nc) % d.H, bi = blockIdx.x / (nc * d.H);
  const int g = h / d.hpg;
  const int t0 = c * Q, valid = min(Q, d.L - t0);
  if (tt0 >= valid) return;
  const int tcount = min(64, valid - tt0);
  const float *cumc = cum + (((size_t)bi * d.H + h) * nc + c) * Q;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;

  for (int i = threadIdx.x; i < 64 * d.N; i += 256) {
    const int r = i / d.N, n = i % d.N;
    cs[r * NS + n] = (r < tcount) ? to_f32(C[(((size_t)bi * d.L + t0 + tt0 + r) * d.G + g) * d.N + n]) : 0.f;
  }
  if (threadIdx.x < 64) cumt[threadIdx.x] = (threadIdx.x < tcount) ? cumc[tt0 + threadIdx.x] : 0.f;

  // Carried-in state: acc = C_t . h_prev[p, :]
  float acc[4][4] = {};
  const float *hp = hprev + (((size_t)bi * nc + c) * d.H + h) * (size_t)d.P * d.N;
  for (int nb = 0; nb < d.N; nb += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      const int pp = i >> 5, nn = i & 31;
      hps[pp * 33 + nn] = (p0 + pp < d.P && nb + nn < d.N) ? hp[(size_t)(p0 + pp) * d.N + nb + nn] : 0.f;
    }
    __syncthreads();
    const int nmax = min(32, d.N - nb);
    for (int nn = 0; nn < nmax; ++nn) {
      float cv[4], hv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) cv[i] = cs[(ty * 4 + i) * NS + nb + nn];
#pragma unroll
      for (int j = 0; j < 4; ++j) hv[j] = hps[(tx * 4 + j) * 33 + nn];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(cv[i], hv[j], acc[i][j]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float e = expf(cumt[ty * 4 + i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] *= e;
  }

  // In-chunk term over source tokens s <= t.
  const int s_end = tt0 + tcount;
  for (int s0 = 0; s0 < s_end; s0 += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * d.N; i += 256) {
      const int k = i / d.N, n = i % d.N;
      bsm[k * NS + n] = (s0 + k < valid) ? to_f32(B[(((size_t)bi * d.L + t0 + s0 + k) * d.G + g) * d.N + n]) : 0.f;
    }
    for (int i = threadIdx.x; i < 32 * 64; i += 256) {
      const int k = i >> 6, pp = i & 63;
      xsm[k * 68 + pp] = (s0 + k < valid && p0 + pp < d.P)
                             ? to_f32(x[(((size_t)bi * d.L + t0 + s0 + k) * d.H + h) * d.P + p0 + pp]) : 0.f;
    }
    if (threadIdx.x < 32) {
      const int s = s0 + threadIdx.x;
      dts[threadIdx.x] = (s < valid) ? dt[((size_t)bi * d.L + t0 + s) * d.H + h] : 0.f;
      cums[threadIdx.x] = (s < valid) ? cumc[s] : 0.f;
    }
    __syncthreads();
    {
      const int r = threadIdx.x >> 2;           // token row within the tile
      const int kb = (threadIdx.x & 3) * 8;     // 8 source tokens per thread
      const int t = tt0 + r;
      for (int kk = 0; kk < 8; ++kk) {
        const int k = kb + kk, s = s0 + k;
        float w = 0.f;
        if (r < tcount && s <= t && s < valid) {
          float g2 = 0.f;
          for (int n = 0; n < d.N; ++n) g2 = fmaf(cs[r * NS + n], bsm[k * NS + n], g2);
          w = expf(cumt[r] - cums[k]) * dts[k] * g2;
        }
        wsm[r * 33 + k] = w;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < 32; ++k) {
      float wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) wv[i] = wsm[(ty * 4 + i) * 33 + k];
      const float4 xv = *reinterpret_cast<const float4 *>(&xsm[k * 68 + tx * 4]);
      const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(wv[i], xa[j], acc[i][j]);
    }
  }

  const float Dh = D[h];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= tcount) continue;
    const size_t row = (((size_t)bi * d.L + t0 + tt0 + r) * d.H + h) * d.P;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = p0 + tx * 4 + j;
      if (p < d.P) y[row + p] = acc[i][j] + Dh * to_f32(x[row + p]);
    }
  }
}

size_t chunk_scan_simt_smem_bytes(int N) {
  const int NS = N + 1;
  const size_t floats = 64 * NS + (size_t)max(32 * NS, 64 * 33) + 64 * 33 + 32 * 68 + 32 + 32 + 64;
  return floats * sizeof(float);
}

// ------------------------------------------------------------------------ launchers
cudaError_t launch_dA_cumsum(const float *dt, const float *A, float *cum, const Dims &d, int Q,
                             int nc, cudaStream_t st) {
  k_dA_cumsum<<<dim3(nc * d.b), 128, 0, st>>>(dt, A, cum, d, Q, nc);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_chunk_state_simt(const T *x, const float *dt, const T *B, const float *cum,
                                    float *states, const Dims &d, int Q, int nc, cudaStream_t st) {
  const dim3 grid(d.b * d.H * nc, ((d.P + 63) / 64) * ((d.N + 63) / 64));
  k_chunk_state_simt<T><<<grid, 256, 0, st>>>(x, dt, B, cum, states, d, Q, nc);
  return cudaGetLastError();
}

cudaError_t launch_state_passing(float *states, const float *cum, const float *init, float *final_state,
                                 float *cstates, const Dims &d, int Q, int nc, cudaStream_t st) {
  const int PN4 = d.P * d.N / 4;
  k_state_passing<<<dim3(d.b * d.H, (PN4 + 255) / 256), 256, 0, st>>>(states, cum, init, final_state, cstates, d, Q,
                                                                        nc);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_chunk_scan_simt(const T *x, const float *dt, const T *B, const T *C, const float *D,
                                   const float *cum, const float *hprev, float *y, const Dims &d, int Q,
                                   int nc, cudaStream_t st) {
  const size_t smem = chunk_scan_simt_smem_bytes(d.N);
  cudaError_t e = cudaFuncSetAttribute(k_chunk_scan_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(d.b * d.H * nc, ((Q + 63) / 64) * ((d.P + 63) / 64));
  k_chunk_scan_simt<T><<<grid, 256, smem, st>>>(x, dt, B, C, D, cum, hprev, y, d, Q, nc);
  return cudaGetLastError();
}

template cudaError_t launch_chunk_state_simt<float>(const float *, const float *, const float *, const float *,
                                                    float *, const Dims &, int, int, cudaStream_t);
template cudaError_t launch_chunk_state_simt<__nv_bfloat16>(const __nv_bfloat16 *, const float *,
                                                            const __nv_bfloat16 *, const float *, float *,
                                                            const Dims &, int, int, cudaStream_t);
template cudaError_t launch_chunk_scan_simt<float>(const float *, const float *, const float *, const float *,
                                                   const float *, const float *, const float *, float *,
                                                   const Dims &, int, int, cudaStream_t);
template cudaError_t launch_chunk_scan_simt<__nv_bfloat16>(const __nv_bfloat16 *, const float *,
                                                           const __nv_bfloat16 *, const __nv_bfloat16 *,
                                                           const float *, const float *, const float *, float *,
                                                           const Dims &, int, int, cudaStream_t);

}  // namespace ssd
