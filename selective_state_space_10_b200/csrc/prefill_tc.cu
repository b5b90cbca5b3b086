// prefill_tc.cu -- chunked SSD prefill on the sm_100a tensor cores (bf16 x/B/C, fp32
// accumulation and state), for headdim P = 64, d_state N = 128, chunk Q in {128, 256}.
//
// The chunked form of "Engineering Hybrid State-Space Models" section 2: inside a chunk
// the semiseparable product Y = (M o C B^T) X, across chunks the state recurrence.
// Three kernels:
//
//  K1 k_chunk_state_tc   S_c^T[n, p] = sum_t B_t[n] * (exp(cum_end - cum_t) dt_t x_t[p])
//                        One CTA per (batch, chunk, group, block of heads).  TMA brings
//                        B_c (once) and each head's x tile (ring of 2 slots); four warps
//                        scale x's rows by the decay weight in fp32 and split the product
//                        into a bf16 high part and a bf16 remainder; one thread issues
//                        tcgen05.mma for both (M = 128 d_state rows, N = 64 channels,
//                        K = Q tokens, accumulated in TMEM), so the state is accurate to
//                        fp32 level rather than bf16 level; four warps stream S_c out in
//                        fp32.  Also writes the chunk's total decay exp(cum_end).
//  K2 k_state_passing_bf16
//                        h_c = exp(cum_end,c) h_{c-1} + S_c over chunks in fp32 (the
//                        first-order recurrence of "Mamba and Selective State Space
//                        Models" section 5); writes the state entering each chunk in bf16
//                        (the next kernel's MMA operand) and the final state in fp32.
//  K3 k_chunk_scan_tc    One CTA per (batch, chunk, 128-row token tile, group, block of
//                        heads).  G = C_tile B_chunk^T is computed once into TMEM.  Per
//                        head: 8 warps turn G into W = G o decay o dt (bf16, causal mask)
//                        in shared memory; tcgen05.mma forms ACC_inter = C_tile h_prev^T
//                        and ACC_intra = W X (double-buffered in TMEM across heads); four
//                        warps write y_t = exp(cum_t) ACC_inter + ACC_intra + D x_t (fp32).
//
// Numerics: every decay exp(cum_t - cum_s), s <= t, is formed so that no intermediate
// leaves the range of the result: inside a 128-token block directly from the
// difference; across blocks as the product of exp(cum_t - cum_r) and exp(cum_r - cum_s)
// with r the last token before the row block (both factors <= 1 when A <= 0, both >= 1
// when A > 0, so no 0 * inf).  All mbarrier waits are bounded (2 s of global time):
// on expiry the kernel raises an error word in the workspace and winds down without
// touching further data.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace ssd {
namespace {

using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int TP = 64;    // headdim handled by the tensor-core path
constexpr int TN = 128;   // d_state handled by the tensor-core path

// ============================================================================ K1
constexpr int K1_SLOTS = 2;
constexpr int K1_THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2-5 scale, warps 6-9 epilogue

struct K1Smem {
  // offsets from the 1024-aligned base
  static constexpr uint32_t bm = 0;  // B chunk: 2 x [Q][128 B]
  // slot s: x (scaled in place to the bf16 high part) at x(), the bf16 remainder at lo()
  static constexpr uint32_t x(int Q, int s) { return 2u * Q * 128u + (uint32_t)s * 2u * Q * 128u; }
  static constexpr uint32_t lo(int Q, int s) { return x(Q, s) + (uint32_t)Q * 128u; }
  static constexpr uint32_t misc(int Q) { return 2u * Q * 128u + K1_SLOTS * 2u * Q * 128u; }
};

struct K1Misc {
  uint64_t b_full;
  uint64_t x_full[K1_SLOTS], scaled[K1_SLOTS], x_free[K1_SLOTS];
  uint64_t acc_full[2], acc_free[2];
  uint32_t tmem;
  int abort_flag;
  float w[2][256];  // decay weights of the current head (double-buffered by head parity)
};

__global__ void __launch_bounds__(K1_THREADS, 1)
k_chunk_state_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_B,
                 const float *__restrict__ dt, const float *__restrict__ A, float *__restrict__ states,
                 float *__restrict__ cdecay, int *err, Dims d, int Q, int nc, int kb, int nhb) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  K1Misc *ms = reinterpret_cast<K1Misc *>(base + K1Smem::misc(Q));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: (bi, c, g, hb) with hb fastest
  int item = blockIdx.x;
  const int hb = item % nhb;
  item /= nhb;
  const int g = item % d.G;
  item /= d.G;
  const int c = item % nc;
  const int bi = item / nc;
  const int h0 = g * d.hpg + hb * kb;
  const int nh = min(kb, d.hpg - hb * kb);
  const int t0 = c * Q;
  const int valid = min(Q, d.L - t0);

  if (threadIdx.x == 0) {
    mbar_init(&ms->b_full, 1);
    for (int s = 0; s < K1_SLOTS; ++s) {
      mbar_init(&ms->x_full[s], 1);
      mbar_init(&ms->scaled[s], 1);
      mbar_init(&ms->x_free[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ms->acc_full[a], 1);
      mbar_init(&ms->acc_free[a], 1);
    }
    ms->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&ms->tmem, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem;
  volatile int *abort_flag = &ms->abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_B);
      mbar_arrive_expect_tx(&ms->b_full, 2u * Q * 128u);
      tma_load_3d(base + K1Smem::bm, &tm_B, &ms->b_full, g * TN, t0, bi);
      tma_load_3d(base + K1Smem::bm + (uint32_t)Q * 128u, &tm_B, &ms->b_full, g * TN + 64, t0, bi);
      int issued = 0;
      for (int k = 0; k < nh; ++k) {
        const int s = k % K1_SLOTS, u = k / K1_SLOTS;
        if (k >= K1_SLOTS && !mbar_wait(&ms->x_free[s], (u - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&ms->x_full[s], (uint32_t)Q * 128u);
        tma_load_3d(base + K1Smem::x(Q, s), &tm_x, &ms->x_full[s], (h0 + k) * TP, t0, bi);
        issued = k + 1;
      }
      if (*abort_flag) {  // let this CTA's own loads land before it exits
        mbar_wait_drain(&ms->b_full, 0);
        for (int k = (issued > K1_SLOTS ? issued - K1_SLOTS : 0); k < issued; ++k)
          mbar_wait_drain(&ms->x_full[k % K1_SLOTS], (k / K1_SLOTS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, TP, /*a MN-major*/ true, /*b MN-major*/ true);
      const uint32_t bm_addr = smem_u32(base + K1Smem::bm);
      bool ok = mbar_wait(&ms->b_full, 0, abort_flag, err);
      for (int k = 0; ok && k < nh; ++k) {
        const int s = k % K1_SLOTS, a = k & 1;
        if (!mbar_wait(&ms->scaled[s], (k / K1_SLOTS) & 1, abort_flag, err)) break;
        if (k >= 2 && !mbar_wait(&ms->acc_free[a], ((k >> 1) - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t x_addr = smem_u32(base + K1Smem::x(Q, s));
        const uint32_t lo_addr = smem_u32(base + K1Smem::lo(Q, s));
        for (int ks = 0; ks < Q / 16; ++ks) {
          // A = B chunk as [M = d_state][K = token], d_state contiguous (two 64-wide blocks Q*128 B apart)
          const uint64_t ad = smem_desc_sw128(bm_addr + ks * 2048u, (uint32_t)Q * 128u, 1024u);
          // B = scaled x as [K = token][N = channel], channel contiguous: high part, then remainder
          const uint64_t bh = smem_desc_sw128(x_addr + ks * 2048u, (uint32_t)Q * 128u, 1024u);
          const uint64_t bl = smem_desc_sw128(lo_addr + ks * 2048u, (uint32_t)Q * 128u, 1024u);
          mma_bf16(tmem + (uint32_t)(a * TP), ad, bh, idesc, ks > 0 ? 1u : 0u);
          mma_bf16(tmem + (uint32_t)(a * TP), ad, bl, idesc, 1u);
        }
        mma_commit(&ms->acc_full[a]);
        mma_commit(&ms->x_free[s]);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------- scale warps (128 threads)
    const int tid = threadIdx.x - 64;
    for (int k = 0; k < nh; ++k) {
      const int s = k % K1_SLOTS, hp = k & 1, h = h0 + k;
      if (warp == 2 && !*abort_flag) {
        // in-chunk cumulative log2-decay, then w_t = exp(cum_end - cum_t) dt_t
        const float a2 = A[h] * kLog2e;
        const int per = Q / 32;
        float c2[8], dtv[8];
        float run = 0.f;
        for (int j = 0; j < per; ++j) {
          const int t = lane * per + j;
          dtv[j] = (t < valid) ? dt[((size_t)bi * d.L + t0 + t) * d.H + h] : 0.f;
          run += dtv[j] * a2;
          c2[j] = run;
        }
        float incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const float excl = incl - run;
        const float cend = __shfl_sync(0xffffffffu, incl, 31);
        for (int j = 0; j < per; ++j) ms->w[hp][lane * per + j] = ex2(cend - (c2[j] + excl)) * dtv[j];
        if (lane == 0) cdecay[((size_t)bi * d.H + h) * nc + c] = ex2(cend);
      }
      named_barrier(1, 128);
      if (!mbar_wait(&ms->x_full[s], (k / K1_SLOTS) & 1, abort_flag, err)) {
        named_barrier(1, 128);
        continue;
      }
      const uint32_t xs = smem_u32(base + K1Smem::x(Q, s));
      const uint32_t ls = smem_u32(base + K1Smem::lo(Q, s));
      for (int unit = tid; unit < Q * 8; unit += 128) {
        const int row = unit >> 3;
        const float wv = ms->w[hp][row];
        const uint32_t off = (uint32_t)unit * 16u;  // rows are 128 B: unit*16 = row*128 + chunk*16
        const uint4 v = ld_shared_v4(xs + off);
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
        uint32_t hi[4], rem[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a0 = __uint_as_float(in[q] << 16) * wv;          // exact x * w in fp32
          const float a1 = __uint_as_float(in[q] & 0xffff0000u) * wv;
          hi[q] = pack_bf16x2(a0, a1);
          const float h0 = __uint_as_float(hi[q] << 16), h1 = __uint_as_float(hi[q] & 0xffff0000u);
          rem[q] = pack_bf16x2(a0 - h0, a1 - h1);
        }
        st_shared_v4(xs + off, hi[0], hi[1], hi[2], hi[3]);
        st_shared_v4(ls + off, rem[0], rem[1], rem[2], rem[3]);
      }
      fence_proxy_async_smem();
      named_barrier(1, 128);
      if (tid == 0) mbar_arrive(&ms->scaled[s]);
    }
  } else {
    // ------------------------------------------------------------- epilogue warps (128 threads)
    const int q = warp & 3;
    const int n = q * 32 + lane;  // d_state row of the accumulator
    const int tid = threadIdx.x - 192;
    for (int k = 0; k < nh; ++k) {
      const int a = k & 1, h = h0 + k;
      const bool ok = mbar_wait(&ms->acc_full[a], (k >> 1) & 1, abort_flag, err);
      tc_fence_after();
      if (ok) {
        float *out = states + (((size_t)bi * nc + c) * d.H + h) * (size_t)(TP * TN) + n;
#pragma unroll
        for (int cg = 0; cg < 2; ++cg) {
          float v[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * TP + cg * 32), v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) out[(size_t)(cg * 32 + j) * TN] = v[j];
        }
      }
      tc_fence_before();
      named_barrier(2, 128);
      if (tid == 0) mbar_arrive(&ms->acc_free[a]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ============================================================================ K2
// grid (b * H, P*N / 8 / 256), block 256: 8 consecutive state elements per thread.
__global__ void __launch_bounds__(256)
k_state_passing_bf16(const float *__restrict__ states, const float *__restrict__ cdecay,
                     __nv_bfloat16 *__restrict__ hprev, float *__restrict__ final_state, Dims d, int nc) {
  const int PN = d.P * d.N;
  const int e = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (e >= PN) return;
  const int h = blockIdx.x % d.H, bi = blockIdx.x / d.H;
  const size_t cstride = (size_t)d.H * PN;
  const size_t off0 = ((size_t)bi * nc * d.H + h) * PN + e;
  const float *dec = cdecay + ((size_t)bi * d.H + h) * nc;
  float hs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float4 s0 = *reinterpret_cast<const float4 *>(states + off0);
  float4 s1 = *reinterpret_cast<const float4 *>(states + off0 + 4);
  for (int c = 0; c < nc; ++c) {
    const size_t off = off0 + (size_t)c * cstride;
    float4 n0 = make_float4(0.f, 0.f, 0.f, 0.f), n1 = n0;
    if (c + 1 < nc) {
      n0 = *reinterpret_cast<const float4 *>(states + off + cstride);
      n1 = *reinterpret_cast<const float4 *>(states + off + cstride + 4);
    }
    uint4 packed;
    packed.x = sm100::pack_bf16x2(hs[0], hs[1]);
    packed.y = sm100::pack_bf16x2(hs[2], hs[3]);
    packed.z = sm100::pack_bf16x2(hs[4], hs[5]);
    packed.w = sm100::pack_bf16x2(hs[6], hs[7]);
    *reinterpret_cast<uint4 *>(hprev + off) = packed;  // state entering chunk c
    const float dc = dec[c];
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) hs[j] = fmaf(dc, hs[j], sv[j]);
    s0 = n0;
    s1 = n1;
  }
  float *fo = final_state + ((size_t)bi * d.H + h) * PN + e;
  *reinterpret_cast<float4 *>(fo) = make_float4(hs[0], hs[1], hs[2], hs[3]);
  *reinterpret_cast<float4 *>(fo + 4) = make_float4(hs[4], hs[5], hs[6], hs[7]);
}

// ============================================================================ K3
constexpr int K3_THREADS = 448;  // warp 0 TMA, 1 MMA, 2-9 W builders, 10-13 output
constexpr int K3_CUMBUF = 3;

struct K3Smem {
  static constexpr uint32_t cm = 0;              // C tile: 2 K-atoms x [128][128 B]      32 KB
  static constexpr uint32_t bw = 32768;          // B rows (for G), then W blocks          64 KB
  static constexpr uint32_t x(int s) { return 98304u + (uint32_t)s * 32768u; }  // 2 x 32 KB
  static constexpr uint32_t hs(int s) { return 163840u + (uint32_t)s * 16384u; } // 2 x 16 KB
  static constexpr uint32_t misc = 196608u;
};

struct K3Misc {
  uint64_t cb_full, g_full, w_full, w_free;
  uint64_t x_full[2], x_free[2], acc_full[2], acc_free[2];
  uint64_t cum_full[K3_CUMBUF], cum_free[K3_CUMBUF];
  uint32_t tmem;
  int abort_flag;
  float c2[K3_CUMBUF][256];   // in-chunk cumulative log2-decay
  float dts[K3_CUMBUF][256];  // dt of each token of the chunk (0 past the end)
  float vf[K3_CUMBUF][128];   // exp(cum_r - cum_s) dt_s for s in the block before the row tile
};

constexpr size_t kK3SmemBytes = 1024 + K3Smem::misc + sizeof(K3Misc);

__global__ void __launch_bounds__(K3_THREADS, 1)
k_chunk_scan_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_C,
                const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_h,
                const float *__restrict__ dt, const float *__restrict__ A, const float *__restrict__ D,
                float *__restrict__ y, int *err, Dims d, int Q, int nc, int kb, int nhb) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  K3Misc *ms = reinterpret_cast<K3Misc *>(base + K3Smem::misc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntt = Q / 128;

  int item = blockIdx.x;
  const int hb = item % nhb;
  item /= nhb;
  const int g = item % d.G;
  item /= d.G;
  const int ti = item % ntt;  // 128-row token tile inside the chunk
  item /= ntt;
  const int c = item % nc;
  const int bi = item / nc;
  const int h0 = g * d.hpg + hb * kb;
  const int nh = min(kb, d.hpg - hb * kb);
  const int t0 = c * Q;
  const int valid = min(Q, d.L - t0);
  if (ti * 128 >= valid) return;  // no rows of this tile exist (whole CTA, before any setup)
  const int nblk = ti + 1;        // source blocks j = 0..ti

  if (threadIdx.x == 0) {
    mbar_init(&ms->cb_full, 1);
    mbar_init(&ms->g_full, 1);
    mbar_init(&ms->w_full, 1);
    mbar_init(&ms->w_free, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ms->x_full[s], 1);
      mbar_init(&ms->x_free[s], 2);  // MMA commit + output warps
      mbar_init(&ms->acc_full[s], 1);
      mbar_init(&ms->acc_free[s], 1);
    }
    for (int s = 0; s < K3_CUMBUF; ++s) {
      mbar_init(&ms->cum_full[s], 1);
      mbar_init(&ms->cum_free[s], 1);
    }
    ms->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&ms->tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem;
  volatile int *abort_flag = &ms->abort_flag;
  const uint32_t TM_G = 0, TM_ACC = 256;  // G: cols [0, 256); acc slot a: inter +128a, intra +128a+64

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_C);
      tma_prefetch_desc(&tm_B);
      tma_prefetch_desc(&tm_h);
      mbar_arrive_expect_tx(&ms->cb_full, 32768u + (uint32_t)nblk * 32768u);
      for (int kn = 0; kn < 2; ++kn)
        tma_load_3d(base + K3Smem::cm + kn * 16384u, &tm_C, &ms->cb_full, g * TN + 64 * kn, t0 + 128 * ti, bi);
      for (int j = 0; j < nblk; ++j)
        for (int kn = 0; kn < 2; ++kn)
          tma_load_3d(base + K3Smem::bw + (uint32_t)kn * nblk * 16384u + j * 16384u, &tm_B, &ms->cb_full,
                      g * TN + 64 * kn, t0 + 128 * j, bi);
      int issued = 0;
      for (int k = 0; k < nh; ++k) {
        const int s = k & 1, u = k >> 1, h = h0 + k;
        if (k >= 2 && !mbar_wait(&ms->x_free[s], (u - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&ms->x_full[s], (uint32_t)nblk * 16384u + 16384u);
        for (int j = 0; j < nblk; ++j)
          tma_load_3d(base + K3Smem::x(s) + j * 16384u, &tm_x, &ms->x_full[s], h * TP, t0 + 128 * j, bi);
        for (int kn = 0; kn < 2; ++kn)
          tma_load_3d(base + K3Smem::hs(s) + kn * 8192u, &tm_h, &ms->x_full[s], 64 * kn, 0, (bi * nc + c) * d.H + h);
        issued = k + 1;
      }
      if (*abort_flag) {  // let this CTA's own loads land before it exits
        mbar_wait_drain(&ms->cb_full, 0);
        for (int k = (issued > 2 ? issued - 2 : 0); k < issued; ++k) mbar_wait_drain(&ms->x_full[k & 1], (k >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t cm = smem_u32(base + K3Smem::cm), bw = smem_u32(base + K3Smem::bw);
      bool ok = mbar_wait(&ms->cb_full, 0, abort_flag, err);
      if (ok) {
        tc_fence_after();
        const uint32_t idg = idesc_bf16_f32(128, 128 * nblk, false, false);
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t ad = smem_desc_sw128(cm + (ks >> 2) * 16384u + (ks & 3) * 32u, 16u, 1024u);
          const uint64_t bd = smem_desc_sw128(bw + (ks >> 2) * (uint32_t)nblk * 16384u + (ks & 3) * 32u, 16u, 1024u);
          mma_bf16(tmem + TM_G, ad, bd, idg, ks > 0 ? 1u : 0u);
        }
        mma_commit(&ms->g_full);
      }
      const uint32_t id_inter = idesc_bf16_f32(128, TP, false, false);
      const uint32_t id_intra = idesc_bf16_f32(128, TP, false, true);
      for (int k = 0; ok && k < nh; ++k) {
        const int s = k & 1, u = k >> 1;
        if (!mbar_wait(&ms->x_full[s], u & 1, abort_flag, err)) break;
        if (k >= 2 && !mbar_wait(&ms->acc_free[s], (u - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + TM_ACC + 128u * s;
        const uint32_t hsa = smem_u32(base + K3Smem::hs(s));
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t ad = smem_desc_sw128(cm + (ks >> 2) * 16384u + (ks & 3) * 32u, 16u, 1024u);
          const uint64_t bd = smem_desc_sw128(hsa + (ks >> 2) * 8192u + (ks & 3) * 32u, 16u, 1024u);
          mma_bf16(acc, ad, bd, id_inter, ks > 0 ? 1u : 0u);
        }
        if (!mbar_wait(&ms->w_full, k & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t xa = smem_u32(base + K3Smem::x(s));
        for (int j = 0; j < nblk; ++j)
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t ad = smem_desc_sw128(bw + j * 32768u + (ks >> 2) * 16384u + (ks & 3) * 32u, 16u, 1024u);
            const uint64_t bd = smem_desc_sw128(xa + j * 16384u + ks * 2048u, 16384u, 1024u);
            mma_bf16(acc + 64, ad, bd, id_intra, (j > 0 || ks > 0) ? 1u : 0u);
          }
        mma_commit(&ms->acc_full[s]);
        mma_commit(&ms->w_free);
        mma_commit(&ms->x_free[s]);
      }
    }
    __syncwarp();
  } else if (warp < 10) {
    // ------------------------------------------------------------- W builders (256 threads)
    const int q = warp & 3, ch = (warp - 2) >> 2;
    const int tl = q * 32 + lane;        // row of the tile (TMEM lane)
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int r = 128 * ti - 1;          // last token before the row tile
    bool g_ready = false;
    for (int k = 0; k < nh; ++k) {
      const int cb = k % K3_CUMBUF, h = h0 + k;
      // (1) cumulative decay of head h for the whole chunk, by one warp
      if (warp == 2) {
        bool ok = true;
        if (k >= K3_CUMBUF) ok = mbar_wait(&ms->cum_free[cb], ((k / K3_CUMBUF) - 1) & 1, abort_flag, err);
        if (ok && !*abort_flag) {
          const float a2 = A[h] * kLog2e;
          const int per = Q / 32;
          float c2[8], dtv[8];
          float run = 0.f;
          for (int j = 0; j < per; ++j) {
            const int t = lane * per + j;
            dtv[j] = (t < valid) ? dt[((size_t)bi * d.L + t0 + t) * d.H + h] : 0.f;
            run += dtv[j] * a2;
            c2[j] = run;
          }
          float incl = run;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
          }
          const float excl = incl - run;
          for (int j = 0; j < per; ++j) {
            ms->c2[cb][lane * per + j] = c2[j] + excl;
            ms->dts[cb][lane * per + j] = dtv[j];
          }
          __syncwarp();
          if (ti > 0) {
            const float c2r = ms->c2[cb][r];
            for (int sidx = lane; sidx < 128 * ti; sidx += 32)
              ms->vf[cb][sidx] = ex2(c2r - ms->c2[cb][sidx]) * ms->dts[cb][sidx];
          }
        }
      }
      named_barrier(1, 256);
      if (tid == 0) mbar_arrive(&ms->cum_full[cb]);
      // (2) wait until G is ready and the previous head's MMAs no longer read W
      if (!g_ready) {
        g_ready = mbar_wait(&ms->g_full, 0, abort_flag, err);
      }
      bool ok = g_ready;
      if (ok && k >= 1) ok = mbar_wait(&ms->w_free, (k - 1) & 1, abort_flag, err);
      tc_fence_after();
      if (ok) {
        const float *c2 = ms->c2[cb];
        const float *dts = ms->dts[cb];
        const int t = 128 * ti + tl;          // chunk-relative row
        const float c2t = c2[t];
        for (int j = 0; j < nblk; ++j) {
          const uint32_t wrow = smem_u32(base + K3Smem::bw) + j * 32768u + ch * 16384u + (uint32_t)tl * 128u;
          const int s0 = 128 * j + 64 * ch;   // first source token of my 64 columns
          if (j == ti && q * 32 + 31 < 64 * ch) {
            // whole warp strictly above the diagonal: zeros
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) st_shared_v4(wrow + ((cc ^ (tl & 7)) << 4), 0u, 0u, 0u, 0u);
            continue;
          }
          float gv[64];
          tmem_ld32(tmem + lane_off + TM_G + (uint32_t)s0, *reinterpret_cast<float(*)[32]>(&gv[0]));
          tmem_ld32(tmem + lane_off + TM_G + (uint32_t)s0 + 32u, *reinterpret_cast<float(*)[32]>(&gv[32]));
          tmem_ld_wait();
          if (j < ti) {
            const float ut = ex2(c2t - c2[r]);
            const float *vf = ms->vf[cb] + s0;
#pragma unroll
            for (int e = 0; e < 64; ++e) gv[e] = gv[e] * vf[e] * ut;
          } else {
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const int sidx = s0 + e;
              gv[e] = (sidx <= t) ? gv[e] * ex2(c2t - c2[sidx]) * dts[sidx] : 0.f;
            }
          }
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            st_shared_v4(wrow + ((cc ^ (tl & 7)) << 4), pack_bf16x2(gv[8 * cc + 0], gv[8 * cc + 1]),
                         pack_bf16x2(gv[8 * cc + 2], gv[8 * cc + 3]), pack_bf16x2(gv[8 * cc + 4], gv[8 * cc + 5]),
                         pack_bf16x2(gv[8 * cc + 6], gv[8 * cc + 7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_barrier(1, 256);
      if (tid == 0) mbar_arrive(&ms->w_full);
    }
  } else {
    // ------------------------------------------------------------- output warps (128 threads)
    const int q = warp & 3;
    const int tl = q * 32 + lane;
    const int t = 128 * ti + tl;
    const int tid = threadIdx.x - 320;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    for (int k = 0; k < nh; ++k) {
      const int s = k & 1, cb = k % K3_CUMBUF, h = h0 + k;
      bool ok = mbar_wait(&ms->cum_full[cb], (k / K3_CUMBUF) & 1, abort_flag, err);
      ok = ok && mbar_wait(&ms->x_full[s], (k >> 1) & 1, abort_flag, err);
      ok = ok && mbar_wait(&ms->acc_full[s], (k >> 1) & 1, abort_flag, err);
      tc_fence_after();
      if (ok) {
        const float et = ex2(ms->c2[cb][t]);
        const float Dh = D[h];
        const uint32_t xrow = smem_u32(base + K3Smem::x(s)) + ti * 16384u + (uint32_t)tl * 128u;
        float *yrow = y + (((size_t)bi * d.L + t0 + t) * d.H + h) * TP;
        const uint32_t acc = tmem + lane_off + TM_ACC + 128u * s;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float vi[32], va[32];
          tmem_ld32(acc + 32u * half, vi);
          tmem_ld32(acc + 64u + 32u * half, va);
          tmem_ld_wait();
          if (t < valid) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int chunk = 4 * half + cc;
              const uint4 xv = ld_shared_v4(xrow + ((chunk ^ (tl & 7)) << 4));
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
              float o[8];
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                const float xl = __uint_as_float(xw[m] << 16), xh = __uint_as_float(xw[m] & 0xffff0000u);
                o[2 * m] = fmaf(et, vi[8 * cc + 2 * m], va[8 * cc + 2 * m]) + Dh * xl;
                o[2 * m + 1] = fmaf(et, vi[8 * cc + 2 * m + 1], va[8 * cc + 2 * m + 1]) + Dh * xh;
              }
              float4 *dst = reinterpret_cast<float4 *>(yrow + 8 * chunk);
              dst[0] = make_float4(o[0], o[1], o[2], o[3]);
              dst[1] = make_float4(o[4], o[5], o[6], o[7]);
            }
          }
        }
      }
      tc_fence_before();
      named_barrier(2, 128);
      if (tid == 0) {
        mbar_arrive(&ms->acc_free[s]);
        mbar_arrive(&ms->x_free[s]);
        mbar_arrive(&ms->cum_free[cb]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================================ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D bf16 tensor map {d0 (contiguous), d1, d2} with a {64, rows, 1} box and 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {64, rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = [] {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
  }();
  return n;
}

// Heads per CTA: the split of a group's heads that fills whole waves of CTAs best.
int pick_heads_per_cta(int base_items, int hpg, int sms) {
  int best_nhb = 1;
  double best = -1.0;
  for (int nhb = 1; nhb <= hpg; ++nhb) {
    const long ctas = (long)base_items * nhb;
    if (ctas > 4L * sms && nhb > 1) break;
    const long waves = (ctas + sms - 1) / sms;
    const double eff = (double)ctas / (double)(waves * sms);
    if (eff > best + 1e-9) {
      best = eff;
      best_nhb = nhb;
    }
  }
  return (hpg + best_nhb - 1) / best_nhb;
}

}  // namespace

bool tc_prefill_supported(const Dims &d, int Q) { return d.P == TP && d.N == TN && (Q == 128 || Q == 256); }

size_t tc_prefill_smem_k1(int Q) { return 1024 + K1Smem::misc(Q) + sizeof(K1Misc); }
size_t tc_prefill_smem_k3() { return kK3SmemBytes; }

cudaError_t launch_tc_prefill(const __nv_bfloat16 *x, const float *dt, const float *A, const __nv_bfloat16 *B,
                              const __nv_bfloat16 *C, const float *D, float *y, float *final_state, float *states,
                              float *cdecay, __nv_bfloat16 *hprev, int *err, const Dims &d, int Q, int nc,
                              cudaStream_t st, const cudaEvent_t *ev) {
  CUtensorMap tm_x1, tm_B1, tm_x3, tm_C3, tm_B3, tm_h3;
  const uint64_t HP = (uint64_t)d.H * d.P, GN = (uint64_t)d.G * d.N;
  if (!make_map(&tm_x1, x, HP, d.L, d.b, Q) || !make_map(&tm_B1, B, GN, d.L, d.b, Q) ||
      !make_map(&tm_x3, x, HP, d.L, d.b, 128) || !make_map(&tm_C3, C, GN, d.L, d.b, 128) ||
      !make_map(&tm_B3, B, GN, d.L, d.b, 128) ||
      !make_map(&tm_h3, hprev, (uint64_t)d.N, (uint64_t)d.P, (uint64_t)d.b * nc * d.H, 64))
    return cudaErrorInvalidValue;
  const int sms = num_sms();
  auto mark = [&](int i) { return ev ? cudaEventRecord(ev[i], st) : cudaSuccess; };
  cudaError_t e = mark(0);
  if (e != cudaSuccess) return e;
  // K1
  {
    const int base_items = d.b * nc * d.G;
    const int kb = pick_heads_per_cta(base_items, d.hpg, sms);
    const int nhb = (d.hpg + kb - 1) / kb;
    const size_t smem = tc_prefill_smem_k1(Q);
    e = cudaFuncSetAttribute(k_chunk_state_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_chunk_state_tc<<<(unsigned)(base_items * nhb), K1_THREADS, smem, st>>>(tm_x1, tm_B1, dt, A, states, cdecay,
                                                                             err, d, Q, nc, kb, nhb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = mark(1)) != cudaSuccess) return e;
  // K2
  {
    const int per_head = d.P * d.N / 8;
    k_state_passing_bf16<<<dim3(d.b * d.H, (per_head + 255) / 256), 256, 0, st>>>(states, cdecay, hprev, final_state,
                                                                                 d, nc);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = mark(2)) != cudaSuccess) return e;
  // K3
  {
    const int ntt = Q / 128;
    const int base_items = d.b * nc * ntt * d.G;
    const int kb = pick_heads_per_cta(base_items, d.hpg, sms);
    const int nhb = (d.hpg + kb - 1) / kb;
    e = cudaFuncSetAttribute(k_chunk_scan_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kK3SmemBytes);
    if (e != cudaSuccess) return e;
    k_chunk_scan_tc<<<(unsigned)(base_items * nhb), K3_THREADS, kK3SmemBytes, st>>>(
        tm_x3, tm_C3, tm_B3, tm_h3, dt, A, D, y, err, d, Q, nc, kb, nhb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return mark(3);
}

}  // namespace ssd
