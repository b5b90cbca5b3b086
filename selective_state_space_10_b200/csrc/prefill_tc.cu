// prefill_tc.cu -- chunked SSD prefill on the sm_100a tensor cores (bf16 x/B/C, fp32
// accumulation and state), for headdim P = 64, d_state N = 128, chunk Q in {128, 256}.
//
// The chunked form of "Engineering Hybrid State-Space Models" section 2: inside a chunk
// the semiseparable product Y = (M o C B^T) X, across chunks the state recurrence.
// Three kernels:
//
//  K1 k_chunk_state_tc   S_c^T[n, p] = sum_t B_t[n] * (exp(cum_end - cum_t) dt_t x_t[p])
//                        One CTA per (batch, chunk, group, block of heads).  TMA brings
//                        B_c (once) and each head's x tile (ring of 2 slots); eight warps
//                        scale x's rows by the decay weight in fp32 and split the product
//                        into a bf16 high part and a bf16 remainder, stored side by side;
//                        one thread issues tcgen05.mma with both as the two 64-wide halves
//                        of N = 128 (M = 128 d_state rows, K = Q tokens), and four warps
//                        add the halves and stream S_c out in fp32, so the state is
//                        accurate to fp32 level rather than bf16 level.  Also writes the
//                        chunk's total decay exp(cum_end).
//  K2 k_state_passing_bf16
//                        h_c = exp(cum_end,c) h_{c-1} + S_c over chunks in fp32 (the
//                        first-order recurrence of "Mamba and Selective State Space
//                        Models" section 5); writes the state entering each chunk in bf16
//                        (the next kernel's MMA operand) and the final state in fp32.
//  K3 k_chunk_scan_tc    One CTA per (batch, chunk, 128-row token tile, group, block of
//                        heads).  G = C_tile B_chunk^T is computed once into TMEM and,
//                        masked, converted once to a head-independent bf16 W (see the
//                        decay factorisation at K3 below); per head, 4 warps scale the
//                        rows of its x tile by the column decay factors, tcgen05.mma forms
//                        ACC_inter = C_tile h_prev^T and ACC_intra = W X' (double-buffered
//                        in TMEM across heads), and 8 warps write
//                        y_t = exp(cum_t) ACC_inter + u_t ACC_intra + D x_t (fp32).
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
#include <stddef.h>

#include <algorithm>
#include <cmath>
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <utility>
#include <vector>

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
constexpr int K1_SLOTS = 3;
constexpr int K1_CUMBUF = 3;
constexpr int K1_THREADS = 480;  // warp 0 TMA, 1 MMA, 2-9 scale, 10-13 epilogue, 14 decay weights

struct K1Smem {
  // offsets from the 1024-aligned base
  // slot s: x (scaled in place to the bf16 high part), directly followed by its remainder
  __host__ __device__ static constexpr uint32_t x(int Q, int s) { return (uint32_t)s * 2u * Q * 128u; }
  __host__ __device__ static constexpr uint32_t lo(int Q, int s) { return x(Q, s) + (uint32_t)Q * 128u; }
  // the B chunk (2 x [Q][128 B]) lands in the last slot and is moved to TMEM before that
  // slot's first use
  __host__ __device__ static constexpr uint32_t bm(int Q) { return x(Q, K1_SLOTS - 1); }
  __host__ __device__ static constexpr uint32_t misc(int Q) { return K1_SLOTS * 2u * Q * 128u; }
};

struct K1Misc {
  uint64_t b_full, b_tmem;
  uint64_t x_full[K1_SLOTS], scaled[K1_SLOTS], x_free[K1_SLOTS];
  uint64_t acc_full[2], acc_free[2];
  uint64_t w_full[K1_CUMBUF], w_free[K1_CUMBUF];
  uint32_t tmem;
  int abort_flag;
  float w[K1_CUMBUF][256];  // decay weights exp(cum_end - cum_t) dt_t of upcoming heads
};

// TMEM columns: two accumulator slots of [high 64 | remainder 64], then B chunk^T (Q / 2).
constexpr uint32_t K1_TM_B = 256, K1_TM_COLS = 512;  // allocation: a power of two >= 256 + Q / 2

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
  grid_dep_launch();  // state passing may be scheduled now; it waits for this grid's results

  if (threadIdx.x == 0) {
    mbar_init(&ms->b_full, 1);
    mbar_init(&ms->b_tmem, 1);
    for (int s = 0; s < K1_SLOTS; ++s) {
      mbar_init(&ms->x_full[s], 1);
      mbar_init(&ms->scaled[s], 1);
      mbar_init(&ms->x_free[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ms->acc_full[a], 1);
      mbar_init(&ms->acc_free[a], 1);
    }
    for (int i = 0; i < K1_CUMBUF; ++i) {
      mbar_init(&ms->w_full[i], 1);
      mbar_init(&ms->w_free[i], 1);
    }
    ms->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&ms->tmem, K1_TM_COLS);
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
      tma_load_3d(base + K1Smem::bm(Q), &tm_B, &ms->b_full, g * TN, t0, bi);
      tma_load_3d(base + K1Smem::bm(Q) + (uint32_t)Q * 128u, &tm_B, &ms->b_full, g * TN + 64, t0, bi);
      int issued = 0;
      for (int k = 0; k < nh; ++k) {
        const int s = k % K1_SLOTS, u = k / K1_SLOTS;
        if (k >= K1_SLOTS && !mbar_wait(&ms->x_free[s], (u - 1) & 1, abort_flag, err)) break;
        // the last slot holds the B chunk until it has been moved to TMEM
        if (k == K1_SLOTS - 1 && !mbar_wait(&ms->b_tmem, 0, abort_flag, err)) break;
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
      // A = B chunk^T from TMEM: [M = d_state lanes][K = token], bf16 pairs along K
      const uint32_t idesc = idesc_bf16_f32(128, 2 * TP, /*a MN-major*/ false, /*b MN-major*/ true);
      bool ok = mbar_wait(&ms->b_tmem, 0, abort_flag, err);
      for (int k = 0; ok && k < nh; ++k) {
        const int s = k % K1_SLOTS, a = k & 1;
        if (!mbar_wait(&ms->scaled[s], (k / K1_SLOTS) & 1, abort_flag, err)) break;
        if (k >= 2 && !mbar_wait(&ms->acc_free[a], ((k >> 1) - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t x_addr = smem_u32(base + K1Smem::x(Q, s));
        for (int ks = 0; ks < Q / 16; ++ks) {
          // B = [K = token][N = (high | remainder) x channel]: two 64-wide blocks Q*128 B apart
          const uint64_t bd = smem_desc_sw128(x_addr + ks * 2048u, (uint32_t)Q * 128u, 1024u);
          mma_bf16_ts(tmem + (uint32_t)(a * 2 * TP), tmem + K1_TM_B + 8u * ks, bd, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&ms->acc_full[a]);
        mma_commit(&ms->x_free[s]);
      }
    }
    __syncwarp();
  } else if (warp < 10) {
    // ------------------------------------------------------------- scale warps (256 threads)
    const int tid = threadIdx.x - 64;
    for (int k = 0; k < nh; ++k) {
      const int s = k % K1_SLOTS, wb = k % K1_CUMBUF;
      bool ok = mbar_wait(&ms->w_full[wb], (k / K1_CUMBUF) & 1, abort_flag, err);
      ok = ok && mbar_wait(&ms->x_full[s], (k / K1_SLOTS) & 1, abort_flag, err);
      if (ok) {
        const uint32_t xs = smem_u32(base + K1Smem::x(Q, s));
        const uint32_t ls = smem_u32(base + K1Smem::lo(Q, s));
        const float *wv_row = ms->w[wb];
#pragma unroll 4
        for (int unit = tid; unit < Q * 8; unit += 256) {
          const float wv = wv_row[unit >> 3];
          const uint32_t off = (uint32_t)unit * 16u;  // rows are 128 B: unit*16 = row*128 + chunk*16
          const uint4 v = ld_shared_v4(xs + off);
          const uint32_t in[4] = {v.x, v.y, v.z, v.w};
          uint32_t hi[4], rem[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a0 = __uint_as_float(in[q] << 16) * wv;  // exact x * w in fp32
            const float a1 = __uint_as_float(in[q] & 0xffff0000u) * wv;
            hi[q] = pack_bf16x2(a0, a1);
            const float h0 = __uint_as_float(hi[q] << 16), h1 = __uint_as_float(hi[q] & 0xffff0000u);
            rem[q] = pack_bf16x2(a0 - h0, a1 - h1);
          }
          st_shared_v4(xs + off, hi[0], hi[1], hi[2], hi[3]);
          st_shared_v4(ls + off, rem[0], rem[1], rem[2], rem[3]);
        }
      }
      fence_proxy_async_smem();
      named_barrier(1, 256);
      if (tid == 0 && ok) {
        mbar_arrive(&ms->scaled[s]);
        mbar_arrive(&ms->w_free[wb]);
      }
    }
  } else if (warp < 14) {
    // ------------------------------------------------------------- epilogue warps (128 threads)
    const int q = warp & 3;
    const int n = q * 32 + lane;  // d_state row of the accumulator
    const int tid = threadIdx.x - 320;
    {
      // First move the B chunk into TMEM as the MMA's A operand: lane n gets B[t][n] for
      // every token, packed in pairs (t even in the low half).  In shared memory (128-byte
      // swizzle) 16-byte chunk j of row t of a 64-wide block sits at chunk j ^ (t & 7).
      bool ok = mbar_wait(&ms->b_full, 0, abort_flag, err);
      if (ok) {
        const uint32_t src = smem_u32(base + K1Smem::bm(Q)) + (uint32_t)(n >> 6) * (uint32_t)Q * 128u +
                             (uint32_t)(n & 7) * 2u;
        const uint32_t j8 = (uint32_t)((n & 63) >> 3);
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        for (int c0 = 0; c0 < Q / 2; c0 += 16) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint32_t t = 2u * (uint32_t)(c0 + e);
            const uint32_t b0 = ld_shared_u16(src + t * 128u + ((j8 ^ (t & 7u)) << 4));
            const uint32_t b1 = ld_shared_u16(src + (t + 1u) * 128u + ((j8 ^ ((t + 1u) & 7u)) << 4));
            pk[e] = b0 | (b1 << 16);
          }
          tmem_st16(tmem + lane_off + K1_TM_B + (uint32_t)c0, pk);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();  // the slot is refilled by TMA after these reads
      tc_fence_before();
      named_barrier(2, 128);
      if (tid == 0 && ok) mbar_arrive(&ms->b_tmem);
    }
    for (int k = 0; k < nh; ++k) {
      const int a = k & 1, h = h0 + k;
      const bool ok = mbar_wait(&ms->acc_full[a], (k >> 1) & 1, abort_flag, err);
      tc_fence_after();
      if (ok) {
        float *out = states + (((size_t)bi * nc + c) * d.H + h) * (size_t)(TP * TN) + n;
#pragma unroll
        for (int cg = 0; cg < 2; ++cg) {
          float vh[32], vl[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * 2 * TP + cg * 32), vh);
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * 2 * TP + TP + cg * 32), vl);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) out[(size_t)(cg * 32 + j) * TN] = vh[j] + vl[j];
        }
      }
      tc_fence_before();
      named_barrier(2, 128);
      if (tid == 0) mbar_arrive(&ms->acc_free[a]);
    }
  } else {
    // ------------------------------------------------------------- decay-weight warp
    // w_t = exp(cum_end - cum_t) dt_t for each upcoming head (ring of K1_CUMBUF), and the
    // chunk's total decay exp(cum_end) for the state-passing kernel.
    // dt and A of head k + 1 are loaded while head k's buffer is awaited and filled
    const int per = Q / 32;
    auto load_head = [&](int k, float (&v)[8], float &a) {
      const int h = h0 + k;
      a = A[h];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int t = lane * per + j;
        v[j] = (j < per && t < valid) ? dt[((size_t)bi * d.L + t0 + t) * d.H + h] : 0.f;
      }
    };
    float dtv[8], dtn[8], acur = 0.f, anxt = 0.f;
    if (nh > 0) load_head(0, dtv, acur);
    for (int k = 0; k < nh; ++k) {
      const int wb = k % K1_CUMBUF, h = h0 + k;
      if (k + 1 < nh) load_head(k + 1, dtn, anxt);
      if (k >= K1_CUMBUF && !mbar_wait(&ms->w_free[wb], ((k / K1_CUMBUF) - 1) & 1, abort_flag, err)) break;
      const float a2 = acur * kLog2e;
      float c2[8];
      float run = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
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
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < per) ms->w[wb][lane * per + j] = ex2(cend - (c2[j] + excl)) * dtv[j];
      if (lane == 0) cdecay[((size_t)bi * d.H + h) * nc + c] = ex2(cend);
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->w_full[wb]);
#pragma unroll
      for (int j = 0; j < 8; ++j) dtv[j] = dtn[j];
      acur = anxt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, K1_TM_COLS);
  }
}

// ============================================================================ K2
// grid (b * H, ceil(P*N/4 / 256)), block 256: one float4 of the state per thread.  The
// chunk states of 8 chunks are loaded before the sequential update so that their
// latencies overlap; the state entering chunk c is stored in bf16, the final state in fp32.
constexpr int K2_BATCH = 8;

__global__ void __launch_bounds__(256)
k_state_passing_bf16(const float *__restrict__ states, const float *__restrict__ cdecay,
                     __nv_bfloat16 *__restrict__ hprev, float *__restrict__ final_state, Dims d, int nc) {
  const int PN4 = d.P * d.N / 4;
  const int e4 = blockIdx.y * blockDim.x + threadIdx.x;
  sm100::grid_dep_launch();  // the chunk scan may start its own set-up meanwhile
  sm100::grid_dep_wait();    // chunk states and decays of the chunk-state kernel
  if (e4 >= PN4) return;
  const int h = blockIdx.x % d.H, bi = blockIdx.x / d.H;
  const size_t cstride = (size_t)d.H * PN4;  // float4s between consecutive chunks
  const size_t off0 = ((size_t)bi * nc * d.H + h) * PN4 + e4;
  const float4 *sp = reinterpret_cast<const float4 *>(states) + off0;
  uint2 *hp = reinterpret_cast<uint2 *>(hprev) + off0;
  const float *dec = cdecay + ((size_t)bi * d.H + h) * nc;
  float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = 0; c0 < nc; c0 += K2_BATCH) {
    float4 sv[K2_BATCH];
    float dc[K2_BATCH];
#pragma unroll
    for (int j = 0; j < K2_BATCH; ++j)
      if (c0 + j < nc) {
        sv[j] = __ldcs(sp + (size_t)(c0 + j) * cstride);
        dc[j] = dec[c0 + j];
      }
#pragma unroll
    for (int j = 0; j < K2_BATCH; ++j)
      if (c0 + j < nc) {
        hp[(size_t)(c0 + j) * cstride] = make_uint2(sm100::pack_bf16x2(hs.x, hs.y), sm100::pack_bf16x2(hs.z, hs.w));
        hs.x = fmaf(dc[j], hs.x, sv[j].x);
        hs.y = fmaf(dc[j], hs.y, sv[j].y);
        hs.z = fmaf(dc[j], hs.z, sv[j].z);
        hs.w = fmaf(dc[j], hs.w, sv[j].w);
      }
  }
  reinterpret_cast<float4 *>(final_state)[((size_t)bi * d.H + h) * PN4 + e4] = hs;
}

// ============================================================================ K3
// Per CTA: one 128-row token tile (chunk-relative rows 128*ti ..) of one chunk, for a block
// of heads of one group.  G = C_tile B_chunk^T (fp32, TMEM) is computed once.
//
// Decay factorisation.  For a row t and a source token s <= t of the chunk, the decay is
// 2^(c2_t - c2_s) with c2 the in-chunk cumulative log2-decay of the head.  With the
// reference token r = 128*ti - 1 (c2_r = 0 for ti = 0: the chunk start) it splits into a
// row factor u_t = 2^(c2_t - c2_r) and a column factor v_s = 2^(c2_r - c2_s) dt_s.  Hence
//     sum_s W_ts x_s = u_t * sum_s (G o mask)_ts (v_s x_s),
// where G o mask (causal) does not depend on the head: it is converted to bf16 once per
// CTA (W_base, kept in TMEM as the A operand of the intra-chunk MMA), and each head only
// scales the rows of its x tile by v_s.  This is exact algebra; it is used when the
// tile's decay range |c2_r - c2_last| is below 100 (then every factor lies in
// [2^-100, 2^100] and all intermediates stay normal fp32).  Heads with a steeper tile
// ("steep" heads) get their own W (W_base times the full decay, in a second TMEM region)
// instead, as a slower exact fallback.
//
// With W in TMEM, shared memory holds only the C tile, the output staging and a ring of
// per-head slots (x tile + h_prev^T): 4 slots for the first row tile, 3 for the second,
// so that several heads' loads are in flight while earlier heads are scaled and stored.
// The D x_t term enters through the accumulator: the scaling warps, which read every raw
// x row anyway, store D x_t / u_t into the intra-chunk accumulator before the MMA adds
// W X' onto it; the output warps then only combine the two accumulators and hand each
// [32 rows][32 channels] tile of y to a TMA store.
constexpr int K3_THREADS = 512;  // warp 0 TMA, 1 MMA (G, inter), 2-5 W/x scaling, 6-13 output, 14 decay
                                 // tables, 15 MMA (intra)
constexpr int K3_CUMBUF = 3;
constexpr int K3_MAXSLOTS = 5;
constexpr float kSteepLog2 = 100.f;

struct K3Smem {
  static constexpr uint32_t cm = 0;  // C tile: 2 K-atoms x [128][128 B]                                32 KB
  // y staging: one [32 rows][32 fp32] tile (128-byte swizzle) per output warp, the source
  // of that warp's TMA store (8 x 4 KB)
  __host__ __device__ static constexpr uint32_t ystage(int w) { return 32768u + (uint32_t)w * 4096u; }
  static constexpr uint32_t misc = 65536u;  // K3Misc, at most 10 KB
  static constexpr uint32_t ring = 75776u;  // slot ring; the B rows for G sit at its end until G is formed
  static constexpr uint32_t end = 231424u;  // 227 KB of dynamic shared memory less the alignment slack
  // slot: nblk x blocks of [128 rows][128 B], then h_prev^T as 2 K-halves of [64][128 B]
  __host__ __device__ static constexpr uint32_t slot_bytes(int nblk) { return (uint32_t)nblk * 16384u + 16384u; }
  __host__ __device__ static constexpr int slots(int nblk) {
    return (end - ring) / slot_bytes(nblk) < (uint32_t)K3_MAXSLOTS ? (int)((end - ring) / slot_bytes(nblk))
                                                                    : K3_MAXSLOTS;
  }
  __host__ __device__ static constexpr uint32_t slot(int nblk, int s) { return ring + (uint32_t)s * slot_bytes(nblk); }
  // B rows for G: 2 K-atoms, each [128 * nblk rows][128 B]
  __host__ __device__ static constexpr uint32_t bm(int nblk) { return end - (uint32_t)nblk * 32768u; }
};
static_assert(K3Smem::slots(1) == 4 && K3Smem::slots(2) == 3, "slot ring depth");
static_assert(K3Smem::ring % 1024 == 0 && K3Smem::bm(1) % 1024 == 0 && K3Smem::bm(2) % 1024 == 0,
              "TMA destinations with 128-byte swizzle must be 1024-byte aligned");

struct K3Misc {
  uint64_t cb_full, g_full, w_ready;
  uint64_t x_full[K3_MAXSLOTS], ops_ready[K3_MAXSLOTS], x_free[K3_MAXSLOTS];
  uint64_t acc_full[2], acc_free[2];
  uint64_t cum_full[K3_CUMBUF], cum_free[K3_CUMBUF];
  uint32_t tmem;
  int abort_flag;
  int steep[K3_CUMBUF];
  float c2ref[K3_CUMBUF];
  // tables are read with 16-byte vector loads: keep every row 16-byte aligned
  alignas(16) float c2[K3_CUMBUF][256];   // in-chunk cumulative log2-decay
  alignas(16) float dts[K3_CUMBUF][256];  // dt of each token of the chunk (0 past the end)
  alignas(16) float v[K3_CUMBUF][256];    // 2^(c2_r - c2_s) dt_s, s < 128 * (ti + 1)
};
static_assert(offsetof(K3Misc, c2) % 16 == 0 && offsetof(K3Misc, v) % 16 == 0, "decay tables must be 16-byte aligned");
static_assert(K3Smem::misc % 16 == 0, "K3Misc must start 16-byte aligned");
static_assert(K3Smem::misc + sizeof(K3Misc) <= K3Smem::ring, "K3Misc overlaps the slot ring");

constexpr size_t kK3SmemBytes = 1024 + K3Smem::end;

// TMEM columns: W_base and a steep head's W (bf16 pairs, 64 columns per 128-token block),
// then two accumulator slots of [inter 64 | intra 64] columns.  G (fp32, 128 * nblk
// columns) occupies the accumulator slots until W_base has been built from it.
constexpr uint32_t K3_TM_WB = 0, K3_TM_WS = 128, K3_TM_ACC = 256;

__global__ void __launch_bounds__(K3_THREADS, 1)
k_chunk_scan_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_C,
                const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_h,
                const __grid_constant__ CUtensorMap tm_y, const float *__restrict__ dt, const float *__restrict__ A,
                const float *__restrict__ D, int *err, Dims d, int Q, int nc, int kb0, int nhb0, int kb1, int nhb1) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  K3Misc *ms = reinterpret_cast<K3Misc *>(base + K3Smem::misc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: (bi, c, g, jb); jb < nhb1 are the second row tile's head blocks (the heavier
  // CTAs, scheduled first), the rest the first tile's
  int item = blockIdx.x;
  const int jb = item % (nhb0 + nhb1);
  item /= nhb0 + nhb1;
  const int g = item % d.G;
  item /= d.G;
  const int c = item % nc;
  const int bi = item / nc;
  const int ti = (jb < nhb1) ? 1 : 0;  // 128-row token tile inside the chunk
  const int hb = (jb < nhb1) ? jb : jb - nhb1;
  const int kb = ti ? kb1 : kb0;
  const int h0 = g * d.hpg + hb * kb;
  const int nh = min(kb, d.hpg - hb * kb);
  const int t0 = c * Q;
  const int valid = min(Q, d.L - t0);
  if (ti * 128 >= valid) return;  // no rows of this tile exist (whole CTA, before any setup)
  const int nblk = ti + 1;        // source blocks j = 0..ti
  const int NS = K3Smem::slots(nblk);
  const uint32_t SB = K3Smem::slot_bytes(nblk);

  if (threadIdx.x == 0) {
    mbar_init(&ms->cb_full, 1);
    mbar_init(&ms->g_full, 1);
    mbar_init(&ms->w_ready, 1);
    for (int s = 0; s < K3_MAXSLOTS; ++s) {
      mbar_init(&ms->x_full[s], 1);
      mbar_init(&ms->ops_ready[s], 1);
      mbar_init(&ms->x_free[s], 2);  // commits of both MMA issuers
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ms->acc_full[a], 2);  // commits of both MMA issuers
      mbar_init(&ms->acc_free[a], 1);
    }
    for (int s = 0; s < K3_CUMBUF; ++s) {
      mbar_init(&ms->cum_full[s], 1);
      mbar_init(&ms->cum_free[s], 2);  // x/W warps + output warps
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

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_C);
      tma_prefetch_desc(&tm_B);
      tma_prefetch_desc(&tm_h);
      tma_prefetch_desc(&tm_y);
      const uint32_t bmo = K3Smem::bm(nblk);
      mbar_arrive_expect_tx(&ms->cb_full, 32768u + (uint32_t)nblk * 32768u);
      for (int kn = 0; kn < 2; ++kn)
        tma_load_3d(base + K3Smem::cm + kn * 16384u, &tm_C, &ms->cb_full, g * TN + 64 * kn, t0 + 128 * ti, bi);
      for (int jj = 0; jj < nblk; ++jj)
        for (int kn = 0; kn < 2; ++kn)
          tma_load_3d(base + bmo + (uint32_t)kn * nblk * 16384u + jj * 16384u, &tm_B, &ms->cb_full,
                      g * TN + 64 * kn, t0 + 128 * jj, bi);
      // x of the first heads is an input: fetch it before waiting for the state-passing
      // kernel, whose chunk-start states (h) are the only thing read from it.  A slot that
      // overlaps the B rows is filled only once G has been formed.
      int pre = 0;
      while (pre < min(nh, NS) && K3Smem::slot(nblk, pre) + SB <= bmo) {
        mbar_arrive_expect_tx(&ms->x_full[pre], SB);
        for (int jj = 0; jj < nblk; ++jj)
          tma_load_3d(base + K3Smem::slot(nblk, pre) + jj * 16384u, &tm_x, &ms->x_full[pre], (h0 + pre) * TP,
                      t0 + 128 * jj, bi);
        ++pre;
      }
      grid_dep_wait();
      bool g_seen = false;
      int issued = 0;
      for (int k = 0; k < nh; ++k) {
        const int s = k % NS, u = k / NS, h = h0 + k;
        const uint32_t so = K3Smem::slot(nblk, s);
        if (k >= pre) {
          if (k >= NS) {
            if (!mbar_wait(&ms->x_free[s], (u - 1) & 1, abort_flag, err)) break;
          } else if (!g_seen) {
            if (!(g_seen = mbar_wait(&ms->g_full, 0, abort_flag, err))) break;
          }
          mbar_arrive_expect_tx(&ms->x_full[s], SB);
          for (int jj = 0; jj < nblk; ++jj)
            tma_load_3d(base + so + jj * 16384u, &tm_x, &ms->x_full[s], h * TP, t0 + 128 * jj, bi);
        }
        for (int kn = 0; kn < 2; ++kn)
          tma_load_3d(base + so + (uint32_t)nblk * 16384u + kn * 8192u, &tm_h, &ms->x_full[s], 64 * kn, 0,
                      (bi * nc + c) * d.H + h);
        issued = k + 1;
      }
      if (*abort_flag) {  // let this CTA's own loads land before it exits
        mbar_wait_drain(&ms->cb_full, 0);
        for (int k = (issued > NS ? issued - NS : 0); k < issued; ++k) mbar_wait_drain(&ms->x_full[k % NS], (k / NS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer: G, then ACC_inter
    // A single thread issues one tcgen05.mma about every 65 ns whatever N is up to 128, so
    // the inter-chunk and intra-chunk products are issued by two warps (this one and warp 15)
    // into their own accumulators; each commits to acc_full and x_free (count 2).
    if (lane == 0) {
      const uint32_t cm = smem_u32(base + K3Smem::cm), bmm = smem_u32(base + K3Smem::bm(nblk));
      bool ok = mbar_wait(&ms->cb_full, 0, abort_flag, err);
      if (ok) {
        tc_fence_after();
        // G = C_tile B^T: M = 128 rows, N = 128 * nblk source tokens, K = d_state
        const uint32_t idg = idesc_bf16_f32(128, 128 * nblk, false, false);
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t ad = smem_desc_sw128(cm + (ks >> 2) * 16384u + (ks & 3) * 32u, 16u, 1024u);
          const uint64_t bd = smem_desc_sw128(bmm + (ks >> 2) * (uint32_t)nblk * 16384u + (ks & 3) * 32u, 16u, 1024u);
          mma_bf16(tmem + K3_TM_ACC, ad, bd, idg, ks > 0 ? 1u : 0u);
        }
        mma_commit(&ms->g_full);
      }
      // G occupies the accumulator columns until W_base has been built from it
      ok = ok && mbar_wait(&ms->w_ready, 0, abort_flag, err);
      const uint32_t id_inter = idesc_bf16_f32(128, TP, false, false);
      for (int k = 0; ok && k < nh; ++k) {
        const int s = k % NS, u = k / NS, a = k & 1;
        if (!mbar_wait(&ms->x_full[s], u & 1, abort_flag, err)) break;
        if (k >= 2 && !mbar_wait(&ms->acc_free[a], ((k >> 1) - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + K3_TM_ACC + 128u * a;
        const uint32_t so = smem_u32(base + K3Smem::slot(nblk, s));
        const uint32_t hsa = so + (uint32_t)nblk * 16384u;
        // ACC_inter = C_tile h_prev^T: K = d_state
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t ad = smem_desc_sw128(cm + (ks >> 2) * 16384u + (ks & 3) * 32u, 16u, 1024u);
          const uint64_t bd = smem_desc_sw128(hsa + (ks >> 2) * 8192u + (ks & 3) * 32u, 16u, 1024u);
          mma_bf16(acc, ad, bd, id_inter, ks > 0 ? 1u : 0u);
        }
        mma_commit(&ms->acc_full[a]);
        mma_commit(&ms->x_free[s]);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------- W build and x scaling (128 threads)
    // Thread (q, lane) owns row tl = 32q + lane of W and of the accumulators (TMEM lane tl);
    // the warp's rows are the 32-token group q of the tile.
    const int q = warp & 3;
    const int tl = q * 32 + lane;
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int t = 128 * ti + tl;  // chunk-relative row
    const int r = 128 * ti - 1;   // reference token (tile start)
    // W_base = G o causal mask in bf16, once
    bool ok = mbar_wait(&ms->g_full, 0, abort_flag, err);
    tc_fence_after();
    if (ok) {
      for (int jj = 0; jj < nblk; ++jj)
        for (int grp = 0; grp < 4; ++grp) {
          const int col0 = 128 * jj + 32 * grp;  // chunk-relative first source column
          uint32_t pk[16];
          if (jj == ti && grp > q) {  // strictly right of the diagonal
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = 0u;
          } else {
            float gg[32];
            tmem_ld32(tmem + lane_off + K3_TM_ACC + (uint32_t)col0, gg);
            tmem_ld_wait();
            if (jj == ti && grp == q) {
#pragma unroll
              for (int e = 0; e < 32; ++e) gg[e] = (col0 + e <= t) ? gg[e] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(gg[2 * e], gg[2 * e + 1]);
          }
          tmem_st16(tmem + lane_off + K3_TM_WB + (uint32_t)(64 * jj + 16 * grp), pk);
        }
      tmem_st_wait();
    }
    tc_fence_before();
    named_barrier(1, 128);
    if (tid == 0 && ok) mbar_arrive(&ms->w_ready);
    for (int k = 0; k < nh; ++k) {
      const int cb = k % K3_CUMBUF, s = k % NS, a = k & 1;
      const float dh = D[h0 + k];
      ok = ok && mbar_wait(&ms->cum_full[cb], (k / K3_CUMBUF) & 1, abort_flag, err);
      const bool steep = ok && ms->steep[cb];
      if (steep) {
        // the head's own W, from W_base and the full decay; W_steep is free once the MMAs of
        // head k-1 (the last that may have read it) are complete
        if (k >= 1) ok = mbar_wait(&ms->x_free[(k - 1) % NS], ((k - 1) / NS) & 1, abort_flag, err);
        tc_fence_after();
        if (ok) {
          const float *c2 = ms->c2[cb];
          const float *dts = ms->dts[cb];
          const float c2t = c2[t];
          for (int jj = 0; jj < nblk; ++jj)
            for (int grp = 0; grp < 4; ++grp) {
              const int col0 = 128 * jj + 32 * grp;
              uint32_t pk[16];
              if (jj == ti && grp > q) {
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = 0u;
              } else {
                tmem_ld16u(tmem + lane_off + K3_TM_WB + (uint32_t)(64 * jj + 16 * grp), pk);
                tmem_ld_wait();
                float gg[32];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  gg[2 * e] = __uint_as_float(pk[e] << 16);
                  gg[2 * e + 1] = __uint_as_float(pk[e] & 0xffff0000u);
                }
                if (jj < ti) {
                  // an earlier block: the reference-token factors (both <= 1 for a decaying head)
                  const float uf = ex2(c2t - c2[r]);
                  const float *vf = ms->v[cb] + col0;
#pragma unroll
                  for (int e = 0; e < 32; ++e) gg[e] *= vf[e] * uf;
                } else {
                  // the tile's own block: one exp of a difference per element (never overflows)
#pragma unroll
                  for (int e = 0; e < 32; ++e) {
                    const int sx = col0 + e;
                    gg[e] = (sx <= t) ? gg[e] * ex2(c2t - c2[sx]) * dts[sx] : 0.f;
                  }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(gg[2 * e], gg[2 * e + 1]);
              }
              tmem_st16(tmem + lane_off + K3_TM_WS + (uint32_t)(64 * jj + 16 * grp), pk);
            }
          tmem_st_wait();
        }
      }
      // Each thread takes row tl of every x block of the slot (the 128-byte swizzle keeps 8
      // consecutive rows on distinct banks).  In the tile's own block it first stores
      // D x_t / u_t into the intra accumulator (the MMA adds W X' onto it); then, unless the
      // head is steep (its W holds the decay), it scales the row by v_s in place.
      ok = ok && mbar_wait(&ms->x_full[s], (k / NS) & 1, abort_flag, err);
      if (k >= 2) ok = ok && mbar_wait(&ms->acc_free[a], ((k >> 1) - 1) & 1, abort_flag, err);
      tc_fence_after();
      if (ok) {
        const uint32_t xs = smem_u32(base + K3Smem::slot(nblk, s));
        const float c2t = ms->c2[cb][t];
        const float dsc = steep ? dh : dh * ex2(ms->c2ref[cb] - c2t);  // D / u_t
        const uint32_t acc_i = tmem + lane_off + K3_TM_ACC + 128u * a + 64u;
        for (int jj = 0; jj < nblk; ++jj) {
          const uint32_t ra = xs + (uint32_t)jj * 16384u + (uint32_t)tl * 128u;
          const float vv = ms->v[cb][128 * jj + tl];
#pragma unroll
          for (int half = 0; half < 2; ++half) {  // channels 32 half .. 32 half + 31
            uint32_t w[16];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint4 in = ld_shared_v4(ra + ((uint32_t)((4 * half + cc) ^ (tl & 7)) << 4));
              w[4 * cc] = in.x;
              w[4 * cc + 1] = in.y;
              w[4 * cc + 2] = in.z;
              w[4 * cc + 3] = in.w;
            }
            if (jj == ti) {
              uint32_t lo[16], hi[16];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                lo[2 * e] = __float_as_uint(__uint_as_float(w[e] << 16) * dsc);
                lo[2 * e + 1] = __float_as_uint(__uint_as_float(w[e] & 0xffff0000u) * dsc);
                hi[2 * e] = __float_as_uint(__uint_as_float(w[8 + e] << 16) * dsc);
                hi[2 * e + 1] = __float_as_uint(__uint_as_float(w[8 + e] & 0xffff0000u) * dsc);
              }
              tmem_st16(acc_i + 32u * half, lo);
              tmem_st16(acc_i + 32u * half + 16u, hi);
            }
            if (!steep) {
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) {
                uint32_t o4[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                  const uint32_t wv = w[4 * cc + m];
                  o4[m] = pack_bf16x2(__uint_as_float(wv << 16) * vv, __uint_as_float(wv & 0xffff0000u) * vv);
                }
                st_shared_v4(ra + ((uint32_t)((4 * half + cc) ^ (tl & 7)) << 4), o4[0], o4[1], o4[2], o4[3]);
              }
            }
          }
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_barrier(1, 128);
      if (tid == 0 && ok) {
        mbar_arrive(&ms->ops_ready[s]);
        mbar_arrive(&ms->cum_free[cb]);
      }
    }
  } else if (warp < 14) {
    // ------------------------------------------------------------- output warps (256 threads)
    // Warp (q, hf) owns rows 32q .. 32q + 31 of the tile (TMEM lane quarter q) and the 32
    // channels [32 hf, 32 hf + 32): y_t = e_t ACC_inter + u_t ACC_intra (the latter already
    // holds D x_t / u_t), written as one swizzled [32][32] fp32 tile and stored by TMA
    // (rows past the end of the sequence are clipped by the tensor map).
    const int q = warp & 3, hf = (warp - 6) >> 2;
    const int tl = q * 32 + lane;
    const int t = 128 * ti + tl;
    const int tid = threadIdx.x - 192;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint8_t *stg = base + K3Smem::ystage(warp - 6);
    const uint32_t srow = smem_u32(stg) + (uint32_t)lane * 128u;
    for (int k = 0; k < nh; ++k) {
      const int a = k & 1, cb = k % K3_CUMBUF, h = h0 + k;
      bool ok = mbar_wait(&ms->cum_full[cb], (k / K3_CUMBUF) & 1, abort_flag, err);
      ok = ok && mbar_wait(&ms->acc_full[a], (k >> 1) & 1, abort_flag, err);
      tc_fence_after();
      float vi[32], va[32];
      float et = 0.f, ut = 0.f;
      if (ok) {
        const uint32_t acc = tmem + lane_off + K3_TM_ACC + 128u * a + 32u * hf;
        tmem_ld32(acc, vi);
        tmem_ld32(acc + 64u, va);
        const float c2t = ms->c2[cb][t];
        et = ex2(c2t);
        ut = ms->steep[cb] ? 1.f : ex2(c2t - ms->c2ref[cb]);
        tmem_ld_wait();
      }
      // the accumulators and decay tables are read: release them before writing y
      tc_fence_before();
      named_barrier(2, 256);
      if (tid == 0 && ok) {
        mbar_arrive(&ms->acc_free[a]);
        mbar_arrive(&ms->cum_free[cb]);
      }
      if (ok) {
        if (lane == 0) tma_store_wait_read();  // the previous head's store has read the tile
        __syncwarp();
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          float o[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) o[m] = fmaf(et, vi[4 * cc + m], ut * va[4 * cc + m]);
          st_shared_v4(srow + ((uint32_t)(cc ^ (lane & 7)) << 4), __float_as_uint(o[0]), __float_as_uint(o[1]),
                       __float_as_uint(o[2]), __float_as_uint(o[3]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_y, stg, h * TP + 32 * hf, t0 + 128 * ti + 32 * q, bi);
          tma_store_commit();
        }
      }
    }
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
  } else if (warp == 15) {
    // ------------------------------------------------------------- MMA issuer: ACC_intra
    // ops_ready implies x_full, acc_free and W_base: the scaling warps waited for all three
    // before storing D x / u into the accumulator this MMA adds onto.
    if (lane == 0) {
      const uint32_t id_intra = idesc_bf16_f32(128, TP, false, true);
      for (int k = 0; k < nh; ++k) {
        const int s = k % NS, u = k / NS, a = k & 1, cb = k % K3_CUMBUF;
        if (!mbar_wait(&ms->ops_ready[s], u & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + K3_TM_ACC + 128u * a;
        const uint32_t so = smem_u32(base + K3Smem::slot(nblk, s));
        // ACC_intra += W X': A from TMEM (W_base, or the head's own W when steep), K = source tokens
        const uint32_t wa = tmem + (ms->steep[cb] ? K3_TM_WS : K3_TM_WB);
        for (int jj = 0; jj < nblk; ++jj)
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t bd = smem_desc_sw128(so + jj * 16384u + ks * 2048u, 16384u, 1024u);
            mma_bf16_ts(acc + 64, wa + (uint32_t)(64 * jj + 8 * ks), bd, id_intra, 1u);  // onto D x / u
          }
        mma_commit(&ms->acc_full[a]);
        mma_commit(&ms->x_free[s]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- decay-table warp
    // dt and A of head k + 1 are loaded while head k's buffer is awaited and filled
    const int per = Q / 32;
    auto load_head = [&](int k, float (&v)[8], float &a) {
      const int h = h0 + k;
      a = A[h];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int tt = lane * per + j;
        v[j] = (j < per && tt < valid) ? dt[((size_t)bi * d.L + t0 + tt) * d.H + h] : 0.f;
      }
    };
    float dtv[8], dtn[8], acur = 0.f, anxt = 0.f;
    if (nh > 0) load_head(0, dtv, acur);
    for (int k = 0; k < nh; ++k) {
      const int cb = k % K3_CUMBUF;
      if (k + 1 < nh) load_head(k + 1, dtn, anxt);
      if (k >= K3_CUMBUF && !mbar_wait(&ms->cum_free[cb], ((k / K3_CUMBUF) - 1) & 1, abort_flag, err)) break;
      const float a2 = acur * kLog2e;
      float c2v[8];
      float run = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        run += dtv[j] * a2;
        c2v[j] = run;
      }
      float incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float vv = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += vv;
      }
      const float excl = incl - run;
      float *c2 = ms->c2[cb];
      float *dts = ms->dts[cb];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < per) {
          c2[lane * per + j] = c2v[j] + excl;
          dts[lane * per + j] = dtv[j];
        }
      __syncwarp();
      const int ncol = 128 * nblk;
      const int last = min(valid, ncol) - 1;
      const float c2r = (ti > 0) ? c2[128 * ti - 1] : 0.f;
      const float range = fabsf(c2r - c2[last]);
      const int steep = !(range < kSteepLog2);  // also catches NaN
      for (int sidx = lane; sidx < ncol; sidx += 32) ms->v[cb][sidx] = ex2(c2r - c2[sidx]) * dts[sidx];
      if (lane == 0) {
        ms->steep[cb] = steep;
        ms->c2ref[cb] = c2r;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->cum_full[cb]);
#pragma unroll
      for (int j = 0; j < 8; ++j) dtv[j] = dtn[j];
      acur = anxt;
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

// 3-D tensor map {d0 (contiguous), d1, d2}, box {inner, rows, 1}, 128-byte swizzle.
bool make_map_t(CUtensorMap *m, CUtensorMapDataType type, uint32_t esize, const void *ptr, uint64_t d0, uint64_t d1,
                uint64_t d2, uint32_t inner, uint32_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
  const cuuint32_t box[3] = {inner, rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, type, 3, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 3-D bf16 tensor map {d0 (contiguous), d1, d2} with a {64, rows, 1} box and 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t rows) {
  return make_map_t(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, d0, d1, d2, 64, rows);
}

int num_sms() {
  static int n = [] {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
  }();
  return n;
}

// Heads per CTA.  A CTA runs a fixed set-up (barriers, TMEM, the chunk's shared
// operands: worth about `overhead` heads) and then its heads one after another; with one
// CTA per SM, the kernel takes about waves x (heads per CTA + overhead).  Pick the split
// of a group's heads that minimises that, preferring more CTAs on ties.
int pick_heads_per_cta(int base_items, int hpg, int sms, double overhead) {
  int best_kb = hpg;
  double best = 1e30;
  for (int nhb = 1; nhb <= hpg; ++nhb) {
    const int kb = (hpg + nhb - 1) / nhb;
    const int nblocks = (hpg + kb - 1) / kb;
    const long ctas = (long)base_items * nblocks;
    const long waves = (ctas + sms - 1) / sms;
    const double cost = (double)waves * (kb + overhead);
    if (cost <= best + 1e-9) {
      best = cost;
      best_kb = kb;
    }
  }
  return best_kb;
}

// Head split of the chunk-scan kernel.  A CTA of the second row tile costs about 1.5x a
// first-tile CTA per head (twice the x tile and the in-chunk product); each also pays a
// fixed set-up (about 1.8 heads).  Candidate splits are scored by simulating the
// hardware's greedy, in-order placement of CTAs onto SMs (one CTA per SM at a time).
struct ScanSplit {
  int kb0, nhb0, kb1, nhb1;
};

double simulate_makespan(int groups, int hpg, int kb0, int kb1, int ntt, int sms) {
  constexpr double kSetup = 1.8, kTile1 = 1.5;
  std::vector<double> free_at(sms, 0.0);
  std::priority_queue<double, std::vector<double>, std::greater<double>> q(free_at.begin(), free_at.end());
  const int nhb0 = (hpg + kb0 - 1) / kb0, nhb1 = ntt > 1 ? (hpg + kb1 - 1) / kb1 : 0;
  double end = 0.0;
  for (int gi = 0; gi < groups; ++gi)
    for (int jj = 0; jj < nhb0 + nhb1; ++jj) {
      const bool t1 = jj < nhb1;
      const int kb = t1 ? kb1 : kb0, hb = t1 ? jj : jj - nhb1;
      const int nh = std::min(kb, hpg - hb * kb);
      const double cost = kSetup + nh * (t1 ? kTile1 : 1.0);
      const double start = q.top();
      q.pop();
      q.push(start + cost);
      end = std::max(end, start + cost);
    }
  return end;
}

ScanSplit pick_scan_split(int groups, int hpg, int ntt, int sms) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, ScanSplit> cache;
  const auto key = std::make_tuple(groups, hpg, ntt, sms);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  ScanSplit best{hpg, 1, hpg, ntt > 1 ? 1 : 0};
  double best_t = 1e300;
  for (int kb1 = 1; kb1 <= hpg; ++kb1) {
    const int kb0 = ntt > 1 ? std::min(hpg, std::max(1, (int)std::lround(kb1 * 1.5))) : kb1;
    const double t = simulate_makespan(groups, hpg, kb0, kb1, ntt, sms);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = {kb0, (hpg + kb0 - 1) / kb0, kb1, ntt > 1 ? (hpg + kb1 - 1) / kb1 : 0};
    }
  }
  cache[key] = best;
  return best;
}

// Launch `kern` on `st`; with `pdl` it may begin while the previous kernel in the stream is
// still running, and must call grid_dep_wait() before it reads that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(dim3 grid, unsigned threads, size_t smem, cudaStream_t st, bool pdl,
                         void (*kern)(KArgs...), Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace

bool tc_prefill_supported(const Dims &d, int Q) { return d.P == TP && d.N == TN && (Q == 128 || Q == 256); }

size_t tc_prefill_smem_k1(int Q) { return 1024 + K1Smem::misc(Q) + sizeof(K1Misc); }
size_t tc_prefill_smem_k3() { return kK3SmemBytes; }

cudaError_t launch_tc_prefill(const __nv_bfloat16 *x, const float *dt, const float *A, const __nv_bfloat16 *B,
                              const __nv_bfloat16 *C, const float *D, float *y, float *final_state, float *states,
                              float *cdecay, __nv_bfloat16 *hprev, int *err, const Dims &d, int Q, int nc,
                              cudaStream_t st, const cudaEvent_t *ev) {
  CUtensorMap tm_x1, tm_B1, tm_x3, tm_C3, tm_B3, tm_h3, tm_y3;
  const uint64_t HP = (uint64_t)d.H * d.P, GN = (uint64_t)d.G * d.N;
  if (!make_map(&tm_x1, x, HP, d.L, d.b, Q) || !make_map(&tm_B1, B, GN, d.L, d.b, Q) ||
      !make_map(&tm_x3, x, HP, d.L, d.b, 128) || !make_map(&tm_C3, C, GN, d.L, d.b, 128) ||
      !make_map(&tm_B3, B, GN, d.L, d.b, 128) ||
      !make_map(&tm_h3, hprev, (uint64_t)d.N, (uint64_t)d.P, (uint64_t)d.b * nc * d.H, 64) ||
      !make_map_t(&tm_y3, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, y, HP, d.L, d.b, 32, 32))
    return cudaErrorInvalidValue;
  const int sms = num_sms();
  auto mark = [&](int i) { return ev ? cudaEventRecord(ev[i], st) : cudaSuccess; };
  // Without per-kernel events the three kernels overlap their set-up with the tail of the
  // one before (programmatic dependent launch); with events between them they run serially.
  const bool pdl = ev == nullptr;
  cudaError_t e = mark(0);
  if (e != cudaSuccess) return e;
  // K1
  {
    const int base_items = d.b * nc * d.G;
    const int kb = pick_heads_per_cta(base_items, d.hpg, sms, 1.0);
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
    const int per_head = d.P * d.N / 4;
    e = launch_after(dim3(d.b * d.H, (per_head + 255) / 256), 256, 0, st, pdl, k_state_passing_bf16, states, cdecay,
                     hprev, final_state, d, nc);
    if (e != cudaSuccess) return e;
  }
  if ((e = mark(2)) != cudaSuccess) return e;
  // K3
  {
    const int ntt = Q / 128;
    const int groups = d.b * nc * d.G;
    const ScanSplit sp = pick_scan_split(groups, d.hpg, ntt, sms);
    e = cudaFuncSetAttribute(k_chunk_scan_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kK3SmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_after(dim3((unsigned)(groups * (sp.nhb0 + sp.nhb1))), K3_THREADS, kK3SmemBytes, st, pdl,
                     k_chunk_scan_tc, tm_x3, tm_C3, tm_B3, tm_h3, tm_y3, dt, A, D, err, d, Q, nc, sp.kb0, sp.nhb0,
                     sp.kb1, sp.nhb1);
    if (e != cudaSuccess) return e;
  }
  return mark(3);
}

}  // namespace ssd
