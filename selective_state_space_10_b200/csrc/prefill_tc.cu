// prefill_tc.cu -- chunked SSD prefill on the sm_100a tensor cores (bf16 x/B/C, fp32
// accumulation and state), for headdim P = 64, d_state N = 128, chunk Q in {128, 256}.
//
// The chunked form of "Engineering Hybrid State-Space Models" section 2: inside a chunk
// the semiseparable product Y = (M o C B^T) X, across chunks the state recurrence.
// Three kernels:
//
//  K1 k_chunk_state_tc   S_c^T[n, p] = sum_t B_t[n] * (exp(cum_end - cum_t) dt_t x_t[p])
//                        One CTA per (batch, chunk, group, block of heads).  While TMA
//                        brings B_c (once) and the first x tiles, the scale warps form the
//                        per-chunk dt.A cumulative sums of the CTA's heads: the in-chunk
//                        cumulative log2-decay c2_t = log2(e) A_h sum_{s<=t} dt_s and dt,
//                        kept in shared memory and written out head-major as one table row
//                        per (batch, head, chunk) for the chunk-scan kernel, plus the
//                        chunk's total decay 2^c2_end for state passing.  Then, per head
//                        (ring of 3 x slots), eight warps scale x's rows by the decay
//                        weight in fp32 and
//                        split the product into a bf16 high part and a bf16 remainder,
//                        stored side by side; one thread issues tcgen05.mma with both as
//                        the two 64-wide halves of N = 128 (M = 128 d_state rows, K = Q
//                        tokens), and four warps add the halves and stream S_c out in
//                        fp32, so the state is accurate to fp32 level rather than bf16.
//  K2 k_state_passing_bf16
//                        h_c = exp(cum_end,c) h_{c-1} + S_c over chunks in fp32 (the
//                        first-order recurrence of "Mamba and Selective State Space
//                        Models" section 5); writes the state entering each chunk in bf16
//                        (the next kernel's MMA operand) and the final state in fp32.
//  K3 k_chunk_scan_tc    One CTA per (batch, chunk, 128-row token tile, group, block of
//                        heads), decay data from K1's table.  G = C_tile B_chunk^T is
//                        computed once into TMEM and, masked, converted once to a
//                        head-independent bf16 W (see the decay factorisation at K3
//                        below); per head, 8 warps scale the rows of its x tile by the
//                        column decay factors, three threads issue tcgen05.mma for
//                        ACC_inter = C_tile h_prev^T and the intra-chunk products W X'
//                        (double-buffered in TMEM across heads), and 8 warps write
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
#include <atomic>
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

// ============================================================================ decay table
// Decay table row of one (batch, head, chunk), floats, 16-byte aligned:
//   [0] D_h, [1] 2^c2_end (the chunk's total decay), [2] c2_end, [3] 0,
//   [4 .. 4+Q) c2_t, the in-chunk cumulative log2-decay through token t,
//   [4+Q .. 4+2Q) dt_t (0 past the end of the sequence, so c2 stays flat there).
__host__ __device__ constexpr int tab_row_floats(int Q) { return 4 + 2 * Q; }
constexpr int kTabHdr = 4;
// ============================================================================ K1
constexpr int K1_SLOTS = 3;
constexpr int K1_THREADS = 448;  // warp 0 TMA, 1 MMA, 2-9 scale (and decay tables), 10-13 epilogue
constexpr int K1_KB_MAX = 10;    // heads per CTA at most (their decay tables stay in shared memory)

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
  uint64_t b_full, b_tmem[2];
  uint64_t x_full[K1_SLOTS], scaled[K1_SLOTS], x_free[K1_SLOTS];
  uint64_t acc_full[2], acc_free[2];
  uint32_t tmem;
  int abort_flag;
  int items_done;  // work items whose MMAs have all completed (advanced by the epilogue warps)
  alignas(16) float tab[K1_KB_MAX][tab_row_floats(256)];  // decay table rows of the current item's heads
};
static_assert(offsetof(K1Misc, tab) % 16 == 0, "bulk-copy destinations must be 16-byte aligned");

// TMEM columns: two accumulator slots of [high 64 | remainder 64], then two buffers for the
// B chunk^T (Q / 2 columns each), so that the next work item's B can be moved in while the
// current item's MMAs still read theirs.
constexpr uint32_t K1_TM_B = 256, K1_TM_COLS = 512;  // allocation: a power of two >= 256 + Q

// One work item: the heads [h0, h0 + nh) of group g for chunk c of batch row bi.
struct K1Item {
  int bi, c, g, h0, nh, t0, valid;
};
__device__ __forceinline__ K1Item k1_item(int item, const Dims &d, int Q, int nc, int kb, int nhb) {
  K1Item w;
  const int hb = item % nhb;
  item /= nhb;
  w.g = item % d.G;
  item /= d.G;
  w.c = item % nc;
  w.bi = item / nc;
  w.h0 = w.g * d.hpg + hb * kb;
  w.nh = min(kb, d.hpg - hb * kb);
  w.t0 = w.c * Q;
  w.valid = min(Q, d.L - w.t0);
  return w;
}

// Bounded wait for a counter in shared memory to reach `target` (sleeping between checks);
// gives up like mbar_wait.
__device__ __forceinline__ bool k1_wait_count(volatile int *cnt, int target, volatile int *abort, int *err) {
  if (*cnt >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (*cnt < target) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > 2000000000ull) {
      *abort = 1;
      if (err) atomicExch(err, 1);
      return false;
    }
    __nanosleep(128);
  }
  return true;
}

// kPersist: a persistent grid for launches with more work items than SMs: CTA j takes items
// j, j + gridDim.x, ... in turn, each role carrying its ring and accumulator counters from
// one item to the next, so that the next item's B chunk, decay tables and first x tiles
// load while the current item's last heads are still being multiplied and written out.
// Otherwise one item per CTA (a compile-time single pass of the same code).
template <bool kPersist>
__global__ void __launch_bounds__(K1_THREADS, 1)
k_chunk_state_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_B,
                 const float *__restrict__ dt, const float *__restrict__ A, const float *__restrict__ D,
                 float *__restrict__ tab, float *__restrict__ cdecay, float *__restrict__ states, int *err, Dims d, int Q,
                 int nc, int kb, int nhb, int nitems) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, and derived from the shared array itself (no integer round trip),
  // so that the compiler keeps every access through it in the shared address space
  uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  K1Misc *ms = reinterpret_cast<K1Misc *>(base + K1Smem::misc(Q));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int my_items = kPersist ? ((int)blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0) : 1;
  auto item_of = [&](int i) { return k1_item((int)blockIdx.x + i * (int)gridDim.x, d, Q, nc, kb, nhb); };

  if (threadIdx.x == 0) {
    mbar_init(&ms->b_full, 1);
    mbar_init(&ms->b_tmem[0], 1);
    mbar_init(&ms->b_tmem[1], 1);
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
    ms->items_done = 0;
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
  // Launched as a programmatic dependent of whatever the stream ran before: the set-up
  // above overlaps that kernel's tail, and nothing global is read or written before it has
  // completed (it may have produced x, dt, B, or still be reading this workspace).
  grid_dep_wait();
  // Only now may state passing be scheduled (it waits for this grid's results).  Its own
  // dependent, the chunk scan, reads x, B and C without waiting: by then the kernel that
  // produced them has completed.
  grid_dep_launch();
  // The device error word starts each prefill at zero.  A kernel of this prefill raises it
  // only after a bounded wait of 2 s has expired, long after this store.
  if (blockIdx.x == 0 && threadIdx.x == 0) *err = 0;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    // Slot K1_SLOTS - 1 also takes each item's B chunk: after the slot's last x has been
    // consumed and the previous B has been moved to TMEM; its next x waits for this B's move.
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_B);
      int gk = 0, issued = 0, nb = 0, last = -1;  // last: global head index of slot K1_SLOTS-1's last x
      bool ok = true;
      for (int i = 0; ok && i < my_items; ++i) {
        const K1Item w = item_of(i);
        if (i > 0 && !mbar_wait(&ms->b_tmem[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, err)) break;
        if (last >= 0 && !mbar_wait(&ms->x_free[K1_SLOTS - 1], (last / K1_SLOTS) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&ms->b_full, 2u * Q * 128u);
        tma_load_3d(base + K1Smem::bm(Q), &tm_B, &ms->b_full, w.g * TN, w.t0, w.bi);
        tma_load_3d(base + K1Smem::bm(Q) + (uint32_t)Q * 128u, &tm_B, &ms->b_full, w.g * TN + 64, w.t0, w.bi);
        nb = i + 1;
        bool b_in_slot = true;
        for (int k = 0; k < w.nh; ++k, ++gk) {
          const int s = gk % K1_SLOTS, u = gk / K1_SLOTS;
          if (gk >= K1_SLOTS && !mbar_wait(&ms->x_free[s], (u - 1) & 1, abort_flag, err)) {
            ok = false;
            break;
          }
          if (s == K1_SLOTS - 1 && b_in_slot) {
            if (!mbar_wait(&ms->b_tmem[i & 1], (i >> 1) & 1, abort_flag, err)) {
              ok = false;
              break;
            }
            b_in_slot = false;
          }
          mbar_arrive_expect_tx(&ms->x_full[s], (uint32_t)Q * 128u);
          tma_load_3d(base + K1Smem::x(Q, s), &tm_x, &ms->x_full[s], (w.h0 + k) * TP, w.t0, w.bi);
          if (s == K1_SLOTS - 1) last = gk;
          issued = gk + 1;
        }
      }
      if (*abort_flag) {  // let this CTA's own loads land before it exits
        if (nb > 0) mbar_wait_drain(&ms->b_full, (uint32_t)((nb - 1) & 1));
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
      int gk = 0;
      bool ok = true;
      for (int i = 0; ok && i < my_items; ++i) {
        const K1Item w = item_of(i);
        if (!(ok = mbar_wait(&ms->b_tmem[i & 1], (i >> 1) & 1, abort_flag, err))) break;
        const uint32_t bcol = K1_TM_B + (uint32_t)(i & 1) * (uint32_t)(Q / 2);
        for (int k = 0; k < w.nh; ++k, ++gk) {
          const int s = gk % K1_SLOTS, a = gk & 1;
          if (!(ok = mbar_wait(&ms->scaled[s], (gk / K1_SLOTS) & 1, abort_flag, err))) break;
          if (gk >= 2 && !(ok = mbar_wait(&ms->acc_free[a], ((gk >> 1) - 1) & 1, abort_flag, err))) break;
          tc_fence_after();
          const uint32_t x_addr = smem_u32(base + K1Smem::x(Q, s));
          for (int ks = 0; ks < Q / 16; ++ks) {
            // B = [K = token][N = (high | remainder) x channel]: two 64-wide blocks Q*128 B apart
            const uint64_t bd = smem_desc_sw128(x_addr + ks * 2048u, (uint32_t)Q * 128u, 1024u);
            mma_bf16_ts(tmem + (uint32_t)(a * 2 * TP), tmem + bcol + 8u * ks, bd, idesc, ks > 0 ? 1u : 0u);
          }
          mma_commit(&ms->acc_full[a]);
          mma_commit(&ms->x_free[s]);
        }
      }
    }
    __syncwarp();
  } else if (warp < 10) {
    // ------------------------------------------------------------- scale warps (256 threads)
    const int tid = threadIdx.x - 64, wl = warp - 2;
    int gk = 0;
    bool ok = true;
    for (int i = 0; i < my_items; ++i) {
      const K1Item w = item_of(i);
      const int bi = w.bi, c = w.c, h0 = w.h0, nh = w.nh, t0 = w.t0, valid = w.valid;
      {
        // Decay tables first (per-chunk dt.A cumulative sums), one head per warp and round:
        // every lane sums Q/32 consecutive tokens, a shuffle scan adds the lanes' totals.
        // All loads of both rounds are issued before the first use.  The previous item's
        // rows are no longer read: these warps have scaled all of its heads.
        const int per = Q / 32;
        float dv[2][8], av[2] = {0.f, 0.f}, dd[2] = {0.f, 0.f};
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int k = wl + 8 * r, h = h0 + k;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int t = lane * per + j;
            dv[r][j] = (k < nh && j < per && t < valid) ? __ldg(dt + ((size_t)bi * d.L + t0 + t) * d.H + h) : 0.f;
          }
          if (k < nh) {
            av[r] = __ldg(A + h);
            dd[r] = __ldg(D + h);
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int k = wl + 8 * r, h = h0 + k;
          if (k >= nh) break;
          const float a2 = av[r] * kLog2e;
          float c2v[8];
          float run = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            run += dv[r][j] * a2;
            c2v[j] = run;
          }
          float incl = run;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float uu = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += uu;
          }
          const float excl = incl - run;
          const float cend = __shfl_sync(0xffffffffu, incl, 31);
          float *row = ms->tab[k];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j < per) {
              row[kTabHdr + lane * per + j] = c2v[j] + excl;
              row[kTabHdr + Q + lane * per + j] = dv[r][j];
            }
          if (lane == 0) {
            const float dec = ex2(cend);
            *reinterpret_cast<float4 *>(row) = make_float4(dd[r], dec, cend, 0.f);
            cdecay[((size_t)bi * d.H + h) * nc + c] = dec;
          }
          __syncwarp();
          // the row, coalesced, for the chunk-scan kernel
          float4 *dst = reinterpret_cast<float4 *>(tab + (((size_t)bi * d.H + h) * nc + c) * (size_t)tab_row_floats(Q));
          for (int j = lane; j < tab_row_floats(Q) / 4; j += 32) dst[j] = reinterpret_cast<const float4 *>(row)[j];
          __syncwarp();
          // then, in place of dt in the shared copy, the weight the scaling below applies to
          // each token: w_t = 2^(c2_end - c2_t) dt_t (0 past the end of the sequence)
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j < per) row[kTabHdr + Q + lane * per + j] = ex2(cend - (c2v[j] + excl)) * dv[r][j];
        }
      }
      // The B chunk into its TMEM buffer (i & 1) as the MMA's A operand, once it has landed
      // and once the item that last used the buffer (i - 2) has finished its MMAs: lane n
      // gets B[t][n] for every token, packed in pairs (t even in the low half), the two
      // warps of a TMEM lane quarter taking half of the columns each.  In shared memory
      // (128-byte swizzle) 16-byte chunk j of row t of a 64-wide block sits at chunk j ^ (t & 7).
      // (The first item's B is moved by the epilogue warps, idle until its first head, so
      // that the move overlaps these tables.)
      if (i > 0) ok = ok && mbar_wait(&ms->b_full, (uint32_t)(i & 1), abort_flag, err);
      ok = ok && (i < 2 || k1_wait_count(&ms->items_done, i - 1, abort_flag, err));
      tc_fence_after();
      if (ok && i > 0) {
        const int q = warp & 3, half = wl >> 2;
        const int n = q * 32 + lane;
        const uint32_t src = smem_u32(base + K1Smem::bm(Q)) + (uint32_t)(n >> 6) * (uint32_t)Q * 128u +
                             (uint32_t)(n & 7) * 2u;
        const uint32_t j8 = (uint32_t)((n & 63) >> 3);
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t bcol = K1_TM_B + (uint32_t)(i & 1) * (uint32_t)(Q / 2);
        for (int c0 = half * (Q / 4); c0 < (half + 1) * (Q / 4); c0 += 16) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint32_t t = 2u * (uint32_t)(c0 + e);
            const uint32_t b0 = ld_shared_u16(src + t * 128u + ((j8 ^ (t & 7u)) << 4));
            const uint32_t b1 = ld_shared_u16(src + (t + 1u) * 128u + ((j8 ^ ((t + 1u) & 7u)) << 4));
            pk[e] = b0 | (b1 << 16);
          }
          tmem_st16(tmem + lane_off + bcol + (uint32_t)c0, pk);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();  // the slot is refilled by TMA after these reads
      tc_fence_before();
      named_barrier(1, 256);  // every head's table row is in shared memory, B is in TMEM
      if (tid == 0 && ok && i > 0) mbar_arrive(&ms->b_tmem[i & 1]);
      // Row t of a slot is scaled by w_t = 2^(c2_end - c2_t) dt_t, kept in its head's table row.
      for (int k = 0; k < nh; ++k, ++gk) {
        const int s = gk % K1_SLOTS;
        ok = ok && mbar_wait(&ms->x_full[s], (gk / K1_SLOTS) & 1, abort_flag, err);
        if (ok) {
          const uint32_t xs = smem_u32(base + K1Smem::x(Q, s));
          const uint32_t ls = smem_u32(base + K1Smem::lo(Q, s));
          const float *tw = ms->tab[k] + kTabHdr + Q;
#pragma unroll 8
          for (int unit = tid; unit < Q * 8; unit += 256) {
            const float wv = tw[unit >> 3];
            const uint32_t off = (uint32_t)unit * 16u;  // rows are 128 B: unit*16 = row*128 + chunk*16
            const uint4 v = ld_shared_v4(xs + off);
            const uint32_t in[4] = {v.x, v.y, v.z, v.w};
            uint32_t hi[4], rem[4];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float a0 = __uint_as_float(in[qq] << 16) * wv;  // exact x * w in fp32
              const float a1 = __uint_as_float(in[qq] & 0xffff0000u) * wv;
              // high part: the top 16 bits (truncation), so a - high is exact in fp32 and is
              // rounded once, to the bf16 remainder
              const uint32_t b0 = __float_as_uint(a0) & 0xffff0000u, b1 = __float_as_uint(a1) & 0xffff0000u;
              hi[qq] = __byte_perm(b0, b1, 0x7632);
              rem[qq] = pack_bf16x2(a0 - __uint_as_float(b0), a1 - __uint_as_float(b1));
            }
            st_shared_v4(xs + off, hi[0], hi[1], hi[2], hi[3]);
            st_shared_v4(ls + off, rem[0], rem[1], rem[2], rem[3]);
          }
        }
        fence_proxy_async_smem();
        named_barrier(1, 256);
        if (tid == 0 && ok) mbar_arrive(&ms->scaled[s]);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue warps (128 threads)
    const int q = warp & 3;
    const int n = q * 32 + lane;  // d_state row of the accumulator
    const int tid = threadIdx.x - 320;
    if (my_items > 0) {
      // The first item's B chunk into TMEM buffer 0 (later items' are moved by the scale
      // warps): lane n gets B[t][n] for every token, packed in pairs.
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
      if (tid == 0 && ok) mbar_arrive(&ms->b_tmem[0]);
    }
    int gk = 0;
    for (int i = 0; i < my_items; ++i) {
      const K1Item w = item_of(i);
      for (int k = 0; k < w.nh; ++k, ++gk) {
        const int a = gk & 1, h = w.h0 + k;
        const bool ok = mbar_wait(&ms->acc_full[a], (gk >> 1) & 1, abort_flag, err);
        tc_fence_after();
        if (ok) {
          // S in the layout of the entering states: [n / 64][p][n % 64] per (batch, chunk, head)
          float *out = states + (((size_t)w.bi * nc + w.c) * d.H + h) * (size_t)(TP * TN) + (n >> 6) * (TP * 64) + (n & 63);
#pragma unroll
          for (int cg = 0; cg < 2; ++cg) {
            float vh[32], vl[32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * 2 * TP + cg * 32), vh);
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * 2 * TP + TP + cg * 32), vl);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) out[(size_t)(cg * 32 + j) * 64] = vh[j] + vl[j];
          }
        }
        tc_fence_before();
        named_barrier(2, 128);
        if (tid == 0) mbar_arrive(&ms->acc_free[a]);
      }
      // every MMA of item i has completed (each head's completion was seen above)
      if (tid == 0) *reinterpret_cast<volatile int *>(&ms->items_done) = i + 1;
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
// State passing: h_c = exp(cum_end,c) h_{c-1} + S_c over the chunks, in fp32 (the
// first-order recurrence of "Mamba and Selective State Space Models" section 5), for every
// float4 column of every (batch, head) state.  Two kernels: for sequences of more than
// K2_ROUND chunks (measured faster there), one wave of CTAs, one per SM: each owns a
// contiguous range of a batch row's state columns (heads x P x N / 4), which for a given
// chunk is one contiguous span of the chunk states.  The spans of several chunks at a time
// are staged in shared memory by bulk copies (one per chunk, issued from different warps,
// since a thread completes about one copy per half microsecond) into two buffers, so the
// next chunks fly while one buffer is read; each thread keeps the running state of its
// columns in registers.
//
// The chunk states S (fp32) and the bf16 entering states of a (batch, chunk, head) share
// one layout, the two 64-wide halves of d_state, [n / 64][p][n % 64] (d_state = 128), so
// that the chunk-scan kernel fetches an entering state with one box; a column index e4
// addresses four consecutive elements of that layout, and the same four elements of a
// [p][n] state (initial, final, exported chunk states) are at state_column_pn(e4).  The
// recurrence starts from `init` (zero if NULL; it may alias final_state: every CTA reads
// the initial values of its columns before it writes any final value); with `cstates`
// non-NULL the state after every chunk is also written there.
constexpr int K2_THREADS = 512;
constexpr int K2_MAX_COLS = 4;                 // columns a thread owns at most
constexpr size_t kK2Buf = 104u * 1024u;        // bytes of a staging buffer
constexpr size_t kK2SmemBytes = 2 * kK2Buf;

__device__ __forceinline__ int state_column_pn(int e4, const Dims &d) {
  const int half = (4 * e4) / (d.P * 64), rem = 4 * e4 - half * d.P * 64;
  return ((rem >> 6) * d.N + half * 64 + (rem & 63)) >> 2;
}

__global__ void __launch_bounds__(K2_THREADS, 1)
k_state_passing_bf16(const float *__restrict__ states, const float *__restrict__ cdecay,
                     __nv_bfloat16 *__restrict__ hprev, const float *init, float *final_state,
                     float *__restrict__ cstates, int *err, Dims d, int nc, int cpc, int parts) {
  extern __shared__ __align__(16) uint8_t k2_smem[];
  __shared__ uint64_t full[2];
  const int PN4 = d.P * d.N / 4;
  const int rowcols = d.H * PN4;  // state columns of one batch row
  const int bi = blockIdx.x / parts, part = blockIdx.x % parts;
  const int col0 = part * cpc, ncol = min(cpc, rowcols - col0);
  const int nwarps = K2_THREADS / 32, warp = threadIdx.x >> 5;
  sm100::grid_dep_launch();  // the chunk scan may start its own set-up meanwhile
  if (ncol <= 0) return;
  const int ks = max(1, min(nc, (int)(kK2Buf / ((size_t)ncol * sizeof(float4)))));  // chunks per stage
  const int nstage = (nc + ks - 1) / ks;
  const size_t cstride = (size_t)rowcols;  // float4s between consecutive chunks
  const float4 *src = reinterpret_cast<const float4 *>(states) + (size_t)bi * nc * cstride + col0;
  float4 *buf0 = reinterpret_cast<float4 *>(k2_smem);
  float4 *buf1 = reinterpret_cast<float4 *>(k2_smem + kK2Buf);
  if (threadIdx.x == 0) {
    sm100::mbar_init(&full[0], nwarps);
    sm100::mbar_init(&full[1], nwarps);
    sm100::mbar_fence_init();
  }
  __syncthreads();
  sm100::grid_dep_wait();  // chunk states and decays of the chunk-state kernel
  // stage st: chunk j of it by lane 0 of warp j % nwarps; every warp arrives with its bytes
  auto issue = [&](int st) {
    float4 *b = (st & 1) ? buf1 : buf0;
    const int c0 = st * ks, cn = min(ks, nc - c0);
    uint32_t bytes = 0;
    for (int j = warp; j < cn; j += nwarps) bytes += (uint32_t)ncol * sizeof(float4);
    sm100::mbar_arrive_expect_tx(&full[st & 1], bytes);
    for (int j = warp; j < cn; j += nwarps)
      sm100::bulk_load(b + (size_t)j * ncol, src + (size_t)(c0 + j) * cstride, (uint32_t)ncol * sizeof(float4),
                       &full[st & 1]);
  };
  if ((threadIdx.x & 31) == 0)
    for (int st = 0; st < 2 && st < nstage; ++st) issue(st);
  // this thread's columns and their running states
  float4 hs[K2_MAX_COLS];
  const float *decp[K2_MAX_COLS];
#pragma unroll
  for (int i = 0; i < K2_MAX_COLS; ++i) {
    const int cl = threadIdx.x + i * K2_THREADS;
    hs[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    decp[i] = cdecay;
    if (cl < ncol) {
      const int col = col0 + cl, h = col / PN4, e4 = col - h * PN4;
      decp[i] = cdecay + ((size_t)bi * d.H + h) * nc;
      if (init) hs[i] = reinterpret_cast<const float4 *>(init)[((size_t)bi * d.H + h) * PN4 + state_column_pn(e4, d)];
    }
  }
  uint2 *hp = reinterpret_cast<uint2 *>(hprev) + (size_t)bi * nc * cstride + col0;
  bool ok = true;
  for (int st = 0; st < nstage; ++st) {
    // bounded wait (1 s): on expiry the error word is raised and the outputs are undefined
    ok = ok && sm100::mbar_wait_drain(&full[st & 1], (uint32_t)((st >> 1) & 1));
    if (!ok && threadIdx.x == 0) atomicExch(err, 1);
    const float4 *b = (st & 1) ? buf1 : buf0;
    const int c0 = st * ks, cn = min(ks, nc - c0);
    if (ok) {
      for (int j = 0; j < cn; ++j) {
        const int c = c0 + j;
#pragma unroll
        for (int i = 0; i < K2_MAX_COLS; ++i) {
          const int cl = threadIdx.x + i * K2_THREADS;
          if (cl < ncol) {
            const float4 sv = b[(size_t)j * ncol + cl];
            const float dc = __ldg(decp[i] + c);
            hp[(size_t)c * cstride + cl] = make_uint2(sm100::pack_bf16x2(hs[i].x, hs[i].y),
                                                      sm100::pack_bf16x2(hs[i].z, hs[i].w));
            hs[i].x = fmaf(dc, hs[i].x, sv.x);
            hs[i].y = fmaf(dc, hs[i].y, sv.y);
            hs[i].z = fmaf(dc, hs[i].z, sv.z);
            hs[i].w = fmaf(dc, hs[i].w, sv.w);
            if (cstates) {  // state after chunk c, in the [p][n] layout
              const int col = col0 + cl, h = col / PN4, e4 = col - h * PN4;
              reinterpret_cast<float4 *>(cstates)[(((size_t)bi * nc + c) * d.H + h) * PN4 + state_column_pn(e4, d)] = hs[i];
            }
          }
        }
      }
    }
    __syncthreads();  // every thread has read this buffer
    if ((threadIdx.x & 31) == 0 && ok && st + 2 < nstage) issue(st + 2);
  }
  if (!ok) {  // let this CTA's own copies land before it exits
    if (threadIdx.x == 0)
      for (int st = 0; st < 2 && st < nstage; ++st) sm100::mbar_wait_drain(&full[st & 1], 0);
    return;
  }
#pragma unroll
  for (int i = 0; i < K2_MAX_COLS; ++i) {
    const int cl = threadIdx.x + i * K2_THREADS;
    if (cl < ncol) {
      const int col = col0 + cl, h = col / PN4, e4 = col - h * PN4;
      reinterpret_cast<float4 *>(final_state)[((size_t)bi * d.H + h) * PN4 + state_column_pn(e4, d)] = hs[i];
    }
  }
}

// Short sequences (at most K2_ROUND chunks): grid (b * H, ceil(P*N/4 / 256)), block 256,
// one float4 column of the state per thread, all of its chunks fetched at once.  The
// update is sequential over chunks, so the time goes in waiting for the chunk states: a
// thread fetches K2_ROUND chunks at once, half into registers and half into shared memory
// by cp.async (which holds no register), so that a CTA has a whole round in flight after
// one issue pass and few CTAs per SM cover the layer.  The state entering chunk c is
// stored in bf16, the final state in fp32.  The recurrence starts from `init` (zero if
// NULL); with `cstates` non-NULL the state after every chunk is also written there in
// fp32.  `init` may be final_state: each thread reads its element before it writes it.
constexpr int K2R_THREADS = 256;
constexpr int K2_REG = 8;              // chunks of a round held in registers
constexpr int K2_STAGED = 8;           // chunks of a round staged in shared memory
constexpr int K2_ROUND = K2_REG + K2_STAGED;
constexpr size_t kK2RSmemBytes = (size_t)K2_STAGED * K2R_THREADS * sizeof(float4);

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// kExport: also store the state after every chunk (cstates non-NULL); a separate
// instantiation, so that the plain prefill's kernel holds no pointer for it.
template <bool kExport>
__global__ void __launch_bounds__(K2R_THREADS, 4)
k_state_passing_rounds(const float *__restrict__ states, const float *__restrict__ cdecay,
                     __nv_bfloat16 *__restrict__ hprev, const float *init, float *final_state,
                     float *__restrict__ cstates, Dims d, int nc) {
  extern __shared__ float4 k2_stage[];  // [K2_STAGED][K2R_THREADS]
  const int PN4 = d.P * d.N / 4;
  const int e4 = blockIdx.y * blockDim.x + threadIdx.x;
  sm100::grid_dep_launch();  // the chunk scan may start its own set-up meanwhile
  sm100::grid_dep_wait();    // chunk states and decays of the chunk-state kernel
  if (e4 >= PN4) return;
  const int h = blockIdx.x % d.H, bi = blockIdx.x / d.H;
  const size_t cstride = (size_t)d.H * PN4;  // float4s between consecutive chunks
  // The chunk states S (fp32) and the bf16 entering states of a (batch, chunk, head) share
  // one layout: the two 64-wide halves of d_state, [n / 64][p][n % 64] (d_state = 128), so
  // that the chunk-scan kernel fetches an entering state with one box.  e4 indexes four
  // consecutive elements of that layout; e4o is the same four elements in a [p][n] state.
  const size_t off0 = ((size_t)bi * nc * d.H + h) * PN4 + e4;
  const float4 *sp = reinterpret_cast<const float4 *>(states) + off0;
  uint2 *hp = reinterpret_cast<uint2 *>(hprev) + off0;
  const int half = (4 * e4) / (d.P * 64), rem = 4 * e4 - half * d.P * 64;
  const int e4o = ((rem >> 6) * d.N + half * 64 + (rem & 63)) >> 2;
  const float *dec = cdecay + ((size_t)bi * d.H + h) * nc;
  const size_t own4 = ((size_t)bi * d.H + h) * PN4 + e4o;  // this element in a [b][H][P][N] state
  float4 hs = init ? reinterpret_cast<const float4 *>(init)[own4] : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 *cs = kExport ? reinterpret_cast<float4 *>(cstates) + ((size_t)bi * nc * d.H + h) * PN4 + e4o : nullptr;
  float4 *stage = k2_stage + threadIdx.x;
  auto step = [&](int c, const float4 &sv) {
    const float dc = __ldg(dec + c);
    hp[(size_t)c * cstride] = make_uint2(sm100::pack_bf16x2(hs.x, hs.y), sm100::pack_bf16x2(hs.z, hs.w));
    hs.x = fmaf(dc, hs.x, sv.x);
    hs.y = fmaf(dc, hs.y, sv.y);
    hs.z = fmaf(dc, hs.z, sv.z);
    hs.w = fmaf(dc, hs.w, sv.w);
    if (kExport) cs[(size_t)c * cstride] = hs;  // state after chunk c
  };
  for (int c0 = 0; c0 < nc; c0 += K2_ROUND) {
    // issue the whole round: chunks c0 .. c0+7 into registers, c0+8 .. c0+15 into shared memory
#pragma unroll
    for (int j = 0; j < K2_STAGED; ++j)
      if (c0 + K2_REG + j < nc) cp_async16(stage + j * K2R_THREADS, sp + (size_t)(c0 + K2_REG + j) * cstride);
    asm volatile("cp.async.commit_group;" ::: "memory");
    float4 sv[K2_REG];
#pragma unroll
    for (int j = 0; j < K2_REG; ++j)
      if (c0 + j < nc) sv[j] = __ldcs(sp + (size_t)(c0 + j) * cstride);
#pragma unroll
    for (int j = 0; j < K2_REG; ++j)
      if (c0 + j < nc) step(c0 + j, sv[j]);
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // this thread's own copies
#pragma unroll
    for (int j = 0; j < K2_STAGED; ++j)
      if (c0 + K2_REG + j < nc) step(c0 + K2_REG + j, stage[j * K2R_THREADS]);
  }
  reinterpret_cast<float4 *>(final_state)[own4] = hs;
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
constexpr int K3_THREADS = 704;  // warp 0 TMA (C, B, x), 1 MMA (G, inter), 2-5 and 17-20 W/x scaling, 6-13 output,
                                 // 14 decay-table loads, 15 MMA (intra, source block 0), 16 MMA (intra, block 1),
                                 // 21 TMA (entering states)
constexpr int K3_CUMBUF = 4;
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
  uint64_t x_full[K3_MAXSLOTS], h_full[K3_MAXSLOTS], ops_ready[K3_MAXSLOTS], x_free[K3_MAXSLOTS];
  uint64_t acc_full[2], acc_free[2];
  uint64_t tab_full[K3_CUMBUF], cum_free[K3_CUMBUF];
  uint32_t tmem;
  int abort_flag;
  alignas(16) float tab[K3_CUMBUF][tab_row_floats(256)];  // decay table rows of upcoming heads (bulk copies)
};
static_assert(offsetof(K3Misc, tab) % 16 == 0, "bulk-copy destinations must be 16-byte aligned");
static_assert(K3Smem::misc % 16 == 0, "K3Misc must start 16-byte aligned");
static_assert(K3Smem::misc + sizeof(K3Misc) <= K3Smem::ring, "K3Misc overlaps the slot ring");

constexpr size_t kK3SmemBytes = 1024 + K3Smem::end;

// One head's decay data for one row tile, read from its table row in shared memory: the
// reference token's c2 (0 before the chunk), and how the tile is factorised:
//   plain -- the tile's decay range is below 2^100: one reference token for all of it;
//   split -- the range is wider but each half of the tile's rows (64 tokens) spans less
//            than 2^100: sources and rows from chunk-relative m = 128*ti + 64 on use the
//            second reference m - 1 (c2ref2) and accumulate apart from the rest;
//   steep -- neither: the head gets its own W with the decay folded in per element.
// Every role derives these identically.
struct TileDecay {
  const float *c2, *dt;
  float c2ref, c2ref2, dcoef;
  bool split, steep;
};
__device__ __forceinline__ TileDecay tile_decay(const float *row, int Q, int ti, int nblk, int valid) {
  TileDecay t;
  t.c2 = row + kTabHdr;
  t.dt = row + kTabHdr + Q;
  t.dcoef = row[0];
  t.c2ref = ti > 0 ? t.c2[128 * ti - 1] : 0.f;
  const int last = min(valid, 128 * nblk) - 1;
  const int m = 128 * ti + 64;
  t.c2ref2 = t.c2[m - 1];
  const bool wide = !(fabsf(t.c2ref - t.c2[last]) < kSteepLog2);  // also catches NaN
  t.split = wide && m <= last && fabsf(t.c2ref - t.c2ref2) < kSteepLog2 && fabsf(t.c2ref2 - t.c2[last]) < kSteepLog2;
  t.steep = wide && !t.split;
  return t;
}

// TMEM columns: W_base (bf16 pairs, 64 columns per 128-token source block), then two
// accumulator buffers of [inter 64 | intra, source block 0: 64 | intra, source block 1: 64]
// columns.  G (fp32, 128 * nblk columns) occupies the buffers until W_base has been built
// from it.  A steep head builds its own W in the other head's buffer (see below).
//
// One thread issues a tcgen05.mma about every 67 ns at N = 64 or 128 (75-94 ns at N = 256,
// measured), and several issuing threads with their own accumulators run concurrently
// (three bursts of 8 complete in about the time of one), so the products of a head
// are spread over up to three issuers of at most 8 MMAs each: C h_prev^T (warp 1), the
// intra-chunk product of source block 0 (warp 15) and of source block 1 (warp 16).
constexpr uint32_t K3_TM_WB = 0, K3_TM_BUF = 128, K3_BUF_COLS = 192;
__device__ __forceinline__ uint32_t k3_buf(int a) { return K3_TM_BUF + K3_BUF_COLS * (uint32_t)a; }

__global__ void __launch_bounds__(K3_THREADS, 1)
k_chunk_scan_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_x2,
                const __grid_constant__ CUtensorMap tm_C,
                const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_h,
                const __grid_constant__ CUtensorMap tm_y, const float *__restrict__ tab, int *err, Dims d, int Q, int nc,
                int kb0, int nhb0, int kb1, int nhb1) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, and derived from the shared array itself (no integer round trip),
  // so that the compiler keeps every access through it in the shared address space
  uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
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
  const uint32_t SBX = (uint32_t)nblk * 16384u;  // the slot's x part; the entering state follows it

  if (threadIdx.x == 0) {
    mbar_init(&ms->cb_full, 1);
    mbar_init(&ms->g_full, 1);
    mbar_init(&ms->w_ready, 1);
    for (int s = 0; s < K3_MAXSLOTS; ++s) {
      mbar_init(&ms->x_full[s], 1);
      mbar_init(&ms->h_full[s], 1);
      mbar_init(&ms->ops_ready[s], 8);  // one arrival per scaling warp
      mbar_init(&ms->x_free[s], 3);  // commits of the three MMA issuers
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ms->acc_full[a], 3);  // commits of the three MMA issuers
      mbar_init(&ms->acc_free[a], 8);  // one arrival per output warp
    }
    for (int s = 0; s < K3_CUMBUF; ++s) {
      mbar_init(&ms->tab_full[s], 1);
      mbar_init(&ms->cum_free[s], 16);  // every x/W warp and every output warp
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
      // x of a head: one box of the tile's 128 * nblk rows (the second row tile's two
      // source blocks are consecutive rows).  The entering states come from warp 21: a
      // thread completes about one TMA box per half microsecond however many it has in
      // flight, so the per-head boxes are spread over two issuing threads.
      const CUtensorMap *xm = nblk == 2 ? &tm_x2 : &tm_x;
      tma_prefetch_desc(xm);
      tma_prefetch_desc(&tm_C);
      tma_prefetch_desc(&tm_B);
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
        mbar_arrive_expect_tx(&ms->x_full[pre], SBX);
        tma_load_3d(base + K3Smem::slot(nblk, pre), xm, &ms->x_full[pre], (h0 + pre) * TP, t0, bi);
        ++pre;
      }
      bool g_seen = false;
      int issued = pre;
      for (int k = pre; k < nh; ++k) {
        const int s = k % NS, u = k / NS, h = h0 + k;
        const uint32_t so = K3Smem::slot(nblk, s);
        if (k >= NS) {
          if (!mbar_wait(&ms->x_free[s], (u - 1) & 1, abort_flag, err)) break;
        } else if (!g_seen) {
          if (!(g_seen = mbar_wait(&ms->g_full, 0, abort_flag, err))) break;
        }
        mbar_arrive_expect_tx(&ms->x_full[s], SBX);
        tma_load_3d(base + so, xm, &ms->x_full[s], h * TP, t0, bi);
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
          mma_bf16(tmem + K3_TM_BUF, ad, bd, idg, ks > 0 ? 1u : 0u);
        }
        mma_commit(&ms->g_full);
      }
      // G occupies the accumulator columns until W_base has been built from it
      ok = ok && mbar_wait(&ms->w_ready, 0, abort_flag, err);
      const uint32_t id_inter = idesc_bf16_f32(128, TP, false, false);
      bool prev_steep = false;
      for (int k = 0; ok && k < nh; ++k) {
        const int s = k % NS, u = k / NS, a = k & 1, cb = k % K3_CUMBUF;
        if (!mbar_wait(&ms->h_full[s], u & 1, abort_flag, err)) break;
        if (k >= 2 && !mbar_wait(&ms->acc_free[a], ((k >> 1) - 1) & 1, abort_flag, err)) break;
        // a steep head k-1 keeps its own W in this head's buffer until its MMAs are done
        if (prev_steep && !mbar_wait(&ms->x_free[(k - 1) % NS], ((k - 1) / NS) & 1, abort_flag, err)) break;
        if (!mbar_wait(&ms->tab_full[cb], (k / K3_CUMBUF) & 1, abort_flag, err)) break;
        prev_steep = tile_decay(ms->tab[cb], Q, ti, nblk, valid).steep;
        tc_fence_after();
        const uint32_t acc = tmem + k3_buf(a);
        const uint32_t so = smem_u32(base + K3Smem::slot(nblk, s));
        const uint32_t hsa = so + SBX;
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
  } else if (warp == 21) {
    // ------------------------------------------------------------- TMA: entering states
    // One box per head (both 64-wide halves of d_state, as the state-passing kernel stores
    // them) into the slot after the head's x, on its own barrier.  The slot is reused once
    // the three MMA issuers have released it; a slot overlapping the B rows only once G
    // has been formed.
    if (lane == 0) {
      tma_prefetch_desc(&tm_h);
      const uint32_t bmo = K3Smem::bm(nblk);
      grid_dep_wait();  // the entering states are the state-passing kernel's output
      bool g_seen = false;
      int issued = 0;
      for (int k = 0; k < nh; ++k) {
        const int s = k % NS, u = k / NS;
        const uint32_t so = K3Smem::slot(nblk, s);
        if (k >= NS) {
          if (!mbar_wait(&ms->x_free[s], (u - 1) & 1, abort_flag, err)) break;
        } else if (so + SB > bmo && !g_seen) {
          if (!(g_seen = mbar_wait(&ms->g_full, 0, abort_flag, err))) break;
        }
        mbar_arrive_expect_tx(&ms->h_full[s], 16384u);
        tma_load_3d(base + so + SBX, &tm_h, &ms->h_full[s], 0, 0, (bi * nc + c) * d.H + h0 + k);
        issued = k + 1;
      }
      if (*abort_flag)  // let this CTA's own loads land before it exits
        for (int k = (issued > NS ? issued - NS : 0); k < issued; ++k) mbar_wait_drain(&ms->h_full[k % NS], (k / NS) & 1);
    }
    __syncwarp();
  } else if (warp < 6 || warp >= 17) {
    // ------------------------------------------------------------- W build and x scaling (256 threads)
    // Two warps per TMEM lane quarter q: thread (q, hh, lane) owns row tl = 32q + lane of W
    // and of the accumulators (TMEM lane tl), and the half hh of the columns: W's 32-column
    // groups 2hh and 2hh + 1, and x's channels 32hh .. 32hh + 31.
    const int q = warp & 3, hh = warp >= 17 ? 1 : 0;
    const int tl = q * 32 + lane;
    const int tid = hh ? (int)threadIdx.x - 17 * 32 + 128 : (int)threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int t = 128 * ti + tl;  // chunk-relative row
    const int r = 128 * ti - 1;   // reference token (tile start)
    // W_base = G o causal mask in bf16, once
    bool ok = mbar_wait(&ms->g_full, 0, abort_flag, err);
    tc_fence_after();
    if (ok) {
      for (int jj = 0; jj < nblk; ++jj)
        for (int grp = 2 * hh; grp < 2 * hh + 2; ++grp) {
          const int col0 = 128 * jj + 32 * grp;  // chunk-relative first source column
          uint32_t pk[16];
          if (jj == ti && grp > q) {  // strictly right of the diagonal
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = 0u;
          } else {
            float gg[32];
            tmem_ld32(tmem + lane_off + K3_TM_BUF + (uint32_t)col0, gg);
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
    named_barrier(1, 256);
    if (tid == 0 && ok) mbar_arrive(&ms->w_ready);
    bool prev_steep = false;
    for (int k = 0; k < nh; ++k) {
      const int cb = k % K3_CUMBUF, s = k % NS, a = k & 1;
      ok = ok && mbar_wait(&ms->tab_full[cb], (k / K3_CUMBUF) & 1, abort_flag, err);
      const TileDecay td = tile_decay(ms->tab[cb], Q, ti, nblk, valid);
      const float dh = td.dcoef;
      const bool steep = ok && td.steep;
      const uint32_t ws_col = k3_buf(a ^ 1);  // a steep head's own W: the other head's buffer
      if (steep) {
        // the head's own W, from W_base and the full decay, built in the buffer of head k-1
        // once the output warps have read that head's accumulators
        if (k >= 1) ok = mbar_wait(&ms->acc_free[a ^ 1], ((k - 1) >> 1) & 1, abort_flag, err);
        tc_fence_after();
        if (ok) {
          const float *c2 = td.c2;
          const float *dts = td.dt;
          const float c2t = c2[t];
          for (int jj = 0; jj < nblk; ++jj)
            for (int grp = 2 * hh; grp < 2 * hh + 2; ++grp) {
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
#pragma unroll
                  for (int e = 0; e < 32; ++e) gg[e] *= ex2(td.c2ref - c2[col0 + e]) * dts[col0 + e] * uf;
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
              tmem_st16(tmem + lane_off + ws_col + (uint32_t)(64 * jj + 16 * grp), pk);
            }
          tmem_st_wait();
        }
      }
      // Each thread takes row tl of every x block of the slot (the 128-byte swizzle keeps 8
      // consecutive rows on distinct banks) and, unless the head is steep (its W holds the
      // decay), scales it by v_s in place as soon as x has landed, keeping the raw values of
      // the tile's own block.  Only then does it wait for the head's accumulator buffer and
      // store D x_t / u_t into the intra accumulator (the MMA adds W X' onto it), so that the
      // scaling is not part of the loop "buffer released -> MMAs -> read out -> released".
      ok = ok && mbar_wait(&ms->x_full[s], (k / NS) & 1, abort_flag, err);
      // A split head's rows and sources from m = 128*ti + 64 on take the second reference,
      // and their D x_t / u_t goes to the second intra accumulator (the first gets 0 for
      // them, and the second gets 0 for the rows before m).
      const bool second = td.split && tl >= 64;
      uint32_t own[16];  // raw x of row tl, channels 32 hh .. 32 hh + 31, in the tile's own block
      if (ok) {
        const uint32_t xs = smem_u32(base + K3Smem::slot(nblk, s));
        for (int jj = 0; jj < nblk; ++jj) {
          const uint32_t ra = xs + (uint32_t)jj * 16384u + (uint32_t)tl * 128u;
          // the column factor in bf16: one packed multiply per pair of channels
          const float vref = (second && jj == ti) ? td.c2ref2 : td.c2ref;
          const float vs = ex2(vref - td.c2[128 * jj + tl]) * td.dt[128 * jj + tl];
          const uint32_t vv2 = pack_bf16x2(vs, vs);
          uint32_t w[16];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint4 in = ld_shared_v4(ra + ((uint32_t)((4 * hh + cc) ^ (tl & 7)) << 4));
            w[4 * cc] = in.x;
            w[4 * cc + 1] = in.y;
            w[4 * cc + 2] = in.z;
            w[4 * cc + 3] = in.w;
          }
          if (jj == ti) {
#pragma unroll
            for (int e = 0; e < 16; ++e) own[e] = w[e];
          }
          if (!steep) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t o4[4];
#pragma unroll
              for (int m = 0; m < 4; ++m) o4[m] = mul_bf16x2(w[4 * cc + m], vv2);
              st_shared_v4(ra + ((uint32_t)((4 * hh + cc) ^ (tl & 7)) << 4), o4[0], o4[1], o4[2], o4[3]);
            }
          }
        }
      }
      if (k >= 2) ok = ok && mbar_wait(&ms->acc_free[a], ((k >> 1) - 1) & 1, abort_flag, err);
      // a steep head k-1 keeps its own W in this head's buffer until its MMAs are done
      if (prev_steep) ok = ok && mbar_wait(&ms->x_free[(k - 1) % NS], ((k - 1) / NS) & 1, abort_flag, err);
      prev_steep = steep;
      tc_fence_after();
      if (ok) {
        const float c2t = td.c2[t];
        const float dsc = steep ? dh : dh * ex2((second ? td.c2ref2 : td.c2ref) - c2t);  // D / u_t
        const uint32_t acc_i = tmem + lane_off + k3_buf(a) + (second ? 128u : 64u);
        if (td.split) {  // the other intra accumulator starts from 0 in this row
          uint32_t z[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) z[e] = 0u;
          const uint32_t acc_z = tmem + lane_off + k3_buf(a) + (second ? 64u : 128u) + 32u * (uint32_t)hh;
          tmem_st16(acc_z, z);
          tmem_st16(acc_z + 16u, z);
        }
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          lo[2 * e] = __float_as_uint(__uint_as_float(own[e] << 16) * dsc);
          lo[2 * e + 1] = __float_as_uint(__uint_as_float(own[e] & 0xffff0000u) * dsc);
          hi[2 * e] = __float_as_uint(__uint_as_float(own[8 + e] << 16) * dsc);
          hi[2 * e + 1] = __float_as_uint(__uint_as_float(own[8 + e] & 0xffff0000u) * dsc);
        }
        tmem_st16(acc_i + 32u * hh, lo);
        tmem_st16(acc_i + 32u * hh + 16u, hi);
        tmem_st_wait();
      }
      // each warp releases its share on its own (no CTA-wide barrier in the head's loop)
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) {
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
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint8_t *stg = base + K3Smem::ystage(warp - 6);
    const uint32_t srow = smem_u32(stg) + (uint32_t)lane * 128u;
    for (int k = 0; k < nh; ++k) {
      const int a = k & 1, cb = k % K3_CUMBUF, h = h0 + k;
      bool ok = mbar_wait(&ms->tab_full[cb], (k / K3_CUMBUF) & 1, abort_flag, err);
      ok = ok && mbar_wait(&ms->acc_full[a], (k >> 1) & 1, abort_flag, err);
      tc_fence_after();
      float vi[32], va[32];
      float et = 0.f, ut = 0.f;
      if (ok) {
        const uint32_t acc = tmem + lane_off + k3_buf(a) + 32u * hf;
        const TileDecay td = tile_decay(ms->tab[cb], Q, ti, nblk, valid);
        const float c2t = td.c2[t];
        et = ex2(c2t);
        ut = td.steep ? 1.f : ex2(c2t - td.c2ref);
        tmem_ld32(acc + 64u, va);
        if (td.split) {  // second accumulator: sources from m on, row factor relative to m - 1
          tmem_ld32(acc + 128u, vi);
          const float ut2 = ex2(c2t - td.c2ref2);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) va[j] = fmaf(ut2, vi[j], ut * va[j]);
          ut = 1.f;
        } else if (nblk > 1) {  // the two source blocks' intra-chunk products share the row factor u_t
          tmem_ld32(acc + 128u, vi);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) va[j] += vi[j];
        }
        tmem_ld32(acc, vi);
        tmem_ld_wait();
      }
      // the accumulators and decay tables are read: release them before writing y
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) {
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
  } else if (warp == 15 || warp == 16) {
    // ------------------------------------------------------------- MMA issuers: ACC_intra
    // Warp 15 forms W_{., 0} X'_0 onto D x / u (stored by the scaling warps), warp 16 the
    // second row tile's W_{., 1} X'_1 into its own accumulator.  ops_ready implies x_full,
    // acc_free and W_base: the scaling warps waited for all three.
    // A split head's K steps are divided at its second reference m = 128*ti + 64 instead:
    // warp 15 takes every source before m (into the first accumulator), warp 16 the
    // sources from m on (into the second).  Both warps commit for every head.
    const int iss = warp - 15;
    if (lane == 0) {
      const uint32_t id_intra = idesc_bf16_f32(128, TP, false, true);
      for (int k = 0; k < nh; ++k) {
        const int s = k % NS, u = k / NS, a = k & 1, cb = k % K3_CUMBUF;
        if (!mbar_wait(&ms->ops_ready[s], u & 1, abort_flag, err)) break;
        if (!mbar_wait(&ms->tab_full[cb], (k / K3_CUMBUF) & 1, abort_flag, err)) break;  // complete already
        tc_fence_after();
        const uint32_t acc = tmem + k3_buf(a) + 64u * (uint32_t)(1 + iss);
        const uint32_t so = smem_u32(base + K3Smem::slot(nblk, s));
        // A from TMEM (W_base, or a steep head's own W in the other buffer), K = source tokens
        const TileDecay td = tile_decay(ms->tab[cb], Q, ti, nblk, valid);
        const uint32_t wbase = tmem + (td.steep ? k3_buf(a ^ 1) : K3_TM_WB);
        // the K steps (16 source tokens each, chunk-relative step index 8*block + ks) of this issuer
        int ks0, ks1;
        if (td.split) {
          ks0 = iss == 0 ? 0 : 8 * ti + 4;
          ks1 = iss == 0 ? 8 * ti + 4 : 8 * nblk;
        } else {
          ks0 = 8 * iss;
          ks1 = iss < nblk ? 8 * iss + 8 : ks0;  // the first row tile has one source block
        }
        for (int kk = ks0; kk < ks1; ++kk) {
          const uint64_t bd = smem_desc_sw128(so + (uint32_t)(kk >> 3) * 16384u + (uint32_t)(kk & 7) * 2048u, 16384u, 1024u);
          // the first accumulator (and a split head's second) adds onto D x / u; a plain
          // head's block-1 accumulator starts from its first step
          mma_bf16_ts(acc, wbase + (uint32_t)(8 * kk), bd, id_intra, (iss == 0 || td.split || kk > ks0) ? 1u : 0u);
        }
        mma_commit(&ms->acc_full[a]);
        mma_commit(&ms->x_free[s]);
      }
    }
    __syncwarp();
  } else if (warp == 14) {
    // ------------------------------------------------------------- decay-table loads
    // One bulk copy per head of its table row (written by the cumulative-sum kernel) into a
    // ring of K3_CUMBUF entries, released by the scaling and the output warps.
    if (lane == 0) {
      const uint32_t tab_bytes = (uint32_t)tab_row_floats(Q) * 4u;
      const float *row0 = tab + (((size_t)bi * d.H + h0) * nc + c) * (size_t)tab_row_floats(Q);
      const size_t head_stride = (size_t)nc * tab_row_floats(Q);
      grid_dep_wait();
      int issued = 0;
      for (int k = 0; k < nh; ++k) {
        const int cb = k % K3_CUMBUF;
        if (k >= K3_CUMBUF && !mbar_wait(&ms->cum_free[cb], ((k / K3_CUMBUF) - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&ms->tab_full[cb], tab_bytes);
        bulk_load(ms->tab[cb], row0 + k * head_stride, tab_bytes, &ms->tab_full[cb]);
        issued = k + 1;
      }
      if (*abort_flag)  // let this CTA's own copies land before it exits
        for (int k = (issued > K3_CUMBUF ? issued - K3_CUMBUF : 0); k < issued; ++k)
          mbar_wait_drain(&ms->tab_full[k % K3_CUMBUF], (k / K3_CUMBUF) & 1);
    }
    __syncwarp();
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

// Encoded tensor maps of recent calls.  A map depends only on its encoding arguments (the
// address, the extents and the box), so a cached one is reused whenever all of them match;
// the cache never dereferences the address.  Serving loops that call the prefill with the
// same buffers every time then skip the host-side encoding.
struct MapKey {
  int type;
  uint32_t esize, inner, rows;
  const void *ptr;
  uint64_t d0, d1, d2;
  bool operator==(const MapKey &o) const {
    return type == o.type && esize == o.esize && inner == o.inner && rows == o.rows && ptr == o.ptr && d0 == o.d0 &&
           d1 == o.d1 && d2 == o.d2;
  }
};
constexpr int kMapCacheSize = 64;
struct MapCache {
  std::mutex mu;
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  int used = 0, next = 0;
};
MapCache &map_cache() {
  static MapCache c;
  return c;
}

// 3-D tensor map {d0 (contiguous), d1, d2}, box {inner, rows, 1}, 128-byte swizzle.
bool make_map_t(CUtensorMap *m, CUtensorMapDataType type, uint32_t esize, const void *ptr, uint64_t d0, uint64_t d1,
                uint64_t d2, uint32_t inner, uint32_t rows) {
  const MapKey k{(int)type, esize, inner, rows, ptr, d0, d1, d2};
  MapCache &c = map_cache();
  {
    std::lock_guard<std::mutex> lock(c.mu);
    for (int i = 0; i < c.used; ++i)
      if (c.key[i] == k) {
        *m = c.map[i];
        return true;
      }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
  const cuuint32_t box[3] = {inner, rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (fn(m, type, 3, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(c.mu);
  const int slot = c.used < kMapCacheSize ? c.used++ : (c.next++ % kMapCacheSize);
  c.key[slot] = k;
  c.map[slot] = *m;
  return true;
}
// 3-D bf16 tensor map {d0 (contiguous), d1, d2} with a {64, rows, 1} box and 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t rows) {
  return make_map_t(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, d0, d1, d2, 64, rows);
}

size_t k1_smem_bytes(int Q) { return 1024 + K1Smem::misc(Q) + sizeof(K1Misc); }

// The kernels' dynamic shared-memory limits, raised once per device (a per-function
// attribute of the current device's module) to the largest size any call launches with:
// chunk_state's for Q = 256, chunk_scan's fixed size.
cudaError_t set_smem_limits_once() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(k_chunk_state_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)k1_smem_bytes(256));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_chunk_state_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)k1_smem_bytes(256));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_chunk_scan_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kK3SmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_state_passing_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kK2SmemBytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
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

// Head split of the chunk-scan kernel.  A CTA of the second row tile costs about 1.26x a
// first-tile CTA per head (twice the x tile and the in-chunk product; measured); each also
// pays a fixed set-up of about 1.8 first-tile heads.  Every pair of head-block sizes is
// scored by simulating the hardware's greedy, in-order placement of CTAs onto SMs (one
// CTA per SM at a time); ties go to the split with fewer CTAs.
struct ScanSplit {
  int kb0, nhb0, kb1, nhb1;
};

double simulate_makespan(int groups, int hpg, int kb0, int kb1, int ntt, int sms) {
  constexpr double kSetup = 1.8, kTile1 = 1.26;
  std::priority_queue<double, std::vector<double>, std::greater<double>> q;
  for (int i = 0; i < sms; ++i) q.push(0.0);
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
  long best_ctas = 0;
  // Only block sizes that give a distinct block count are worth scoring.
  std::vector<int> sizes;
  for (int nb = 1; nb <= hpg; ++nb) {
    const int kb = (hpg + nb - 1) / nb;
    if (sizes.empty() || sizes.back() != kb) sizes.push_back(kb);
  }
  for (int kb1 : (ntt > 1 ? sizes : std::vector<int>{hpg}))
    for (int kb0 : sizes) {
      const int nhb0 = (hpg + kb0 - 1) / kb0, nhb1 = ntt > 1 ? (hpg + kb1 - 1) / kb1 : 0;
      const long ctas = (long)groups * (nhb0 + nhb1);
      const double t = simulate_makespan(groups, hpg, kb0, kb1, ntt, sms);
      if (t < best_t - 1e-9 || (t < best_t + 1e-9 && ctas < best_ctas)) {
        best_t = t;
        best_ctas = ctas;
        best = {kb0, nhb0, kb1, nhb1};
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

size_t tc_prefill_smem_k1(int Q) { return k1_smem_bytes(Q); }
size_t tc_prefill_table_floats(const Dims &d, int Q, int nc) { return (size_t)d.b * d.H * nc * tab_row_floats(Q); }
size_t tc_prefill_smem_k3() { return kK3SmemBytes; }

cudaError_t launch_tc_prefill(const __nv_bfloat16 *x, const float *dt, const float *A, const __nv_bfloat16 *B,
                              const __nv_bfloat16 *C, const float *D, const float *init, float *y, float *final_state,
                              float *cstates, float *tab, float *states, float *cdecay, __nv_bfloat16 *hprev, int *err,
                              const Dims &d, int Q, int nc, cudaStream_t st, const cudaEvent_t *ev) {
  CUtensorMap tm_x1, tm_B1, tm_x3, tm_x3b, tm_C3, tm_B3, tm_h3, tm_y3;
  const uint64_t HP = (uint64_t)d.H * d.P, GN = (uint64_t)d.G * d.N;
  if (!make_map(&tm_x1, x, HP, d.L, d.b, Q) || !make_map(&tm_B1, B, GN, d.L, d.b, Q) ||
      !make_map(&tm_x3, x, HP, d.L, d.b, 128) || !make_map(&tm_x3b, x, HP, d.L, d.b, 256) ||
      !make_map(&tm_C3, C, GN, d.L, d.b, 128) ||
      !make_map(&tm_B3, B, GN, d.L, d.b, 128) ||
      !make_map(&tm_h3, hprev, 64, 2 * (uint64_t)d.P, (uint64_t)d.b * nc * d.H, 2 * d.P) ||
      !make_map_t(&tm_y3, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, y, HP, d.L, d.b, 32, 32))
    return cudaErrorInvalidValue;
  const int sms = num_sms();
  auto mark = [&](int i) { return ev ? cudaEventRecord(ev[i], st) : cudaSuccess; };
  // Without per-kernel events each kernel overlaps its set-up with the tail of the one
  // before (programmatic dependent launch); with events between them they run serially.
  const bool pdl = ev == nullptr;
  cudaError_t e = mark(0);
  if (e != cudaSuccess) return e;
  if ((e = set_smem_limits_once()) != cudaSuccess) return e;
  // K1
  {
    const int base_items = d.b * nc * d.G;
    const int kb = std::min(K1_KB_MAX, pick_heads_per_cta(base_items, d.hpg, sms, 1.0));
    const int nhb = (d.hpg + kb - 1) / kb;
    const int nitems = base_items * nhb;
    if (nitems > sms)  // more items than SMs: a persistent grid, one CTA per SM
      e = launch_after(dim3((unsigned)sms), K1_THREADS, tc_prefill_smem_k1(Q), st, pdl, k_chunk_state_tc<true>, tm_x1,
                       tm_B1, dt, A, D, tab, cdecay, states, err, d, Q, nc, kb, nhb, nitems);
    else
      e = launch_after(dim3((unsigned)nitems), K1_THREADS, tc_prefill_smem_k1(Q), st, pdl, k_chunk_state_tc<false>,
                       tm_x1, tm_B1, dt, A, D, tab, cdecay, states, err, d, Q, nc, kb, nhb, nitems);
    if (e != cudaSuccess) return e;
  }
  if ((e = mark(1)) != cudaSuccess) return e;
  // K2
  {
    if (nc <= K2_ROUND) {  // every chunk of a column fetched at once by its thread
      const int per_head = d.P * d.N / 4;
      const dim3 grid(d.b * d.H, (per_head + K2R_THREADS - 1) / K2R_THREADS);
      e = cstates ? launch_after(grid, K2R_THREADS, kK2RSmemBytes, st, pdl, k_state_passing_rounds<true>, states,
                                 cdecay, hprev, init, final_state, cstates, d, nc)
                  : launch_after(grid, K2R_THREADS, kK2RSmemBytes, st, pdl, k_state_passing_rounds<false>, states,
                                 cdecay, hprev, init, final_state, cstates, d, nc);
    } else {
      // one wave: the batch rows' state columns split evenly over the SMs, at most
      // K2_MAX_COLS per thread (more CTAs, in several waves, past that)
      const long rowcols = (long)d.H * d.P * d.N / 4;
      const long per_sm = ((long)d.b * rowcols + sms - 1) / sms;
      const int cpc = (int)std::min<long>((long)K2_MAX_COLS * K2_THREADS, std::max<long>(per_sm, 1));
      const int parts = (int)((rowcols + cpc - 1) / cpc);
      e = launch_after(dim3((unsigned)(d.b * parts)), K2_THREADS, kK2SmemBytes, st, pdl, k_state_passing_bf16, states,
                       cdecay, hprev, init, final_state, cstates, err, d, nc, cpc, parts);
    }
    if (e != cudaSuccess) return e;
  }
  if ((e = mark(2)) != cudaSuccess) return e;
  // K3
  {
    const int ntt = Q / 128;
    const int groups = d.b * nc * d.G;
    const ScanSplit sp = pick_scan_split(groups, d.hpg, ntt, sms);
    e = launch_after(dim3((unsigned)(groups * (sp.nhb0 + sp.nhb1))), K3_THREADS, kK3SmemBytes, st, pdl,
                     k_chunk_scan_tc, tm_x3, tm_x3b, tm_C3, tm_B3, tm_h3, tm_y3, (const float *)tab, err, d, Q, nc, sp.kb0,
                     sp.nhb0, sp.kb1, sp.nhb1);
    if (e != cudaSuccess) return e;
  }
  return mark(3);
}

}  // namespace ssd
