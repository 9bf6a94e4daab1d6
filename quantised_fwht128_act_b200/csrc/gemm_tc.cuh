// IQ8R linear on the 5th-generation tensor cores (tcgen05, kind::i8) for
// prefill-sized M: the one place the layer is a dense contraction.
//
// y[m][n] = a[m] * s2[n] / 128 * sum_g s1[n][g] * P[m][n][g] (trunk) or
// a[m] / 128 * sum_g s[n][g] * P[m][n][g] (lm_head), P the exact int32 dot
// product over 256-K (128-K) block g -- the W8A8 linear of "Qwen3.8-27B IQ8R
// + DFlash2 -- radiance container" (rows "Weights" and "Activations"). The
// u8 sub-scale changes every 256 of K, so each block's int32 result leaves
// the tensor core and is promoted into an fp32 sum by the epilogue.
//
// Design (sm_100a, one CTA per SM, persistent over output tiles):
//  - operands swapped so the per-row weight scales are per thread: the MMA's
//    M side is a 128-row weight tile (TMEM lanes), its N side BM <= 256
//    tokens (TMEM columns); D[n][m] = sum_k W[n][k] * Xq[m][k], both K-major;
//  - warp 0 (one lane) loads 128-K slices of both operands with 2-D TMA
//    (128-byte swizzle) into a 4-stage ring, activations evict-last in L2
//    (they are reused by every weight tile); the output is stored streaming
//    (evict-first) so it does not push out weight tiles other CTAs still read;
//  - warp 1 owns the tensor memory: it allocates 2..8 int32 accumulators of
//    BM columns (as many as 512 columns hold, so the epilogue may lag several
//    blocks behind on small tiles) and one lane issues tcgen05.mma (4 per
//    stage, K = 32 each), always accumulating, one accumulator per 256-K block
//    in turn, committing to mbarriers;
//  - warps 2..9 are the epilogue: warp e covers TMEM lanes 32 (warp % 4) of
//    column group e / 4 (half the tile's tokens). The accumulators start each block at the bits of
//    1.5 * 2^23, so the int32 sums read back (tcgen05.ld) are the floats
//    1.5 * 2^23 + P: one packed f32x2 subtract makes P exact and one packed
//    f32x2 FMA adds P times the row's sub-scale into fp32 registers; the
//    epilogue writes the bias back (tcgen05.st) before releasing the buffer.
//    At the tile's end it applies a[m] * s2[n] / 128 and stores bf16. Tiles walk the token dimension fastest, so concurrently
//    running CTAs share weight tiles and the activations stay in L2.
#pragma once

#include <cuda.h>

#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kTcBN = 128;            // weight rows per tile (MMA M)
constexpr int kTcMaxBM = 256;         // tokens per tile (MMA N)
constexpr int kTcStageK = 128;        // K bytes per stage: one 128-byte swizzle row
constexpr int kTcStages = 4;          // stages of the largest (BM = 256) stage size
constexpr int kTcMaxStages = 12;      // smaller token tiles get more, smaller stages
constexpr int kTcMaxAcc = 8;          // TMEM accumulators: 512 columns / bm, at most 8
constexpr int kTcEpiWarps = 8;                 // 4 TMEM lane quarters x kTcGroups column groups
constexpr int kTcGroups = kTcEpiWarps / 4;
constexpr int kTcThreads = (2 + kTcEpiWarps) * 32;
constexpr int kTcStageA = kTcBN * kTcStageK;                // 16 KB
constexpr int kTcStageB = kTcMaxBM * kTcStageK;             // 32 KB
constexpr int kTcStageBytes = kTcStageA + kTcStageB;        // 48 KB
constexpr int kTcRingBytes = kTcStages * kTcStageBytes;     // 192 KB for the operand ring
// ring, then barriers (2 x 12 + 2 x 8 + 1) x 8 B, the TMEM address and flags, 2 x 256
// activation scales; plus 1 KB to align the ring to 1024 bytes
constexpr int kTcSmemBytes = kTcRingBytes + 4096 + 1024;
// Small token tiles (BM <= 64: verify blocks and few-token lm_head calls):
// two CTAs an SM, each with half the operand ring and at most 256 TMEM
// columns, so one CTA's stalls (unit boundaries, the epilogue) are covered
// by the other's weight stream. Measured on B200 at BM = 32: verify8/16
// 36 -> 27 us a GEMM, lm_head M = 8 213 -> 143 us.
constexpr int kTcRingBytesSmall = 96 * 1024;
__host__ __device__ constexpr int tc_ctas_per_sm(int bmax) { return bmax <= 64 ? 2 : 1; }
__host__ __device__ constexpr int tc_ring_bytes(int bmax) { return bmax <= 64 ? kTcRingBytesSmall : kTcRingBytes; }
__host__ __device__ constexpr int tc_smem_bytes(int bmax) { return tc_ring_bytes(bmax) + 4096 + 1024; }
// Split-K partial tiles: fp32 [BM][128] per unit, BM <= 128 when split.
constexpr int kTcSplitMaxBM = 128;

struct TcParams {
  int64_t m;          // tokens
  int64_t n;          // weight rows
  int k;              // K (multiple of 256 for the trunk, 128 for lm_head)
  int bm;             // tokens per tile: multiple of 16, 16..256
  int fmt;            // 0 trunk, 1 lm_head
  int rotated;
  int64_t tiles_m;    // token tiles
  int64_t tiles;      // output tiles (tiles_m x weight tiles)
  int splits;         // K ranges per tile (split-K), >= 1; a unit is (tile, split)
  int64_t units;      // tiles x splits
  int stages;         // operand ring depth (stage = 16 KB weights + bm x 128 tokens)
  int nacc;           // TMEM accumulators of bm columns (2 .. kTcMaxAcc)
  int stage_bytes;
  int stream_w;       // 1: weights are read once (one token tile): evict-first
  float* ws;          // split > 1: fp32 [units][128][bm] partial tiles
  const float* xs;    // [m] activation scales
  const uint8_t* sub; // [n][k/256]
  const uint16_t* scale;  // [n] or [n][k/128]
  uint16_t* y;        // [m][n], or nullptr in partials mode
  int32_t* partials;  // [m][n][k/G] in partials mode
  uint32_t tmem_cols; // columns allocated: 2 * bm rounded up to a power of two >= 32
  int weights_after_wait;  // 1: no weight tile before the previous kernel completes
};

// ------------------------------------------------------------ tcgen05 / TMA

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand stored as rows of
// 128 bytes with the 128-byte swizzle (8-row atoms of 1024 bytes): start
// address >> 4, leading offset 1 (unused for swizzled K-major), stride 1024 B
// between 8-row groups, descriptor version 1, swizzle mode 2 (128 B).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor, kind::i8: s32 accumulator, signed int8 A and B,
// both K-major, M = 128, N = bm.
__device__ __forceinline__ uint32_t umma_idesc_i8(int bm) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(bm >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The mbarrier arrives once every tcgen05 op this thread issued before has
// completed (MMAs reading shared memory and writing TMEM).
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns starting at taddr.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns, all set to v.
__device__ __forceinline__ void tmem_st16_fill(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
      "%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The accumulators start every block at the bits of 1.5 * 2^23 (as an int32)
// instead of 0, so the MMA's exact int32 sum P (|P| < 2^22) lands in the
// float 1.5 * 2^23 + P, and subtracting 1.5 * 2^23 recovers P exactly.
constexpr uint32_t kTcBiasBits = 0x4B400000u;
constexpr float kTcBias = 12582912.0f;

// Two fp32 lanes in one 64-bit register: Blackwell's packed f32x2 add and
// fma do both halves in one instruction, each rounded like the scalar op.
__device__ __forceinline__ uint64_t u2_pack(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ uint64_t f2_splat(float v) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// ------------------------------------------------------------------ kernel

// BMAX: the largest token tile the instance handles (256, or 128 for the
// split-K capable instance, whose epilogue keeps half the registers).
template <int FMT, bool PARTIALS, int BMAX>
__global__ void __launch_bounds__(kTcThreads, tc_ctas_per_sm(BMAX))
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                   const TcParams p) {
  constexpr int kCols = BMAX / kTcGroups;  // most tokens per epilogue column group
  constexpr bool kCanSplit = BMAX <= kTcSplitMaxBM && !PARTIALS;
  constexpr int G = FMT == 0 ? kGroupTrunk : kGroupHead;
  constexpr int SPB = G / kTcStageK;  // stages per scale block: 2 (trunk) or 1 (lm_head)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled TMA tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + tc_ring_bytes(BMAX));
  uint64_t* empty = full + kTcMaxStages;
  uint64_t* acc_full = empty + kTcMaxStages;
  uint64_t* acc_empty = acc_full + kTcMaxAcc;
  uint64_t* mma_done = acc_empty + kTcMaxAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  float* sa = reinterpret_cast<float*>(tmem_slot + 4);  // [2][kTcMaxBM] activation scales per tile
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = p.k;
  const int ng = K / G;                // scale blocks per row
  const int bm = p.bm;
  const int S = kCanSplit ? p.splits : 1;  // instances that never split keep the plain tile loop
  const int nst = p.stages;
  const int nacc = p.nacc;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int st = 0; st < nst; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    for (int b = 0; b < nacc; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kTcEpiWarps);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // set-up above overlaps the previous kernel's tail. Its outputs (the
  // activation codes and scales) are read only after it has completed, and
  // this kernel's own outputs are written only after that too; the producer
  // streams the first ring of weight tiles before it waits (the weights are
  // no earlier kernel's output, unless the caller says otherwise)
  pdl_launch_dependents();
  if (warp != 0 || p.weights_after_wait) pdl_wait();

  // A unit is one output tile over one K range: blocks [g0, g1) of the tile's
  // ng scale blocks, split s of S (the tile's K split evenly in blocks).
  auto unit_range = [&](int64_t u, int64_t& tile, int& split, int& g0, int& g1) {
    tile = u / S;
    split = static_cast<int>(u - tile * S);
    g0 = static_cast<int>((static_cast<int64_t>(split) * ng) / S);
    g1 = static_cast<int>((static_cast<int64_t>(split + 1) * ng) / S);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = p.stream_w ? l2_policy_evict_first() : l2_policy_evict_normal();
      const uint64_t pol_x = l2_policy_evict_last();
      const uint32_t tx = kTcStageA + bm * kTcStageK;
      // the first `pre` stages' weight tiles go out before the wait for the
      // previous kernel; their activation tiles follow it
      uint32_t pre = 0;
      if (!p.weights_after_wait) {
        for (int64_t u = blockIdx.x; u < p.units && pre < static_cast<uint32_t>(nst); u += gridDim.x) {
          int64_t tile;
          int split, g0, g1;
          unit_range(u, tile, split, g0, g1);
          const int n0 = static_cast<int>((tile / p.tiles_m) * kTcBN);
          for (int kb = g0 * SPB; kb < g1 * SPB && pre < static_cast<uint32_t>(nst); ++kb, ++pre) {
            mbar_arrive_expect_tx(&full[pre], tx);
            tma_load_2d(stage_base + pre * p.stage_bytes, &tmap_w, kb * kTcStageK, n0, &full[pre], pol_w);
          }
        }
        pdl_wait();
      }
      uint32_t it = 0;   // stages issued
      int st = 0;        // ring slot of stage `it`
      uint32_t ph = 0;   // its use count & 1
      bool ok = true;
      for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        int64_t tile;
        int split, g0, g1;
        unit_range(u, tile, split, g0, g1);
        const int m0 = static_cast<int>((tile % p.tiles_m) * bm);
        const int n0 = static_cast<int>((tile / p.tiles_m) * kTcBN);
        for (int kb = g0 * SPB; kb < g1 * SPB; ++kb, ++it) {
          uint8_t* sp = stage_base + st * p.stage_bytes;
          if (it < pre) {
            // armed and its weight tile issued before the wait
            tma_load_2d(sp + kTcStageA, &tmap_x, kb * kTcStageK, m0, &full[st], pol_x);
            if (++st == nst) {
              st = 0;
              ph ^= 1u;
            }
            continue;
          }
          if (s_abort || (it >= static_cast<uint32_t>(nst) && !mbar_wait(&empty[st], ph ^ 1u, kDevErrTcEmpty))) {
            s_abort = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[st], tx);
          tma_load_2d(sp, &tmap_w, kb * kTcStageK, n0, &full[st], pol_w);
          tma_load_2d(sp + kTcStageA, &tmap_x, kb * kTcStageK, m0, &full[st], pol_x);
          if (++st == nst) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      // never leave with a copy still landing in this CTA's shared memory
      // (stages armed before the wait count as issued: their weight tiles are)
      if (it < pre) it = pre;
      const uint32_t first = it > static_cast<uint32_t>(nst) ? it - nst : 0u;
      for (uint32_t j = first; j < it; ++j)
        if (!mbar_wait(&full[j % nst], (j / nst) & 1u, kDevErrTcDrain)) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(bm);
      uint32_t it = 0;   // stages consumed
      int st = 0;        // ring slot of stage `it`
      uint32_t ph = 0;   // its use count & 1
      int buf = 0;       // accumulator of the current block
      uint32_t aph = 0;  // its use count & 1
      bool ok = true;
      for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        int64_t tile;
        int split, g0, g1;
        unit_range(u, tile, split, g0, g1);
        for (int kb = g0 * SPB; kb < g1 * SPB && ok; ++kb, ++it) {
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * bm);
          if (kb % SPB == 0) {
            // the accumulator must have been drained by the epilogue and
            // reset to the bias (the epilogue seeds all of them at the start)
            if (s_abort || !mbar_wait(&acc_empty[buf], aph, kDevErrTcAccEmpty)) {
              s_abort = 1;
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (s_abort || !mbar_wait(&full[st], ph, kDevErrTcFull)) {
            s_abort = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(stage_base + st * p.stage_bytes);
          const uint32_t b_addr = a_addr + kTcStageA;
#pragma unroll
          for (int k = 0; k < kTcStageK / 32; ++k) {
            // advancing K by 32 bytes inside the swizzle atom moves the start address
            umma_i8(d_tmem, umma_desc_sw128(a_addr + 32 * k), umma_desc_sw128(b_addr + 32 * k), idesc, 1u);
          }
          umma_commit(&empty[st]);  // the stage can be refilled once these MMAs have read it
          if (++st == nst) {
            st = 0;
            ph ^= 1u;
          }
          if (kb % SPB == SPB - 1) {
            umma_commit(&acc_full[buf]);  // the block's int32 sums are complete
            if (++buf == nacc) {
              buf = 0;
              aph ^= 1u;
            }
          }
        }
      }
      // every MMA issued here, complete or not, must be finished before the
      // tensor memory is released
      if (it > 0) {
        umma_commit(mma_done);
        mbar_wait(mma_done, 0u, kDevErrTcDrain);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;          // 0 .. kTcEpiWarps - 1
    const int q = e >> 2;            // column group: tokens [q * cols, (q + 1) * cols) of the tile
    const int lq = warp & 3;         // TMEM lane quarter this warp may access
    const int cols = bm / kTcGroups; // tokens per column group (a multiple of 16 when bm is of 32)
    const int rloc = lq * 32 + lane; // this thread's row within the weight tile
    const uint32_t lane_addr = static_cast<uint32_t>(lq * 32) << 16;
    const float rot = p.rotated ? 0.0078125f : 1.0f;
    constexpr int kSD = BMAX >= 256 ? 4 : 8;  // blocks of scale prefetch
    auto load_scale = [&](int64_t i) -> uint32_t {
      return FMT == 0 ? static_cast<uint32_t>(__ldg(p.sub + i)) : static_cast<uint32_t>(__ldg(p.scale + i));
    };
    // seed every accumulator with the bias (this warp's lanes and columns)
    for (int b = 0; b < nacc; ++b) {
      const uint32_t t0 = tmem_base + lane_addr + static_cast<uint32_t>(b * bm + q * cols);
      for (int c = 0; c < cols; c += 16) tmem_st16_fill(t0 + c, kTcBiasBits);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int b = 0; b < nacc; ++b) mbar_arrive(&acc_empty[b]);
    const uint64_t neg_bias = f2_splat(-kTcBias);
    int buf = 0;       // accumulator of the current block
    uint32_t aph = 0;  // its use count & 1
    int par = 0;
    bool failed = false;
    for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x, par ^= 1) {
      int64_t tile;
      int split, g0, g1;
      unit_range(u, tile, split, g0, g1);
      const int64_t m0 = (tile % p.tiles_m) * bm;
      const int64_t n0 = (tile / p.tiles_m) * kTcBN;
      const int64_t n = n0 + rloc;  // this thread's weight row
      const bool nvalid = n < p.n;
      // activation scales of the tile's tokens, shared by all epilogue warps
      if (!PARTIALS) {
        for (int i = e * 32 + lane; i < bm; i += kTcEpiWarps * 32)
          sa[par * kTcMaxBM + i] = (m0 + i < p.m) ? p.xs[m0 + i] : 0.0f;
      }
      float s2f = 0.0f;
      if (FMT == 0 && !PARTIALS && nvalid) s2f = bf16_bits_to_float(p.scale[n]);
      uint64_t acc[kCols / 2];  // fp32 pairs
#pragma unroll
      for (int j = 0; j < kCols / 2; ++j) acc[j] = 0ull;
      // the row's block scales, loaded kSD blocks ahead of use: while the
      // weight stream keeps HBM busy a scattered load takes microseconds
      uint32_t sq[kSD];
#pragma unroll
      for (int i = 0; i < kSD; ++i) sq[i] = (!PARTIALS && nvalid && g0 + i < g1) ? load_scale(n * ng + g0 + i) : 0u;
      for (int gb = g0; gb < g1; gb += kSD)
#pragma unroll
      for (int i = 0; i < kSD; ++i) {
        const int g = gb + i;
        if (g >= g1) break;
        const uint64_t sg = f2_splat(FMT == 0 ? static_cast<float>(sq[i]) : bf16_bits_to_float(static_cast<uint16_t>(sq[i])));
        if (!PARTIALS && nvalid && g + kSD < g1) sq[i] = load_scale(n * ng + g + kSD);
        if (!failed) {
          bool bad = s_abort != 0;
          if (!bad) bad = !mbar_wait(&acc_full[buf], aph, kDevErrTcAccFull);
          failed = !__all_sync(0xffffffffu, !bad);
          if (failed && lane == 0) s_abort = 1;
        }
        tc_fence_after();
        const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(buf * bm + q * cols);
        // with few columns per thread, chunk c + 1 loads while chunk c is
        // converted and summed; with many, registers are kept for the sums
        constexpr bool kPipe = kCols <= 64;
        uint32_t rn[16];
        if (kPipe && !failed) {
          tmem_ld16(tbase, rn);
          tmem_wait_ld();
        }
#pragma unroll
        for (int c = 0; c < kCols; c += 16) {
          if (c < cols) {
            uint32_t r[16];
            if (kPipe) {
#pragma unroll
              for (int j = 0; j < 16; ++j) r[j] = rn[j];
              if (!failed && c + 16 < cols) tmem_ld16(tbase + c + 16, rn);
            } else if (!failed) {
              tmem_ld16(tbase + c, r);
              tmem_wait_ld();
            }
            tmem_st16_fill(tbase + c, kTcBiasBits);  // reset for the block after next
            if (failed) continue;
            if (PARTIALS) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int64_t m = m0 + q * cols + c + j;
                if (nvalid && m < p.m)
                  p.partials[(m * p.n + n) * ng + g] = static_cast<int32_t>(r[j] - kTcBiasBits);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; j += 2) {
                const uint64_t v = f2_add(u2_pack(r[j], r[j + 1]), neg_bias);  // exact: P
                acc[(c + j) / 2] = f2_fma(v, sg, acc[(c + j) / 2]);
              }
            }
            if (kPipe && c + 16 < cols) tmem_wait_ld();
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        if (++buf == nacc) {
          buf = 0;
          aph ^= 1u;
        }
      }
      if (PARTIALS) continue;
      if (kCanSplit && S > 1) {
        // split-K: publish this unit's fp32 partial tile, row-major [128][bm]
        // (this thread's row, its column group: cols consecutive floats); a
        // second kernel adds the S partials of every tile in split order
        float* wsu = p.ws + static_cast<size_t>(u) * kTcBN * bm + static_cast<size_t>(rloc) * bm + q * cols;
#pragma unroll
        for (int j = 0; j < kCols; j += 4) {
          if (j < cols) {
            float a0, a1, a2, a3;
            f2_unpack(acc[j / 2], a0, a1);
            f2_unpack(acc[j / 2 + 1], a2, a3);
            __stcg(reinterpret_cast<float4*>(wsu + j), make_float4(a0, a1, a2, a3));
          }
        }
        continue;
      }
      // all epilogue warps have staged their part of sa before anyone reads it
      named_barrier(1, kTcEpiWarps * 32);
      if (!failed && nvalid) {
        const float rs = (FMT == 0 ? s2f : 1.0f) * rot;
#pragma unroll
        for (int j = 0; j < kCols; j += 2) {
          float a0, a1;
          f2_unpack(acc[j / 2], a0, a1);
          const int64_t m = m0 + q * cols + j;
          if (j < cols && m < p.m)
            __stcs(p.y + m * p.n + n, float_to_bf16_bits_rn(a0 * sa[par * kTcMaxBM + q * cols + j] * rs));
          if (j + 1 < cols && m + 1 < p.m)
            __stcs(p.y + (m + 1) * p.n + n, float_to_bf16_bits_rn(a1 * sa[par * kTcMaxBM + q * cols + j + 1] * rs));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(p.tmem_cols)
                 : "memory");
  }
}

}  // namespace iq8r
