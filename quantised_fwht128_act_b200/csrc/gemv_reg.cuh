// Weight-streaming IQ8R GEMV for one or two tokens, streamed by per-lane
// vector loads into registers (the decode step).
//
// y[m][n] = a[m] * s2[n] * sum_g s1[n][g] * P[m][n][g] / 128 (trunk) or
// a[m] / 128 * sum_g s[n][g] * P[m][n][g] (lm_head), P the exact int32 dot
// product of int8 codes over block g -- the W8A8 linear of "Qwen3.8-27B
// IQ8R + DFlash2 -- radiance container" (rows "Weights" and "Activations").
// At one or two tokens the layer is bound by streaming the int8 codes from
// HBM (the page's "Speed" section: the IQ8R decode step runs as fast as
// FP8's, the same bytes a weight).
//
// Design (sm_100a):
//  - persistent grid, one CTA per SM, each CTA a contiguous range of rows;
//    its 16 warps claim rows from a counter in shared memory;
//  - a unit is half of a 5 KB row (5 steps of 512 bytes: 16 bytes a lane a
//    step); each warp keeps three units in flight in registers, loaded with
//    16-byte non-coherent loads that bypass L1. When a unit's dot products
//    are done its registers are refilled at once with the warp's next unit.
//    On B200 this streams at the copy bandwidth across back-to-back
//    launches, where 1-D bulk copies into shared-memory stages lost about a
//    third of it (issuing a bulk copy can hold the issuing warp for a
//    microsecond when the SM's copy engine is busy, and the first refills
//    of a launch came late);
//  - the block scales of the CTA's rows (u8 sub-scales and bf16 row scales,
//    or the lm_head's bf16 scales) are one bulk copy into shared memory at
//    the start; the activation codes are rotated and quantised here (fused)
//    or copied in;
//  - programmatic dependent launch: the first units of weights are loaded
//    before the wait for the previous kernel (unless the caller said that
//    kernel wrote the weights); activations, outputs and everything else
//    come after it;
//  - arithmetic as gemv_kernel's: dp4a per 16 bytes; trunk: each block's
//    int32 sum scaled by its u8 sub-scale in int32 (exact), folded to int64
//    every unit; lm_head: one fp32 fma a step with the block's scale, in K
//    order; one fp32 scale product and one bf16 rounding per output. The
//    outputs are the same bits as gemv_kernel's.
#pragma once

#include "act_quant.cuh"
#include "gemv.cuh"
#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kRegWarps = 16;
constexpr int kRegPartSteps = 5;  // 512-byte steps a unit
constexpr int kRegUnits = 3;      // units in flight a warp
constexpr int kRegPartBytes = kRegPartSteps * 512;

// Launch shape (host, see gemv_reg_plan).
struct RegPlan {
  int64_t rows_base;  // rows a CTA; the first rows_extra CTAs take one more
  int64_t rows_extra;
  int parts;          // units a row
  int sc_bytes;       // shared-memory window of the CTA's block scales
  int smem;           // dynamic shared memory
};

// 16 bytes of streamed weights: read-only for the kernel, not kept in L1.
__device__ __forceinline__ int4 ldg_weights(const int8_t* p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
// The same through the coherent path, for weights the previous kernel on
// the stream may have written (read only after waiting for it).
__device__ __forceinline__ int4 ldg_weights_coherent(const int8_t* p) {
  int4 v;
  asm volatile("ld.global.L1::no_allocate.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// AFTER: the caller said the previous kernel on the stream wrote the weights
// (IQ8R_PATH_FLAG_WEIGHTS_WRITTEN): they are read through the coherent path,
// and only after waiting for that kernel. A template parameter, so each
// instance has a single form of the load (a runtime choice between the two
// can cost a wait on every load).
template <int MT, int FMT, bool FUSED, bool AFTER>
__global__ void __launch_bounds__(kRegWarps * 32, 1) gemv_reg_kernel(const LinearArgs a, const RegPlan p) {
  constexpr int G = FMT == 0 ? kGroupTrunk : kGroupHead;
  constexpr int PS = kRegPartSteps;
  constexpr int NB = kRegUnits;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t prebar;
  __shared__ int counter;
  __shared__ float red[MT * 32];

  const int K = static_cast<int>(a.k);
  const int64_t N = a.n;
  const int M = static_cast<int>(a.m);
  const int ng = K / G;
  const int lane = threadIdx.x & 31;
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  uint8_t* scw = smem + gemv_align128(MT * K);  // block scales of the CTA's rows
  const int64_t bid = blockIdx.x;
  const int64_t r0 = bid * p.rows_base + (bid < p.rows_extra ? bid : p.rows_extra);
  const int R = static_cast<int>(p.rows_base + (bid < p.rows_extra ? 1 : 0));
  // trunk: [s1 of the rows: R * ng bytes][s2 of the rows: 2R bytes], each in
  // its 16-byte window; lm_head: the rows' bf16 scales, 2 * R * ng bytes
  const int s1_win = gemv_align16(R * ng + 32);

  // one lane: the bulk copies of the scale windows
  auto issue_scales = [&]() {
    GemvWindow w0, w1{nullptr, nullptr, 0u};
    if (FMT == 0) {
      w0 = window_copy_plan(scw, a.sub, N * ng, r0 * ng, (r0 + R) * ng, true);
      w1 = window_copy_plan(scw + s1_win, reinterpret_cast<const uint8_t*>(a.scale), 2 * N, 2 * r0, 2 * (r0 + R),
                            true);
    } else {
      w0 = window_copy_plan(scw, reinterpret_cast<const uint8_t*>(a.scale), 2 * N * ng, 2 * r0 * ng,
                            2 * (r0 + R) * ng, true);
    }
    mbar_arrive_expect_tx(&prebar, w0.bytes + w1.bytes);
    for (uint32_t off = 0; off < w0.bytes; off += kGemvMaxCopy)
      bulk_g2s_default(w0.dst + off, w0.src + off, min(static_cast<uint32_t>(kGemvMaxCopy), w0.bytes - off), &prebar);
    if (w1.bytes) bulk_g2s_default(w1.dst, w1.src, w1.bytes, &prebar);
  };

  if (threadIdx.x == 0) {
    mbar_init(&prebar, 1);
    counter = 0;
    fence_barrier_init();
    if (!AFTER) issue_scales();
  }
  {  // token rows past M are zero (their codes never reach an output anyway)
    int4* pad = reinterpret_cast<int4*>(act + M * K);
    const int n16 = (MT - M) * K / 16;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) pad[i] = make_int4(0, 0, 0, 0);
  }
  __syncthreads();
  pdl_launch_dependents();

  // Units: the warp claims whole rows (lane 0, shared counter) and takes
  // their parts in order. Row -1: no more work.
  int cur_row = -1;
  int cur_part = 0;
  auto next_unit = [&](int& row, int& part) {
    if (cur_row >= 0 && cur_part + 1 < p.parts) {
      ++cur_part;
    } else {
      int c = 0;
      if (lane == 0) c = atomicAdd(&counter, 1);
      c = __shfl_sync(0xffffffffu, c, 0);
      cur_row = c < R ? c : -1;
      cur_part = 0;
    }
    row = cur_row;
    part = cur_part;
  };
  int4 buf[NB][PS];
  int brow[NB] = {};
  int bpart[NB] = {};
  // Loads carry no per-lane guard (an inline-assembly load cannot be
  // predicated, so a guard on each would be a branch on each): a step past
  // the row's end reads the row's last 16 bytes instead, and its weights are
  // zeroed where they are used.
  auto load = [&](int j) {
    if (brow[j] < 0) return;
    const int8_t* src = a.codes + (r0 + brow[j]) * K;
    const int k0 = bpart[j] * kRegPartBytes + lane * 16;
#pragma unroll
    for (int u = 0; u < PS; ++u) {
      const int kk = min(k0 + u * 512, K - 16);
      buf[j][u] = AFTER ? ldg_weights_coherent(src + kk) : ldg_weights(src + kk);
    }
  };

  // The first units hold only weights, which no earlier kernel writes: they
  // stream while the previous kernel on the stream finishes (unless the
  // caller said that kernel wrote them).
  if (AFTER) {
    pdl_wait();
    if (threadIdx.x == 0) issue_scales();
  }
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    next_unit(brow[j], bpart[j]);
    load(j);
  }
  pdl_wait();

  float xscale[MT];
  if (FUSED) {
    gemv_fused_act<MT>(a, act, xscale, red);
  } else {
    const int n16 = M * K / 16;
    for (int i = threadIdx.x; i < n16; i += blockDim.x)
      reinterpret_cast<int4*>(act)[i] = reinterpret_cast<const int4*>(a.xq)[i];
#pragma unroll
    for (int m = 0; m < MT; ++m) xscale[m] = m < M ? a.xs[m] : 0.0f;
    __syncthreads();
  }
  bool failed = !__all_sync(0xffffffffu, mbar_wait(&prebar, 0u, kDevErrGemvFull));
  const float rot = a.rotated ? 0.0078125f : 1.0f;
  // scales start inside their 16-byte windows (see window_copy_plan)
  const uint8_t* s1w = scw + ((r0 * ng) & 15);
  const uint16_t* s2w = reinterpret_cast<const uint16_t*>(scw + s1_win + ((2 * r0) & 15));
  const uint16_t* shw = reinterpret_cast<const uint16_t*>(scw + ((2 * r0 * ng) & 15));

  long long racc[MT];  // trunk: the row's sum so far
  float facc[MT];      // lm_head: the lane's sum so far
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    racc[m] = 0;
    facc[m] = 0.0f;
  }
  bool live = !failed;
  while (live) {
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (brow[j] < 0) {
        live = false;
        break;
      }
      const int row = brow[j];
      const int part = bpart[j];
      int acc32[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc32[m] = 0;
      if (part == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          racc[m] = 0;
          facc[m] = 0.0f;
        }
      }
      auto step = [&](int u) {
        const int kr = (part * PS + u) * 512 + lane * 16;
        const bool in = kr < K;  // past the row's end: zero weights (the products are 0)
        const int kk = in ? kr : K - 16;
        const int4 wv = in ? buf[j][u] : make_int4(0, 0, 0, 0);
        if (FMT == 0) {
          const int s1 = s1w[row * ng + kk / G];
#pragma unroll
          for (int m = 0; m < MT; ++m)
            acc32[m] += s1 * dot16(wv, *reinterpret_cast<const int4*>(act + m * K + kk));  // <= 5 steps of 255 * 16 * 127^2
        } else {
          const float s = bf16_bits_to_float(shw[row * ng + kk / G]);
#pragma unroll
          for (int m = 0; m < MT; ++m)
            facc[m] =
                fmaf(static_cast<float>(dot16(wv, *reinterpret_cast<const int4*>(act + m * K + kk))), s, facc[m]);
        }
      };
#pragma unroll
      for (int u = 0; u < PS; ++u) step(u);
      // the registers are free again: the warp's next unit streams into them
      next_unit(brow[j], bpart[j]);
      load(j);
      if (FMT == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) racc[m] += acc32[m];
      }
      if (part == p.parts - 1) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          float yv;
          if (FMT == 0) {
            long long v = racc[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            yv = __ll2float_rn(v) * xscale[m] * bf16_bits_to_float(s2w[row]) * rot;
          } else {
            float v = facc[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            yv = v * xscale[m] * rot;
          }
          if (lane == m && m < M) a.y[static_cast<int64_t>(m) * N + r0 + row] = float_to_bf16_bits_rn(yv);
        }
      }
    }
  }
  // the scale copy has landed before the CTA leaves (it writes shared memory)
  if (failed && threadIdx.x == 0) mbar_wait(&prebar, 0u, kDevErrGemvDrain);
}

}  // namespace iq8r
