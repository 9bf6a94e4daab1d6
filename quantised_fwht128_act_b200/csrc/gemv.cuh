// Weight-streaming IQ8R GEMV for small M, streaming through shared-memory
// stages filled by bulk copies. The library runs it for the partial sums
// (the debug twin below), for a GEMV forced at three to eight tokens, and
// where the register-streaming kernel (gemv_reg.cuh, the one- and two-token
// path) does not fit; its fused activation prologue (gemv_fused_act) and
// dot16 serve both.
//
// y[m][n] = a[m] * s2[n] * sum_g s1[n][g] * P[m][n][g] / 128 (trunk) or
// a[m] / 128 * sum_g s[n][g] * P[m][n][g] (lm_head), P the exact int32 dot
// product of int8 codes over block g -- the W8A8 linear of "Qwen3.8-27B IQ8R
// + DFlash2 -- radiance container" (rows "Weights" and "Activations").
// At M <= 8 the layer is bound by streaming the int8 codes from HBM (the
// page's "Speed" section: the IQ8R decode step runs as fast as FP8's, the
// same bytes a weight).
//
// Design (sm_100a), warp-autonomous streaming:
//  - persistent grid, one CTA per SM, each CTA a contiguous range of tiles
//    (balanced to one tile). A tile is RT whole weight rows (contiguous in
//    memory), or, when a row is longer than a stage, one row in K chunks;
//  - no producer warp: each warp (16 a CTA for one or two tokens, else 8)
//    owns D private stage buffers and keeps them full itself. One lane
//    claims the next tile from a per-CTA
//    counter and issues 1-D bulk copies (TMA engine) of the stage's codes and
//    scales (u8 sub-scales + bf16 row scales, or the lm_head's bf16 group
//    scales) completing on the buffer's mbarrier, weights evict-first in L2.
//    Only the activation codes are shared, loaded once;
//  - the warp consumes stages in the order it issued them: per 512-byte step
//    each lane holds 16 bytes of K; loads for 4 steps are issued before any
//    dp4a; activation registers are reused across the RG rows computed
//    together; the lane's partial is scaled by its block's u8 sub-scale in
//    int32 (exact) and folded into int64 every 16 steps;
//  - epilogue per tile: warp shuffles, the fp32 scale product and one bf16
//    rounding per output.
// PARTIALS instantiates the same loads and dp4a chains but reduces each
// block's 16 (or 8) lanes and writes P instead of y (the debug twin).
#pragma once

#include <type_traits>

#include "act_quant.cuh"
#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kGemvMaxWarps = 16;

// Warps per CTA: more warps hide more load latency; large token tiles need
// the registers of fewer threads.
__host__ __device__ constexpr int gemv_warps(int mt) { return mt <= 2 ? 16 : 8; }
constexpr int kGemvMaxDepth = 4;          // stage buffers per warp
constexpr int kGemvMaxRowsPerTile = 32;
constexpr int kGemvMaxCopy = 16 * 1024;   // bytes per bulk copy

// 512-byte steps whose loads are issued together: 4, fewer when the loaded
// int4 registers (MT activations + RG weights per step) would crowd out the rest.
__host__ __device__ constexpr int gemv_unroll(int mt, int rg) {
  return 96 / (4 * (mt + rg)) >= 4 ? 4 : (96 / (4 * (mt + rg)) >= 2 ? 2 : 1);
}

__host__ __device__ constexpr int gemv_align128(int x) { return (x + 127) & ~127; }
__host__ __device__ constexpr int gemv_align16(int x) { return (x + 15) & ~15; }

// Runtime shape of one launch (chosen on the host, see gemv_plan).
struct GemvPlan {
  int warps;        // warps per CTA (each streams its own stages)
  int rt;           // rows per tile
  int kc;           // bytes of K per stage: K, or a chunk when one row is split
  int depth;        // stage buffers per warp
  int stage_bytes;  // codes + scales of one stage, 128-aligned
  int sc_off;       // offset of the scales within a stage
  int s2_off;       // offset of the trunk's row scales within a stage
  int pre;          // trunk: 1 = the CTA's row scales are loaded once, up front
  int pre_s1;       // pre: bytes of the sub-scale window in shared memory
  int pre_bytes;    // pre: sub-scale window + row-scale window
  int smem;         // total dynamic shared memory
};

// Scale bytes of one stage: sub-scales (or group scales) for rt rows x kc,
// then (trunk) rt bf16 row scales. Each is fetched as the 16-byte-aligned
// window around its bytes, hence up to 32 bytes of slack per array.
__host__ __device__ constexpr int gemv_s1_window(int rt, int kc) { return gemv_align16(rt * (kc / kGroupTrunk) + 32); }
__host__ __device__ constexpr int gemv_sc_bytes(int fmt, int rt, int kc) {
  return fmt == 0 ? gemv_s1_window(rt, kc) + gemv_align16(2 * rt + 32)
                  : gemv_align16(rt * (kc / kGroupHead) * 2 + 32);
}

__host__ __device__ inline GemvPlan gemv_plan_for(int mt, int fmt, int k, int rt, int kc, int depth, int warps) {
  GemvPlan p{};
  p.warps = warps;
  p.rt = rt;
  p.kc = kc;
  p.depth = depth;
  p.sc_off = gemv_align16(rt * kc);
  p.s2_off = p.sc_off + gemv_s1_window(rt, kc);
  p.stage_bytes = gemv_align128(p.sc_off + gemv_sc_bytes(fmt, rt, kc));
  // [act MT*K][warps x depth stages][barriers: warps x depth + 1][counter]
  p.smem = gemv_align128(mt * k) + warps * depth * p.stage_bytes + 8 * (warps * depth + 2) + 16;
  return p;
}

// Stage size: as many whole rows as fit `target` bytes (at most 32), else one
// row in chunks of `target` (a multiple of 512) bytes.
__host__ __device__ inline GemvPlan gemv_plan(int mt, int fmt, int k, int target, int depth, int warps) {
  if (k <= target) {
    int rt = target / k;
    if (rt > kGemvMaxRowsPerTile) rt = kGemvMaxRowsPerTile;
    return gemv_plan_for(mt, fmt, k, rt, k, depth, warps);
  }
  return gemv_plan_for(mt, fmt, k, 1, target & ~511, depth, warps);
}

__device__ __forceinline__ int dot16(const int4 w, const int4 x) {
  int p = __dp4a(w.x, x.x, 0);
  p = __dp4a(w.y, x.y, p);
  p = __dp4a(w.z, x.z, p);
  p = __dp4a(w.w, x.w, p);
  return p;
}

// One issued stage, as the issuing lane described it to its warp.
struct GemvStage {
  int64_t tile;  // -1: nothing issued
  int chunk;
};

// Fused prologue: rotate and quantise the M token rows of x (bf16) into the
// shared activation buffer, one fp32 scale per token, with the same
// arithmetic as the standalone activation kernel (see act_quant.cuh): pass 1
// finds each token's amax, pass 2 repeats the identical transform and
// quantises. Every CTA does this for itself; CTA 0 writes the codes and scales
// back when asked. Called by all threads.
template <int MT>
__device__ __forceinline__ void gemv_fused_act(const LinearArgs& a, int8_t* act, float* xscale, float* red) {
  const int K = static_cast<int>(a.k);
  const int M = static_cast<int>(a.m);
  const int slots = K / kActSlot;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int iters = (slots + blockDim.x - 1) / blockDim.x;
  if (MT <= 2 && iters == 1) {
    // every thread holds at most one slot per token: one load and one
    // transform, kept in registers across the CTA-wide amax
    float v[MT][kActSlot];
    float mx1[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      mx1[m] = 0.0f;
      const int s = threadIdx.x;
      if (m < M && s < slots) {
        act_load_slot(a.x + static_cast<int64_t>(m) * K + s * kActSlot, v[m], false);
      } else {
#pragma unroll
        for (int i = 0; i < kActSlot; ++i) v[m][i] = 0.0f;
      }
      if (a.rotated) act_fwht_slot(v[m], lane);
      mx1[m] = act_slot_absmax(v[m]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx1[m] = fmaxf(mx1[m], __shfl_xor_sync(0xffffffffu, mx1[m], o));
      if (lane == 0) red[m * 32 + warp] = mx1[m];
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) {
        xscale[m] = 0.0f;
        continue;
      }
      float amax = 0.0f;
      for (int w = 0; w < nwarps; ++w) amax = fmaxf(amax, red[m * 32 + w]);
      const float inv = act_inv(amax);
      xscale[m] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
      act_prescale_slot(v[m], amax);
      if (static_cast<int>(threadIdx.x) < slots) act_store_slot(act + m * K + threadIdx.x * kActSlot, v[m], inv);
    }
  } else {
  float mx[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    mx[m] = 0.0f;
    if (m >= M) continue;
    const uint16_t* xr = a.x + static_cast<int64_t>(m) * K;
    for (int j = 0; j < iters; ++j) {
      const int s = threadIdx.x + j * blockDim.x;
      float v[kActSlot];
      if (s < slots) {
        act_load_slot(xr + s * kActSlot, v, false);
      } else {
#pragma unroll
        for (int i = 0; i < kActSlot; ++i) v[i] = 0.0f;
      }
      if (a.rotated) act_fwht_slot(v, lane);  // whole 8-lane groups are in or out
      mx[m] = fmaxf(mx[m], act_slot_absmax(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx[m] = fmaxf(mx[m], __shfl_xor_sync(0xffffffffu, mx[m], o));
    if (lane == 0) red[m * 32 + warp] = mx[m];
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m >= M) {
      xscale[m] = 0.0f;
      continue;
    }
    float amax = 0.0f;
    for (int w = 0; w < nwarps; ++w) amax = fmaxf(amax, red[m * 32 + w]);
    const float inv = act_inv(amax);
    xscale[m] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
    const uint16_t* xr = a.x + static_cast<int64_t>(m) * K;
    for (int j = 0; j < iters; ++j) {
      const int s = threadIdx.x + j * blockDim.x;
      float v[kActSlot];
      if (s < slots) {
        act_load_slot(xr + s * kActSlot, v, false);
      } else {
#pragma unroll
        for (int i = 0; i < kActSlot; ++i) v[i] = 0.0f;
      }
      if (a.rotated) act_fwht_slot(v, lane);
      act_prescale_slot(v, amax);
      if (s < slots) act_store_slot(act + m * K + s * kActSlot, v, inv);
    }
  }
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    if (a.xq_out) {
      const int n16 = M * K / 16;
      for (int i = threadIdx.x; i < n16; i += blockDim.x)
        reinterpret_cast<int4*>(a.xq_out)[i] = reinterpret_cast<const int4*>(act)[i];
    }
    if (a.xs_out && threadIdx.x < M) a.xs_out[threadIdx.x] = xscale[threadIdx.x < MT ? threadIdx.x : 0];
  }
}

template <int MT, int RG, int FMT, bool PARTIALS, bool FUSED>
__global__ void __launch_bounds__(gemv_warps(MT) * 32, 1)
    gemv_kernel(const LinearArgs a, const GemvPlan p, int64_t tiles_base, int64_t tiles_extra) {
  constexpr int G = FMT == 0 ? kGroupTrunk : kGroupHead;
  constexpr int LPB = G / 16;  // lanes per block within a 512-byte step
  constexpr int kGemvUnroll = gemv_unroll(MT, RG);
  // one or two tokens, one row at a time: stage rows of up to kRegSteps x 512
  // bytes are consumed from registers (see below)
  constexpr bool kRegStage = MT <= 2 && RG == 1;
  constexpr int kRegSteps = 10;

  extern __shared__ __align__(128) uint8_t smem[];
  const int K = static_cast<int>(a.k);
  const int64_t N = a.n;
  const int M = static_cast<int>(a.m);
  const int ng = K / G;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  uint8_t* bufs = smem + gemv_align128(MT * K) + warp * p.depth * p.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + gemv_align128(MT * K) + p.warps * p.depth * p.stage_bytes);
  uint64_t* full = bars + warp * p.depth;
  uint64_t* actbar = bars + p.warps * p.depth;
  uint64_t* prebar = actbar + 1;
  int* counter = reinterpret_cast<int*>(actbar + 2);
  // trunk scales of the CTA's rows, when loaded up front: [s1 window][s2 window]
  uint8_t* pre_sc = smem + p.smem - p.pre_bytes;

  const int64_t bid = blockIdx.x;
  const int64_t t0 = bid * tiles_base + (bid < tiles_extra ? bid : tiles_extra);
  const int64_t t1 = t0 + tiles_base + (bid < tiles_extra ? 1 : 0);
  const int nchunks = (K + p.kc - 1) / p.kc;
  const bool pre = FMT == 0 && !PARTIALS && p.pre;
  const int64_t crow0 = t0 * p.rt;                          // the CTA's first row
  const int64_t crow1 = min(t1 * p.rt, N);                  // and one past its last

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.warps * p.depth; ++s) mbar_init(&bars[s], 1);
    mbar_init(actbar, 1);
    mbar_init(prebar, 1);
    *counter = 0;
    fence_barrier_init();
    if (pre && crow1 > crow0) {
      // one copy each for the sub-scales and the row scales of all the CTA's
      // rows (16-byte windows; plain loads only past the arrays' last 16 bytes)
      const GemvWindow w0 = window_copy_plan(pre_sc, a.sub, N * ng, crow0 * ng, crow1 * ng, true);
      const GemvWindow w1 = window_copy_plan(pre_sc + p.pre_s1, reinterpret_cast<const uint8_t*>(a.scale), 2 * N,
                                             2 * crow0, 2 * crow1, true);
      mbar_arrive_expect_tx(prebar, w0.bytes + w1.bytes);
      if (w0.bytes) bulk_g2s_default(w0.dst, w0.src, w0.bytes, prebar);
      if (w1.bytes) bulk_g2s_default(w1.dst, w1.src, w1.bytes, prebar);
    }
  }
  // token rows past M are zero (their codes never reach an output anyway)
  {
    int4* pad = reinterpret_cast<int4*>(act + M * K);
    const int n16 = (MT - M) * K / 16;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) pad[i] = make_int4(0, 0, 0, 0);
  }
  __syncthreads();
  pdl_launch_dependents();
  const uint64_t pol = l2_policy_evict_first();

  // ---- issuing (lane 0): claim work, fill stage buffer `b`
  int64_t cur_tile = -1;  // tile whose chunks are being issued
  int cur_chunk = 0;
  GemvStage issued[kGemvMaxDepth];
  uint32_t uses[kGemvMaxDepth];
#pragma unroll
  for (int b = 0; b < kGemvMaxDepth; ++b) {
    issued[b].tile = -1;
    issued[b].chunk = 0;
    uses[b] = 0;
  }
  auto issue = [&](int b) {
    // advance to the next (tile, chunk); lane 0 claims tiles, all lanes learn
    int64_t tile = -1;
    int chunk = 0;
    if (cur_tile >= 0 && cur_chunk + 1 < nchunks) {
      tile = cur_tile;
      chunk = cur_chunk + 1;
    } else {
      int claimed = 0;
      if (lane == 0) claimed = atomicAdd(counter, 1);
      claimed = __shfl_sync(0xffffffffu, claimed, 0);
      tile = t0 + claimed < t1 ? t0 + claimed : -1;
    }
    cur_tile = tile;
    cur_chunk = chunk;
    issued[b].tile = tile;
    issued[b].chunk = chunk;
    if (tile < 0) return;
    // every lane computes the stage descriptor; lane 0 arms the barrier, then
    // lanes 0, 1, 2 issue the codes, sub-scale and row-scale copies at once
    const int64_t row0 = tile * p.rt;
    const int rows = static_cast<int>(min(static_cast<int64_t>(p.rt), N - row0));
    const int len = min(p.kc, K - chunk * p.kc);
    uint8_t* st = bufs + b * p.stage_bytes;
    const int cbytes = rows * len;
    GemvWindow w0{nullptr, nullptr, 0u}, w1{nullptr, nullptr, 0u};
    if (!PARTIALS && !pre && lane < 3) {
      const int gb = len / G;
      const int64_t o0 = row0 * ng + chunk * (p.kc / G);  // first scale of the stage, in elements
      if (FMT == 0) {
        w0 = window_copy_plan(st + p.sc_off, a.sub, N * ng, o0, o0 + rows * gb, lane == 1);
        // every chunk carries the row scales: the epilogue runs on the last
        w1 = window_copy_plan(st + p.s2_off, reinterpret_cast<const uint8_t*>(a.scale), 2 * N, 2 * row0,
                              2 * (row0 + rows), lane == 2);
      } else {
        w0 = window_copy_plan(st + p.sc_off, reinterpret_cast<const uint8_t*>(a.scale), 2 * N * ng, 2 * o0,
                              2 * (o0 + rows * gb), lane == 1);
      }
    }
    __syncwarp();  // plain tails (if any) are written before the arrive
    if (lane == 0) mbar_arrive_expect_tx(&full[b], static_cast<uint32_t>(cbytes) + w0.bytes + w1.bytes);
    __syncwarp();
    if (lane == 0) {
      const int8_t* src = a.codes + row0 * K + chunk * p.kc;  // rows x len, contiguous
      for (int off = 0; off < cbytes; off += kGemvMaxCopy)
        bulk_g2s(st + off, src + off, static_cast<uint32_t>(min(kGemvMaxCopy, cbytes - off)), &full[b], pol);
    } else if (lane == 1 && w0.bytes) {
      bulk_g2s(w0.dst, w0.src, w0.bytes, &full[b], pol);
    } else if (lane == 2 && w1.bytes) {
      bulk_g2s(w1.dst, w1.src, w1.bytes, &full[b], pol);
    }
  };

  // the first stages hold only weights, which no earlier kernel writes: they
  // stream while the previous kernel on the stream finishes (unless the
  // caller said that kernel wrote them)
  if (a.weights_after_wait) pdl_wait();
  for (int b = 0; b < p.depth; ++b) issue(b);
  pdl_wait();
  if (!FUSED && threadIdx.x == 0) {
    mbar_arrive_expect_tx(actbar, static_cast<uint32_t>(M * K));
    bulk_g2s_default(act, a.xq, static_cast<uint32_t>(M * K), actbar);
  }

  // activation codes: computed here (fused) while the first stages stream,
  // or on their way by bulk copy
  float xscale[MT];
  bool failed = false;  // warp-uniform: a wait ran out; stop computing
  if (FUSED) {
    __shared__ float red[MT * 32];
    gemv_fused_act<MT>(a, act, xscale, red);
  } else {
#pragma unroll
    for (int m = 0; m < MT; ++m) xscale[m] = (!PARTIALS && m < M) ? a.xs[m] : 0.0f;
    const bool ok = mbar_wait(actbar, 0u, kDevErrGemvFull);
    failed = !__all_sync(0xffffffffu, ok);
  }
  if (pre && crow1 > crow0 && !failed) {
    const bool ok = mbar_wait(prebar, 0u, kDevErrGemvFull);
    failed = !__all_sync(0xffffffffu, ok);
  }
  const float rot = a.rotated ? 0.0078125f : 1.0f;

  // Sums of the row group in flight: int64 (trunk) or fp32 (lm_head). They
  // carry across chunks only for one-row tiles; whole-row tiles have one chunk.
  long long racc[RG][MT];
  float facc[RG][MT];
  int b = 0;
  while (issued[b].tile >= 0) {
    const int64_t tile = issued[b].tile;
    const int chunk = issued[b].chunk;
    if (!failed) {
      const bool ok = mbar_wait(&full[b], uses[b] & 1u, kDevErrGemvFull);
      failed = !__all_sync(0xffffffffu, ok);
    }
    const uint8_t* st = bufs + b * p.stage_bytes;
    const int64_t row0 = tile * p.rt;
    const int rows = static_cast<int>(min(static_cast<int64_t>(p.rt), N - row0));
    const int len = min(p.kc, K - chunk * p.kc);
    const int gb = len / G;
    // scales start inside their 16-byte window (see window_copy_plan)
    const int64_t so = row0 * ng + chunk * (p.kc / G);
    const uint8_t* sc = pre ? pre_sc + ((crow0 * ng) & 15) + (so - crow0 * ng)
                            : st + p.sc_off + (FMT == 0 ? (so & 15) : ((2 * so) & 15));
    const uint16_t* s2p = pre ? reinterpret_cast<const uint16_t*>(pre_sc + p.pre_s1 + ((2 * crow0) & 15)) +
                                    (row0 - crow0)
                              : reinterpret_cast<const uint16_t*>(st + p.s2_off + ((2 * row0) & 15));
    const int sstride = pre ? ng : gb;  // scales per row in the stage (or in the CTA's preloaded rows)
    const int nsteps = (len + 511) / 512;
    bool refilled = false;
    if (kRegStage && rows == 1 && nsteps <= kRegSteps) {
      // one row (chunk) of at most 5 KB: pull it and its scales into
      // registers, hand the buffer straight back to the copy engine, then
      // compute -- the copy of the next tile overlaps this tile's arithmetic
      int4 wv[kRegSteps];
      uint32_t scv[kRegSteps];
#pragma unroll
      for (int u = 0; u < kRegSteps; ++u) {
        const int o = u * 512 + lane * 16;
        const bool vr = u < nsteps && !failed && o < len;
        wv[u] = vr ? *reinterpret_cast<const int4*>(st + o) : make_int4(0, 0, 0, 0);
        scv[u] = 0u;
        if (!PARTIALS && vr)
          scv[u] = FMT == 0 ? static_cast<uint32_t>(sc[o / G])
                            : static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(sc)[o / G]);
      }
      const uint16_t s2b = (FMT == 0 && !PARTIALS) ? s2p[0] : 0;
      __syncwarp();
      uses[b] += 1;
      if (!failed) {
        issue(b);
      } else {
        issued[b].tile = -1;
      }
      refilled = true;
      if (chunk == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          racc[0][m] = 0;
          facc[0][m] = 0.0f;
        }
      }
      int acc32[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc32[m] = 0;
#pragma unroll
      for (int u = 0; u < kRegSteps; ++u) {
        if (u < nsteps) {
          const int o = u * 512 + lane * 16;
          const bool valid = !failed && o < len;
          const int kk = chunk * p.kc + o;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const int4 xv = valid ? *reinterpret_cast<const int4*>(act + m * K + kk) : make_int4(0, 0, 0, 0);
            int q = dot16(wv[u], xv);
            if (PARTIALS) {
#pragma unroll
              for (int off = 1; off < LPB; off <<= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
              if (valid && m < M && (lane & (LPB - 1)) == 0)
                a.partials[(static_cast<int64_t>(m) * N + row0) * ng + kk / G] = q;
            } else if (FMT == 0) {
              acc32[m] += static_cast<int>(scv[u]) * q;  // <= 10 steps of 255 * 16 * 127^2 < 2^31
            } else {
              facc[0][m] = fmaf(static_cast<float>(q), bf16_bits_to_float(static_cast<uint16_t>(scv[u])), facc[0][m]);
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) racc[0][m] += acc32[m];
      if (!PARTIALS && chunk == nchunks - 1) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          float yv;
          if (FMT == 0) {
            long long v = racc[0][m];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            yv = __ll2float_rn(v) * xscale[m] * bf16_bits_to_float(s2b) * rot;
          } else {
            float v = facc[0][m];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            yv = v * xscale[m] * rot;
          }
          if (lane == m && !failed && m < M) a.y[static_cast<int64_t>(m) * N + row0] = float_to_bf16_bits_rn(yv);
        }
      }
    }
    for (int r0 = 0; r0 < (refilled ? 0 : rows); r0 += RG) {
      if (chunk == 0) {
#pragma unroll
        for (int i = 0; i < RG; ++i)
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            racc[i][m] = 0;
            facc[i][m] = 0.0f;
          }
      }
      int acc32[RG][MT];
#pragma unroll
      for (int i = 0; i < RG; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc32[i][m] = 0;
      int since = 0;
      for (int t0s = 0; t0s < nsteps; t0s += kGemvUnroll) {
        // loads for kGemvUnroll steps first, then the dot products
        int4 xv[kGemvUnroll][MT];
        int4 wv[kGemvUnroll][RG];
        int s1v[kGemvUnroll][RG];
        float sfv[kGemvUnroll][RG];
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
          const int o = (t0s + u) * 512 + lane * 16;
          const bool valid = !failed && o < len;  // uniform per 256-byte half-warp
          const int kk = chunk * p.kc + o;
#pragma unroll
          for (int m = 0; m < MT; ++m)
            xv[u][m] = valid ? *reinterpret_cast<const int4*>(act + m * K + kk) : make_int4(0, 0, 0, 0);
#pragma unroll
          for (int i = 0; i < RG; ++i) {
            const int rl = r0 + i;
            const bool vr = valid && rl < rows;
            wv[u][i] = vr ? *reinterpret_cast<const int4*>(st + rl * len + o) : make_int4(0, 0, 0, 0);
            s1v[u][i] = 0;
            sfv[u][i] = 0.0f;
            if (!PARTIALS && vr) {
              if (FMT == 0)
                s1v[u][i] = sc[rl * sstride + o / G];
              else
                sfv[u][i] = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(sc)[rl * sstride + o / G]);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
#pragma unroll
          for (int i = 0; i < RG; ++i) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              int q = dot16(wv[u][i], xv[u][m]);
              if (PARTIALS) {
                // LPB lanes make one block: 16 (trunk) or 8 (lm_head)
#pragma unroll
                for (int off = 1; off < LPB; off <<= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
                const int o = (t0s + u) * 512 + lane * 16;
                if (!failed && o < len && r0 + i < rows && m < M && (lane & (LPB - 1)) == 0)
                  a.partials[(static_cast<int64_t>(m) * N + row0 + r0 + i) * ng + (chunk * p.kc + o) / G] = q;
              } else if (FMT == 0) {
                acc32[i][m] += s1v[u][i] * q;  // |s1 * q| <= 255 * 16 * 127^2 < 2^26
              } else {
                facc[i][m] = fmaf(static_cast<float>(q), sfv[u][i], facc[i][m]);
              }
            }
          }
        }
        if (FMT == 0 && !PARTIALS) {
          since += kGemvUnroll;
          if (since >= 16) {  // 16 steps < 2^30: fold before int32 can overflow
            since = 0;
#pragma unroll
            for (int i = 0; i < RG; ++i)
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                racc[i][m] += acc32[i][m];
                acc32[i][m] = 0;
              }
          }
        }
      }
      if (FMT == 0 && !PARTIALS) {
#pragma unroll
        for (int i = 0; i < RG; ++i)
#pragma unroll
          for (int m = 0; m < MT; ++m) racc[i][m] += acc32[i][m];
      }
      // ---- epilogue once the tile's last chunk is in
      if (!PARTIALS && chunk == nchunks - 1) {
        uint16_t s2b[RG];
#pragma unroll
        for (int i = 0; i < RG; ++i)
          s2b[i] = (FMT == 0 && r0 + i < rows) ? s2p[r0 + i] : 0;
#pragma unroll
        for (int i = 0; i < RG; ++i) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            float yv;
            if (FMT == 0) {
              long long v = racc[i][m];
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
              yv = __ll2float_rn(v) * xscale[m] * bf16_bits_to_float(s2b[i]) * rot;
            } else {
              float v = facc[i][m];
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
              yv = v * xscale[m] * rot;
            }
            if (lane == i * MT + m && !failed && r0 + i < rows && m < M)
              a.y[static_cast<int64_t>(m) * N + row0 + r0 + i] = float_to_bf16_bits_rn(yv);
          }
        }
      }
    }
    // the buffer is consumed: refill it (the chunk's data is no longer read)
    if (!refilled) {
      __syncwarp();
      uses[b] += 1;
      if (!failed) {
        issue(b);
      } else {
        issued[b].tile = -1;
      }
    }
    b = b + 1 == p.depth ? 0 : b + 1;
    if (failed) {
      // drain: never leave with a copy still landing in this warp's buffers
      for (int j = 0; j < p.depth; ++j)
        if (issued[j].tile >= 0) {
          mbar_wait(&full[j], uses[j] & 1u, kDevErrGemvDrain);
          issued[j].tile = -1;
        }
      break;
    }
  }
  if (!FUSED && threadIdx.x == 0) mbar_wait(actbar, 0u, kDevErrGemvDrain);  // the shared copies have landed
  if (pre && crow1 > crow0 && threadIdx.x == 0) mbar_wait(prebar, 0u, kDevErrGemvDrain);
}

}  // namespace iq8r
