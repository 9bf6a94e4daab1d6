// The drafter's codebook linear: 4-bit indices into 16 integer levels with a
// bf16 scale per (row, 128 of K), in the rotated domain ("Qwen3.8-27B IQ8R +
// DFlash2 -- radiance container": the "Speculator" row and the dflash recipe
// lines of "How this file was made", table=-127;-97;...;97;127 group=128
// scale=bf16 transform=fwht128).
//
// y[m][n] = a[m] / 128 * sum_g s[n][g] * P[m][n][g], P the exact int32 dot
// product of the activation codes with the levels of block g -- the lm_head
// formula with the codes looked up.
//
// Weight-streaming GEMV (half the bytes of the int8 formats): each warp owns
// whole rows; a lane reads 16 bytes = 32 indices a step through the read-only
// path, the loads of a row chunk (up to 4 KB) issued before any arithmetic
// and the next row's issued before this row's arithmetic. Indices become
// int8 levels with byte permutes: the low 3 bits pick a byte of the lower or
// the upper half of the table, and the permute's sign-replicate mode turns
// bit 3 into the byte mask that chooses between them.
#pragma once

#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kCb4Warps = 16;
constexpr int kCb4ChunkSteps = 8;  // 8 x 512 bytes of indices: K up to 8192 in one chunk

// The table as bytes: levels 0-3, 4-7, 8-11, 12-15 (little-endian words).
__device__ __forceinline__ uint32_t cb4_word(int w) {
  switch (w) {
    case 0: return 0xC6B59F81u;  // -127 -97 -75 -58
    case 1: return 0xFAEEE2D5u;  // -43 -30 -18 -6
    case 2: return 0x2B1E1206u;  // 6 18 30 43
    default: return 0x7F614B3Au;  // 58 75 97 127
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 8 indices (one word, index j in bits 4j..4j+3) -> 8 int8 levels (2 words).
// A permute reads only the low 16 bits of its selector, so one mask of the
// whole word gives the selectors of indices 0-3 and, shifted, of 4-7.
__device__ __forceinline__ void cb4_decode8(uint32_t w, uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3,
                                            uint32_t& out0, uint32_t& out1) {
  const uint32_t w4 = w << 4;
  const uint32_t sel = w & 0x77777777u;  // the low 3 bits of every index
  // indices 0-3
  const uint32_t lo0 = prmt(t0, t1, sel), hi0 = prmt(t2, t3, sel);
  // byte k = 0xFF where index k has bit 3 set: the sign-replicate selectors
  // read bit 3 of index 2j from (w << 4) and of index 2j + 1 from w
  const uint32_t m0 = prmt(w4, w, 0xD9C8u);
  out0 = (lo0 & ~m0) | (hi0 & m0);
  // indices 4-7
  const uint32_t s1 = sel >> 16;
  const uint32_t lo1 = prmt(t0, t1, s1), hi1 = prmt(t2, t3, s1);
  const uint32_t m1 = prmt(w4, w, 0xFBEAu);
  out1 = (lo1 & ~m1) | (hi1 & m1);
}

// One row chunk of STEPS x 512 index bytes (lane: STEPS x 16 bytes) against
// the staged activation codes: per-block partial sums (PARTIALS) or the fp32
// sum of s * P into facc. EXACT: every chunk is full (K / 2 a multiple of
// STEPS x 512), so no lane is past the row's end.
template <int MT, bool PARTIALS, int STEPS, bool EXACT>
__device__ __forceinline__ void cb4_rows_step(const LinearArgs& a, const int8_t* act, const int4 (&buf)[STEPS],
                                              const uint32_t (&scl)[STEPS],
                                              int64_t row, int s0, int nsteps, int kb, int K, int M, int64_t N,
                                              int ng, int lane, uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3,
                                              float (&facc)[MT]) {
#pragma unroll
  for (int u = 0; u < STEPS; ++u) {
    if (s0 + u >= nsteps) break;               // warp-uniform
    const int o = (s0 + u) * 512 + lane * 16;  // index bytes; weights 2 * o ..
    const bool valid = EXACT || o < kb;        // whole 4-lane blocks in or out (kb % 64 == 0)
    const uint32_t wv[4] = {static_cast<uint32_t>(buf[u].x), static_cast<uint32_t>(buf[u].y),
                            static_cast<uint32_t>(buf[u].z), static_cast<uint32_t>(buf[u].w)};
    uint32_t lv[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) cb4_decode8(wv[i], t0, t1, t2, t3, lv[2 * i], lv[2 * i + 1]);
    const int kk = valid ? 2 * o : 0;          // first weight of the lane's 32
    const int blk = kk / kGroupHead;           // the 32 share one 128-block
    const float sb = valid ? bf16_bits_to_float(static_cast<uint16_t>(scl[u])) : 0.0f;  // loaded with the codes
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int4 x0 = *reinterpret_cast<const int4*>(act + m * K + kk);
      const int4 x1 = *reinterpret_cast<const int4*>(act + m * K + kk + 16);
      int q = __dp4a(static_cast<int>(lv[0]), x0.x, 0);
      q = __dp4a(static_cast<int>(lv[1]), x0.y, q);
      q = __dp4a(static_cast<int>(lv[2]), x0.z, q);
      q = __dp4a(static_cast<int>(lv[3]), x0.w, q);
      q = __dp4a(static_cast<int>(lv[4]), x1.x, q);
      q = __dp4a(static_cast<int>(lv[5]), x1.y, q);
      q = __dp4a(static_cast<int>(lv[6]), x1.z, q);
      q = __dp4a(static_cast<int>(lv[7]), x1.w, q);
      q = valid ? q : 0;
      if (PARTIALS) {
        // 4 lanes make one 128-block
        q += __shfl_xor_sync(0xffffffffu, q, 1);
        q += __shfl_xor_sync(0xffffffffu, q, 2);
        if (valid && (lane & 3) == 0 && m < M) a.partials[(static_cast<int64_t>(m) * N + row) * ng + blk] = q;
      } else {
        facc[m] = fmaf(static_cast<float>(q), sb, facc[m]);
      }
    }
  }
}

// Rows of at most STEPS x 512 index bytes are kept DEPTH rows ahead in
// registers (a warp's rows: gw, gw + nw, ...): the row computed now was
// loaded DEPTH - 1 rows earlier. Longer rows (STEPS chunks each) go one chunk
// ahead. EXACT: K / 2 is a multiple of STEPS x 512, so every chunk is full and
// the masks and clamps drop out.
template <int MT, bool PARTIALS, int STEPS, bool EXACT>
__global__ void __launch_bounds__(kCb4Warps * 32, 1) cb4_gemv_kernel(const LinearArgs a) {
  constexpr int DEPTH = STEPS <= 5 ? 3 : 2;
  extern __shared__ __align__(16) uint8_t smem[];
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  const int K = static_cast<int>(a.k);
  const int M = static_cast<int>(a.m);
  const int64_t N = a.n;
  const int ng = K / kGroupHead;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint8_t* codes = reinterpret_cast<const uint8_t*>(a.codes);
  const int kb = K / 2;                       // index bytes a row
  const int nsteps = (kb + 511) / 512;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kCb4Warps + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kCb4Warps;

  // a row chunk's codes and the scale of each lane's block, loaded together
  // (a scale fetched only when needed would wait behind the weight stream).
  // Within a row every lane loads unconditionally, lanes and steps past the
  // row's end from its first bytes: the arithmetic masks them, and no select
  // on a load's result makes the warp wait for the data it is prefetching.
  auto load = [&](int64_t row, int s0, int4 (&buf)[STEPS], uint32_t (&scl)[STEPS]) {
    if (row >= N) return;  // warp-uniform; the slot is never computed
#pragma unroll
    for (int u = 0; u < STEPS; ++u) {
      int o = (s0 + u) * 512 + lane * 16;
      if (!EXACT) o = o < kb ? o : 0;
      buf[u] = __ldg(reinterpret_cast<const int4*>(codes + row * kb + o));
      if (!PARTIALS) scl[u] = static_cast<uint32_t>(__ldg(a.scale + row * ng + (2 * o) / kGroupHead));
    }
  };

  pdl_launch_dependents();
  // the weights are no earlier kernel's output: the first rows' loads go
  // out before waiting for the kernel that writes the activation codes
  int4 ring[DEPTH][STEPS];
  uint32_t rsc[DEPTH][STEPS];
#pragma unroll
  for (int d = 0; d < DEPTH; ++d) {
#pragma unroll
    for (int u = 0; u < STEPS; ++u) {
      ring[d][u] = make_int4(0, 0, 0, 0);
      rsc[d][u] = 0u;
    }
  }
  const bool whole = nsteps <= STEPS;
  if (a.weights_after_wait) pdl_wait();  // the caller says that kernel wrote them
  if (whole) {
#pragma unroll
    for (int d = 0; d < DEPTH; ++d) load(gw + d * nw, 0, ring[d], rsc[d]);
  }
  pdl_wait();
  for (int i = threadIdx.x; i < MT * K / 16; i += blockDim.x) {
    const int m = (i * 16) / K;
    reinterpret_cast<int4*>(act)[i] =
        m < M ? __ldg(reinterpret_cast<const int4*>(a.xq) + i) : make_int4(0, 0, 0, 0);
  }
  __syncthreads();
  const uint32_t t0 = cb4_word(0), t1 = cb4_word(1), t2 = cb4_word(2), t3 = cb4_word(3);
  const float rot = a.rotated ? 0.0078125f : 1.0f;

  auto finish = [&](int64_t row, float (&facc)[MT]) {
    if (PARTIALS) return;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = facc[m];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == m && m < M) a.y[static_cast<int64_t>(m) * N + row] = float_to_bf16_bits_rn(v * a.xs[m] * rot);
    }
  };

  if (whole) {
    for (int64_t base = gw; base < N; base += DEPTH * nw) {
#pragma unroll
      for (int d = 0; d < DEPTH; ++d) {
        const int64_t row = base + d * nw;
        if (row >= N) break;
        float facc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) facc[m] = 0.0f;
        cb4_rows_step<MT, PARTIALS, STEPS, EXACT>(a, act, ring[d], rsc[d], row, 0, nsteps, kb, K, M, N, ng, lane,
                                                 t0, t1, t2, t3, facc);
        load(row + DEPTH * nw, 0, ring[d], rsc[d]);  // this slot's next row
        finish(row, facc);
      }
    }
  } else {
    // long rows, STEPS x 512 index bytes a chunk, two chunk buffers
    for (int64_t row = gw; row < N; row += nw) {
      float facc[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) facc[m] = 0.0f;
      load(row, 0, ring[0], rsc[0]);
      for (int s0 = 0; s0 < nsteps; s0 += 2 * STEPS) {
        if (s0 + STEPS < nsteps) load(row, s0 + STEPS, ring[1], rsc[1]);
        cb4_rows_step<MT, PARTIALS, STEPS, EXACT>(a, act, ring[0], rsc[0], row, s0, nsteps, kb, K, M, N, ng, lane,
                                                 t0, t1, t2, t3, facc);
        if (s0 + STEPS >= nsteps) break;
        if (s0 + 2 * STEPS < nsteps) load(row, s0 + 2 * STEPS, ring[0], rsc[0]);
        cb4_rows_step<MT, PARTIALS, STEPS, EXACT>(a, act, ring[1], rsc[1], row, s0 + STEPS, nsteps, kb, K, M, N, ng,
                                                 lane, t0, t1, t2, t3, facc);
      }
      finish(row, facc);
    }
  }
}

}  // namespace iq8r
