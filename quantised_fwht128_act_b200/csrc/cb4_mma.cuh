// The drafter's codebook linear for 2..16 tokens on mma.sync m16n8k32 s8.
//
// A warp owns a group of 16 weight rows over half of K. Lane (g, t) (group
// g = lane / 4, t = lane % 4) loads 16 index bytes (32 weights) of rows g
// and g + 8 at index-byte offset 64 s + 16 t of step s, so a quad covers one
// 128-weight scale block per step. The dot product does not depend on the
// order of K: MMA i of a step takes the lane's weights 8i..8i+7 (decoded
// word i: a0/a2 for row g, a1/a3 for row g + 8) and the same eight K
// positions of token g's activation codes (b0/b1), so A and B agree for
// every t. Each step's four MMAs give the exact int32 block sums P of rows
// g, g + 8 and tokens 2t, 2t + 1, which are scaled by the block's bf16
// scale into fp32. The two halves of K meet in shared memory, added in
// order.
#pragma once

#include "cb4_gemv.cuh"

namespace iq8r {

constexpr int kCb4MmaWarps = 8;  // 4 row groups x 2 halves of K
constexpr int kCb4MmaDepth = 4;  // steps in flight a lane

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NT token tiles of 8 (M <= 8 * NT).
template <int NT>
__global__ void __launch_bounds__(kCb4MmaWarps * 32, 2) cb4_mma_kernel(const LinearArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int K = static_cast<int>(a.k);
  const int M = static_cast<int>(a.m);
  const int64_t N = a.n;
  const int ast = K + 16;  // activation row stride: 16-byte skew, no bank conflicts
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  float* red = reinterpret_cast<float*>(smem + 8 * NT * ast);  // [4 groups][32 lanes][4 NT]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int kb = K / 2;         // index bytes a row
  const int steps = K / 128;    // scale blocks a row
  const int ng = steps;
  const int half = warp & 1;
  const int s0 = half == 0 ? 0 : steps / 2;
  const int s1 = half == 0 ? steps / 2 : steps;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * 4 + (warp >> 1)) * 16;
  // rows past N load row N - 1 (valid memory) and are never stored
  const int64_t ra = min(row0 + g, N - 1), rb = min(row0 + g + 8, N - 1);
  const uint8_t* codes = reinterpret_cast<const uint8_t*>(a.codes);
  const uint8_t* pa = codes + ra * kb + 16 * t;
  const uint8_t* pb = codes + rb * kb + 16 * t;
  const uint16_t* qa = a.scale + ra * ng;
  const uint16_t* qb = a.scale + rb * ng;

  int4 wa[kCb4MmaDepth], wb[kCb4MmaDepth];
  uint32_t sa[kCb4MmaDepth], sb[kCb4MmaDepth];
  auto load = [&](int d, int s) {
    if (s < s1) {
      wa[d] = __ldg(reinterpret_cast<const int4*>(pa + 64 * s));
      wb[d] = __ldg(reinterpret_cast<const int4*>(pb + 64 * s));
      sa[d] = __ldg(qa + s);
      sb[d] = __ldg(qb + s);
    }
  };
  pdl_launch_dependents();
  // the weights are no earlier kernel's output: the first steps' loads go
  // out before waiting for the kernel that writes the activation codes
  // (unless the caller said that kernel wrote them)
  if (a.weights_after_wait) pdl_wait();
#pragma unroll
  for (int d = 0; d < kCb4MmaDepth; ++d) load(d, s0 + d);
  pdl_wait();
  for (int i = threadIdx.x; i < 8 * NT * (K / 16); i += blockDim.x) {
    const int m = i / (K / 16), c = i - m * (K / 16);
    const int4 v = m < M ? __ldg(reinterpret_cast<const int4*>(a.xq + static_cast<int64_t>(m) * K) + c)
                         : make_int4(0, 0, 0, 0);
    *reinterpret_cast<int4*>(act + m * ast + 16 * c) = v;
  }
  __syncthreads();
  const uint32_t t0 = cb4_word(0), t1 = cb4_word(1), t2 = cb4_word(2), t3 = cb4_word(3);

  float facc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) facc[nt][j] = 0.0f;

  for (int sbase = s0; sbase < s1; sbase += kCb4MmaDepth) {
#pragma unroll
    for (int d = 0; d < kCb4MmaDepth; ++d) {
      const int s = sbase + d;
      if (s >= s1) break;  // warp-uniform
      const uint32_t wA[4] = {static_cast<uint32_t>(wa[d].x), static_cast<uint32_t>(wa[d].y),
                              static_cast<uint32_t>(wa[d].z), static_cast<uint32_t>(wa[d].w)};
      const uint32_t wB[4] = {static_cast<uint32_t>(wb[d].x), static_cast<uint32_t>(wb[d].y),
                              static_cast<uint32_t>(wb[d].z), static_cast<uint32_t>(wb[d].w)};
      const float fa = bf16_bits_to_float(static_cast<uint16_t>(sa[d]));
      const float fb = bf16_bits_to_float(static_cast<uint16_t>(sb[d]));
      load(d, s + kCb4MmaDepth);  // this slot's next step
      uint32_t aLo[4], aHi[4], bLo[4], bHi[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        cb4_decode8(wA[i], t0, t1, t2, t3, aLo[i], aHi[i]);
        cb4_decode8(wB[i], t0, t1, t2, t3, bLo[i], bHi[i]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int8_t* xr = act + (nt * 8 + g) * ast + 64 * 2 * s + 32 * t;  // weights 128 s + 32 t ..
        const int4 x0 = *reinterpret_cast<const int4*>(xr);
        const int4 x1 = *reinterpret_cast<const int4*>(xr + 16);
        const uint32_t xw[8] = {static_cast<uint32_t>(x0.x), static_cast<uint32_t>(x0.y),
                                static_cast<uint32_t>(x0.z), static_cast<uint32_t>(x0.w),
                                static_cast<uint32_t>(x1.x), static_cast<uint32_t>(x1.y),
                                static_cast<uint32_t>(x1.z), static_cast<uint32_t>(x1.w)};
        int dd[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 4; ++i) mma_s8_16832(dd, aLo[i], bLo[i], aHi[i], bHi[i], xw[2 * i], xw[2 * i + 1]);
        facc[nt][0] = fmaf(static_cast<float>(dd[0]), fa, facc[nt][0]);
        facc[nt][1] = fmaf(static_cast<float>(dd[1]), fa, facc[nt][1]);
        facc[nt][2] = fmaf(static_cast<float>(dd[2]), fb, facc[nt][2]);
        facc[nt][3] = fmaf(static_cast<float>(dd[3]), fb, facc[nt][3]);
      }
    }
  }
  // the second half's sums meet the first's in shared memory
  float* rw = red + ((warp >> 1) * 32 + lane) * 4 * NT;
  if (half == 1) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) rw[nt * 4 + j] = facc[nt][j];
  }
  __syncthreads();
  if (half == 1) return;
  const float rot = a.rotated ? 0.0078125f : 1.0f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = nt * 8 + 2 * t + (j & 1);
      const int64_t r = row0 + g + (j >> 1) * 8;
      const float v = facc[nt][j] + rw[nt * 4 + j];
      if (m < M && r < N) a.y[static_cast<int64_t>(m) * N + r] = float_to_bf16_bits_rn(v * a.xs[m] * rot);
    }
  }
}

}  // namespace iq8r
