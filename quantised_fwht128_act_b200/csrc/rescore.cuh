// Candidate rescoring: the outputs of the IQ8R linear for a short list of
// weight rows per token. "Qwen3.8-27B IQ8R + DFlash2 -- radiance container",
// table row "Speculator": 32 candidates come from the drafter's 2-bit
// vocabulary head, and the model's int8 head (a bf16 scale per 128 of K)
// re-scores them. The arithmetic is the linear's exactly -- the
// same exact int32 block sums P and the same epilogue -- evaluated only at
// out[t][j] = y[t][cand[t][j]].
//
// One CTA per (token, 32 candidates), one warp per candidate: the token's
// activation codes are staged once in shared memory, each warp streams its
// weight row in 512-byte steps (16 bytes a lane, read-only path) and the
// trunk sums s1 * P in int32 / int64 exactly like the GEMV, so trunk results
// are the GEMV's bits. The work is a gather of 32 rows a token: latency-
// bound, not a streaming kernel.
#pragma once

#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kRescoreWarps = 32;  // candidates per CTA

struct RescoreArgs {
  const int8_t* xq;       // [m][k]
  const float* xs;        // [m]
  int64_t m;
  const int8_t* codes;    // [n][k]
  const uint8_t* sub;     // [n][k/256] (trunk)
  const uint16_t* scale;  // [n] (trunk) or [n][k/128] (G128)
  int64_t n;
  int k;
  int rotated;
  const int32_t* cand;    // [m][kc]
  int kc;
  uint16_t* out;          // [m][kc] bf16
};

template <int FMT>
__global__ void __launch_bounds__(kRescoreWarps * 32) rescore_kernel(const RescoreArgs a) {
  constexpr int G = FMT == 0 ? kGroupTrunk : kGroupHead;
  extern __shared__ __align__(16) uint8_t smem[];
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = a.k;
  const int ng = K / G;
  // the token's codes, once per CTA (K is a multiple of 128, so of 16)
  for (int i = threadIdx.x; i < K / 16; i += blockDim.x)
    reinterpret_cast<int4*>(act)[i] = __ldg(reinterpret_cast<const int4*>(a.xq + t * K) + i);
  __syncthreads();
  const int j = blockIdx.y * kRescoreWarps + warp;
  if (j >= a.kc) return;
  const int64_t c = a.cand[t * a.kc + j];
  if (c < 0 || c >= a.n) {
    if (lane == 0) {
      set_device_error(kDevErrRescoreIndex);
      a.out[t * a.kc + j] = 0;
    }
    return;
  }
  const int8_t* wrow = a.codes + c * K;
  long long racc = 0;
  int acc32 = 0;
  float facc = 0.0f;
  const int nsteps = (K + 511) / 512;
  for (int s = 0; s < nsteps; ++s) {
    const int o = s * 512 + lane * 16;
    if (o < K) {  // uniform per half-warp: K is a multiple of 256
      const int4 w = __ldg(reinterpret_cast<const int4*>(wrow + o));
      const int4 x = *reinterpret_cast<const int4*>(act + o);
      int q = __dp4a(w.x, x.x, 0);
      q = __dp4a(w.y, x.y, q);
      q = __dp4a(w.z, x.z, q);
      q = __dp4a(w.w, x.w, q);
      if (FMT == 0) {
        acc32 += static_cast<int>(__ldg(a.sub + c * ng + o / G)) * q;  // < 2^26 a step
      } else {
        facc = fmaf(static_cast<float>(q), bf16_bits_to_float(__ldg(a.scale + c * ng + o / G)), facc);
      }
    }
    if (FMT == 0 && (s & 15) == 15) {  // 16 steps < 2^30: fold before int32 can overflow
      racc += acc32;
      acc32 = 0;
    }
  }
  const float rot = a.rotated ? 0.0078125f : 1.0f;
  float yv;
  if (FMT == 0) {
    long long v = racc + acc32;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    yv = __ll2float_rn(v) * a.xs[t] * bf16_bits_to_float(a.scale[c]) * rot;
  } else {
    float v = facc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    yv = v * a.xs[t] * rot;
  }
  if (lane == 0) a.out[t * a.kc + j] = float_to_bf16_bits_rn(yv);
}

}  // namespace iq8r
