// The tensor-core GEMM's split-K second pass (see gemm_tc.cuh): adds the
// fp32 partial tiles of each output tile in split order, so the result does
// not depend on timing, and applies the scale epilogue.
#pragma once

#include "gemm_tc.cuh"

namespace iq8r {

// Split-K second pass: y[m][n] = bf16(sum over splits, in split order, of
// the fp32 partial tiles, times a[m] * s2[n] / 128 (trunk) or a[m] / 128
// (lm_head)). One thread: one weight row of one tile, 4 consecutive tokens;
// consecutive threads take consecutive token quads of a row, so each warp
// reads whole 128-byte runs of the partial tiles, and a thread issues the
// loads of all its splits before it adds them (in split order).
constexpr int kTcReduceThreads = 256;
constexpr int kTcReduceBatch = 8;  // splits whose loads are in flight together
template <int FMT>
__global__ void __launch_bounds__(kTcReduceThreads) tc_split_reduce_kernel(const TcParams p) {
  pdl_wait();  // the partial tiles come from the kernel before
  const int quads = p.bm / 4;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= p.tiles * kTcBN * quads) return;
  const int64_t tile = i / (kTcBN * quads);
  const int rem = static_cast<int>(i - tile * kTcBN * quads);
  const int r = rem / quads;
  const int c = rem - r * quads;
  const int64_t m0 = (tile % p.tiles_m) * p.bm + 4 * c;
  const int64_t n = (tile / p.tiles_m) * kTcBN + r;
  if (n >= p.n || m0 >= p.m) return;
  const size_t sstride = static_cast<size_t>(kTcBN) * p.bm;
  const float* w = p.ws + static_cast<size_t>(tile) * p.splits * sstride + static_cast<size_t>(r) * p.bm + 4 * c;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int sp0 = 0; sp0 < p.splits; sp0 += kTcReduceBatch) {
    float4 v[kTcReduceBatch];
#pragma unroll
    for (int t = 0; t < kTcReduceBatch; ++t)
      if (sp0 + t < p.splits) v[t] = __ldcg(reinterpret_cast<const float4*>(w + (sp0 + t) * sstride));
#pragma unroll
    for (int t = 0; t < kTcReduceBatch; ++t)
      if (sp0 + t < p.splits) {
        acc[0] += v[t].x;
        acc[1] += v[t].y;
        acc[2] += v[t].z;
        acc[3] += v[t].w;
      }
  }
  const float rs = (FMT == 0 ? bf16_bits_to_float(p.scale[n]) : 1.0f) * (p.rotated ? 0.0078125f : 1.0f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t m = m0 + j;
    if (m < p.m) __stcs(p.y + m * p.n + n, float_to_bf16_bits_rn(acc[j] * p.xs[m] * rs));
  }
}

}  // namespace iq8r
