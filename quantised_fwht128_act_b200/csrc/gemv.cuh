// Weight-streaming IQ8R GEMV for small M (decode and short verify blocks).
//
// y[m][n] = a[m] * s2[n] * sum_g s1[n][g] * P[m][n][g] / 128 (trunk) or
// a[m] / 128 * sum_g s[n][g] * P[m][n][g] (lm_head), P the exact int32 dot
// product of int8 codes over block g -- the W8A8 linear of "Qwen3.8-27B IQ8R
// + DFlash2 -- radiance container" (rows "Weights" and "Activations").
// At M <= 8 the layer is bound by streaming the int8 codes from HBM (the
// page's "Speed" section: the IQ8R decode step runs as fast as FP8's, the
// same bytes a weight).
//
// Design (sm_100a):
//  - persistent grid, one CTA per SM, each CTA a contiguous range of 8-row
//    tiles (balanced to one tile);
//  - warp 8 is the producer: one lane streams each tile in 2 KB-of-K chunks
//    (8 rows x 2 KB = 16 KB stage) with 1-D bulk copies (TMA engine) into a
//    ring of up to 12 stages, completion counted on mbarriers, weights
//    marked evict-first in L2;
//  - warps 0..7 consume: the activation codes [MT][K] sit in shared memory;
//    a warp owns RG rows and every WK-th 512-byte step of K; each lane does
//    4 dp4a per 16 bytes per token, multiplies the lane's partial by its
//    block's u8 sub-scale in int32 (exact) and folds into int64 per chunk;
//  - epilogue: warp shuffle (and, when WK > 1, a shared-memory) reduction,
//    then the fp32 scale product and one bf16 rounding.
// PARTIALS instantiates the same loads and dp4a chains but reduces each
// block's 16 (or 8) lanes and writes P instead of y (the debug twin).
#pragma once

#include <type_traits>

#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kGemvRows = 8;         // rows per tile
constexpr int kGemvKC = 2048;        // bytes of K per chunk
constexpr int kGemvStageBytes = kGemvRows * kGemvKC;
constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvThreads = (kGemvConsumerWarps + 1) * 32;
constexpr int kGemvMaxStages = 12;

template <int MT>
struct GemvShape {
  static constexpr int RG = MT == 1 ? 1 : (MT == 2 ? 2 : 4);  // rows per warp
  static constexpr int WR = kGemvRows / RG;                    // warps along rows
  static constexpr int WK = kGemvConsumerWarps / WR;           // warps along K
  static constexpr int STEPS = kGemvKC / 512;                  // 512-byte steps per chunk
  static constexpr int SPW = STEPS / WK;                       // steps per warp per chunk
};

__host__ __device__ constexpr int gemv_align128(int x) { return (x + 127) & ~127; }

// Shared memory bytes for a given MT, K and stage count.
__host__ __device__ constexpr int gemv_smem_bytes(int mt, int k, int stages, int red_bytes) {
  return gemv_align128(mt * k) + stages * kGemvStageBytes + 2 * stages * 8 + red_bytes + 128;
}

template <int MT, int FMT>
__host__ __device__ constexpr int gemv_red_bytes() {
  // [2 buffers][WK][WR][RG][MT] of int64 (trunk) or float (lm_head)
  return 2 * GemvShape<MT>::WK * GemvShape<MT>::WR * GemvShape<MT>::RG * MT * (FMT == 0 ? 8 : 4);
}

__device__ __forceinline__ int dot16(const int4 w, const int4 x) {
  int p = __dp4a(w.x, x.x, 0);
  p = __dp4a(w.y, x.y, p);
  p = __dp4a(w.z, x.z, p);
  p = __dp4a(w.w, x.w, p);
  return p;
}

template <int MT, int FMT, bool PARTIALS>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_kernel(const LinearArgs a, int stages, int64_t tiles_base, int64_t tiles_extra) {
  using S = GemvShape<MT>;
  constexpr int G = FMT == 0 ? kGroupTrunk : kGroupHead;
  using Red = typename std::conditional<FMT == 0, long long, float>::type;

  extern __shared__ __align__(128) uint8_t smem[];
  const int K = static_cast<int>(a.k);
  const int64_t N = a.n;
  const int M = static_cast<int>(a.m);
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  uint8_t* ring = smem + gemv_align128(MT * K);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + stages * kGemvStageBytes);
  uint64_t* empty = full + stages;
  Red* red = reinterpret_cast<Red*>(empty + stages);
  // Set by any role whose bounded wait ran out; everyone then skips further
  // waits but still reaches every barrier, so the CTA always finishes.
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t bid = blockIdx.x;
  const int64_t t0 = bid * tiles_base + (bid < tiles_extra ? bid : tiles_extra);
  const int64_t t1 = t0 + tiles_base + (bid < tiles_extra ? 1 : 0);
  const int nchunks = (K + kGemvKC - 1) / kGemvKC;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvConsumerWarps);
    }
    fence_barrier_init();
  }
  // activation codes -> shared memory; token rows >= M are zero
  {
    const int per_row = K / 16;
    for (int i = threadIdx.x; i < MT * per_row; i += blockDim.x) {
      const int m = i / per_row;
      const int c = i - m * per_row;
      int4 v = make_int4(0, 0, 0, 0);
      if (m < M) v = __ldg(reinterpret_cast<const int4*>(a.xq + static_cast<int64_t>(m) * K) + c);
      reinterpret_cast<int4*>(act + m * K)[c] = v;
    }
  }
  __syncthreads();

  if (warp == kGemvConsumerWarps) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t tile = t0; tile < t1 && ok; ++tile) {
        const int64_t row0 = tile * kGemvRows;
        const int rows = static_cast<int>(min(static_cast<int64_t>(kGemvRows), N - row0));
        for (int c = 0; c < nchunks; ++c) {
          const int slot = static_cast<int>(it % stages);
          const uint32_t use = it / stages;
          if (s_abort || (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1u, kDevErrGemvEmpty))) {
            s_abort = 1;
            ok = false;
            break;
          }
          const int len = min(kGemvKC, K - c * kGemvKC);
          mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(rows * len));
          uint8_t* dst = ring + slot * kGemvStageBytes;
          const int8_t* src = a.codes + row0 * K + c * kGemvKC;
          for (int r = 0; r < rows; ++r)
            bulk_g2s(dst + r * kGemvKC, src + static_cast<int64_t>(r) * K, static_cast<uint32_t>(len), &full[slot],
                     pol);
          ++it;
        }
      }
      // never leave with a copy still landing in this CTA's shared memory
      const uint32_t first = it > static_cast<uint32_t>(stages) ? it - stages : 0u;
      for (uint32_t j = first; j < it; ++j)
        if (!mbar_wait(&full[j % stages], (j / stages) & 1u, kDevErrGemvDrain)) break;
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int wr = warp % S::WR;
  const int wk = warp / S::WR;
  float xscale[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) xscale[m] = (!PARTIALS && m < M) ? a.xs[m] : 0.0f;
  const float rot = a.rotated ? 0.0078125f : 1.0f;
  const int ng = K / G;

  uint32_t it = 0;
  int par = 0;
  bool failed = false;  // warp-uniform
  for (int64_t tile = t0; tile < t1; ++tile, par ^= 1) {
    const int64_t row0 = tile * kGemvRows + wr * S::RG;
    long long acc64[S::RG][MT];
    float accf[S::RG][MT];
#pragma unroll
    for (int i = 0; i < S::RG; ++i)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        acc64[i][m] = 0;
        accf[i][m] = 0.0f;
      }
    for (int c = 0; c < nchunks; ++c, ++it) {
      const int slot = static_cast<int>(it % stages);
      const int len = min(kGemvKC, K - c * kGemvKC);
      // scales for this lane's steps, fetched before the data arrives
      int sc_i[S::RG][S::SPW];
      float sc_f[S::RG][S::SPW];
#pragma unroll
      for (int i = 0; i < S::RG; ++i)
#pragma unroll
        for (int u = 0; u < S::SPW; ++u) {
          const int o = (wk + S::WK * u) * 512 + lane * 16;
          const int64_t row = row0 + i;
          const bool v = o < len && row < N;
          const int kk = c * kGemvKC + o;
          sc_i[i][u] = 0;
          sc_f[i][u] = 0.0f;
          if (!PARTIALS && v) {
            if (FMT == 0)
              sc_i[i][u] = __ldg(a.sub + row * ng + (kk >> 8));
            else
              sc_f[i][u] = bf16_bits_to_float(__ldg(a.scale + row * ng + (kk >> 7)));
          }
        }
      if (!failed) {
        bool bad = s_abort != 0;
        if (!bad) bad = !mbar_wait(&full[slot], (it / stages) & 1u, kDevErrGemvFull);
        failed = __any_sync(0xffffffffu, bad);
        if (failed && lane == 0) s_abort = 1;
      }
      const uint8_t* stage = ring + slot * kGemvStageBytes;
      int acc32[S::RG][MT];
#pragma unroll
      for (int i = 0; i < S::RG; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc32[i][m] = 0;
#pragma unroll
      for (int u = 0; u < S::SPW; ++u) {
        const int o = (wk + S::WK * u) * 512 + lane * 16;
        const bool valid = !failed && o < len;  // uniform per 256-byte half-warp
        int4 xv[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m)
          xv[m] = valid ? *reinterpret_cast<const int4*>(act + m * K + c * kGemvKC + o) : make_int4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < S::RG; ++i) {
          if (row0 + i >= N) continue;  // warp-uniform
          const int4 wv = valid ? *reinterpret_cast<const int4*>(stage + (wr * S::RG + i) * kGemvKC + o)
                                : make_int4(0, 0, 0, 0);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int p = dot16(wv, xv[m]);
            if (PARTIALS) {
              // 16 lanes (trunk) or 8 lanes (lm_head) make one block
#pragma unroll
              for (int off = 1; off < G / 16; off <<= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
              if (valid && m < M && (lane & (G / 16 - 1)) == 0) {
                const int g = (c * kGemvKC + o) / G;
                a.partials[(static_cast<int64_t>(m) * N + row0 + i) * ng + g] = p;
              }
            } else if (FMT == 0) {
              acc32[i][m] += sc_i[i][u] * p;  // <= 255 * 16 * 127^2 per step
            } else {
              accf[i][m] = fmaf(static_cast<float>(p), sc_f[i][u], accf[i][m]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (FMT == 0 && !PARTIALS) {
#pragma unroll
        for (int i = 0; i < S::RG; ++i)
#pragma unroll
          for (int m = 0; m < MT; ++m) acc64[i][m] += acc32[i][m];
      }
    }
    if (PARTIALS) continue;

    // ------------------------------------------------------------ epilogue
    Red tot[S::RG][MT];
#pragma unroll
    for (int i = 0; i < S::RG; ++i)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        Red v;
        if (FMT == 0)
          v = acc64[i][m];
        else
          v = accf[i][m];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        tot[i][m] = v;
      }
    if (S::WK > 1) {
      Red* rb = red + par * (S::WK * S::WR * S::RG * MT);
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < S::RG; ++i)
#pragma unroll
          for (int m = 0; m < MT; ++m) rb[((wk * S::WR + wr) * S::RG + i) * MT + m] = tot[i][m];
      }
      named_barrier(1, kGemvConsumerWarps * 32);
      if (wk == 0 && lane < S::RG * MT) {
        const int i = lane / MT;
        const int m = lane % MT;
        Red v = 0;
#pragma unroll
        for (int w = 0; w < S::WK; ++w) v += rb[((w * S::WR + wr) * S::RG + i) * MT + m];
        const int64_t row = row0 + i;
        if (!failed && m < M && row < N) {
          float yv;
          if (FMT == 0)
            yv = __ll2float_rn(static_cast<long long>(v)) * xscale[m] * bf16_bits_to_float(a.scale[row]) * rot;
          else
            yv = static_cast<float>(v) * xscale[m] * rot;
          a.y[static_cast<int64_t>(m) * N + row] = float_to_bf16_bits_rn(yv);
        }
      }
    } else if (lane == 0 && !failed) {
#pragma unroll
      for (int i = 0; i < S::RG; ++i) {
        const int64_t row = row0 + i;
        if (row >= N) continue;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m >= M) continue;
          float yv;
          if (FMT == 0)
            yv = __ll2float_rn(static_cast<long long>(tot[i][m])) * xscale[m] *
                 bf16_bits_to_float(a.scale[row]) * rot;
          else
            yv = static_cast<float>(tot[i][m]) * xscale[m] * rot;
          a.y[static_cast<int64_t>(m) * N + row] = float_to_bf16_bits_rn(yv);
        }
      }
    }
  }
}

}  // namespace iq8r
