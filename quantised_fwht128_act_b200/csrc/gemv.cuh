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
//  - warp 8 is the producer. One lane issues every copy with 1-D bulk copies
//    (TMA engine) completing on mbarriers: the activation codes once, then
//    per tile its scales (u8 sub-scales and bf16 row scales, or the lm_head's
//    bf16 group scales) into a 4-slot scale ring, and the tile's codes in
//    2 KB-of-K chunks (8 rows x 2 KB = 16 KB stage) into a ring of up to 12
//    stages, weights marked evict-first in L2;
//  - warps 0..7 consume from shared memory only: a warp owns RG rows and
//    every WK-th 512-byte step of K; each lane does 4 dp4a per 16 bytes per
//    token, scales the lane's partial by its block's u8 sub-scale in int32
//    (exact) and folds it into int64 once per chunk;
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
constexpr int kGemvScaleSlots = 4;

template <int MT>
struct GemvShape {
  static constexpr int RG = MT == 1 ? 1 : (MT == 2 ? 2 : 4);  // rows per warp
  static constexpr int WR = kGemvRows / RG;                    // warps along rows
  static constexpr int WK = kGemvConsumerWarps / WR;           // warps along K
  static constexpr int STEPS = kGemvKC / 512;                  // 512-byte steps per chunk
  static constexpr int SPW = STEPS / WK;                       // steps per warp per chunk
};

__host__ __device__ constexpr int gemv_align128(int x) { return (x + 127) & ~127; }
__host__ __device__ constexpr int gemv_align16(int x) { return (x + 15) & ~15; }

// One tile's scales in shared memory. Trunk: [8][ng] u8 sub-scales, padded
// to 16 bytes, then [8] bf16 row scales. lm_head: [8][ng] bf16 group scales.
__host__ __device__ constexpr int gemv_s2_offset(int k) { return gemv_align16(kGemvRows * (k / kGroupTrunk)); }
__host__ __device__ constexpr int gemv_scale_slot_bytes(int fmt, int k) {
  return fmt == 0 ? gemv_s2_offset(k) + 2 * kGemvRows : gemv_align16(kGemvRows * (k / kGroupHead) * 2);
}

template <int MT, int FMT>
__host__ __device__ constexpr int gemv_red_bytes() {
  // [2 buffers][WK][WR][RG][MT] of int64 (trunk) or float (lm_head)
  return 2 * GemvShape<MT>::WK * GemvShape<MT>::WR * GemvShape<MT>::RG * MT * (FMT == 0 ? 8 : 4);
}

struct GemvSmem {
  int ring, scales, bars, red, total;
};

// Shared memory map: [act MT*K][ring][scale slots][barriers][reduction].
__host__ __device__ constexpr GemvSmem gemv_smem_layout(int mt, int fmt, int k, int stages, int red_bytes) {
  const int ring = gemv_align128(mt * k);
  const int scales = ring + stages * kGemvStageBytes;
  const int bars = scales + kGemvScaleSlots * gemv_scale_slot_bytes(fmt, k);
  const int red = gemv_align16(bars + 8 * (2 * stages + 2 * kGemvScaleSlots + 1));
  return GemvSmem{ring, scales, bars, red, red + red_bytes};
}

__device__ __forceinline__ int dot16(const int4 w, const int4 x) {
  int p = __dp4a(w.x, x.x, 0);
  p = __dp4a(w.y, x.y, p);
  p = __dp4a(w.z, x.z, p);
  p = __dp4a(w.w, x.w, p);
  return p;
}

// Bytes of [src, src + bytes) that go by bulk copy: the whole 16-byte
// multiple when src is 16-byte aligned, else none.
__device__ __forceinline__ int bulk_part(const void* src, int bytes) {
  return (reinterpret_cast<uintptr_t>(src) & 15u) == 0 ? (bytes & ~15) : 0;
}

// Plain byte copy of the part bulk_part leaves (done before the arrive, so
// the barrier's release orders it for the consumers).
__device__ __forceinline__ void plain_tail(uint8_t* dst, const uint8_t* src, int from, int bytes) {
  for (int b = from; b < bytes; ++b) dst[b] = __ldg(src + b);
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
  const int ng = K / G;
  const GemvSmem L = gemv_smem_layout(MT, FMT, K, stages, gemv_red_bytes<MT, FMT>());
  const int slot_bytes = gemv_scale_slot_bytes(FMT, K);
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  uint8_t* ring = smem + L.ring;
  uint8_t* scl = smem + L.scales;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + stages;
  uint64_t* sfull = empty + stages;
  uint64_t* sempty = sfull + kGemvScaleSlots;
  uint64_t* actbar = sempty + kGemvScaleSlots;
  Red* red = reinterpret_cast<Red*>(smem + L.red);
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
    for (int s = 0; s < kGemvScaleSlots; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], kGemvConsumerWarps);
    }
    mbar_init(actbar, 1);
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kGemvConsumerWarps) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      // the M token rows of activation codes, contiguous [M][K]
      mbar_arrive_expect_tx(actbar, static_cast<uint32_t>(M * K));
      bulk_g2s_default(act, a.xq, static_cast<uint32_t>(M * K), actbar);
      uint32_t it = 0;
      uint32_t lt = 0;
      bool ok = true;
      for (int64_t tile = t0; tile < t1 && ok; ++tile, ++lt) {
        const int64_t row0 = tile * kGemvRows;
        const int rows = static_cast<int>(min(static_cast<int64_t>(kGemvRows), N - row0));
        if (!PARTIALS) {
          const int ss = static_cast<int>(lt % kGemvScaleSlots);
          const uint32_t suse = lt / kGemvScaleSlots;
          if (s_abort || (suse > 0 && !mbar_wait(&sempty[ss], (suse - 1) & 1u, kDevErrGemvEmpty))) {
            s_abort = 1;
            ok = false;
            break;
          }
          uint8_t* dst = scl + ss * slot_bytes;
          const uint8_t* src0;
          int bytes0;
          if (FMT == 0) {
            src0 = a.sub + row0 * ng;
            bytes0 = rows * ng;
          } else {
            src0 = reinterpret_cast<const uint8_t*>(a.scale + row0 * ng);
            bytes0 = rows * ng * 2;
          }
          const int nb0 = bulk_part(src0, bytes0);
          plain_tail(dst, src0, nb0, bytes0);
          int nb1 = 0;
          const uint8_t* src1 = nullptr;
          uint8_t* dst1 = dst + gemv_s2_offset(K);
          if (FMT == 0) {
            src1 = reinterpret_cast<const uint8_t*>(a.scale + row0);
            nb1 = bulk_part(src1, rows * 2);
            plain_tail(dst1, src1, nb1, rows * 2);
          }
          mbar_arrive_expect_tx(&sfull[ss], static_cast<uint32_t>(nb0 + nb1));
          if (nb0) bulk_g2s(dst, src0, static_cast<uint32_t>(nb0), &sfull[ss], pol);
          if (nb1) bulk_g2s(dst1, src1, static_cast<uint32_t>(nb1), &sfull[ss], pol);
        }
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
      bool drained = mbar_wait(actbar, 0u, kDevErrGemvDrain);
      const uint32_t first = it > static_cast<uint32_t>(stages) ? it - stages : 0u;
      for (uint32_t j = first; j < it && drained; ++j)
        drained = mbar_wait(&full[j % stages], (j / stages) & 1u, kDevErrGemvDrain);
      if (!PARTIALS) {
        const uint32_t sfirst = lt > static_cast<uint32_t>(kGemvScaleSlots) ? lt - kGemvScaleSlots : 0u;
        for (uint32_t j = sfirst; j < lt && drained; ++j)
          drained = mbar_wait(&sfull[j % kGemvScaleSlots], (j / kGemvScaleSlots) & 1u, kDevErrGemvDrain);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int wr = warp % S::WR;
  const int wk = warp / S::WR;
  // token rows past M are zero (their codes never reach an output anyway)
  {
    int4* pad = reinterpret_cast<int4*>(act + M * K);
    const int n16 = (MT - M) * K / 16;
    for (int i = threadIdx.x; i < n16; i += kGemvConsumerWarps * 32) pad[i] = make_int4(0, 0, 0, 0);
  }
  named_barrier(1, kGemvConsumerWarps * 32);
  float xscale[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) xscale[m] = (!PARTIALS && m < M) ? a.xs[m] : 0.0f;
  const float rot = a.rotated ? 0.0078125f : 1.0f;

  bool failed = false;  // warp-uniform
  {
    bool bad = s_abort != 0;
    if (!bad) bad = !mbar_wait(actbar, 0u, kDevErrGemvFull);
    failed = __any_sync(0xffffffffu, bad);
    if (failed && lane == 0) s_abort = 1;
  }

  uint32_t it = 0;
  uint32_t lt = 0;
  int par = 0;
  for (int64_t tile = t0; tile < t1; ++tile, ++lt, par ^= 1) {
    const int64_t wrow0 = tile * kGemvRows + wr * S::RG;  // this warp's first row
    const int ss = static_cast<int>(lt % kGemvScaleSlots);
    const uint8_t* ts = scl + ss * slot_bytes;
    if (!PARTIALS && !failed) {
      bool bad = s_abort != 0;
      if (!bad) bad = !mbar_wait(&sfull[ss], (lt / kGemvScaleSlots) & 1u, kDevErrGemvFull);
      failed = __any_sync(0xffffffffu, bad);
      if (failed && lane == 0) s_abort = 1;
    }
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
        const int kk = c * kGemvKC + o;
        const int g = kk / G;
        int4 xv[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m)
          xv[m] = valid ? *reinterpret_cast<const int4*>(act + m * K + kk) : make_int4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < S::RG; ++i) {
          if (wrow0 + i >= N) continue;  // warp-uniform
          const int rl = wr * S::RG + i;  // row within the tile
          const int4 wv = valid ? *reinterpret_cast<const int4*>(stage + rl * kGemvKC + o) : make_int4(0, 0, 0, 0);
          int s1 = 0;
          float sf = 0.0f;
          if (!PARTIALS && valid) {
            if (FMT == 0)
              s1 = ts[rl * ng + g];
            else
              sf = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(ts)[rl * ng + g]);
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int p = dot16(wv, xv[m]);
            if (PARTIALS) {
              // 16 lanes (trunk) or 8 lanes (lm_head) make one block
#pragma unroll
              for (int off = 1; off < G / 16; off <<= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
              if (valid && m < M && (lane & (G / 16 - 1)) == 0)
                a.partials[(static_cast<int64_t>(m) * N + wrow0 + i) * ng + g] = p;
            } else if (FMT == 0) {
              acc32[i][m] += s1 * p;  // <= 255 * 16 * 127^2 per step, <= 4 steps
            } else {
              accf[i][m] = fmaf(static_cast<float>(p), sf, accf[i][m]);
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
    const uint16_t* s2 = reinterpret_cast<const uint16_t*>(ts + gemv_s2_offset(K));
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
        const int64_t row = wrow0 + i;
        if (!failed && m < M && row < N) {
          float yv;
          if (FMT == 0)
            yv = __ll2float_rn(static_cast<long long>(v)) * xscale[m] * bf16_bits_to_float(s2[wr * S::RG + i]) * rot;
          else
            yv = static_cast<float>(v) * xscale[m] * rot;
          a.y[static_cast<int64_t>(m) * N + row] = float_to_bf16_bits_rn(yv);
        }
      }
    } else if (lane == 0 && !failed) {
#pragma unroll
      for (int i = 0; i < S::RG; ++i) {
        const int64_t row = wrow0 + i;
        if (row >= N) continue;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m >= M) continue;
          float yv;
          if (FMT == 0)
            yv = __ll2float_rn(static_cast<long long>(tot[i][m])) * xscale[m] *
                 bf16_bits_to_float(s2[wr * S::RG + i]) * rot;
          else
            yv = static_cast<float>(tot[i][m]) * xscale[m] * rot;
          a.y[static_cast<int64_t>(m) * N + row] = float_to_bf16_bits_rn(yv);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sempty[ss]);  // this warp is done with the tile's scales
  }
}

}  // namespace iq8r
