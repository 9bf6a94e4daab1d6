// Activation rotate + int8 quantise: the activations are int8 in the same
// rotated domain as the weights, W8A8 ("Qwen3.8-27B IQ8R + DFlash2 --
// radiance container", table row "Activations"), one fp32 scale per token:
// a = amax / 127, codes rint(x' * (127 / amax)) clamped to +-127, a row with
// amax below 2^-64 first multiplied by 2^64 (exact; see act_inv).
//
// One CTA per token row. A thread owns "slots" of 16 consecutive elements
// (two 16-byte bf16 loads, one 16-byte int8 store). A 128-chunk is 8 slots
// held by 8 consecutive lanes, so fwht128's seven butterfly stages run as
// h = 1, 2, 4, 8 inside the thread and h = 16, 32, 64 across lanes (xor 1,
// 2, 4; or, in the one-CTA-a-row kernel, through a shared-memory exchange),
// in that order, each an IEEE add or subtract: the result is bit-identical
// to the sequential radix-2 transform.
#pragma once

#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kActSlot = 16;           // elements per slot
constexpr int kActRegMaxK = 16384;     // register path up to this K
constexpr int kActRegMaxThreads = 256;  // its CTA size limit (8 slots a thread cover K = 16384)
constexpr int kActTwoPassThreads = 256;

__device__ __forceinline__ void act_load_slot(const uint16_t* p, float (&v)[kActSlot], bool streaming) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  uint4 lo, hi;
  if (streaming) {
    lo = __ldcs(q);
    hi = __ldcs(q + 1);
  } else {
    lo = __ldg(q);
    hi = __ldg(q + 1);
  }
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// fwht128 of the chunk this lane's slot belongs to (8 lanes per chunk).
__device__ __forceinline__ void act_fwht_slot(float (&v)[kActSlot], int lane) {
#pragma unroll
  for (int h = 1; h < kActSlot; h <<= 1) {
#pragma unroll
    for (int i = 0; i < kActSlot; ++i) {
      if ((i & h) == 0) {
        const float a = v[i];
        const float b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int b = 1; b < 8; b <<= 1) {
    const bool upper = (lane & b) != 0;
#pragma unroll
    for (int i = 0; i < kActSlot; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], b);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
}

// The same transform with h = 16, 32, 64 through shared memory instead of
// shuffles. After the in-thread stages, each 8-lane group (one 128-chunk,
// lane q holding elements 16q..16q+15) exchanges its chunk so that lane q
// holds elements 16p + 2q + b (p = 0..7, b = 0, 1) as t[2p + b]; h = 16, 32,
// 64 are then register butterflies over p with strides 1, 2, 4, in that
// order, each the same add or subtract. Layout of a group's 128 floats:
// element 16p + i at 8i + 4(i / 4) + p, groups kActXStride floats apart, so
// the scalar writes (fixed i, the warp's 32 lanes) and the 16-byte reads
// (fixed offset, 8 lanes a phase) fall in distinct banks. xb: the warp's
// 4 * kActXStride floats, 16-byte aligned.
constexpr int kActXStride = 152;  // floats a group (128 + 24; 152 = 24 mod 32)
constexpr int kActCStride = 144;  // bytes a group of codes (128 + 16)

__device__ __forceinline__ void act_fwht_slot_xchg(float (&v)[kActSlot], float* xb, int lane) {
#pragma unroll
  for (int h = 1; h < kActSlot; h <<= 1) {
#pragma unroll
    for (int i = 0; i < kActSlot; ++i) {
      if ((i & h) == 0) {
        const float a = v[i];
        const float b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
    }
  }
  const int q = lane & 7;
  float* gb = xb + (lane >> 3) * kActXStride;
  __syncwarp();  // earlier readers of the buffer are done
#pragma unroll
  for (int i = 0; i < kActSlot; ++i) gb[8 * i + 4 * (i >> 2) + q] = v[i];
  __syncwarp();
  // elements i = 2q (then 2q + 1), p = 0..7: 16 consecutive floats
  const float4* r = reinterpret_cast<const float4*>(gb + 16 * q + 4 * (q >> 1));
  float f[kActSlot];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 w = r[c];
    f[4 * c] = w.x;
    f[4 * c + 1] = w.y;
    f[4 * c + 2] = w.z;
    f[4 * c + 3] = w.w;
  }
  // f[8b + p] is element 16p + 2q + b
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      if ((p & h) == 0) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const float x0 = f[8 * b + p];
          const float x1 = f[8 * b + p + h];
          f[8 * b + p] = __fadd_rn(x0, x1);
          f[8 * b + p + h] = __fsub_rn(x0, x1);
        }
      }
    }
  }
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    v[2 * p] = f[p];
    v[2 * p + 1] = f[8 + p];
  }
}

// The code of one value: rint(v * inv). No clamp is needed for a finite
// row: |v| <= amax (after the same prescale as amax) and inv = RN(127 /
// amax), so |v * inv| <= 127 (1 + 2^-24) and its rounding to the nearest
// integer is at most 127 in magnitude; the clamp to +-127 of the definition
// never acts. (Non-finite rows are outside the definition.)
__device__ __forceinline__ int act_code(float v, float inv) { return __float2int_rn(__fmul_rn(v, inv)); }

// Low bytes of four codes, in order, as one word (two byte permutes).
__device__ __forceinline__ uint32_t act_pack4(int q0, int q1, int q2, int q3) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(q0), static_cast<uint32_t>(q1), 0x0040u);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(q2), static_cast<uint32_t>(q3), 0x0040u);
  return __byte_perm(lo, hi, 0x5410u);
}

// Quantise a slot left by act_fwht_slot_xchg (t[2p + b] = element
// 16p + 2q + b) and store the group's codes in element order: pairs of bytes
// into the group's cb window (conflict-free: groups 36 words apart), then
// each lane's own 16 bytes to p (when `in`).
__device__ __forceinline__ void act_store_slot_xchg(int8_t* out, const float (&t)[kActSlot], float inv,
                                                    uint8_t* cb, int lane, bool in) {
  const int q = lane & 7;
  uint8_t* gc = cb + (lane >> 3) * kActCStride;
  __syncwarp();  // earlier readers of the buffer are done
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int c0 = act_code(t[2 * p], inv);  // in -127..127 (see act_code)
    const int c1 = act_code(t[2 * p + 1], inv);
    *reinterpret_cast<uint16_t*>(gc + 16 * p + 2 * q) =
        static_cast<uint16_t>(__byte_perm(static_cast<uint32_t>(c0), static_cast<uint32_t>(c1), 0x0040u));
  }
  __syncwarp();
  if (in) *reinterpret_cast<uint4*>(out) = *reinterpret_cast<const uint4*>(gc + 16 * q);
}

// A row whose amax is below 2^-64 is quantised after an exact multiplication
// by 2^64, so that 127 / amax stays finite down to the smallest subnormal
// (it overflows below 127 / FLT_MAX). For every row whose 127 / amax is
// finite this changes no code: (x' c) * (127 / (amax c)) is the same real
// number as x' * (127 / amax). The scale a = amax / 127 is unchanged.
constexpr float kActTiny = 0x1p-64f;
constexpr float kActPrescale = 0x1p64f;

// 127 / amax for the codes (after the prescale), 0 for a zero row.
__device__ __forceinline__ float act_inv(float amax) {
  return amax > 0.0f ? __fdiv_rn(127.0f, amax < kActTiny ? __fmul_rn(amax, kActPrescale) : amax) : 0.0f;
}

// The prescale of a tiny row's values (uniform across the row's threads).
__device__ __forceinline__ void act_prescale_slot(float (&v)[kActSlot], float amax) {
  if (amax < kActTiny) {
#pragma unroll
    for (int i = 0; i < kActSlot; ++i) v[i] = __fmul_rn(v[i], kActPrescale);
  }
}

__device__ __forceinline__ float act_slot_absmax(const float (&v)[kActSlot]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kActSlot; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

__device__ __forceinline__ void act_store_slot(int8_t* p, const float (&v)[kActSlot], float inv) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = act_pack4(act_code(v[4 * i], inv), act_code(v[4 * i + 1], inv), act_code(v[4 * i + 2], inv),
                     act_code(v[4 * i + 3], inv));
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// CTA-wide max of non-negative floats; every thread gets the result.
__device__ __forceinline__ float act_block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  float m = 0.0f;
  for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[w]);
  return m;
}

// K <= kActRegMaxK: the row stays in registers (J slots per thread).
template <int J>
__global__ void __launch_bounds__(kActRegMaxThreads) act_quant_reg_kernel(const uint16_t* __restrict__ x, int k, int rotate,
                                                            int8_t* __restrict__ xq, float* __restrict__ xs) {
  __shared__ float red[32];
  // per warp: the chunk exchange of the transform and the codes' reorder
  __shared__ __align__(16) float xbuf[kActRegMaxThreads / 32][4 * kActXStride];
  __shared__ __align__(16) uint8_t cbuf[kActRegMaxThreads / 32][4 * kActCStride];
  pdl_launch_dependents();  // the next kernel may start its set-up
  const int64_t row = blockIdx.x;
  const int slots = k / kActSlot;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint16_t* xr = x + row * k;
  float v[J][kActSlot];
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int s = threadIdx.x + j * blockDim.x;
    if (s < slots) {
      act_load_slot(xr + s * kActSlot, v[j], true);
    } else {
#pragma unroll
      for (int i = 0; i < kActSlot; ++i) v[j][i] = 0.0f;
    }
    if (rotate) act_fwht_slot_xchg(v[j], xbuf[warp], lane);  // whole 8-lane groups are in or out
    amax = fmaxf(amax, act_slot_absmax(v[j]));
  }
  amax = act_block_max(amax, red);
  const float inv = act_inv(amax);
  int8_t* qr = xq + row * k;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int s = threadIdx.x + j * blockDim.x;
    act_prescale_slot(v[j], amax);
    if (rotate) {
      act_store_slot_xchg(qr + s * kActSlot, v[j], inv, cbuf[warp], lane, s < slots);
    } else if (s < slots) {
      act_store_slot(qr + s * kActSlot, v[j], inv);
    }
  }
  if (threadIdx.x == 0) xs[row] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

// Few tokens: a row is shared by the C CTAs of one thread-block cluster
// (blockIdx.x = part of the row, blockIdx.y = token), each holding whole
// 128-chunks in registers (J slots per thread). The token's amax is the max
// of the C CTA maxima, read from each other's shared memory (DSMEM), so the
// row is read from HBM once and C SMs share it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_shared_cluster_f32(const float* p, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(p)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

template <int J>
__global__ void __launch_bounds__(1024) act_quant_cluster_kernel(const uint16_t* __restrict__ x, int k,
                                                                 int slots_per_part, int rotate,
                                                                 int8_t* __restrict__ xq, float* __restrict__ xs) {
  __shared__ float red[32];
  pdl_launch_dependents();  // the next kernel may start its set-up
  __shared__ float part_max;
  const int64_t row = blockIdx.y;
  const int slots = k / kActSlot;
  const int lane = threadIdx.x & 31;
  const int s0 = blockIdx.x * slots_per_part;
  const int s1 = min(slots, s0 + slots_per_part);
  const uint16_t* xr = x + row * k;
  float v[J][kActSlot];
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int s = s0 + threadIdx.x + j * blockDim.x;
    if (s < s1) {
      act_load_slot(xr + s * kActSlot, v[j], true);
    } else {
#pragma unroll
      for (int i = 0; i < kActSlot; ++i) v[j][i] = 0.0f;
    }
    if (rotate) act_fwht_slot(v[j], lane);  // parts and J-steps hold whole 8-lane groups
    amax = fmaxf(amax, act_slot_absmax(v[j]));
  }
  amax = act_block_max(amax, red);
  if (threadIdx.x == 0) part_max = amax;
  cluster_sync_all();  // every part's maximum is in its shared memory
  float g = 0.0f;
  for (uint32_t r = 0; r < gridDim.x; ++r) g = fmaxf(g, ld_shared_cluster_f32(&part_max, r));
  cluster_sync_all();  // no CTA leaves while another still reads its maximum
  const float inv = act_inv(g);
  int8_t* qr = xq + row * k;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int s = s0 + threadIdx.x + j * blockDim.x;
    act_prescale_slot(v[j], g);
    if (s < s1) act_store_slot(qr + s * kActSlot, v[j], inv);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) xs[row] = g > 0.0f ? __fdiv_rn(g, 127.0f) : 0.0f;
}

// Any K: pass 1 finds amax, pass 2 reloads the row (now in L2), repeats the
// identical transform and quantises.
__global__ void __launch_bounds__(kActTwoPassThreads) act_quant_2pass_kernel(const uint16_t* __restrict__ x, int k,
                                                                             int rotate, int8_t* __restrict__ xq,
                                                                             float* __restrict__ xs) {
  __shared__ float red[32];
  pdl_launch_dependents();  // the next kernel may start its set-up
  const int64_t row = blockIdx.x;
  const int slots = k / kActSlot;
  const int lane = threadIdx.x & 31;
  const uint16_t* xr = x + row * static_cast<int64_t>(k);
  const int iters = (slots + blockDim.x - 1) / blockDim.x;
  float v[kActSlot];
  float amax = 0.0f;
  for (int j = 0; j < iters; ++j) {
    const int s = threadIdx.x + j * blockDim.x;
    if (s < slots) {
      act_load_slot(xr + static_cast<int64_t>(s) * kActSlot, v, false);
    } else {
#pragma unroll
      for (int i = 0; i < kActSlot; ++i) v[i] = 0.0f;
    }
    if (rotate) act_fwht_slot(v, lane);
    amax = fmaxf(amax, act_slot_absmax(v));
  }
  amax = act_block_max(amax, red);
  const float inv = act_inv(amax);
  int8_t* qr = xq + row * static_cast<int64_t>(k);
  for (int j = 0; j < iters; ++j) {
    const int s = threadIdx.x + j * blockDim.x;
    if (s < slots) {
      act_load_slot(xr + static_cast<int64_t>(s) * kActSlot, v, false);
    } else {
#pragma unroll
      for (int i = 0; i < kActSlot; ++i) v[i] = 0.0f;
    }
    if (rotate) act_fwht_slot(v, lane);
    act_prescale_slot(v, amax);
    if (s < slots) act_store_slot(qr + static_cast<int64_t>(s) * kActSlot, v, inv);
  }
  if (threadIdx.x == 0) xs[row] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

}  // namespace iq8r
