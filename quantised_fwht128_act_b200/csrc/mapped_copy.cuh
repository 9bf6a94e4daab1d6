// Copies between pinned, device-mapped host memory and device memory, as a
// kernel: a step's input copy, its layer and its output copy then chain
// under programmatic dependent launch (a copy node between two kernels on a
// stream would end their overlap, and every step would pay a cold start).
//
// IN (host -> device): each thread reads its first kMapCopyAhead 16-byte
// pieces of the host buffer before the wait for the previous kernel (nothing
// before this launch writes them: the caller filled the host buffer before
// the call), and stores them after it (the previous kernel may still read
// the device buffer). OUT (device -> host): everything after the wait.
#pragma once

#include "iq8r_device.cuh"

namespace iq8r {

constexpr int kMapCopyThreads = 128;
constexpr int kMapCopyAhead = 4;

template <bool IN>
__global__ void __launch_bounds__(kMapCopyThreads) mapped_copy_kernel(const uint16_t* src, uint16_t* dst,
                                                                      int64_t n) {
  const int64_t n16 = n / 8;  // whole 16-byte pieces
  const int4* s = reinterpret_cast<const int4*>(src);
  int4* d = reinterpret_cast<int4*>(dst);
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  pdl_launch_dependents();
  int4 v[kMapCopyAhead];
  if (IN) {
#pragma unroll
    for (int j = 0; j < kMapCopyAhead; ++j) {
      const int64_t i = t + j * stride;
      if (i < n16) v[j] = s[i];
    }
  }
  pdl_wait();
  if (IN) {
#pragma unroll
    for (int j = 0; j < kMapCopyAhead; ++j) {
      const int64_t i = t + j * stride;
      if (i < n16) d[i] = v[j];
    }
  }
  for (int64_t i = t + (IN ? kMapCopyAhead * stride : 0); i < n16; i += stride) d[i] = s[i];
  // the last n % 8 elements
  if (t < n - n16 * 8) dst[n16 * 8 + t] = src[n16 * 8 + t];
}

}  // namespace iq8r
