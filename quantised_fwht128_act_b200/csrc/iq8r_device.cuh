// Device-side helpers shared by the IQ8R kernels: the error word, bounded
// mbarrier waits and 1-D bulk (TMA engine) copies. Inline PTX for sm_100a.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "iq8r_internal.h"

namespace iq8r {

// One word per device. A kernel whose bounded wait runs out stores the
// wait's code here (first writer wins) and leaves; the host reads and clears
// it through iq8r_get_device_error.
__device__ uint32_t g_device_error;

// Upper bound on any single wait inside a kernel, in SM clock cycles
// (about a second at B200 clocks). Waits normally last nanoseconds to
// microseconds; running out means the partner role is gone. The SM's own
// cycle counter is used because it is cheap to read inside a polling loop.
constexpr uint64_t kWaitLimitCycles = 2000ull * 1000ull * 1000ull;

__device__ __forceinline__ void set_device_error(uint32_t code) {
  atomicCAS(&g_device_error, 0u, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (bulk copy) proxy.
// Programmatic dependent launch. A kernel launched with programmatic stream
// serialisation may start while the stream's previous kernel is finishing;
// pdl_wait() blocks until that kernel has completed and its writes are
// visible, so everything before it may only read data no earlier kernel
// writes (the weights). pdl_launch_dependents() lets the next kernel start
// once every CTA of this one has issued it or exited. Both are no-ops for a
// plain launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// One poll of the barrier. A thread whose phase is not complete yet may be
// suspended (not spinning, so it leaves issue slots to working warps) for up
// to kSuspendHintNs before the poll reports "not yet".
constexpr uint32_t kSuspendHintNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Has the phase with the given parity completed? Never blocks.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// limit_cycles SM cycles. On timeout: record `code` and return false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t code,
                                          uint64_t limit_cycles = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (static_cast<uint64_t>(clock64() - t0) > limit_cycles) {
      set_device_error(code);
      return false;
    }
  }
}

// L2 policy for data read exactly once (streamed weights).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> shared through the TMA engine; completion is
// counted in bytes on `bar`. dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Same, with the default L2 policy (data that other CTAs read too).
__device__ __forceinline__ void bulk_g2s_default(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Plan the copy of bytes [o0, o1) of a 16-byte-aligned array of `total`
// bytes into dst as the 16-byte-aligned window [o0 & ~15, ...) around them,
// one bulk copy; dst[(o0 & 15) + i] is then byte o0 + i. Only bytes past the
// last whole 16 of the array (the final rows of a matrix) go by plain loads,
// done here (by the lane with copy_tail) before the caller's arrive.
struct GemvWindow {
  const uint8_t* src;
  uint8_t* dst;
  uint32_t bytes;
};
__device__ __forceinline__ GemvWindow window_copy_plan(uint8_t* dst, const uint8_t* base, int64_t total, int64_t o0,
                                                       int64_t o1, bool copy_tail) {
  const int64_t w0 = o0 & ~int64_t(15);
  const int64_t e16 = total & ~int64_t(15);
  int64_t w1 = (o1 + 15) & ~int64_t(15);
  if (w1 > e16) {
    w1 = e16;
    if (copy_tail)
      for (int64_t b = (w0 > e16 ? w0 : e16); b < o1; ++b) dst[b - w0] = __ldg(base + b);
  }
  GemvWindow w{base + w0, dst, w1 > w0 ? static_cast<uint32_t>(w1 - w0) : 0u};
  return w;
}

// Named barrier over `threads` threads (a multiple of 32), id 1..15.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// float -> bf16 bits, round to nearest even (finite and inf inputs).
__device__ __forceinline__ uint16_t float_to_bf16_bits_rn(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

}  // namespace iq8r
