// Launchers for the IQ8R kernels. All device code lives in this one
// translation unit so the per-device error word is a single symbol.

#include <algorithm>
#include <atomic>
#include <string>

#include <cudaTypedefs.h>

#include "act_quant.cuh"
#include "gemm_tc.cuh"
#include "tc_split_reduce.cuh"
#include "gemv.cuh"
#include "gemv_reg.cuh"
#include "mapped_copy.cuh"
#include "cb4_gemv.cuh"
#include "cb4_mma.cuh"
#include "rescore.cuh"
#include "iq8r_device.cuh"
#include "iq8r_internal.h"

namespace iq8r {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kGemvY = 0, kGemvPartials = 1, kGemvFused = 2;  // what a GEMV launch produces

struct DeviceInfo {
  int num_sms = 0;
  int smem_optin = 0;
};

DeviceInfo g_dev[kMaxDevices];
std::atomic<int> g_dev_ready[kMaxDevices];

cudaError_t device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (g_dev_ready[dev].load(std::memory_order_acquire) == 0) {
    DeviceInfo d;
    e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    g_dev[dev] = d;
    g_dev_ready[dev].store(1, std::memory_order_release);
  }
  *out = g_dev[dev];
  return cudaSuccess;
}

// Raise a kernel's dynamic shared memory limit once per device (and again
// only if a larger size is asked for). `configured` must be distinct for
// every kernel: kernels of one signature share a function-pointer type, so
// the caller owns the cache (a static inside its own template instance).
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, std::atomic<int>* configured) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (configured[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) configured[dev].store(bytes, std::memory_order_release);
  return e;
}

// Static shared memory and alignment slack kept out of the dynamic budget.
constexpr int kSmemReserve = 2048;

// Stage size and depth for a token tile of `mt`: the shared memory left after
// the activation codes is split over the warps; each gets two or more stages
// of up to 16 KB of codes (whole rows when they fit). rt == 0: no fit.
GemvPlan gemv_choose(int mt, int fmt, int k, const DeviceInfo& d) {
  GemvPlan none{};
  const int warps = gemv_warps(mt);
  const int budget = d.smem_optin - kSmemReserve;
  const int avail = budget - gemv_align128(mt * k) - 8 * (warps * kGemvMaxDepth + 1) - 16;
  if (avail <= 0) return none;
  const int per_warp = avail / warps;
  // one or two tokens: a stage holds at most 10 steps of 512 bytes, the
  // register-staged consumer's limit
  const int cap = mt <= 2 ? 10 * 512 : 16 * 1024;
  for (int target = std::min(cap, (per_warp / 2) & ~511); target >= 512; target -= 512) {
    GemvPlan p = gemv_plan(mt, fmt, k, target, 2, warps);
    const int depth = std::min(kGemvMaxDepth, per_warp / p.stage_bytes);
    if (depth < 2) continue;
    p = gemv_plan(mt, fmt, k, target, depth, warps);
    if (p.smem <= budget) return p;
  }
  return none;
}

template <int MT, int RG, int FMT, int MODE>
cudaError_t launch_gemv_t(const LinearArgs& a, const GemvPlan& plan, const DeviceInfo& d, cudaStream_t stream) {
  auto kernel = gemv_kernel<MT, RG, FMT, MODE == kGemvPartials, MODE == kGemvFused>;
  const int64_t tiles = (a.n + plan.rt - 1) / plan.rt;
  const int64_t grid = std::min<int64_t>(d.num_sms, tiles);
  GemvPlan p = plan;
  if (FMT == 0 && MODE != kGemvPartials) {
    // the trunk's scales of a CTA's rows are small: load them once, up front,
    // instead of two more copies with every stage
    const int64_t rows = (tiles + grid - 1) / grid * p.rt;
    const int64_t ng = a.k / kGroupTrunk;
    const int64_t s1b = gemv_align16(static_cast<int>(std::min<int64_t>(rows * ng, 1 << 20)) + 32);
    const int64_t s2b = gemv_align16(static_cast<int>(std::min<int64_t>(2 * rows, 1 << 20)) + 32);
    const int64_t base = gemv_align16(p.smem);
    if (base + s1b + s2b <= d.smem_optin - kSmemReserve) {
      p.pre = 1;
      p.pre_s1 = static_cast<int>(s1b);
      p.pre_bytes = static_cast<int>(s1b + s2b);
      p.smem = static_cast<int>(base + s1b + s2b);
    }
  }
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = ensure_smem(kernel, p.smem, configured);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the kernel's first weight stages stream
  // while the stream's previous kernel drains (the kernel waits for it before
  // touching activations or outputs)
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(p.warps * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a, p, tiles / grid, tiles % grid);
}

// The register-streaming GEMV's shape (one or two tokens): rows_base == 0
// when its activation codes and scale window do not fit shared memory.
RegPlan gemv_reg_plan(const LinearArgs& a, int mt, const DeviceInfo& d) {
  RegPlan p{};
  if (mt > 2 || a.n < 1) return p;
  const int64_t ng = a.k / (a.fmt == 0 ? kGroupTrunk : kGroupHead);
  const int64_t grid = std::min<int64_t>(d.num_sms, a.n);
  const int64_t rmax = (a.n + grid - 1) / grid;
  const int64_t sc = a.fmt == 0 ? gemv_align16(static_cast<int>(std::min<int64_t>(rmax * ng, 1 << 24)) + 32) +
                                      gemv_align16(static_cast<int>(std::min<int64_t>(2 * rmax, 1 << 24)) + 32)
                                : gemv_align16(static_cast<int>(std::min<int64_t>(2 * rmax * ng, 1 << 24)) + 32);
  const int64_t smem = gemv_align128(static_cast<int>(mt * a.k)) + sc;
  if (rmax * ng > (1 << 22) || smem > d.smem_optin - kSmemReserve) return p;
  p.rows_base = a.n / grid;
  p.rows_extra = a.n % grid;
  p.parts = static_cast<int>((a.k + kRegPartBytes - 1) / kRegPartBytes);
  p.sc_bytes = static_cast<int>(sc);
  p.smem = static_cast<int>(smem);
  return p;
}

template <int MT, int FMT, bool FUSED, bool AFTER>
cudaError_t launch_gemv_reg_t(const LinearArgs& a, const RegPlan& p, const DeviceInfo& d, cudaStream_t stream) {
  auto kernel = gemv_reg_kernel<MT, FMT, FUSED, AFTER>;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = ensure_smem(kernel, p.smem, configured);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the first units of weights stream while
  // the stream's previous kernel drains (the kernel waits for it before
  // touching activations or outputs)
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(d.num_sms, a.n)));
  cfg.blockDim = dim3(kRegWarps * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a, p);
}

template <int FMT, int MODE>
cudaError_t launch_gemv_mt(const LinearArgs& a, int mt, const DeviceInfo& d, cudaStream_t stream) {
  if (MODE != kGemvPartials) {
    const RegPlan rp = gemv_reg_plan(a, mt, d);
    if (rp.parts > 0) {
      constexpr bool fused = MODE == kGemvFused;
      if (a.weights_after_wait)
        return mt == 1 ? launch_gemv_reg_t<1, FMT, fused, true>(a, rp, d, stream)
                       : launch_gemv_reg_t<2, FMT, fused, true>(a, rp, d, stream);
      return mt == 1 ? launch_gemv_reg_t<1, FMT, fused, false>(a, rp, d, stream)
                     : launch_gemv_reg_t<2, FMT, fused, false>(a, rp, d, stream);
    }
  }
  const GemvPlan p = gemv_choose(mt, FMT, static_cast<int>(a.k), d);
  if (p.rt == 0) return cudaErrorInvalidConfiguration;
  // rows computed together: up to 1, 2 or 4 by token count, never past a tile
  const int pref = mt <= 2 ? 2 : 4;
  const int rg = std::min(pref, p.rt) >= 4 ? 4 : (std::min(pref, p.rt) >= 2 ? 2 : 1);
  switch (mt) {
    case 1:
      return rg == 1 ? launch_gemv_t<1, 1, FMT, MODE>(a, p, d, stream)
                     : launch_gemv_t<1, 2, FMT, MODE>(a, p, d, stream);
    case 2:
      return rg == 1 ? launch_gemv_t<2, 1, FMT, MODE>(a, p, d, stream)
                     : launch_gemv_t<2, 2, FMT, MODE>(a, p, d, stream);
    case 4:
      return rg == 1   ? launch_gemv_t<4, 1, FMT, MODE>(a, p, d, stream)
             : rg == 2 ? launch_gemv_t<4, 2, FMT, MODE>(a, p, d, stream)
                       : launch_gemv_t<4, 4, FMT, MODE>(a, p, d, stream);
    default:
      return rg == 1   ? launch_gemv_t<8, 1, FMT, MODE>(a, p, d, stream)
             : rg == 2 ? launch_gemv_t<8, 2, FMT, MODE>(a, p, d, stream)
                       : launch_gemv_t<8, 4, FMT, MODE>(a, p, d, stream);
  }
}

int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// Largest token tile (1, 2, 4 or 8) whose activation codes leave room for a
// two-stage ring.
int gemv_max_mt(int64_t k, const DeviceInfo& d) {
  if (k > (int64_t(1) << 24)) return 0;
  for (int mt = 8; mt >= 1; mt >>= 1)
    if (gemv_choose(mt, 0, static_cast<int>(k), d).rt && gemv_choose(mt, 1, static_cast<int>(k), d).rt) return mt;
  return 0;
}

}  // namespace

template <int J>
cudaError_t launch_act_cluster_t(const uint16_t* x, int64_t m, int k, int parts, int slots_per_part, int threads,
                                 int rotate, int8_t* xq, float* xs, cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(parts), static_cast<unsigned>(m));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(parts);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, act_quant_cluster_kernel<J>, x, k, slots_per_part, rotate, xq, xs);
}

cudaError_t launch_act_quant(const uint16_t* x, int64_t m, int64_t k, int rotate, int8_t* xq, float* xs,
                             cudaStream_t stream) {
  if (m == 0) return cudaSuccess;
  const int slots = static_cast<int>(k / kActSlot);
  const unsigned grid = static_cast<unsigned>(m);
  DeviceInfo d;
  cudaError_t e = device_info(&d);
  if (e != cudaSuccess) return e;
  // fewer tokens than SMs: spread each row over a cluster of up to 8 CTAs
  const int64_t chunks = k / kRot;
  const int parts = static_cast<int>(std::min<int64_t>({8, chunks, (d.num_sms + m - 1) / m}));
  if (parts > 1 && m <= 65535) {
    const int spp = static_cast<int>((chunks + parts - 1) / parts) * (kRot / kActSlot);
    const int threads = std::min(1024, (spp + 31) / 32 * 32);
    const int j = (spp + threads - 1) / threads;
    const int kk = static_cast<int>(k);
    // every part must own at least one chunk: parts * spp covers the row
    // and (parts - 1) * spp < slots
    if (j <= 3 && static_cast<int64_t>(parts - 1) * spp < slots) {
      switch (j) {
        case 1: e = launch_act_cluster_t<1>(x, m, kk, parts, spp, threads, rotate, xq, xs, stream); break;
        case 2: e = launch_act_cluster_t<2>(x, m, kk, parts, spp, threads, rotate, xq, xs, stream); break;
        default: e = launch_act_cluster_t<3>(x, m, kk, parts, spp, threads, rotate, xq, xs, stream); break;
      }
      return e;
    }
  }
  if (k <= kActRegMaxK) {
    // J slots a thread, the CTA a multiple of 32 threads (at most
    // kActRegMaxThreads): the choice with the fewest idle slots, which still
    // run the butterflies and shuffles (K = 5120: 2 x 160, not 3 x 128)
    int j = 0, threads = 0;
    int64_t idle = -1;
    for (int jj = 1; jj <= 8; ++jj) {
      const int t = ((slots + jj - 1) / jj + 31) / 32 * 32;
      const int64_t w = static_cast<int64_t>(jj) * t - slots;
      if (t <= kActRegMaxThreads && (idle < 0 || w < idle)) {
        j = jj;
        threads = t;
        idle = w;
      }
    }
    const int kk = static_cast<int>(k);
    switch (j) {
      case 1: act_quant_reg_kernel<1><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
      case 2: act_quant_reg_kernel<2><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
      case 3: act_quant_reg_kernel<3><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
      case 4: act_quant_reg_kernel<4><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
      case 5: act_quant_reg_kernel<5><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
      case 6: act_quant_reg_kernel<6><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
      case 7: act_quant_reg_kernel<7><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
      default: act_quant_reg_kernel<8><<<grid, threads, 0, stream>>>(x, kk, rotate, xq, xs); break;
    }
  } else {
    act_quant_2pass_kernel<<<grid, kActTwoPassThreads, 0, stream>>>(x, static_cast<int>(k), rotate, xq, xs);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemv(const LinearArgs& a, cudaStream_t stream) {
  if (a.m == 0 || a.n == 0) return cudaSuccess;
  DeviceInfo d;
  cudaError_t e = device_info(&d);
  if (e != cudaSuccess) return e;
  const int step = gemv_max_mt(a.k, d);
  if (step == 0) return cudaErrorInvalidConfiguration;
  const int64_t ng = a.k / (a.fmt == 0 ? kGroupTrunk : kGroupHead);
  for (int64_t m0 = 0; m0 < a.m; m0 += step) {
    const int mg = static_cast<int>(std::min<int64_t>(step, a.m - m0));
    LinearArgs s = a;
    s.m = mg;
    s.xq = a.xq + m0 * a.k;
    if (a.xs) s.xs = a.xs + m0;
    if (a.y) s.y = a.y + m0 * a.n;
    if (a.x) s.x = a.x + m0 * a.k;
    if (a.xq_out) s.xq_out = a.xq_out + m0 * a.k;
    if (a.xs_out) s.xs_out = a.xs_out + m0;
    if (a.partials) s.partials = a.partials + m0 * a.n * ng;
    const int mt = next_pow2(mg);
    const bool part = a.partials != nullptr;
    const int mode = part ? kGemvPartials : (a.x ? kGemvFused : kGemvY);
    if (a.fmt == 0)
      e = mode == kGemvPartials ? launch_gemv_mt<0, kGemvPartials>(s, mt, d, stream)
          : mode == kGemvFused  ? launch_gemv_mt<0, kGemvFused>(s, mt, d, stream)
                                : launch_gemv_mt<0, kGemvY>(s, mt, d, stream);
    else
      e = mode == kGemvPartials ? launch_gemv_mt<1, kGemvPartials>(s, mt, d, stream)
          : mode == kGemvFused  ? launch_gemv_mt<1, kGemvFused>(s, mt, d, stream)
                                : launch_gemv_mt<1, kGemvY>(s, mt, d, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

bool gemv_supported(int64_t k, std::string* why) {
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) {
    if (why) *why = "cannot query the current device";
    return false;
  }
  if (gemv_max_mt(k, d) == 0) {
    if (why) *why = "K too large for the GEMV's shared-memory activation buffer";
    return false;
  }
  return true;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
std::atomic<int> g_encode_ready{0};

// cuTensorMapEncodeTiled from the driver the runtime is using (no link to
// libcuda needed).
cudaError_t get_encode_tiled(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  if (g_encode_ready.load(std::memory_order_acquire) == 0) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || p == nullptr) return cudaErrorNotSupported;
    g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    g_encode_ready.store(1, std::memory_order_release);
  }
  *fn = g_encode_tiled;
  return cudaSuccess;
}

// Row-major int8 [rows][k] as 2-D TMA tiles of [box_rows][128 bytes], 128-byte
// swizzle, out-of-range rows read as zeros.
cudaError_t make_tmap_i8(CUtensorMap* map, const void* base, int64_t rows, int64_t k, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  cudaError_t e = get_encode_tiled(&encode);
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcStageK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Split-K workspace: the fp32 partial tiles of the units, in an array of the
// library's device image (made when the module is loaded on a device, kept
// for the process), so no call allocates. Its address is looked up once per
// device.
constexpr size_t kTcWsBytes = size_t(16) << 20;
static __device__ __align__(256) float g_tc_ws_array[kTcWsBytes / sizeof(float)];
float* g_tc_ws[kMaxDevices];
std::atomic<int> g_tc_ws_ready[kMaxDevices];

cudaError_t tc_workspace(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (g_tc_ws_ready[dev].load(std::memory_order_acquire) == 0) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_tc_ws_array);
    if (e != cudaSuccess) return e;
    g_tc_ws[dev] = static_cast<float*>(ptr);
    g_tc_ws_ready[dev].store(1, std::memory_order_release);
  }
  *out = g_tc_ws[dev];
  return cudaSuccess;
}

// Fixed scratch of the no-allocation entry point: split-K partial tiles in a
// static device array (part of the module image, so nothing is allocated at
// call time). Its address is looked up once per device.
constexpr size_t kNoAllocWsBytes = size_t(8) << 20;
static __device__ __align__(256) float g_noalloc_ws[kNoAllocWsBytes / sizeof(float)];
float* g_noalloc_ptr[kMaxDevices];
std::atomic<int> g_noalloc_ready[kMaxDevices];

cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (g_noalloc_ready[dev].load(std::memory_order_acquire) == 0) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_ws);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<float*>(ptr);
    g_noalloc_ready[dev].store(1, std::memory_order_release);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

// Cost, in scale blocks, of the busiest CTA when `units` units of a tile
// split S ways are dealt round-robin to min(sms, units) persistent CTAs;
// a split unit also pays about half a block for its partial tile.
double tc_split_cost(int64_t tiles, int ng, int S, int sms) {
  const int64_t units = tiles * S;
  const int64_t grid = std::min<int64_t>(sms, units);
  double worst = 0.0;
  for (int64_t c = 0; c < grid; ++c) {
    double t = 0.0;
    for (int64_t u = c; u < units; u += grid) {
      const int64_t sp = u % S;
      t += static_cast<double>((sp + 1) * ng / S - sp * ng / S) + 0.25 + (S > 1 ? 0.5 : 0.0);
    }
    worst = std::max(worst, t);
  }
  return worst;
}

// A launch that may begin while the stream's previous kernel drains (the
// kernel waits for it before reading that kernel's outputs).
cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int FMT, bool PARTIALS, int BMAX>
cudaError_t launch_tc_t(const CUtensorMap& tw, const CUtensorMap& tx, const TcParams& p, int grid,
                        cudaStream_t stream) {
  auto kernel = gemm_tc_kernel<FMT, PARTIALS, BMAX>;
  constexpr int smem = tc_smem_bytes(BMAX);
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = ensure_smem(kernel, smem, configured);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(grid), dim3(kTcThreads), smem, stream, attr);
  e = cudaLaunchKernelEx(&cfg, kernel, tw, tx, p);
  if (e != cudaSuccess || p.splits <= 1) return e;
  const int64_t threads = p.tiles * kTcBN * (p.bm / 4);
  cudaLaunchConfig_t rcfg = pdl_config(dim3(static_cast<unsigned>((threads + kTcReduceThreads - 1) / kTcReduceThreads)),
                                       dim3(kTcReduceThreads), 0, stream, attr);
  return cudaLaunchKernelEx(&rcfg, tc_split_reduce_kernel<FMT>, p);
}

}  // namespace

bool gemm_tc_supported(const LinearArgs& a, std::string* why) {
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) {
    if (why) *why = "cannot query the current device";
    return false;
  }
  if (d.smem_optin < kTcSmemBytes + 1024) {
    if (why) *why = "not enough shared memory per block for the tensor-core kernel";
    return false;
  }
  if (a.k % kTcStageK) {
    if (why) *why = "K must be a multiple of 128";
    return false;
  }
  return true;
}

cudaError_t launch_gemm_tc(const LinearArgs& a, cudaStream_t stream, bool fixed_scratch, bool* too_big) {
  if (too_big) *too_big = false;
  if (a.m == 0 || a.n == 0) return cudaSuccess;
  DeviceInfo d;
  cudaError_t e = device_info(&d);
  if (e != cudaSuccess) return e;
  TcParams p{};
  p.m = a.m;
  p.n = a.n;
  p.k = static_cast<int>(a.k);
  // tokens per tile: each of the kTcGroups column groups needs a multiple of 16
  constexpr int64_t kBmStep = 16 * kTcGroups;
  p.bm = a.m >= kTcMaxBM ? kTcMaxBM : static_cast<int>((a.m + kBmStep - 1) / kBmStep * kBmStep);
  p.fmt = a.fmt;
  p.rotated = a.rotated;
  p.tiles_m = (a.m + p.bm - 1) / p.bm;
  p.tiles = p.tiles_m * ((a.n + kTcBN - 1) / kTcBN);
  p.stage_bytes = kTcStageA + p.bm * kTcStageK;
  const int bmax = p.bm <= 32 ? 32 : (p.bm <= 64 ? 64 : (p.bm <= kTcSplitMaxBM ? kTcSplitMaxBM : kTcMaxBM));
  const int slots = d.num_sms * tc_ctas_per_sm(bmax);
  p.stages = std::min(kTcMaxStages, tc_ring_bytes(bmax) / p.stage_bytes);
  p.stream_w = p.tiles_m == 1 ? 1 : 0;
  // split K when there are too few tiles to fill the SMs
  const int ng = static_cast<int>(a.k / (a.fmt == 0 ? kGroupTrunk : kGroupHead));
  p.splits = 1;
  if (p.bm <= kTcSplitMaxBM && a.partials == nullptr) {
    double best = tc_split_cost(p.tiles, ng, 1, slots);
    for (int S = 2; S <= std::min(ng, 32); ++S) {
      if (static_cast<size_t>(p.tiles) * S * p.bm * kTcBN * sizeof(float) > kTcWsBytes) break;
      const double c = tc_split_cost(p.tiles, ng, S, slots);
      if (c < 0.95 * best) {
        best = c;
        p.splits = S;
      }
    }
  }
  p.units = p.tiles * p.splits;
  if (p.splits > 1) {
    if (fixed_scratch) {
      // the same plan as the allocating path; refuse it if the fixed array
      // cannot hold its partial tiles (nothing is launched)
      const size_t need = static_cast<size_t>(p.units) * kTcBN * p.bm * sizeof(float);
      if (need > kNoAllocWsBytes) {
        if (too_big) *too_big = true;
        return cudaSuccess;
      }
      e = noalloc_scratch(&p.ws);
    } else {
      e = tc_workspace(&p.ws);
    }
    if (e != cudaSuccess) return e;
  }
  p.xs = a.xs;
  p.sub = a.sub;
  p.scale = a.scale;
  p.y = a.y;
  p.partials = a.partials;
  p.weights_after_wait = a.weights_after_wait;
  // accumulators: the 512 TMEM columns shared by the CTAs resident on an SM
  p.nacc = std::max(2, std::min(kTcMaxAcc, 512 / (p.bm * tc_ctas_per_sm(bmax))));
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(p.nacc * p.bm)) cols <<= 1;
  p.tmem_cols = cols;
  CUtensorMap tw, tx;
  e = make_tmap_i8(&tw, a.codes, a.n, a.k, kTcBN);
  if (e != cudaSuccess) return e;
  e = make_tmap_i8(&tx, a.xq, a.m, a.k, p.bm);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(std::min<int64_t>(slots, p.units));
  const bool part = a.partials != nullptr;
  if (p.bm <= 32) {
    if (a.fmt == 0)
      return part ? launch_tc_t<0, true, 32>(tw, tx, p, grid, stream)
                  : launch_tc_t<0, false, 32>(tw, tx, p, grid, stream);
    return part ? launch_tc_t<1, true, 32>(tw, tx, p, grid, stream)
                : launch_tc_t<1, false, 32>(tw, tx, p, grid, stream);
  }
  if (p.bm <= 64) {
    if (a.fmt == 0)
      return part ? launch_tc_t<0, true, 64>(tw, tx, p, grid, stream)
                  : launch_tc_t<0, false, 64>(tw, tx, p, grid, stream);
    return part ? launch_tc_t<1, true, 64>(tw, tx, p, grid, stream)
                : launch_tc_t<1, false, 64>(tw, tx, p, grid, stream);
  }
  if (p.bm <= kTcSplitMaxBM) {
    if (a.fmt == 0)
      return part ? launch_tc_t<0, true, kTcSplitMaxBM>(tw, tx, p, grid, stream)
                  : launch_tc_t<0, false, kTcSplitMaxBM>(tw, tx, p, grid, stream);
    return part ? launch_tc_t<1, true, kTcSplitMaxBM>(tw, tx, p, grid, stream)
                : launch_tc_t<1, false, kTcSplitMaxBM>(tw, tx, p, grid, stream);
  }
  if (a.fmt == 0)
    return part ? launch_tc_t<0, true, kTcMaxBM>(tw, tx, p, grid, stream)
                : launch_tc_t<0, false, kTcMaxBM>(tw, tx, p, grid, stream);
  return part ? launch_tc_t<1, true, kTcMaxBM>(tw, tx, p, grid, stream)
              : launch_tc_t<1, false, kTcMaxBM>(tw, tx, p, grid, stream);
}

// The mma.sync codebook kernel stages 16 tokens of codes (and its
// reduction buffer) in shared memory.
bool cb4_mma_fits(int64_t k, const DeviceInfo& d) {
  return 16 * (k + 16) + 4 * 32 * 4 * 2 * 4 <= d.smem_optin - kSmemReserve;
}

template <int MT, bool PARTIALS, int STEPS, bool EXACT>
cudaError_t launch_cb4_s(const LinearArgs& a, const DeviceInfo& d, cudaStream_t stream) {
  auto kernel = cb4_gemv_kernel<MT, PARTIALS, STEPS, EXACT>;
  const int smem = MT * static_cast<int>(a.k);
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = ensure_smem(kernel, smem, configured);
  if (e != cudaSuccess) return e;
  const int64_t rows_per_cta = kCb4Warps;
  const int grid = static_cast<int>(std::min<int64_t>(d.num_sms, (a.n + rows_per_cta - 1) / rows_per_cta));
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(grid), dim3(kCb4Warps * 32), static_cast<size_t>(smem), stream, attr);
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

// Row chunk of 4, 5 or 8 steps of 512 index bytes (K up to 4096, 5120 or
// longer), the exact instance when K / 2 is a multiple of the chunk; the
// partial sums (tests) use the general 8-step instance only.
template <int MT, bool PARTIALS, int STEPS>
cudaError_t launch_cb4_e(const LinearArgs& a, const DeviceInfo& d, cudaStream_t stream) {
  if ((a.k / 2) % (STEPS * 512) == 0) return launch_cb4_s<MT, PARTIALS, STEPS, true>(a, d, stream);
  return launch_cb4_s<MT, PARTIALS, STEPS, false>(a, d, stream);
}

template <int MT, bool PARTIALS>
cudaError_t launch_cb4_t(const LinearArgs& a, const DeviceInfo& d, cudaStream_t stream) {
  const int64_t steps = (a.k / 2 + 511) / 512;
  if constexpr (PARTIALS) {
    return launch_cb4_s<MT, PARTIALS, 8, false>(a, d, stream);
  } else {
    if (steps > 5) return launch_cb4_e<MT, PARTIALS, 8>(a, d, stream);
    if (steps == 5) return launch_cb4_e<MT, PARTIALS, 5>(a, d, stream);
    return launch_cb4_e<MT, PARTIALS, 4>(a, d, stream);
  }
}

template <int NT>
cudaError_t launch_cb4_mma_t(const LinearArgs& a, const DeviceInfo& d, cudaStream_t stream) {
  auto kernel = cb4_mma_kernel<NT>;
  const int smem = 8 * NT * (static_cast<int>(a.k) + 16) + 4 * 32 * 4 * NT * 4;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = ensure_smem(kernel, smem, configured);
  if (e != cudaSuccess) return e;
  const int64_t groups = (a.n + 15) / 16;
  const unsigned grid = static_cast<unsigned>((groups + 3) / 4);
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(grid), dim3(kCb4MmaWarps * 32), static_cast<size_t>(smem), stream, attr);
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

// The codebook format. Two or more tokens: mma.sync, 16 tokens a launch
// (their codes staged in shared memory); one token, and the partial sums:
// the dp4a kernel, up to 8 tokens a launch.
cudaError_t launch_cb4(const LinearArgs& a, cudaStream_t stream) {
  if (a.m == 0 || a.n == 0) return cudaSuccess;
  DeviceInfo d;
  cudaError_t e = device_info(&d);
  if (e != cudaSuccess) return e;
  const int64_t ng = a.k / kGroupHead;
  if (a.partials == nullptr && a.m >= 2 && cb4_mma_fits(a.k, d)) {
    for (int64_t m0 = 0; m0 < a.m; m0 += 16) {
      const int mg = static_cast<int>(std::min<int64_t>(16, a.m - m0));
      LinearArgs s = a;
      s.m = mg;
      s.xq = a.xq + m0 * a.k;
      s.xs = a.xs + m0;
      s.y = a.y + m0 * a.n;
      e = mg > 8 ? launch_cb4_mma_t<2>(s, d, stream) : launch_cb4_mma_t<1>(s, d, stream);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  for (int64_t m0 = 0; m0 < a.m; m0 += 8) {
    const int mg = static_cast<int>(std::min<int64_t>(8, a.m - m0));
    LinearArgs s = a;
    s.m = mg;
    s.xq = a.xq + m0 * a.k;
    if (a.xs) s.xs = a.xs + m0;
    if (a.y) s.y = a.y + m0 * a.n;
    if (a.partials) s.partials = a.partials + m0 * a.n * ng;
    const int mt = next_pow2(mg);
    const bool part = a.partials != nullptr;
    switch (mt) {
      case 1: e = part ? launch_cb4_t<1, true>(s, d, stream) : launch_cb4_t<1, false>(s, d, stream); break;
      case 2: e = part ? launch_cb4_t<2, true>(s, d, stream) : launch_cb4_t<2, false>(s, d, stream); break;
      case 4: e = part ? launch_cb4_t<4, true>(s, d, stream) : launch_cb4_t<4, false>(s, d, stream); break;
      default: e = part ? launch_cb4_t<8, true>(s, d, stream) : launch_cb4_t<8, false>(s, d, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

bool cb4_supported(int64_t k, std::string* why) {
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) {
    if (why) *why = "cannot query the current device";
    return false;
  }
  if (8 * k > d.smem_optin - kSmemReserve) {
    if (why) *why = "k too large for the codebook kernel (8 tokens of codes must fit in shared memory)";
    return false;
  }
  return true;
}

cudaError_t launch_rescore(const LinearArgs& a, const int32_t* cand, int kc, uint16_t* out, cudaStream_t stream) {
  if (a.m == 0 || kc == 0) return cudaSuccess;
  RescoreArgs r{};
  r.xq = a.xq;
  r.xs = a.xs;
  r.m = a.m;
  r.codes = a.codes;
  r.sub = a.sub;
  r.scale = a.scale;
  r.n = a.n;
  r.k = static_cast<int>(a.k);
  r.rotated = a.rotated;
  r.cand = cand;
  r.kc = kc;
  r.out = out;
  const dim3 grid(static_cast<unsigned>(a.m), static_cast<unsigned>((kc + kRescoreWarps - 1) / kRescoreWarps));
  const size_t smem = static_cast<size_t>(a.k);
  if (a.fmt == 0) {
    static std::atomic<int> configured[kMaxDevices];
    cudaError_t e = ensure_smem(rescore_kernel<0>, static_cast<int>(smem), configured);
    if (e != cudaSuccess) return e;
    rescore_kernel<0><<<grid, kRescoreWarps * 32, smem, stream>>>(r);
  } else {
    static std::atomic<int> configured[kMaxDevices];
    cudaError_t e = ensure_smem(rescore_kernel<1>, static_cast<int>(smem), configured);
    if (e != cudaSuccess) return e;
    rescore_kernel<1><<<grid, kRescoreWarps * 32, smem, stream>>>(r);
  }
  return cudaGetLastError();
}

namespace {

// One thread waits on a barrier that nothing will ever arrive on; the
// bounded wait must give up after limit_ns and record the self-test code.
__global__ void wait_selftest_kernel(uint64_t limit_cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait(&bar, 0u, kDevErrSelftest, limit_cycles);
  }
}

}  // namespace

cudaError_t launch_mapped_copy(const uint16_t* src, uint16_t* dst, int64_t n, bool host_to_device,
                               cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  DeviceInfo d;
  cudaError_t e = device_info(&d);
  if (e != cudaSuccess) return e;
  // enough CTAs that an input copy is read ahead of the wait in one piece
  // per thread-slot (at most kMapCopyAhead x 16 bytes a thread), at most one an SM
  const int64_t per_cta = static_cast<int64_t>(kMapCopyThreads) * kMapCopyAhead * 8;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(d.num_sms, (n + per_cta - 1) / per_cta));
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(static_cast<unsigned>(grid)), dim3(kMapCopyThreads), 0, stream, attr);
  return host_to_device ? cudaLaunchKernelEx(&cfg, mapped_copy_kernel<true>, src, dst, n)
                        : cudaLaunchKernelEx(&cfg, mapped_copy_kernel<false>, src, dst, n);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream) {
  // cycles at no more than 2 GHz: the wait lasts at most about limit_ns
  wait_selftest_kernel<<<1, 32, 0, stream>>>(2 * limit_ns);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(uint32_t* err) {
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *err = v;
  return cudaSuccess;
}

}  // namespace iq8r
