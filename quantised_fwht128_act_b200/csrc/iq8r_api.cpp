// The C ABI of libiq8r: argument checks, dispatch and error reporting.
// Every entry point validates before touching the GPU, so a bad call
// returns IQ8R_ERR_INVALID_ARG and launches nothing.

#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/iq8r.h"
#include "iq8r_internal.h"

namespace {

thread_local std::string t_last_error;

iq8r_status fail(iq8r_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

iq8r_status ok() {
  t_last_error.clear();
  return IQ8R_OK;
}

iq8r_status cuda_fail(cudaError_t e, const char* where) {
  return fail(IQ8R_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxK = int64_t(1) << 30;
constexpr int64_t kMaxGridRows = (int64_t(1) << 31) - 1;
// iq8r_linear_bf16 fuses the activation quantiser into the GEMV up to this
// many activation elements (M * K); beyond it two launches are cheaper.
constexpr int64_t kFuseMaxElems = 16384;
// Above this many tokens the automatic choice is the tensor-core GEMM.
constexpr int64_t kGemvMaxM = 2;

iq8r_status check_weight(const iq8r_weight* w, const char* fn) {
  if (!w) return fail(IQ8R_ERR_INVALID_ARG, "%s: weight is NULL", fn);
  if (w->fmt != IQ8R_FMT_G256_U8_BF16 && w->fmt != IQ8R_FMT_G128_BF16 && w->fmt != IQ8R_FMT_CB4_G128)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: unknown weight format %d", fn, w->fmt);
  if (w->rotated != 0 && w->rotated != 1)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: rotated must be 0 or 1", fn);
  const int64_t g = w->fmt == IQ8R_FMT_G256_U8_BF16 ? iq8r::kGroupTrunk : iq8r::kGroupHead;
  if (w->n <= 0 || w->k <= 0) return fail(IQ8R_ERR_INVALID_ARG, "%s: n and k must be positive", fn);
  if (w->k % g) return fail(IQ8R_ERR_INVALID_ARG, "%s: k = %lld is not a multiple of %lld", fn, (long long)w->k, (long long)g);
  if (w->k > kMaxK) return fail(IQ8R_ERR_INVALID_ARG, "%s: k = %lld exceeds 2^30", fn, (long long)w->k);
  if (!w->codes || !w->scale) return fail(IQ8R_ERR_INVALID_ARG, "%s: weight codes or scale is NULL", fn);
  if (w->fmt == IQ8R_FMT_G256_U8_BF16 && !w->sub_scale)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: the trunk format needs sub_scale", fn);
  if (!aligned16(w->codes) || !aligned16(w->scale) || (w->sub_scale && !aligned16(w->sub_scale)))
    return fail(IQ8R_ERR_INVALID_ARG, "%s: weight codes, sub_scale and scale must be 16-byte aligned", fn);
  return IQ8R_OK;
}

iq8r::LinearArgs make_args(const int8_t* xq, const float* xs, int64_t m, const iq8r_weight* w) {
  iq8r::LinearArgs a{};
  a.xq = xq;
  a.xs = xs;
  a.m = m;
  a.fmt = w->fmt;
  a.rotated = w->rotated;
  a.n = w->n;
  a.k = w->k;
  a.codes = w->codes;
  a.sub = w->sub_scale;
  a.scale = w->scale;
  return a;
}

// Choose and launch a kernel for y or partials. fixed_scratch: the
// no-allocation variant (split-K scratch from the static array).
iq8r_status run_linear(const iq8r::LinearArgs& args, int32_t path_and_flags, const char* fn, cudaStream_t stream,
                       bool fixed_scratch = false) {
  const int32_t path = path_and_flags & ~IQ8R_PATH_FLAG_WEIGHTS_WRITTEN;
  if (path != IQ8R_PATH_AUTO && path != IQ8R_PATH_GEMV && path != IQ8R_PATH_TC)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: unknown path %d", fn, path_and_flags);
  iq8r::LinearArgs a = args;
  a.weights_after_wait = (path_and_flags & IQ8R_PATH_FLAG_WEIGHTS_WRITTEN) ? 1 : 0;
  if (a.m == 0) return ok();
  std::string why;
  if (a.fmt == IQ8R_FMT_CB4_G128) {
    // the codebook format has one kernel, the weight-streaming GEMV
    if (path == IQ8R_PATH_TC) return fail(IQ8R_ERR_UNSUPPORTED, "%s: the codebook format runs on the GEMV only", fn);
    if (!iq8r::cb4_supported(a.k, &why)) return fail(IQ8R_ERR_UNSUPPORTED, "%s: %s", fn, why.c_str());
    const cudaError_t e = iq8r::launch_cb4(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return ok();
  }
  bool use_tc = false;
  if (path == IQ8R_PATH_TC) {
    if (!iq8r::gemm_tc_supported(a, &why)) return fail(IQ8R_ERR_UNSUPPORTED, "%s: %s", fn, why.c_str());
    use_tc = true;
  } else if (path == IQ8R_PATH_AUTO) {
    use_tc = a.m > kGemvMaxM && iq8r::gemm_tc_supported(a, nullptr);
  }
  if (!use_tc && !iq8r::gemv_supported(a.k, &why)) {
    if (path == IQ8R_PATH_AUTO && iq8r::gemm_tc_supported(a, nullptr))
      use_tc = true;
    else
      return fail(IQ8R_ERR_UNSUPPORTED, "%s: %s", fn, why.c_str());
  }
  bool too_big = false;
  const cudaError_t e = use_tc ? iq8r::launch_gemm_tc(a, stream, fixed_scratch, &too_big) : iq8r::launch_gemv(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  if (too_big)
    return fail(IQ8R_ERR_UNSUPPORTED, "%s: the split-K plan needs more scratch than the fixed array holds", fn);
  return ok();
}

// y for iq8r_linear / iq8r_linear_ex / iq8r_linear_noalloc.
iq8r_status linear_y(const char* fn, const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w,
                     uint16_t* y_bf16, int32_t path, cudaStream_t stream, bool fixed_scratch) {
  iq8r_status st = check_weight(w, fn);
  if (st != IQ8R_OK) return st;
  if (m < 0 || m > kMaxGridRows) return fail(IQ8R_ERR_INVALID_ARG, "%s: m = %lld out of range", fn, (long long)m);
  if (m == 0) return ok();
  if (!xq || !x_scale || !y_bf16) return fail(IQ8R_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if (!aligned16(xq) || !aligned16(y_bf16)) return fail(IQ8R_ERR_INVALID_ARG, "%s: xq and y must be 16-byte aligned", fn);
  iq8r::LinearArgs a = make_args(xq, x_scale, m, w);
  a.y = y_bf16;
  return run_linear(a, path, fn, stream, fixed_scratch);
}

}  // namespace

extern "C" {

int32_t iq8r_version(void) { return 100; }

const char* iq8r_last_error(void) { return t_last_error.c_str(); }

iq8r_status iq8r_packed_sizes(int32_t fmt, int64_t n, int64_t k, size_t* codes_bytes, size_t* sub_bytes,
                              size_t* scale_bytes) {
  if (fmt != IQ8R_FMT_G256_U8_BF16 && fmt != IQ8R_FMT_G128_BF16 && fmt != IQ8R_FMT_CB4_G128)
    return fail(IQ8R_ERR_INVALID_ARG, "iq8r_packed_sizes: unknown format %d", fmt);
  const int64_t g = fmt == IQ8R_FMT_G256_U8_BF16 ? iq8r::kGroupTrunk : iq8r::kGroupHead;
  if (n < 0 || k < 0 || k % g)
    return fail(IQ8R_ERR_INVALID_ARG, "iq8r_packed_sizes: need n >= 0 and k a non-negative multiple of %lld",
                (long long)g);
  if (codes_bytes)
    *codes_bytes = static_cast<size_t>(n) * static_cast<size_t>(fmt == IQ8R_FMT_CB4_G128 ? k / 2 : k);
  if (fmt == IQ8R_FMT_G256_U8_BF16) {
    if (sub_bytes) *sub_bytes = static_cast<size_t>(n) * static_cast<size_t>(k / iq8r::kGroupTrunk);
    if (scale_bytes) *scale_bytes = 2 * static_cast<size_t>(n);
  } else {
    if (sub_bytes) *sub_bytes = 0;
    if (scale_bytes) *scale_bytes = 2 * static_cast<size_t>(n) * static_cast<size_t>(k / iq8r::kGroupHead);
  }
  return ok();
}

iq8r_status iq8r_pack(int32_t fmt, int32_t rotate, const uint16_t* w_bf16, int64_t n, int64_t k, int8_t* codes,
                      uint8_t* sub_scale, uint16_t* scale, int32_t n_threads) {
  return iq8r_pack_ex(fmt, rotate, IQ8R_RULE_RTN, w_bf16, n, k, codes, sub_scale, scale, n_threads);
}

iq8r_status iq8r_pack_ex(int32_t fmt, int32_t rotate, int32_t rule, const uint16_t* w_bf16, int64_t n, int64_t k,
                         int8_t* codes, uint8_t* sub_scale, uint16_t* scale, int32_t n_threads) {
  const char* fn = "iq8r_pack";
  if (rule != IQ8R_RULE_RTN && rule != IQ8R_RULE_SEARCH)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: unknown rule %d", fn, rule);
  if (fmt != IQ8R_FMT_G256_U8_BF16 && fmt != IQ8R_FMT_G128_BF16 && fmt != IQ8R_FMT_CB4_G128)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: unknown format %d", fn, fmt);
  if (rotate != 0 && rotate != 1) return fail(IQ8R_ERR_INVALID_ARG, "%s: rotate must be 0 or 1", fn);
  const int64_t g = fmt == IQ8R_FMT_G256_U8_BF16 ? iq8r::kGroupTrunk : iq8r::kGroupHead;
  if (n < 0 || k <= 0 || k % g)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: need n >= 0 and k a positive multiple of %lld", fn, (long long)g);
  if (n == 0) return ok();
  if (!w_bf16 || !codes || !scale) return fail(IQ8R_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if (fmt == IQ8R_FMT_G256_U8_BF16 && !sub_scale)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: the trunk format needs sub_scale", fn);
  iq8r::pack_rows(fmt, rotate != 0, rule, w_bf16, n, k, codes, fmt == IQ8R_FMT_G256_U8_BF16 ? sub_scale : nullptr,
                  scale, n_threads);
  return ok();
}

iq8r_status iq8r_rotate_quant_act(const uint16_t* x_bf16, int64_t m, int64_t k, int32_t rotate, int8_t* xq,
                                  float* x_scale, cudaStream_t stream) {
  const char* fn = "iq8r_rotate_quant_act";
  if (rotate != 0 && rotate != 1) return fail(IQ8R_ERR_INVALID_ARG, "%s: rotate must be 0 or 1", fn);
  if (m < 0 || m > kMaxGridRows) return fail(IQ8R_ERR_INVALID_ARG, "%s: m = %lld out of range", fn, (long long)m);
  if (k <= 0 || k % iq8r::kRot || k > kMaxK)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: k = %lld must be a positive multiple of 128 up to 2^30", fn, (long long)k);
  if (m == 0) return ok();
  if (!x_bf16 || !xq || !x_scale) return fail(IQ8R_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if (!aligned16(x_bf16) || !aligned16(xq)) return fail(IQ8R_ERR_INVALID_ARG, "%s: x and xq must be 16-byte aligned", fn);
  const cudaError_t e = iq8r::launch_act_quant(x_bf16, m, k, rotate, xq, x_scale, stream);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

iq8r_status iq8r_linear_ex(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w, uint16_t* y_bf16,
                           int32_t path, cudaStream_t stream) {
  return linear_y("iq8r_linear", xq, x_scale, m, w, y_bf16, path, stream, false);
}

iq8r_status iq8r_linear_noalloc(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w,
                                uint16_t* y_bf16, cudaStream_t stream) {
  return linear_y("iq8r_linear_noalloc", xq, x_scale, m, w, y_bf16, IQ8R_PATH_AUTO, stream, true);
}

iq8r_status iq8r_linear_bf16(const uint16_t* x_bf16, int64_t m, const iq8r_weight* w, uint16_t* y_bf16,
                             int8_t* xq_out, float* x_scale_out, cudaStream_t stream) {
  const char* fn = "iq8r_linear_bf16";
  iq8r_status st = check_weight(w, fn);
  if (st != IQ8R_OK) return st;
  if (m < 0 || m > kMaxGridRows) return fail(IQ8R_ERR_INVALID_ARG, "%s: m = %lld out of range", fn, (long long)m);
  if (w->k % iq8r::kRot) return fail(IQ8R_ERR_INVALID_ARG, "%s: k must be a multiple of 128", fn);
  if (m == 0) return ok();
  if (!x_bf16 || !y_bf16) return fail(IQ8R_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if (!aligned16(x_bf16) || !aligned16(y_bf16) || (xq_out && !aligned16(xq_out)))
    return fail(IQ8R_ERR_INVALID_ARG, "%s: x, y and xq_out must be 16-byte aligned", fn);
  std::string why;
  // One launch when the activation is small enough that every CTA redoing
  // its rotation is cheap, or when there is nowhere to stage the codes.
  const bool small = m * w->k <= kFuseMaxElems;
  const bool staged = xq_out && x_scale_out;
  if (w->fmt != IQ8R_FMT_CB4_G128 && m <= 8 && (small || m <= kGemvMaxM || !staged) &&
      iq8r::gemv_supported(w->k, &why)) {
    // one launch: every CTA rotates and quantises x itself, then streams W
    iq8r::LinearArgs a = make_args(nullptr, nullptr, m, w);
    a.y = y_bf16;
    a.x = x_bf16;
    a.xq_out = xq_out;
    a.xs_out = x_scale_out;
    const cudaError_t e = iq8r::launch_gemv(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return ok();
  }
  if (!staged)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: this call needs xq_out and x_scale_out (the codes are staged there)", fn);
  cudaError_t e = iq8r::launch_act_quant(x_bf16, m, w->k, w->rotated, xq_out, x_scale_out, stream);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  iq8r::LinearArgs a = make_args(xq_out, x_scale_out, m, w);
  a.y = y_bf16;
  return run_linear(a, IQ8R_PATH_AUTO, fn, stream);
}

// Largest copies the host-buffer entry makes as mapped-copy kernels.
constexpr size_t kMappedInMaxBytes = 64 * 1024;
constexpr size_t kMappedOutMaxBytes = 1024 * 1024;

// The device address of pinned host memory mapped into the current device's
// address space, or nullptr (pageable or device memory, or an unknown
// pointer). The query's own error state is cleared.
static void* mapped_host(const void* p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

iq8r_status iq8r_linear_bf16_host(const uint16_t* x_host, int64_t m, const iq8r_weight* w, uint16_t* x_dev,
                                  uint16_t* y_dev, uint16_t* y_host, int8_t* xq_out, float* x_scale_out,
                                  cudaStream_t stream) {
  const char* fn = "iq8r_linear_bf16_host";
  iq8r_status st = check_weight(w, fn);
  if (st != IQ8R_OK) return st;
  if (m < 0 || m > kMaxGridRows) return fail(IQ8R_ERR_INVALID_ARG, "%s: m = %lld out of range", fn, (long long)m);
  if (w->k % iq8r::kRot) return fail(IQ8R_ERR_INVALID_ARG, "%s: k must be a multiple of 128", fn);
  if (m == 0) return ok();
  if (!x_host || !y_host || !x_dev || !y_dev) return fail(IQ8R_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if (!aligned16(x_dev) || !aligned16(y_dev) || (xq_out && !aligned16(xq_out)))
    return fail(IQ8R_ERR_INVALID_ARG, "%s: x_dev, y_dev and xq_out must be 16-byte aligned", fn);
  const size_t xb = static_cast<size_t>(m) * static_cast<size_t>(w->k) * 2;
  const size_t yb = static_cast<size_t>(m) * static_cast<size_t>(w->n) * 2;
  // Small copies between pinned host buffers that the device can address
  // run as kernels chained with the layer (see mapped_copy.cuh): there a
  // step's cost is latency, which the chaining hides. Large inputs, or
  // anything else (pageable memory, an unaligned view): copy calls. (On
  // B200 a 557 KB input read through the mapping ran at about 5 GB/s, where
  // the copy engines stream it; reads of host memory by the device are
  // round trips, writes are not.)
  const bool small = xb <= kMappedInMaxBytes && yb <= kMappedOutMaxBytes;
  const uint16_t* xm = small ? static_cast<const uint16_t*>(mapped_host(x_host)) : nullptr;
  uint16_t* ym = small ? static_cast<uint16_t*>(mapped_host(y_host)) : nullptr;
  if (xm && ym && aligned16(xm) && aligned16(ym)) {
    cudaError_t e = iq8r::launch_mapped_copy(xm, x_dev, m * w->k, true, stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    st = iq8r_linear_bf16(x_dev, m, w, y_dev, xq_out, x_scale_out, stream);
    if (st != IQ8R_OK) return st;
    e = iq8r::launch_mapped_copy(y_dev, ym, m * w->n, false, stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return ok();
  }
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  st = iq8r_linear_bf16(x_dev, m, w, y_dev, xq_out, x_scale_out, stream);
  if (st != IQ8R_OK) return st;
  e = cudaMemcpyAsync(y_host, y_dev, yb, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

iq8r_status iq8r_linear(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w, uint16_t* y_bf16,
                        cudaStream_t stream) {
  return iq8r_linear_ex(xq, x_scale, m, w, y_bf16, IQ8R_PATH_AUTO, stream);
}

iq8r_status iq8r_linear_partials(const int8_t* xq, int64_t m, const iq8r_weight* w, int64_t n0, int64_t n1,
                                 int32_t* p, int32_t path, cudaStream_t stream) {
  const char* fn = "iq8r_linear_partials";
  iq8r_status st = check_weight(w, fn);
  if (st != IQ8R_OK) return st;
  if (m < 0 || m > kMaxGridRows) return fail(IQ8R_ERR_INVALID_ARG, "%s: m = %lld out of range", fn, (long long)m);
  if (n0 < 0 || n1 <= n0 || n1 > w->n)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: need 0 <= n0 < n1 <= n (n0=%lld n1=%lld n=%lld)", fn, (long long)n0,
                (long long)n1, (long long)w->n);
  if (m == 0) return ok();
  if (!xq || !p) return fail(IQ8R_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if (!aligned16(xq) || !aligned16(p)) return fail(IQ8R_ERR_INVALID_ARG, "%s: xq and p must be 16-byte aligned", fn);
  iq8r_weight sub = *w;
  sub.n = n1 - n0;
  sub.codes = w->codes + n0 * (w->fmt == IQ8R_FMT_CB4_G128 ? w->k / 2 : w->k);
  // the partials need no scales, but the argument block carries valid ones
  if (w->fmt == IQ8R_FMT_G256_U8_BF16) {
    sub.sub_scale = w->sub_scale + n0 * (w->k / iq8r::kGroupTrunk);
    sub.scale = w->scale + n0;
  } else {
    sub.scale = w->scale + n0 * (w->k / iq8r::kGroupHead);
  }
  if (!aligned16(sub.codes)) return fail(IQ8R_ERR_INVALID_ARG, "%s: codes of row n0 must be 16-byte aligned", fn);
  iq8r::LinearArgs a = make_args(xq, nullptr, m, &sub);
  a.partials = p;
  return run_linear(a, path, fn, stream);
}

iq8r_status iq8r_rescore(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w,
                         const int32_t* cand, int64_t n_cand, uint16_t* out_bf16, cudaStream_t stream) {
  const char* fn = "iq8r_rescore";
  iq8r_status st = check_weight(w, fn);
  if (st != IQ8R_OK) return st;
  if (m < 0 || m > kMaxGridRows) return fail(IQ8R_ERR_INVALID_ARG, "%s: m = %lld out of range", fn, (long long)m);
  if (n_cand < 0 || n_cand > 65535 * 32)
    return fail(IQ8R_ERR_INVALID_ARG, "%s: n_cand = %lld out of range", fn, (long long)n_cand);
  if (w->k > 48 * 1024) return fail(IQ8R_ERR_UNSUPPORTED, "%s: k above 49152 is not supported", fn);
  if (w->fmt == IQ8R_FMT_CB4_G128) return fail(IQ8R_ERR_UNSUPPORTED, "%s: not for the codebook format", fn);
  if (m == 0 || n_cand == 0) return ok();
  if (!xq || !x_scale || !cand || !out_bf16) return fail(IQ8R_ERR_INVALID_ARG, "%s: NULL buffer", fn);
  if (!aligned16(xq)) return fail(IQ8R_ERR_INVALID_ARG, "%s: xq must be 16-byte aligned", fn);
  iq8r::LinearArgs a = make_args(xq, x_scale, m, w);
  const cudaError_t e = iq8r::launch_rescore(a, cand, static_cast<int>(n_cand), out_bf16, stream);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

iq8r_status iq8r_get_device_error(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "iq8r_get_device_error: stream");
  uint32_t code = 0;
  e = iq8r::read_and_clear_device_error(&code);
  if (e != cudaSuccess) return cuda_fail(e, "iq8r_get_device_error: read");
  if (code == 0) return ok();
  const char* what = "unknown wait";
  switch (code) {
    case iq8r::kDevErrGemvFull: what = "GEMV consumer waiting for a weight stage"; break;
    case iq8r::kDevErrGemvEmpty: what = "GEMV producer waiting for a free ring slot"; break;
    case iq8r::kDevErrGemvDrain: what = "GEMV producer draining its copies"; break;
    case iq8r::kDevErrTcFull: what = "TC GEMM waiting for an operand stage"; break;
    case iq8r::kDevErrTcEmpty: what = "TC GEMM waiting for a free operand slot"; break;
    case iq8r::kDevErrTcAccFull: what = "TC GEMM epilogue waiting for an accumulator"; break;
    case iq8r::kDevErrTcAccEmpty: what = "TC GEMM MMA waiting for a drained accumulator"; break;
    case iq8r::kDevErrTcDrain: what = "TC GEMM draining its copies"; break;
    case iq8r::kDevErrSelftest: what = "self-test wait (expected)"; break;
    case iq8r::kDevErrRescoreIndex:
      return fail(IQ8R_ERR_INVALID_ARG, "iq8r_rescore: a candidate index was outside [0, n) (its output is 0)");
    default: break;
  }
  return fail(IQ8R_ERR_DEVICE_TIMEOUT, "device wait timed out: %s (code 0x%x)", what, code);
}

iq8r_status iq8r_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream) {
  if (limit_ns < 1000 || limit_ns > 100 * 1000 * 1000)
    return fail(IQ8R_ERR_INVALID_ARG, "iq8r_selftest_wait_timeout: limit_ns must be in [1e3, 1e8]");
  const cudaError_t e = iq8r::launch_wait_selftest(static_cast<uint64_t>(limit_ns), stream);
  if (e != cudaSuccess) return cuda_fail(e, "iq8r_selftest_wait_timeout");
  return ok();
}

}  // extern "C"
