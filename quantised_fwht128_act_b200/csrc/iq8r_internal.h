// Internal interface between the C ABI (iq8r_api.cpp, host C++) and the
// CUDA launchers (iq8r_kernels.cu). Not installed; not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>

#include <cuda_runtime_api.h>

namespace iq8r {

constexpr int kGroupTrunk = 256;  // u8 sub-scale block of the trunk format
constexpr int kGroupHead = 128;   // bf16 scale block of the lm_head format
// The drafter's 16-level codebook: a 4-bit index i stands for kCb4Table[i]
// (the dflash recipe lines of the IQ8R page, "How this file was made").
constexpr int kCb4Table[16] = {-127, -97, -75, -58, -43, -30, -18, -6, 6, 18, 30, 43, 58, 75, 97, 127};
constexpr int kRot = 128;         // fwht128 acts on each 128 of K

// Device error word values (0 = no error). The low byte names the wait.
enum DeviceError : uint32_t {
  kDevErrNone = 0,
  kDevErrGemvFull = 0x101,    // GEMV consumer: weight stage never arrived
  kDevErrGemvEmpty = 0x102,   // GEMV producer: ring slot never released
  kDevErrGemvDrain = 0x103,   // GEMV producer: copy in flight at exit
  kDevErrTcFull = 0x201,      // TC GEMM: operand stage never arrived
  kDevErrTcEmpty = 0x202,     // TC GEMM: operand slot never released
  kDevErrTcAccFull = 0x203,   // TC GEMM: accumulator never committed
  kDevErrTcAccEmpty = 0x204,  // TC GEMM: accumulator never drained
  kDevErrTcDrain = 0x205,     // TC GEMM: copy in flight at exit
  kDevErrSelftest = 0x301,    // self-test wait that nothing satisfies
  kDevErrRescoreIndex = 0x401,  // rescoring: a candidate row index outside [0, n)
};

struct LinearArgs {
  const int8_t* xq;      // [m][k]
  const float* xs;       // [m]
  int64_t m;
  int fmt;               // 0 = G256 trunk, 1 = G128 lm_head
  int rotated;
  int64_t n;
  int64_t k;
  const int8_t* codes;   // [n][k]
  const uint8_t* sub;    // [n][k/256] (G256)
  const uint16_t* scale; // [n] (G256) or [n][k/128] (G128)
  uint16_t* y;           // [m][n] bf16, or nullptr in partials mode
  int32_t* partials;     // [m][n][k/G] in partials mode, else nullptr
  // fused mode (x given): the kernel rotates and quantises x itself
  const uint16_t* x;     // [m][k] bf16, or nullptr
  int8_t* xq_out;        // [m][k] codes written back when not null
  float* xs_out;         // [m] scales written back when not null
  // 1: the weights may come from the previous kernel on the stream; read
  // them only after it has completed (no read-ahead under programmatic launch)
  int weights_after_wait;
};

// Launchers (iq8r_kernels.cu). They validate nothing: the ABI layer has.
cudaError_t launch_act_quant(const uint16_t* x, int64_t m, int64_t k, int rotate, int8_t* xq,
                             float* xs, cudaStream_t stream);
cudaError_t launch_gemv(const LinearArgs& a, cudaStream_t stream);
bool gemv_supported(int64_t k, std::string* why);
// fixed_scratch: split-K partials go to the static no-allocation array; a
// plan that needs more than it holds sets *too_big and launches nothing.
cudaError_t launch_gemm_tc(const LinearArgs& a, cudaStream_t stream, bool fixed_scratch = false,
                           bool* too_big = nullptr);
bool gemm_tc_supported(const LinearArgs& a, std::string* why);
cudaError_t read_and_clear_device_error(uint32_t* err);
// n bf16 values from src to dst by a kernel (programmatic launch), one of
// them pinned host memory mapped into the device's address space (its
// device address), both 16-byte aligned (mapped_copy.cuh).
cudaError_t launch_mapped_copy(const uint16_t* src, uint16_t* dst, int64_t n, bool host_to_device,
                               cudaStream_t stream);
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream);
// The drafter's codebook format (cb4_gemv.cuh): y or partials.
cudaError_t launch_cb4(const LinearArgs& a, cudaStream_t stream);
bool cb4_supported(int64_t k, std::string* why);
// out[t][j] = y[t][cand[t][j]] (see rescore.cuh)
cudaError_t launch_rescore(const LinearArgs& a, const int32_t* cand, int kc, uint16_t* out, cudaStream_t stream);

// Host packer (iq8r_pack.cpp).
void pack_rows(int fmt, bool rotate, int rule, const uint16_t* w, int64_t n, int64_t k, int8_t* codes,
               uint8_t* sub, uint16_t* scale, int n_threads);

}  // namespace iq8r
