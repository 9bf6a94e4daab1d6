/*
 * libiq8r -- the IQ8R rotated W8A8 linear layer on NVIDIA B200 (sm_100a).
 *
 * The layer, as the "radiance" model cards describe it:
 *
 *  - "Qwen3.8-27B IQ8R + DFlash2 -- radiance container", table row "Weights":
 *    the trunk linears hold int8 codes in -127..127 with one u8 scale for
 *    every row and 256-wide block of K, below one bf16 scale per row, every
 *    128 of K first rotated by a Hadamard transform without normalisation;
 *    the lm_head holds int8 codes with one bf16 scale for every row and
 *    128-wide block of K.
 *  - same page, table row "Activations": the activations are int8 too, in
 *    the same rotated domain (W8A8).
 *  - same page, "How this file was made": the recipe rules
 *    "codes=i8 group=256 scale=u8 scale2=bf16 block2=1x* transform=fwht128
 *    clamp=sym" (trunk) and "codes=i8 group=128 scale=bf16 clamp=sym"
 *    (lm_head).
 *
 * Notation. W is a bf16 weight [N][K] (out x in), x a bf16 activation [M][K],
 * H the 128x128 Sylvester Hadamard matrix (H[i][j] = (-1)^popcount(i&j),
 * unnormalised, H H = 128 I), T(.) applies H to every consecutive 128 of K.
 * y = x W^T is computed as (1/128) T(x) T(W)^T on int8 codes.
 *
 * Where the pages are silent the library follows stated definitions:
 *  - the fp32 transform runs radix-2 butterflies h = 1, 2, ..., 64 in that
 *    order, (a, b) -> (a + b, a - b), round-to-nearest-even, no fused ops;
 *  - activations carry one fp32 scale per token: a = amax / 127,
 *    codes = clamp(rint(x' * (127 / amax)), -127, 127); a row with amax
 *    below 2^-64 is first multiplied by 2^64 (exact), which keeps 127 / amax
 *    finite down to bf16 subnormals and changes no code where it was finite;
 *    rows whose x' is not finite are outside the definition;
 *  - trunk weights: step d[n][g] = s2[n] * s1[n][g], s2 = bf16 of
 *    R[n] / 32385 rounded up (R = row absmax of T(W)), s1 = min(255,
 *    ceil(A[n][g] / (127 * s2))) (A = absmax of the 256-block);
 *  - lm_head weights: s[n][g] = bf16 of A[n][g] / 127 rounded up;
 *  - round-half-to-even wherever a value is rounded to nearest.
 *
 * Conventions for every call:
 *  - The caller owns every buffer. Hot calls allocate nothing.
 *  - Device pointers must be device memory of the current CUDA device and
 *    16-byte aligned; tensors are dense and row-major as stated.
 *  - A bad argument returns IQ8R_ERR_INVALID_ARG, launches nothing and sets
 *    the thread's message (iq8r_last_error). A failed launch returns
 *    IQ8R_ERR_CUDA.
 *  - GPU calls are asynchronous and ordered on `stream` (0 = the legacy
 *    default stream). Kernels never trap: a bounded wait that runs out sets
 *    a device error word that iq8r_get_device_error reports.
 */
#ifndef IQ8R_H_
#define IQ8R_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  IQ8R_OK = 0,
  IQ8R_ERR_INVALID_ARG = 1,    /* bad shape, pointer, alignment or format */
  IQ8R_ERR_UNSUPPORTED = 2,    /* valid request this build cannot serve */
  IQ8R_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
  IQ8R_ERR_DEVICE_TIMEOUT = 4  /* a kernel's bounded wait ran out */
} iq8r_status;

typedef enum {
  /* trunk: int8 codes, u8 sub-scale per (row, 256 of K), bf16 scale per row */
  IQ8R_FMT_G256_U8_BF16 = 0,
  /* lm_head: int8 codes, bf16 scale per (row, 128 of K) */
  IQ8R_FMT_G128_BF16 = 1,
  /* the drafter's linears: 4-bit indices into the 16 levels
   * -127 -97 -75 -58 -43 -30 -18 -6 6 18 30 43 58 75 97 127 (IQ8R page,
   * "How this file was made", the dflash recipe lines), two a byte with the
   * even K position in the low nibble, and a bf16 scale per (row, 128 of K);
   * y as for G128 with the codes' levels. Packed by nearest level (ties to
   * the larger) under s = bf16 of A / 127 rounded up (IQ8R_RULE_RTN) or the
   * searched scale (IQ8R_RULE_SEARCH). Weight-streaming kernels only (no
   * IQ8R_PATH_TC): one token on dp4a, two or more on mma.sync (16 tokens a
   * launch); not for iq8r_rescore. */
  IQ8R_FMT_CB4_G128 = 2
} iq8r_format;

/* Kernel choice for iq8r_linear_ex. AUTO picks by M. */
typedef enum {
  IQ8R_PATH_AUTO = 0,
  IQ8R_PATH_GEMV = 1,   /* weight-streaming dp4a GEMV, M handled 8 rows at a time */
  IQ8R_PATH_TC = 2,     /* tcgen05 kind::i8 tensor-core GEMM */
  /* Flag, OR-ed into the path of iq8r_linear_ex: the weight arrays may have
   * been written by the kernel just before this call on the stream, so read
   * them only after that kernel has completed (see iq8r_weight). */
  IQ8R_PATH_FLAG_WEIGHTS_WRITTEN = 0x100
} iq8r_path;

/* A packed weight on the device. Not owned by the library.
 *   codes     int8 [n][k], K contiguous (row-major), values -127..127; for
 *             IQ8R_FMT_CB4_G128 the packed indices, u8 [n][k/2]
 *   sub_scale u8   [n][k/256] for IQ8R_FMT_G256_U8_BF16; NULL for G128
 *   scale     bf16 [n] (G256) or [n][k/128] (G128), as raw 16-bit patterns
 *   rotated   1 if the codes live in the fwht128 domain (the output is then
 *             multiplied by 1/128); 0 for a plain int8 weight.
 * k must be a multiple of 256 (G256) or 128 (G128); codes, sub_scale and
 * scale must be 16-byte aligned (the arrays' base addresses).
 *
 * Read-ahead of the weights. The linear calls launch their kernels with
 * programmatic dependent launch: the weight-streaming kernels start copying
 * weight tiles while the previous kernel on the stream is still finishing,
 * and wait for it only before they read the activations. So the weight
 * arrays must not be written by the kernel that immediately precedes a
 * linear call on the same stream (for example a device-side repack or
 * update): write them earlier, synchronise, or pass
 * IQ8R_PATH_FLAG_WEIGHTS_WRITTEN to iq8r_linear_ex, which makes every kernel
 * wait for the previous one before its first weight read. */
typedef struct {
  int32_t fmt;
  int32_t rotated;
  int64_t n;
  int64_t k;
  const int8_t* codes;
  const uint8_t* sub_scale;
  const uint16_t* scale;
} iq8r_weight;

/* Byte sizes of the three packed arrays for an [n][k] weight of `fmt`
 * (sub_bytes is 0 for G128). Host only; any pointer may be NULL. */
iq8r_status iq8r_packed_sizes(int32_t fmt, int64_t n, int64_t k, size_t* codes_bytes,
                              size_t* sub_bytes, size_t* scale_bytes);

/* Round-to-nearest packing of a bf16 weight (the recipes' "rtn"; the pages'
 * own GPTQ fit needs calibration Hessians and is not part of this library).
 * Host memory in and out, synchronous.
 *   w_bf16    bf16 [n][k] host, raw 16-bit patterns
 *   rotate    1: apply fwht128 to each 128 of K first (k % 128 == 0)
 *   codes     int8 [n][k] host (out)
 *   sub_scale u8 [n][k/256] host (out; G256 only, NULL for G128)
 *   scale     bf16 [n] (G256) or [n][k/128] (G128) host (out)
 *   n_threads host threads to use; <= 0 picks the hardware concurrency.
 * Trunk: a u8 scale for each row and 256 of K below a bf16 row scale (IQ8R
 * page, "Weights"); lm_head: a bf16 scale for each row and 128 of K (same
 * row).
 * Output is byte-identical to the stated definition in the file comment. */
iq8r_status iq8r_pack(int32_t fmt, int32_t rotate, const uint16_t* w_bf16, int64_t n, int64_t k,
                      int8_t* codes, uint8_t* sub_scale, uint16_t* scale, int32_t n_threads);

/* Packing rules: IQ8R_RULE_RTN is iq8r_pack's. IQ8R_RULE_SEARCH is the
 * recipes' "rule=search" (one scale per 128 columns, chosen by a search for
 * the least error: "Qwen3.8-Flash-Next, IQR-V4 -- radiance container", row
 * "Trunk"), in this reading: per group, the RTN scale (the smallest that clips
 * nothing) and the 15 next smaller ones are tried, and the one with the least
 * sum of (w' - code * step)^2 over the group (in double, added in order)
 * is kept, ties going to the larger scale. For the trunk the candidates are
 * s1, s1 - 1, ... (>= 1) under the unchanged row scale s2; for G128 and the
 * codebook format they are s and the next smaller bf16 values, and for the
 * codebook each value's term uses its nearest level at that scale. */
typedef enum { IQ8R_RULE_RTN = 0, IQ8R_RULE_SEARCH = 1 } iq8r_rule;

/* iq8r_pack with a packing rule (same arguments otherwise). */
iq8r_status iq8r_pack_ex(int32_t fmt, int32_t rotate, int32_t rule, const uint16_t* w_bf16, int64_t n,
                         int64_t k, int8_t* codes, uint8_t* sub_scale, uint16_t* scale, int32_t n_threads);

/* Rotate and quantise activations: int8 in the weights' rotated domain,
 * W8A8 (IQ8R page, "Activations"), one fp32 scale per token.
 *   x_bf16  device bf16 [m][k], raw 16-bit patterns, 16-byte aligned
 *   m >= 0 (0 launches nothing), k % 128 == 0, 0 < k <= 2^30
 *   rotate  1: x' = T(x) in fp32; 0: x' = x
 *   xq      device int8 [m][k] (out), 16-byte aligned
 *   x_scale device fp32 [m] (out): a = amax(|x'|) / 127 (0 for a zero row)
 * Codes and scales are bit-identical to the stated definition. */
iq8r_status iq8r_rotate_quant_act(const uint16_t* x_bf16, int64_t m, int64_t k, int32_t rotate,
                                  int8_t* xq, float* x_scale, cudaStream_t stream);

/* y = x W^T on int8 codes, the scale epilogue fused, bf16 out.
 *   xq      device int8 [m][w->k] from iq8r_rotate_quant_act (same rotate
 *           setting as the weight), 16-byte aligned
 *   x_scale device fp32 [m]
 *   m >= 0 (0 launches nothing)
 *   y_bf16  device bf16 [m][w->n] (out), 16-byte aligned
 * Trunk:   y[m][n] = bf16_rn(a[m] * s2[n] * sum_g s1[n][g] * P[m][n][g] / 128)
 * lm_head: y[m][n] = bf16_rn(a[m] / 128 * sum_g s[n][g] * P[m][n][g])
 * with P the exact int32 dot product of the codes over block g (256 or 128
 * of K); /128 only when w->rotated. The sum over g is carried in fp32 or
 * exact integers, so y matches the float64 value to within its bf16
 * rounding plus ~1e-6 of the output's scale.
 * Kernels: m <= 2 streams the weights through the GEMV (16-byte loads into
 * registers, three half rows in flight a warp, the rows' block scales in
 * shared memory); larger m runs the
 * tensor-core GEMM (measured on B200: from 3 tokens on it is as fast or
 * faster, at every workload shape). When the GEMM has fewer output tiles than SMs it splits
 * K: the fp32 partial tiles go to a per-device workspace, a 16 MiB array in
 * the library's device image (loaded with the module; no call allocates),
 * and a second kernel adds them in a fixed order, so the result does not
 * depend on timing. The first call on a device looks up the array's address
 * and sets kernel attributes: make it before any stream capture. Calls on
 * different streams that both split K and overlap in time share that
 * workspace and race; order them on one stream. Results are the same bits
 * from call to call. */
iq8r_status iq8r_linear(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w,
                        uint16_t* y_bf16, cudaStream_t stream);

/* The whole layer from bf16 activations: rotate + quantise x (as
 * iq8r_rotate_quant_act, rotating iff w->rotated) and then iq8r_linear.
 * For m <= 2, for m <= 8 with m * k <= 16384, and when xq_out and
 * x_scale_out are not given (m <= 8 only), this is one kernel: every CTA of
 * the weight-streaming GEMV rotates and quantises x itself while its first
 * weight tiles stream in. Otherwise the codes are staged in xq_out /
 * x_scale_out and iq8r_linear consumes them; give the staging buffers for
 * long K (a verify block), where that is the faster way.
 *   x_bf16      device bf16 [m][w->k], 16-byte aligned (w->k % 128 == 0)
 *   y_bf16      device bf16 [m][w->n] (out), 16-byte aligned
 *   xq_out      device int8 [m][w->k] (out) or NULL: the activation codes
 *   x_scale_out device fp32 [m] (out) or NULL: the activation scales
 * For m > 8 xq_out / x_scale_out must be given. Codes and y are the same
 * bits either way, and the same as the two-call path. */
iq8r_status iq8r_linear_bf16(const uint16_t* x_bf16, int64_t m, const iq8r_weight* w, uint16_t* y_bf16,
                             int8_t* xq_out, float* x_scale_out, cudaStream_t stream);

/* The layer from host memory in one call: queues on `stream` the copy of
 * x_host (bf16 [m][w->k]) into x_dev, iq8r_linear_bf16 from x_dev into
 * y_dev, and the copy of y_dev back into y_host (bf16 [m][w->n]), and returns
 * without waiting (synchronise the stream before reading y_host). This is
 * the whole step of a caller whose activations live in host memory, with
 * one crossing of the ABI instead of three.
 *   x_host, y_host  host buffers; page-locked (cudaHostAlloc / pinned) for the
 *                   copies to be asynchronous, else the copies are synchronous
 *   x_dev, y_dev    caller-owned device buffers of the same sizes, 16-byte aligned
 *   xq_out, x_scale_out  as for iq8r_linear_bf16 (needed where it needs them)
 * When x is at most 64 KB and y at most 1 MB (a decode step), both host
 * buffers are page-locked, mapped into the current device's address space
 * (every page-locked allocation is, under unified addressing) and 16-byte
 * aligned, the two copies are small kernels that read x_host and write
 * y_host through the mapping, chained with the layer by programmatic
 * dependent launch, so back-to-back calls overlap as device-only calls do;
 * x_host is read before the previous kernel on the stream has finished (the
 * caller has filled it before the call). Otherwise they are copy calls (the
 * copy engines move large buffers faster than the device's reads of host
 * memory do).
 * Arguments are checked before the first copy is queued; a failure after
 * that returns the failing call's status. Nothing is allocated. */
iq8r_status iq8r_linear_bf16_host(const uint16_t* x_host, int64_t m, const iq8r_weight* w, uint16_t* x_dev,
                                  uint16_t* y_dev, uint16_t* y_host, int8_t* xq_out, float* x_scale_out,
                                  cudaStream_t stream);

/* iq8r_linear with an explicit kernel choice (tests and measurement).
 * path: IQ8R_PATH_AUTO, _GEMV or _TC, optionally OR IQ8R_PATH_FLAG_WEIGHTS_WRITTEN
 * (weights written by the previous kernel on the stream; see iq8r_weight).
 * Any other value returns IQ8R_ERR_INVALID_ARG. */
iq8r_status iq8r_linear_ex(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w,
                           uint16_t* y_bf16, int32_t path, cudaStream_t stream);

/* iq8r_linear that allocates nothing (no counterpart on the pages; an
 * interface for callers that must not allocate, e.g. inside their own
 * memory pools or graphs). Same arguments, same kernel choice and same
 * split plan as iq8r_linear, so y is the same bits; but the split-K partial
 * tiles go to a fixed array of 8 MiB of its own in the library's device
 * image (separate from iq8r_linear's workspace).
 *   - Set-up: the first call on a device looks up that array's address
 *     (cudaGetSymbolAddress) and sets kernel attributes; make it before any
 *     stream capture. No call allocates or frees device memory.
 *   - A call whose split plan needs more than 8 MiB of partial tiles
 *     (units x 128 x tokens-per-tile x 4 bytes) returns
 *     IQ8R_ERR_UNSUPPORTED and launches nothing; iq8r_linear handles it.
 *   - Nothing in the array needs to start at zero: every partial tile is
 *     written in full before the second pass reads it.
 *   - There is one array per device: calls that overlap in time (different
 *     streams, or other threads) race on it; order them on one stream. */
iq8r_status iq8r_linear_noalloc(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w,
                                uint16_t* y_bf16, cudaStream_t stream);

/* Candidate rescoring: the linear's outputs for a short list of weight rows
 * per token, out[t][j] = y[t][cand[t][j]] with y as iq8r_linear defines it
 * (same block sums, same epilogue). The IQ8R page, row "Speculator": 32
 * candidates a position come from the drafter's 2-bit head, and the int8
 * head of the model itself re-scores them.
 *   xq, x_scale  as for iq8r_linear (xq 16-byte aligned)
 *   w            any IQ8R weight (the lm_head: G128); k <= 49152
 *   cand         device int32 [m][n_cand], row indices in [0, w->n)
 *   out_bf16     device bf16 [m][n_cand] (out)
 * One launch, one warp per candidate. Trunk-format results are the same bits
 * as the GEMV path of iq8r_linear. A candidate outside [0, n) gets output 0
 * and makes the next iq8r_get_device_error return IQ8R_ERR_INVALID_ARG; no
 * out-of-range row is read. */
iq8r_status iq8r_rescore(const int8_t* xq, const float* x_scale, int64_t m, const iq8r_weight* w,
                         const int32_t* cand, int64_t n_cand, uint16_t* out_bf16, cudaStream_t stream);

/* Debug twin of iq8r_linear: writes the exact per-block int32 partial sums
 * P[i][j][g] = sum_{k in block g} xq[i][k] * codes[n0 + j][k] for rows
 * n0 <= n < n1 instead of y, computed by the same kernel code as the
 * chosen path (0 <= n0 < n1 <= w->n; block = 256 for G256, 128 for G128).
 *   p  device int32 [m][n1 - n0][k / block] (out), 16-byte aligned */
iq8r_status iq8r_linear_partials(const int8_t* xq, int64_t m, const iq8r_weight* w, int64_t n0,
                                 int64_t n1, int32_t* p, int32_t path, cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the current device's error
 * word. IQ8R_OK if no kernel reported a problem since the last call;
 * IQ8R_ERR_DEVICE_TIMEOUT if a bounded wait ran out (the message names the
 * kernel and the wait); IQ8R_ERR_INVALID_ARG if iq8r_rescore met a candidate
 * index out of range; IQ8R_ERR_CUDA if the stream itself failed. */
iq8r_status iq8r_get_device_error(cudaStream_t stream);

/* Failure-path self-test (no counterpart on the pages). Launches one
 * kernel whose bounded wait waits on a barrier that nothing arrives on, so
 * it gives up after limit_ns (1e3..1e8 ns) and records a self-test code; the
 * next iq8r_get_device_error then returns IQ8R_ERR_DEVICE_TIMEOUT and the
 * context stays usable. It exercises the same wait that every pipelined
 * kernel uses, without faulting or hanging the GPU. */
iq8r_status iq8r_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream);

/* The calling thread's message for its last failed call ("" if none).
 * Valid until the thread's next libiq8r call. */
const char* iq8r_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t iq8r_version(void);

#ifdef __cplusplus
}
#endif

#endif /* IQ8R_H_ */
