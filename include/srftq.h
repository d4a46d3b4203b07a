/*
 * srftq.h -- C ABI of the B200 rotate-then-quantize KV-cache codec (libsrftq.so).
 *
 * The codec is the one of "When Quantization Is Free" (technical summary):
 * every head-dim vector x of an fp16 KV cache is rotated by
 * SRFT(x) = pack(F diag(s) x) (Methodology 1; F the unitary DFT, s a fixed
 * random sign vector), rescaled per channel by lambda, quantised with group
 * absmax to signed int4 (two codes per byte) or int8 (Methodology 2, steps
 * 1-5; Methodology 3 for per-channel + per-group scaling), and
 * dequantised by the exact inverse. The SRHT variant replaces F by the
 * normalised Walsh-Hadamard matrix ("HyperQuant", Methodology 1: H D x).
 *
 * Conventions shared by every call
 * --------------------------------
 * Shapes: a call covers S slices (e.g. layer x {K,V}) of N rows, each row
 * holding H heads of d-element vectors. Vector (s, r, h) of an array with
 * slice stride T rows lives at element offset ((s*T + r)*H + h) * per_vector.
 *
 *   x       fp16 (IEEE binary16 bit patterns)  [S][T_x][H][d]
 *   codes   uint8                               [S][T_o][H][d*bits/8]
 *   scales  fp16 bit patterns                   [S][T_o][H][d/group]
 *   signs   int8, one row per (slice, head)     [S][H][d]   (< 0 means -1,
 *           anything else +1)
 *   lambda  float32, one row per (slice, head)  [S][H][d]   (finite, > 0)
 *
 * Packed coordinate order of the rotated vector y (d reals):
 *   y_0 = X_0, y_1 = X_{d/2}, y_{2k} = sqrt2 Re X_k, y_{2k+1} = sqrt2 Im X_k
 *   (0 < k < d/2), X = F (s * x) with kernel exp(-2 pi i k n / d) / sqrt(d).
 * SRHT: y = H_d (s * x) / sqrt(d), Sylvester natural order.
 *
 * Quantiser (per vector, per group g of `group` consecutive coordinates):
 *   w_j = y_j / lambda_j;  a_g = max |w_j|;  qmax = 7 (int4) or 127 (int8)
 *   sigma_g = fp16 round-to-nearest-even of (a_g / qmax), saturated at 65504
 *   q_j = clamp(round-half-even(w_j / sigma_g), -qmax, qmax); 0 if sigma_g == 0
 *   int4: element 2k in the low nibble of byte k, 2k+1 in the high nibble.
 * Dequantiser: x_hat = s * R^T (lambda * sigma * q), rounded to fp16.
 *
 * Ownership and execution: every pointer is a device pointer owned by the
 * caller; the library allocates no device memory and keeps no per-call
 * state. Calls enqueue work on `stream` (a cudaStream_t; NULL = legacy
 * default stream) and return without synchronising: SRFTQ_OK means
 * "launched". A call with zero vectors launches nothing. Every other
 * successful call launches exactly one kernel.
 *
 * Errors: argument errors are detected on the host before anything is
 * launched and return a negative status. A launch failure returns
 * SRFTQ_ERR_CUDA. Device-side guards (bounded waits) record into a
 * library-wide word read by srftq_check_device(); they never trap.
 *
 * Alignment: every pointer must be 16-byte aligned; slice strides are in
 * rows and must be >= N (slices may not overlap). Inputs and outputs must
 * not overlap (no in-place use). Non-finite inputs give unspecified codes,
 * never a fault.
 *
 * Supported: d in {16, 32, 64, 128, 256}; group a power of two with
 * 8 <= group <= d (group = d is one scale per vector, the per-token
 * scaling the pages compare against); bits in {4, 8}; heads >= 1; rotation
 * SRFT or SRHT.
 */
#ifndef SRFTQ_H
#define SRFTQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
#define SRFTQ_OK                0
#define SRFTQ_ERR_INVALID_ARG  (-1)  /* null pointer, bad size, overlap  */
#define SRFTQ_ERR_UNSUPPORTED  (-2)  /* d / group / bits / rotation       */
#define SRFTQ_ERR_MISALIGNED   (-3)  /* pointer not 16-byte aligned       */
#define SRFTQ_ERR_CUDA         (-4)  /* CUDA runtime or driver error      */
#define SRFTQ_ERR_DEVICE_CHECK (-5)  /* a device-side guard fired         */

/* Rotation kinds. */
#define SRFTQ_ROT_SRFT 0  /* sign-randomised real-packed FFT (Methodology 1) */
#define SRFTQ_ROT_SRHT 1  /* sign-randomised Walsh-Hadamard ("HyperQuant")  */

/* Codec configuration: head dimension, heads per row, group size, code
 * width and rotation kind. Plain data; the caller owns it. */
typedef struct srftq_desc {
    int32_t d;
    int32_t heads;
    int32_t group;
    int32_t bits;
    int32_t rotation;
} srftq_desc;

/*
 * srftq_quantize -- rotate, rescale and quantise S x N x H vectors.
 * "When Quantization Is Free", Methodology 2, steps 1-5 (load and sign,
 * FFT, Hermitian pack, lambda / group absmax / round, nibble packing).
 *
 *   x        [S][x_slice_stride_rows][H][d] fp16, read-only
 *   signs    [S][H][d] int8;  lambda [S][H][d] float32
 *   codes    [S][out_slice_stride_rows][H][d*bits/8] uint8, written
 *   scales   [S][out_slice_stride_rows][H][d/group] fp16, written
 * Only rows 0..n_rows-1 of every slice are read or written.
 */
int srftq_quantize(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                   const uint16_t* x, int64_t x_slice_stride_rows,
                   const int8_t* signs, const float* lambda,
                   uint8_t* codes, uint16_t* scales,
                   int64_t out_slice_stride_rows, void* stream);

/*
 * srftq_dequantize -- the inverse of srftq_quantize: unpack, multiply by
 * the group scale and lambda, apply R^T (inverse real FFT or WHT), multiply
 * by the signs, round to fp16. Implied by the cache use in "When
 * Quantization Is Free" (Methodology 2, the cache that holds the codes;
 * Problem Statement, the cost of de-rotation).
 *
 *   codes, scales as written by srftq_quantize, slice stride in_slice_stride_rows
 *   xhat     [S][out_slice_stride_rows][H][d] fp16, written
 */
int srftq_dequantize(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                     const uint8_t* codes, const uint16_t* scales,
                     int64_t in_slice_stride_rows,
                     const int8_t* signs, const float* lambda,
                     uint16_t* xhat, int64_t out_slice_stride_rows, void* stream);

/*
 * srftq_calibrate_lambda -- per-channel lambda from calibration rows.
 * lambda_out[s][h][j] = sqrt(mean over rows r < n_cal of y_{s,r,h,j}^2),
 * 1 where that sum is zero; y is the rotation of x (no lambda). The
 * statistic is the calibrated per-channel scale of "When Quantization Is
 * Free", Methodology 2 step 4 and Methodology 3 (the pages leave the
 * statistic open; the root mean square is the reading taken). The sum is
 * accumulated in float64 in a fixed order, so the result is deterministic.
 *
 *   x          [S][x_slice_stride_rows][H][d] fp16 (rows 0..n_cal-1 read)
 *   lambda_out [S][H][d] float32, written
 */
int srftq_calibrate_lambda(const srftq_desc* desc, int64_t n_slices, int64_t n_cal,
                           const uint16_t* x, int64_t x_slice_stride_rows,
                           const int8_t* signs, float* lambda_out, void* stream);

/*
 * srftq_rotate -- the rotation alone, float32 out (parity and debugging).
 * y = R (s * x), divided by lambda when lambda_or_null is not NULL.
 * "When Quantization Is Free", Methodology 1 (SRFT definition).
 *
 *   y_out [S][n_rows][H][d] float32, contiguous, written
 */
int srftq_rotate(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                 const uint16_t* x, int64_t x_slice_stride_rows,
                 const int8_t* signs, const float* lambda_or_null,
                 float* y_out, void* stream);

/*
 * srftq_dequantize_rotated -- dequantises into the rotated domain: for every
 * vector, yhat'_j = lambda_j * sigma_g(j) * q_j (fp16, round to nearest
 * even), the reconstruction R xhat of the cached vector with neither the
 * inverse transform nor the signs applied. R is orthogonal ("When
 * Quantization Is Free", Methodology 1), so attention can score the rotated
 * query R q against these vectors, (R q) . yhat' = q . xhat, accumulate the
 * value vectors in the rotated domain and undo the rotation once per output
 * with srftq_unrotate. desc->rotation is not used (no transform runs).
 *
 *   codes  [S][in_stride][H][d*bits/8], scales [S][in_stride][H][d/group]
 *   lambda [S][H][d] float32 (the quantiser's)
 *   out    [S][out_stride][H][d] fp16, written
 *
 * Same argument rules as srftq_dequantize (signs are not read).
 */
int srftq_dequantize_rotated(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                             const uint8_t* codes, const uint16_t* scales,
                             int64_t in_slice_stride_rows, const float* lambda, uint16_t* out,
                             int64_t out_slice_stride_rows, void* stream);

/*
 * srftq_unrotate -- the inverse rotation x = s * R^T y, float32 in and out
 * (y in the packed rotated coordinates of srftq_rotate without lambda).
 * "When Quantization Is Free", Methodology 1 (R orthogonal, R^T = R^-1).
 *
 *   y [S][y_stride][H][d] float32, signs [S][H][d] int8,
 *   x [S][x_stride][H][d] float32, written (must not overlap y or signs)
 */
int srftq_unrotate(const srftq_desc* desc, int64_t n_slices, int64_t n_rows, const float* y,
                   int64_t y_slice_stride_rows, const int8_t* signs, float* x,
                   int64_t x_slice_stride_rows, void* stream);

/*
 * srftq_decode_attention -- one decode step of attention, fused with
 * dequantisation, for d = 128. For every sequence b < n_seq and KV head h,
 * the q_per_kv (1, 2, 4 or 8) query heads h*q_per_kv + g attend over the
 * n_ctx cached tokens of the quantised K and V caches:
 *   out = sum_t softmax_t(softmax_scale * q . khat_t) vhat_t
 * with khat, vhat what srftq_dequantize would return (before its fp16
 * rounding). R is orthogonal ("When Quantization Is Free", Methodology 1),
 * so the kernel rotates each query once with the K signs, reads only codes
 * and scales, and undoes the V rotation once per output: it never writes a
 * dequantised cache and runs no inverse transform per token. Arithmetic is
 * float32, except the key scores for int4 codes with q_per_kv = 1 and
 * group >= 16. There the rotated query is held as integers, exact to 2^-22
 * of its largest value in each run of 16 coordinates, and multiplied with
 * the codes on the integer tensor cores.
 *
 *   q        [n_seq][heads*q_per_kv][d] fp16
 *   k_codes, v_codes    rows of [heads][d*bits/8] uint8; k_scales, v_scales
 *            rows of [heads][d/group] fp16; token t of sequence b is row
 *            t*tok_stride_rows + b*seq_stride_rows (strides >= 0)
 *   k_signs, v_signs [heads][d] int8; k_lambda, v_lambda [heads][d] float32
 *            (the quantiser's, for the one slice each cache is)
 *   out      [n_seq][heads*q_per_kv][d] float32, written; must not overlap
 *            an input. It doubles as the call's scratch: the first of the
 *            call's three kernels writes the rotated queries there, the
 *            second overwrites them with the rotated-domain outputs and the
 *            third unrotates those in place, so `out` holds the result only
 *            once the call's work on `stream` is complete.
 *
 * Returns SRFTQ_ERR_UNSUPPORTED for d != 128 or another q_per_kv, and
 * SRFTQ_ERR_INVALID_ARG for n_ctx < 1 or bad pointers and strides; every
 * pointer must be 16-byte aligned (SRFTQ_ERR_MISALIGNED).
 */
int srftq_decode_attention(const srftq_desc* desc, int64_t n_seq, int64_t n_ctx, int32_t q_per_kv,
                           const uint16_t* q, const uint8_t* k_codes, const uint16_t* k_scales,
                           const int8_t* k_signs, const float* k_lambda, const uint8_t* v_codes,
                           const uint16_t* v_scales, const int8_t* v_signs,
                           const float* v_lambda, int64_t tok_stride_rows,
                           int64_t seq_stride_rows, float softmax_scale, float* out,
                           void* stream);

/*
 * Dense-rotation codec: the Householder variant of "When Quantization Is
 * Free" (Methodology 3, Householder rotations: k = d/2 reflectors at
 * d = 256 give practically lossless quantisation; Key Results, lossless
 * regime), and any other orthogonal rotation given as a matrix. The codec
 * after the rotation is the one above (lambda, group absmax, fp16 scale,
 * rounding, packing; the dequantiser applies R^T). d in {64, 128, 256};
 * desc->rotation selects the base of srftq_householder_rotation and is not
 * read by the other dense calls. Same ownership, stream, error and
 * alignment rules as above.
 *
 * Rotation matrices are float32 [S][H][d][d], row n giving output
 * coordinate n (y = R x). The dense codec reads a rotation as an "operand":
 * [S][H][2][d][d] fp16 bit patterns, part 0 = fp16_rn(R) ("hi"), part 1 =
 * fp16_rn(R - hi) ("lo"), so hi + lo carries R to about 2^-22.
 */

/*
 * srftq_householder_rotation -- R = H(v_1) H(v_2) ... H(v_k) B for every
 * (slice, head), with H(v) = I - 2 v v^T / (v^T v) and B the signed base
 * rotation of desc->rotation (SRFT or SRHT matrix times diag(s)): the
 * learned reflectors act on top of the fixed SRFT base, H(v_k) first. k = 0
 * gives B itself (the FFT / WHT rotation as a matrix). Computed in double,
 * stored in float32. A reflector that is exactly zero is skipped.
 *
 *   reflectors   [S][H][k][d] float32 (may be NULL when k = 0)
 *   signs        [S][H][d] int8
 *   rotation_out [S][H][d][d] float32, written; must not overlap the inputs
 * One launch (one block per (slice, head)). 0 <= k <= 65536.
 */
int srftq_householder_rotation(const srftq_desc* desc, int64_t n_slices, int32_t n_reflectors,
                               const float* reflectors, const int8_t* signs,
                               float* rotation_out, void* stream);

/*
 * srftq_dense_operand -- splits float32 rotations [S][H][d][d] into the
 * fp16 operand [S][H][2][d][d] (hi, lo) the dense codec reads. One launch.
 */
int srftq_dense_operand(const srftq_desc* desc, int64_t n_slices, const float* rotation,
                        uint16_t* operand_out, void* stream);

/*
 * srftq_calibrate_lambda_dense -- lambda_out[s][h][n] = sqrt(mean over rows
 * r < n_cal of y_n^2), y = R x (R = hi + lo of the operand), 1 where the
 * sum is zero; float64 sums in a fixed order (deterministic). One launch.
 */
int srftq_calibrate_lambda_dense(const srftq_desc* desc, int64_t n_slices, int64_t n_cal,
                                 const uint16_t* x, int64_t x_slice_stride_rows,
                                 const uint16_t* operand, float* lambda_out, void* stream);

/*
 * srftq_quantize_dense -- y = R x per vector, then the codec's quantiser:
 * w = y / lambda, sigma = fp16(absmax / qmax), q = clamp(rne(w / sigma)).
 * Arguments and layouts as srftq_quantize, with the operand in place of the
 * signs. One launch.
 */
int srftq_quantize_dense(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                         const uint16_t* x, int64_t x_slice_stride_rows, const uint16_t* operand,
                         const float* lambda, uint8_t* codes, uint16_t* scales,
                         int64_t out_slice_stride_rows, void* stream);

/*
 * srftq_dequantize_dense -- xhat = R^T (lambda * sigma * q), rounded to
 * fp16. Arguments and layouts as srftq_dequantize, with the operand in
 * place of the signs. One launch.
 */
int srftq_dequantize_dense(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                           const uint8_t* codes, const uint16_t* scales,
                           int64_t in_slice_stride_rows, const uint16_t* operand,
                           const float* lambda, uint16_t* xhat, int64_t out_slice_stride_rows,
                           void* stream);

/* Human-readable text for a status code (static storage, never NULL). */
const char* srftq_status_string(int status);

/*
 * srftq_check_device -- reads and clears, in one atomic step on `stream`,
 * the library-wide device guard word of the current device, then
 * synchronises `stream` and returns SRFTQ_OK if no guard fired since the
 * last check, SRFTQ_ERR_DEVICE_CHECK if one did (a bounded wait gave up),
 * SRFTQ_ERR_CUDA on a runtime error. The step is one one-thread kernel on
 * `stream`: codec work still running on other streams cannot lose a bit
 * (a bit set after the step is reported by the next check). Work on other
 * streams is not waited for; synchronise them first to include it.
 */
int srftq_check_device(void* stream);

/*
 * srftq_probe_wait_timeout -- exercises the device-side failure path. Launches
 * one thread that waits on a shared-memory barrier nothing ever arrives on,
 * polling it `polls` times (1 <= polls <= 4194304, the codec kernels' own
 * limit) before it gives up and records the timeout in the guard word, as
 * every codec kernel does when one of its waits runs out. Nothing faults and
 * the context stays usable: the next srftq_check_device on the same stream
 * returns SRFTQ_ERR_DEVICE_CHECK (and clears the word). Returns
 * SRFTQ_ERR_INVALID_ARG for `polls` out of range, SRFTQ_ERR_CUDA if the
 * launch fails, else SRFTQ_OK (launched, asynchronous).
 */
int srftq_probe_wait_timeout(uint32_t polls, void* stream);

/*
 * srftq_debug_checks -- 1 if this library was built with the device-side
 * index checks (SRFTQ_DEBUG_CHECKS; the in-tree libsrftq_debug.so), else 0.
 * In that build every kernel checks each global-memory index it computes
 * (vector slots, TMA tile coordinates) against the call's extents before the
 * access; a failed check skips the access and records bit 1 of the guard
 * word, which srftq_check_device reports as SRFTQ_ERR_DEVICE_CHECK. Nothing
 * traps. The release build compiles the checks away.
 */
int srftq_debug_checks(void);

/*
 * srftq_probe_index_check -- exercises that check on the device: one thread
 * checks `index` against [0, limit) as the kernels check theirs (no memory
 * is accessed). In the debug build an index outside the range is recorded,
 * and the next srftq_check_device on the stream returns
 * SRFTQ_ERR_DEVICE_CHECK; in the release build nothing is recorded.
 * Returns SRFTQ_ERR_CUDA if the launch fails, else SRFTQ_OK.
 */
int srftq_probe_index_check(int64_t index, int64_t limit, void* stream);

/* Library version as 10000*major + 100*minor + patch. */
int srftq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SRFTQ_H */
