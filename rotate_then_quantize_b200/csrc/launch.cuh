// Host-side launch layer: tensor-map encoding, kernel configuration and
// dispatch over the compile-time shapes. Each head dimension d is compiled
// in its own translation unit (launch_d*.cu) from launch_impl.cuh.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/srftq.h"

namespace srftq {

struct QuantCall {
  int32_t heads, group, bits, rotation;
  int64_t n_slices, n_rows;
  const uint16_t* x;
  int64_t x_slice_stride_rows;
  const int8_t* signs;
  const float* lambda;
  uint8_t* codes;
  uint16_t* scales;
  int64_t out_slice_stride_rows;
  cudaStream_t stream;
};

struct DequantCall {
  int32_t heads, group, bits, rotation;
  int64_t n_slices, n_rows;
  const uint8_t* codes;
  const uint16_t* scales;
  int64_t in_slice_stride_rows;
  const int8_t* signs;
  const float* lambda;
  uint16_t* xhat;
  int64_t out_slice_stride_rows;
  cudaStream_t stream;
};

struct RotateCall {
  int32_t heads, rotation;
  int64_t n_slices, n_rows;
  const uint16_t* x;
  int64_t x_slice_stride_rows;
  const int8_t* signs;
  const float* lambda;
  float* y;
  cudaStream_t stream;
};

struct RotDequantCall {
  int32_t heads, group, bits;
  int64_t n_slices, n_rows;
  const uint8_t* codes;
  const uint16_t* scales;
  int64_t in_slice_stride_rows;
  const float* lambda;
  uint16_t* out;
  int64_t out_slice_stride_rows;
  cudaStream_t stream;
};

struct UnrotateCall {
  int32_t heads, rotation;
  int64_t n_slices, n_rows;
  const float* y;
  int64_t y_slice_stride_rows;
  const int8_t* signs;
  float* x;
  int64_t x_slice_stride_rows;
  cudaStream_t stream;
};

struct AttnCall {
  int32_t heads, group, bits, rotation, q_per_kv;
  int64_t n_seq, n_ctx, tok_stride_rows, seq_stride_rows;
  float scale;
  const uint16_t* q;
  const uint8_t* k_codes;
  const uint16_t* k_scales;
  const int8_t* k_signs;
  const float* k_lambda;
  const uint8_t* v_codes;
  const uint16_t* v_scales;
  const int8_t* v_signs;
  const float* v_lambda;
  float* out;
  cudaStream_t stream;
};

struct CalibCall {
  int32_t heads, rotation;
  int64_t n_slices, n_cal;
  const uint16_t* x;
  int64_t x_slice_stride_rows;
  const int8_t* signs;
  float* lambda_out;
  cudaStream_t stream;
};

// Dense-rotation codec (launch_dense.cu).
struct HouseholderCall {
  int32_t d, heads, rotation, n_reflectors;
  int64_t n_slices;
  const float* reflectors;
  const int8_t* signs;
  float* rot;
  cudaStream_t stream;
};

struct OperandCall {
  int32_t d, heads;
  int64_t n_slices;
  const float* rot;
  uint16_t* operand;
  cudaStream_t stream;
};

struct DenseCall {
  int32_t d, heads, group, bits;
  int64_t n_slices, n_rows, in_stride_rows, out_stride_rows;
  const uint16_t* x;
  const uint8_t* codes_in;
  const uint16_t* scales_in;
  uint8_t* codes;
  uint16_t* scales;
  uint16_t* xhat;
  const uint16_t* operand;
  const float* lambda;
  cudaStream_t stream;
};

struct DenseCalibCall {
  int32_t d, heads;
  int64_t n_slices, n_cal, x_stride_rows;
  const uint16_t* x;
  const uint16_t* operand;
  float* lambda_out;
  cudaStream_t stream;
};

int launch_householder(const HouseholderCall& c);
int launch_dense_operand(const OperandCall& c);
int launch_quantize_dense(const DenseCall& c);
int launch_dequantize_dense(const DenseCall& c);
int launch_calibrate_dense(const DenseCalibCall& c);

// Services the per-d units get from the API unit.
struct Runtime {
  // Encodes a rank-4 tiled tensor map; returns 0 on success.
  static int encode_4d(CUtensorMap* map, CUtensorMapDataType dtype, void* base,
                       const uint64_t dims[4], const uint64_t strides_bytes[3],
                       const uint32_t box[4], CUtensorMapSwizzle swz);
  static int num_sms();          // streaming multiprocessors of the current device
  static unsigned* guard_word(); // device address of the guard word, current device
};

template <int D> int launch_quantize(const QuantCall& c);
template <int D> int launch_dequantize(const DequantCall& c);
template <int D> int launch_rotate(const RotateCall& c);
template <int D> int launch_calibrate(const CalibCall& c);
template <int D> int launch_dequantize_rotated(const RotDequantCall& c);
template <int D> int launch_unrotate(const UnrotateCall& c);

// Decode attention over the quantised cache in the rotated domain, d = 128
// (launch_attention.cu).
int launch_decode_attention_d128(const AttnCall& c);

// d = 256 has its own kernels (two threads per vector; launch_d256.cu).
template <> int launch_quantize<256>(const QuantCall& c);
template <> int launch_dequantize<256>(const DequantCall& c);
template <> int launch_rotate<256>(const RotateCall& c);
template <> int launch_calibrate<256>(const CalibCall& c);
template <> int launch_unrotate<256>(const UnrotateCall& c);

}  // namespace srftq
