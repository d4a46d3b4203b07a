// Kernels and launchers for head dimension d = 256 (two role warps per block
// for the codec; groups of 8 to 256 coordinates).
#include "aux256.cuh"
#include "launch_split.cuh"

namespace srftq {

template <>
int launch_quantize<256>(const QuantCall& c) {
  return dispatch_split<256>(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto r_) {
    return quantize_split_impl<256, decltype(b_)::value, decltype(g_)::value,
                               decltype(r_)::value>(c);
  });
}

template <>
int launch_dequantize<256>(const DequantCall& c) {
  return dispatch_split<256>(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto r_) {
    return dequantize_split_impl<256, decltype(b_)::value, decltype(g_)::value,
                                 decltype(r_)::value>(c);
  });
}

template <>
int launch_rotate<256>(const RotateCall& c) {
  const int64_t total = c.n_slices * c.n_rows * c.heads;
  if (total == 0) return SRFTQ_OK;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  RotateArgs a{c.n_slices, c.n_rows, c.x_slice_stride_rows, c.heads, c.x, c.signs, c.lambda, c.y,
               guard};
  const int64_t want = (2 * total + 127) / 128;
  const int64_t cap = int64_t(Runtime::num_sms()) * 16;
  const int grid = int(want < cap ? want : cap);
  if (c.rotation == kSRFT)
    rotate256_kernel<kSRFT><<<grid, 128, 0, c.stream>>>(a);
  else
    rotate256_kernel<kSRHT><<<grid, 128, 0, c.stream>>>(a);
  return finish_launch();
}

template <>
int launch_calibrate<256>(const CalibCall& c) {
  const int64_t blocks = c.n_slices * c.heads * kCalibCluster;   // one cluster per (slice, head)
  if (blocks == 0) return SRFTQ_OK;
  if (blocks > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  CalibArgs a{c.n_cal, c.x_slice_stride_rows, c.heads, c.x, c.signs, c.lambda_out, c.n_slices,
              guard};
  if (c.rotation == kSRFT)
    calibrate256_kernel<kSRFT><<<int(blocks), 128, 0, c.stream>>>(a);
  else
    calibrate256_kernel<kSRHT><<<int(blocks), 128, 0, c.stream>>>(a);
  return finish_launch();
}

template <>
int launch_unrotate<256>(const UnrotateCall& c) {
  const int64_t total = c.n_slices * c.n_rows * c.heads;
  if (total == 0) return SRFTQ_OK;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  UnrotateArgs a{c.n_slices, c.n_rows, c.y_slice_stride_rows, c.x_slice_stride_rows, c.heads,
                 c.y, c.signs, c.x, guard};
  const int64_t want = (2 * total + 127) / 128;
  const int64_t cap = int64_t(Runtime::num_sms()) * 16;
  const int grid = int(want < cap ? want : cap);
  if (c.rotation == kSRFT)
    unrotate256_kernel<kSRFT><<<grid, 128, 0, c.stream>>>(a);
  else
    unrotate256_kernel<kSRHT><<<grid, 128, 0, c.stream>>>(a);
  return finish_launch();
}

}  // namespace srftq

template int srftq::launch_dequantize_rotated<256>(const srftq::RotDequantCall&);
