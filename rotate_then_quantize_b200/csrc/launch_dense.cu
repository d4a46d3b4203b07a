// Launchers of the dense-rotation codec (dense.cuh): the Householder rotation
// builder, the operand split, and the quantise / dequantise / calibration
// products, for d in {64, 128, 256}.
#include "dense.cuh"
#include "launch_impl.cuh"

namespace srftq {

namespace {

template <typename F>
int by_dense_d(int d, F&& f) {
  switch (d) {
    case 64: return f(Int<64>{});
    case 128: return f(Int<128>{});
    case 256: return f(Int<256>{});
    default: return SRFTQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

int launch_householder(const HouseholderCall& c) {
  if (c.n_slices == 0) return SRFTQ_OK;
  const int64_t blocks = c.n_slices * c.heads;
  if (blocks > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  HouseholderArgs a{c.heads, c.n_reflectors, c.reflectors, c.signs, c.rot};
  return by_dense_d(c.d, [&](auto d_) {
    constexpr int D = decltype(d_)::value;
    if (c.rotation == kSRFT)
      householder_kernel<D, kSRFT><<<int(blocks), D, 0, c.stream>>>(a);
    else
      householder_kernel<D, kSRHT><<<int(blocks), D, 0, c.stream>>>(a);
    return finish_launch();
  });
}

int launch_dense_operand(const OperandCall& c) {
  const int64_t mats = c.n_slices * c.heads;
  if (mats == 0) return SRFTQ_OK;
  const int64_t total = mats * c.d * c.d;
  const int64_t want = (total + 255) / 256;
  const int64_t cap = int64_t(Runtime::num_sms()) * 8;
  operand_kernel<<<int(want < cap ? want : cap), 256, 0, c.stream>>>(c.rot, c.operand, mats,
                                                                       c.d * c.d);
  return finish_launch();
}

template <bool QUANT>
int launch_dense_codec(const DenseCall& c) {
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  const int64_t tiles = (c.n_rows + kDenseRows - 1) / kDenseRows;
  const int64_t blocks = c.n_slices * c.heads * tiles;
  if (blocks > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  DenseArgs a{c.n_slices, c.n_rows, c.in_stride_rows, c.out_stride_rows, c.heads, tiles,
              c.x,        c.codes_in, c.scales_in,  c.codes,           c.scales, c.xhat,
              c.operand,  c.lambda};
  return by_dense_d(c.d, [&](auto d_) {
    constexpr int D = decltype(d_)::value;
    int rc = SRFTQ_ERR_UNSUPPORTED;
    static_for<0, 2>([&](auto b_) {
      constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
      static_for<3, ilog2(D) + 1>([&](auto lg_) {
        constexpr int G = 1 << decltype(lg_)::value;
        if (c.bits == BITS && c.group == G) {
          constexpr auto K = dense_gemm_kernel<D, BITS, G, QUANT>;
          constexpr int smem = DenseTile<D>::kBytes;
          int bps = 0;
          rc = prepare_kernel<K>(smem, kDenseThreads, &bps);
          if (rc != SRFTQ_OK) return;
          K<<<int(blocks), kDenseThreads, smem, c.stream>>>(a);
          rc = finish_launch();
        }
      });
    });
    return rc;
  });
}

int launch_quantize_dense(const DenseCall& c) { return launch_dense_codec<true>(c); }
int launch_dequantize_dense(const DenseCall& c) { return launch_dense_codec<false>(c); }

int launch_calibrate_dense(const DenseCalibCall& c) {
  const int64_t blocks = c.n_slices * c.heads;
  if (blocks == 0) return SRFTQ_OK;
  if (blocks > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  DenseCalibArgs a{c.n_cal, c.x_stride_rows, c.heads, c.x, c.operand, c.lambda_out};
  return by_dense_d(c.d, [&](auto d_) {
    constexpr int D = decltype(d_)::value;
    constexpr auto K = dense_calibrate_kernel<D>;
    constexpr int smem = DenseTile<D>::kBytes;
    int bps = 0;
    const int rc = prepare_kernel<K>(smem, kDenseThreads, &bps);
    if (rc != SRFTQ_OK) return rc;
    K<<<int(blocks), kDenseThreads, smem, c.stream>>>(a);
    return finish_launch();
  });
}

}  // namespace srftq
