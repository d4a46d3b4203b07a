// Launchers of the dense-rotation codec: the Householder rotation builder,
// the operand split and the calibration product (dense.cuh, CUDA cores), and
// the tensor-core quantiser and dequantiser (dense_mma.cuh,
// dense_mma_dequant.cuh), for d in {64, 128, 256}.
#include "dense.cuh"
#include "dense_mma.cuh"
#include "dense_mma_dequant.cuh"
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
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  HouseholderArgs a{c.heads, c.n_reflectors, c.reflectors, c.signs, c.rot, c.n_slices, guard};
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

constexpr int kDenseEpiGroups = 2;

template <int D, int BITS, int G>
int quantize_dense_mma(const DenseCall& c) {
  using L = DenseMma<D, kDenseEpiGroups>;
  const int64_t row_blocks = (c.n_rows + 127) / 128;
  const int64_t total = c.n_slices * c.heads * row_blocks;
  if (total > INT_MAX || c.n_rows > INT_MAX || c.n_slices * c.heads * 2 * D > INT_MAX)
    return SRFTQ_ERR_UNSUPPORTED;
  CUtensorMap tm_x, tm_op;
  {
    // x [S][T][H][d] fp16: boxes of 64 elements x 1 head x 128 rows
    const uint64_t dims[4] = {uint64_t(D), uint64_t(c.heads), uint64_t(c.n_rows),
                              uint64_t(c.n_slices)};
    const uint64_t str[3] = {uint64_t(2 * D), uint64_t(c.heads) * 2 * D,
                             uint64_t(c.in_stride_rows) * c.heads * 2 * D};
    const uint32_t box[4] = {64u, 1u, 128u, 1u};
    if (Runtime::encode_4d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT16, const_cast<uint16_t*>(c.x),
                           dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) != 0)
      return SRFTQ_ERR_CUDA;
  }
  {
    // operand [S][H][2][d][d] fp16 as a 2-D array of rows of d elements (a
    // rank-4 map with two unit dimensions): boxes of 64 columns x d rows
    const uint64_t dims[4] = {uint64_t(D), uint64_t(c.n_slices * c.heads * 2 * D), 1, 1};
    const uint64_t str[3] = {uint64_t(2 * D), uint64_t(2 * D) * c.n_slices * c.heads * 2 * D,
                             uint64_t(2 * D) * c.n_slices * c.heads * 2 * D};
    const uint32_t box[4] = {64u, uint32_t(D), 1u, 1u};
    if (Runtime::encode_4d(&tm_op, CU_TENSOR_MAP_DATA_TYPE_UINT16,
                           const_cast<uint16_t*>(c.operand), dims, str, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) != 0)
      return SRFTQ_ERR_CUDA;
  }
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  DenseMmaArgs a{c.n_rows, row_blocks, c.n_slices, c.heads, c.codes, c.scales,
                 c.out_stride_rows, c.lambda, guard};
  constexpr auto K = quantize_dense_mma_kernel<D, BITS, G, kDenseEpiGroups>;
  constexpr int smem = L::kBytes + kSmemSlack;
  int bps = 0;
  const int rc = prepare_kernel<K>(smem, L::kThreads, &bps);
  if (rc != SRFTQ_OK) return rc;
  // the same number of CTAs for every head (CTA c serves head c % H), at
  // most one per (slice, row block) of a head
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int64_t steps = c.n_slices * row_blocks;
  int64_t per_head = cap / c.heads;
  if (per_head < 1) per_head = 1;
  if (per_head > steps) per_head = steps;
  const int grid = int(per_head * c.heads);
  K<<<grid, L::kThreads, smem, c.stream>>>(tm_x, tm_op, a);
  return finish_launch();
}

int launch_quantize_dense(const DenseCall& c) {
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  return by_dense_d(c.d, [&](auto d_) {
    constexpr int D = decltype(d_)::value;
    int rc = SRFTQ_ERR_UNSUPPORTED;
    static_for<0, 2>([&](auto b_) {
      constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
      static_for<3, ilog2(D) + 1>([&](auto lg_) {
        constexpr int G = 1 << decltype(lg_)::value;
        if (c.bits == BITS && c.group == G) rc = quantize_dense_mma<D, BITS, G>(c);
      });
    });
    return rc;
  });
}
template <int D, int BITS, int G>
int dequantize_dense_mma(const DenseCall& c) {
  using L = DenseDeq<D, BITS>;
  const int64_t row_blocks = (c.n_rows + 127) / 128;
  const int64_t total = c.n_slices * c.heads * row_blocks;
  if (total > INT_MAX || c.n_rows > INT_MAX || c.n_slices * c.heads * 2 * D > INT_MAX)
    return SRFTQ_ERR_UNSUPPORTED;
  CUtensorMap tm_c, tm_op;
  {
    // codes [S][T][H][d*bits/8] bytes: boxes of (up to) 128 bytes x 1 head x 128 rows
    const uint64_t dims[4] = {uint64_t(L::kCB), uint64_t(c.heads), uint64_t(c.n_rows),
                              uint64_t(c.n_slices)};
    const uint64_t str[3] = {uint64_t(L::kCB), uint64_t(c.heads) * L::kCB,
                             uint64_t(c.in_stride_rows) * c.heads * L::kCB};
    const uint32_t box[4] = {uint32_t(L::kCSpan), 1u, 128u, 1u};
    if (Runtime::encode_4d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8,
                           const_cast<uint8_t*>(c.codes_in), dims, str, box,
                           swizzle_mode(L::kCSpan)) != 0)
      return SRFTQ_ERR_CUDA;
  }
  {
    // operand [S][H][2][d][d] fp16 as a 2-D array of rows of d elements:
    // boxes of 64 columns x 64 rows
    const uint64_t dims[4] = {uint64_t(D), uint64_t(c.n_slices * c.heads * 2 * D), 1, 1};
    const uint64_t str[3] = {uint64_t(2 * D), uint64_t(2 * D) * c.n_slices * c.heads * 2 * D,
                             uint64_t(2 * D) * c.n_slices * c.heads * 2 * D};
    const uint32_t box[4] = {64u, 64u, 1u, 1u};
    if (Runtime::encode_4d(&tm_op, CU_TENSOR_MAP_DATA_TYPE_UINT16,
                           const_cast<uint16_t*>(c.operand), dims, str, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) != 0)
      return SRFTQ_ERR_CUDA;
  }
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  DenseDeqArgs a{c.n_rows, row_blocks, c.n_slices, c.heads, c.scales_in, c.in_stride_rows,
                 c.xhat, c.out_stride_rows, c.lambda, guard};
  constexpr auto K = dequantize_dense_mma_kernel<D, BITS, G>;
  constexpr int smem = L::kBytes + kSmemSlack;
  int bps = 0;
  const int rc = prepare_kernel<K>(smem, L::kThreads, &bps);
  if (rc != SRFTQ_OK) return rc;
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int64_t steps = c.n_slices * row_blocks;
  int64_t per_head = cap / c.heads;
  if (per_head < 1) per_head = 1;
  if (per_head > steps) per_head = steps;
  const int grid = int(per_head * c.heads);
  K<<<grid, L::kThreads, smem, c.stream>>>(tm_c, tm_op, a);
  return finish_launch();
}

int launch_dequantize_dense(const DenseCall& c) {
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  return by_dense_d(c.d, [&](auto d_) {
    constexpr int D = decltype(d_)::value;
    int rc = SRFTQ_ERR_UNSUPPORTED;
    static_for<0, 2>([&](auto b_) {
      constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
      static_for<3, ilog2(D) + 1>([&](auto lg_) {
        constexpr int G = 1 << decltype(lg_)::value;
        if (c.bits == BITS && c.group == G) rc = dequantize_dense_mma<D, BITS, G>(c);
      });
    });
    return rc;
  });
}

int launch_calibrate_dense(const DenseCalibCall& c) {
  // one cluster of kDenseCalibCluster blocks per (slice, head)
  const int64_t blocks = c.n_slices * c.heads * kDenseCalibCluster;
  if (blocks == 0) return SRFTQ_OK;
  if (blocks > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  DenseCalibArgs a{c.n_cal, c.x_stride_rows, c.heads, c.x, c.operand, c.lambda_out, c.n_slices,
                   guard};
  return by_dense_d(c.d, [&](auto d_) {
    constexpr int D = decltype(d_)::value;
    constexpr auto K = dense_calibrate_kernel<D>;
    constexpr int smem = DenseTile<D>::kBytes;
    const int rc = prepare_smem<K>(smem);
    if (rc != SRFTQ_OK) return rc;
    K<<<int(blocks), kDenseThreads, smem, c.stream>>>(a);
    return finish_launch();
  });
}

}  // namespace srftq
