// Kernels and launchers for head dimension d = 128. The SRFT quantiser with
// groups of up to 64 runs on the tensor cores (codec_mma.cuh); the SRHT
// quantiser, groups of 128 and both dequantisers run the one-thread-per-vector
// kernels of codec.cuh.
#include "codec_mma.cuh"
#include "launch_impl.cuh"

// 0 routes the SRFT quantiser to the one-thread kernel as well.
#ifndef SRFTQ_MMA128
#define SRFTQ_MMA128 0
#endif

namespace srftq {
namespace {

// Epilogue groups of four warps of the tensor-core quantiser.
#ifndef SRFTQ_MMA_EPI
#define SRFTQ_MMA_EPI 1
#endif
constexpr int kEpiGroups = SRFTQ_MMA_EPI;

template <int BITS, int G>
int quantize_mma_impl(const QuantCall& c) {
  using S = Shape<128, BITS, G>;
  using L = MmaLayout<BITS, G, kEpiGroups>;
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  if (c.n_rows > INT_MAX || c.n_slices > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  int64_t total = 0;
  const TileGeom g = make_geom(c.n_slices, c.n_rows, c.heads, &total);
  if (total > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  const uint32_t hpt = 1u << g.hpt_log2, rpt = uint32_t(kTileRows) >> g.hpt_log2;

  CUtensorMap tm_x, tm_c;
  {
    const uint64_t dims[4] = {128u, uint64_t(c.heads), uint64_t(c.n_rows), uint64_t(c.n_slices)};
    const uint64_t str[3] = {uint64_t(S::XB), uint64_t(c.heads) * S::XB,
                             uint64_t(c.x_slice_stride_rows) * c.heads * S::XB};
    const uint32_t box[4] = {64u, hpt, rpt, 1u};
    if (Runtime::encode_4d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT16, const_cast<uint16_t*>(c.x), dims,
                           str, box, CU_TENSOR_MAP_SWIZZLE_128B) != 0)
      return SRFTQ_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {uint64_t(S::CB), uint64_t(c.heads), uint64_t(c.n_rows),
                              uint64_t(c.n_slices)};
    const uint64_t str[3] = {uint64_t(S::CB), uint64_t(c.heads) * S::CB,
                             uint64_t(c.out_slice_stride_rows) * c.heads * S::CB};
    const uint32_t box[4] = {uint32_t(S::C_SPAN), hpt, rpt, 1u};
    if (Runtime::encode_4d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.codes, dims, str, box,
                           swizzle_mode(S::C_SPAN)) != 0)
      return SRFTQ_ERR_CUDA;
  }
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  QuantArgs a;
  a.g = g;
  a.signs = c.signs;
  a.lambda = c.lambda;
  a.codes = c.codes;
  a.scales = c.scales;
  a.out_slice_stride_rows = c.out_slice_stride_rows;
  a.guard = guard;

  constexpr auto K = quantize_mma_kernel<BITS, G, kEpiGroups>;
  const int smem = L::kBytes + kSmemSlack;
  int bps = 0;
  const int rc = prepare_kernel<K>(smem, L::kThreads, &bps);
  if (rc != SRFTQ_OK) return rc;
  // one CTA per SM: each holds all 512 columns of its SM's tensor memory
  const int64_t blocks = (total + L::kSub - 1) / L::kSub;
  const int64_t sms = Runtime::num_sms();
  const int grid = int(blocks < sms ? blocks : sms);
  K<<<grid, L::kThreads, smem, c.stream>>>(tm_x, tm_c, a);
  return finish_launch();
}

}  // namespace

template <>
int launch_quantize<128>(const QuantCall& c) {
  if (SRFTQ_MMA128 && c.rotation == kSRFT && c.group <= 64)
    return dispatch_config<64>(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto) {
      return quantize_mma_impl<decltype(b_)::value, decltype(g_)::value>(c);
    });
  return dispatch_config<128>(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto r_) {
    return quantize_impl<128, decltype(b_)::value, decltype(g_)::value, decltype(r_)::value>(c);
  });
}

}  // namespace srftq

template int srftq::launch_dequantize<128>(const srftq::DequantCall&);
template int srftq::launch_rotate<128>(const srftq::RotateCall&);
template int srftq::launch_calibrate<128>(const srftq::CalibCall&);
