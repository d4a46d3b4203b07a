// Launchers of the two-warp codec kernels (codec_split.cuh).
#pragma once

#include "codec_split.cuh"
#include "launch_impl.cuh"

namespace srftq {

// Blocks per SM the register budget of the two-warp kernels is sized for:
// d = 256 keeps half a vector (128 coordinates) per thread in 4 blocks
// (8 warps) with the full 255 registers.
constexpr int kSplitMinBlocks = 4;

// Rank-4 tensor maps over (d-bytes-or-elements, H, N, S); an x box is one
// 128-byte piece (64 fp16) of HPT heads x RPT rows, a code box one piece of
// C_SPAN bytes.
template <typename S>
int encode_split_x(CUtensorMap* tm, const uint16_t* base, int64_t H, int64_t N, int64_t Sl,
                   int64_t slice_stride_rows, uint32_t hpt, uint32_t rpt) {
  const uint64_t dims[4] = {uint64_t(2 * S::DH), uint64_t(H), uint64_t(N), uint64_t(Sl)};
  const uint64_t str[3] = {uint64_t(S::XB), uint64_t(H) * S::XB,
                           uint64_t(slice_stride_rows) * H * S::XB};
  const uint32_t box[4] = {uint32_t(S::X_SPAN / 2), hpt, rpt, 1u};
  return Runtime::encode_4d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT16, const_cast<uint16_t*>(base), dims,
                            str, box, swizzle_mode(S::X_SPAN));
}

template <typename S>
int encode_split_codes(CUtensorMap* tm, const uint8_t* base, int64_t H, int64_t N, int64_t Sl,
                       int64_t slice_stride_rows, uint32_t hpt, uint32_t rpt) {
  const uint64_t dims[4] = {uint64_t(S::CB), uint64_t(H), uint64_t(N), uint64_t(Sl)};
  const uint64_t str[3] = {uint64_t(S::CB), uint64_t(H) * S::CB,
                           uint64_t(slice_stride_rows) * H * S::CB};
  const uint32_t box[4] = {uint32_t(S::C_SPAN), hpt, rpt, 1u};
  return Runtime::encode_4d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<uint8_t*>(base), dims,
                            str, box, swizzle_mode(S::C_SPAN));
}

template <int D, int BITS, int G, int ROT>
int quantize_split_impl(const QuantCall& c) {
  using S = SplitShape<D, BITS, G>;
  using Lay = SplitLayout<D, BITS, G, true>;
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  if (c.n_rows > INT_MAX || c.n_slices > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  int64_t total = 0;
  const TileGeom g = make_geom(c.n_slices, c.n_rows, c.heads, &total);
  if (total > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  const uint32_t hpt = 1u << g.hpt_log2, rpt = uint32_t(kTileRows) >> g.hpt_log2;
  CUtensorMap tm_x, tm_c;
  if (encode_split_x<S>(&tm_x, c.x, c.heads, c.n_rows, c.n_slices, c.x_slice_stride_rows, hpt,
                        rpt) != 0 ||
      encode_split_codes<S>(&tm_c, c.codes, c.heads, c.n_rows, c.n_slices,
                            c.out_slice_stride_rows, hpt, rpt) != 0)
    return SRFTQ_ERR_CUDA;
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

  constexpr auto K = quantize_split_kernel<D, BITS, G, ROT, kSplitMinBlocks>;
  const int smem = Lay::kBytes + kSmemSlack;
  int bps = 0;
  const int rc = prepare_kernel<K>(smem, 64, &bps);
  if (rc != SRFTQ_OK) return rc;
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int grid = int(total < cap ? total : cap);
  K<<<grid, 64, smem, c.stream>>>(tm_x, tm_c, a);
  return finish_launch();
}

template <int D, int BITS, int G, int ROT>
int dequantize_split_impl(const DequantCall& c) {
  using S = SplitShape<D, BITS, G>;
  using Lay = SplitLayout<D, BITS, G, false>;
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  if (c.n_rows > INT_MAX || c.n_slices > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  int64_t total = 0;
  const TileGeom g = make_geom(c.n_slices, c.n_rows, c.heads, &total);
  if (total > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  const uint32_t hpt = 1u << g.hpt_log2, rpt = uint32_t(kTileRows) >> g.hpt_log2;
  CUtensorMap tm_c, tm_x;
  if (encode_split_codes<S>(&tm_c, c.codes, c.heads, c.n_rows, c.n_slices,
                            c.in_slice_stride_rows, hpt, rpt) != 0 ||
      encode_split_x<S>(&tm_x, c.xhat, c.heads, c.n_rows, c.n_slices, c.out_slice_stride_rows,
                        hpt, rpt) != 0)
    return SRFTQ_ERR_CUDA;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  DequantArgs a;
  a.g = g;
  a.signs = c.signs;
  a.lambda = c.lambda;
  a.codes = c.codes;
  a.scales = c.scales;
  a.in_slice_stride_rows = c.in_slice_stride_rows;
  a.xhat = c.xhat;
  a.out_slice_stride_rows = c.out_slice_stride_rows;
  a.guard = guard;

  constexpr auto K = dequantize_split_kernel<D, BITS, G, ROT, kSplitMinBlocks>;
  const int smem = Lay::kBytes + kSmemSlack;
  int bps = 0;
  const int rc = prepare_kernel<K>(smem, 64, &bps);
  if (rc != SRFTQ_OK) return rc;
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int grid = int(total < cap ? total : cap);
  K<<<grid, 64, smem, c.stream>>>(tm_c, tm_x, a);
  return finish_launch();
}

// Calls f(Int<BITS>, Int<G>, Int<ROT>) for the run-time configuration, groups
// of 8 .. GMAX coordinates.
template <int GMAX, typename F>
int dispatch_split(int bits, int group, int rot, F&& f) {
  int rc = SRFTQ_ERR_UNSUPPORTED;
  static_for<0, 2>([&](auto b_) {
    constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
    static_for<3, ilog2(GMAX) + 1>([&](auto lg_) {
      constexpr int G = 1 << decltype(lg_)::value;
      static_for<0, 2>([&](auto r_) {
        constexpr int ROT = decltype(r_)::value;
        if (bits == BITS && group == G && rot == ROT) rc = f(Int<BITS>{}, Int<G>{}, Int<ROT>{});
      });
    });
  });
  return rc;
}

}  // namespace srftq
