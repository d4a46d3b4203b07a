// Kernels and launchers for head dimension d = 256 (two role warps per block
// for the codec; groups of 8 to 64 coordinates).
#include "aux256.cuh"
#include "codec256.cuh"
#include "launch_impl.cuh"

namespace srftq {
namespace {

// d = 256 codec launch shape: blocks of two role warps, 4 blocks (8 warps)
// per SM with the full register budget.
constexpr int kMinBlocks256 = 4;

// Calls f(Int<BITS>, Int<G>, Int<ROT>) for the run-time configuration.
template <typename F>
int dispatch_config256(int bits, int group, int rot, F&& f) {
  int rc = SRFTQ_ERR_UNSUPPORTED;
  static_for<0, 2>([&](auto b_) {
    constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
    static_for<3, 7>([&](auto lg_) {
      constexpr int G = 1 << decltype(lg_)::value;
      static_for<0, 2>([&](auto r_) {
        constexpr int ROT = decltype(r_)::value;
        if (bits == BITS && group == G && rot == ROT) rc = f(Int<BITS>{}, Int<G>{}, Int<ROT>{});
      });
    });
  });
  return rc;
}

// Rank-4 tensor maps over (d-bytes-or-elements, H, N, S); a box is one
// 128-byte piece of HPT heads x RPT rows (a tile of 32 vectors).
int encode_x256(CUtensorMap* tm, const uint16_t* base, int64_t H, int64_t N, int64_t S,
                int64_t slice_stride_rows, uint32_t hpt, uint32_t rpt) {
  const uint64_t dims[4] = {256u, uint64_t(H), uint64_t(N), uint64_t(S)};
  const uint64_t str[3] = {512u, uint64_t(H) * 512u, uint64_t(slice_stride_rows) * H * 512u};
  const uint32_t box[4] = {64u, hpt, rpt, 1u};
  return Runtime::encode_4d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT16, const_cast<uint16_t*>(base), dims,
                            str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

int encode_codes256(CUtensorMap* tm, const uint8_t* base, int cb, int64_t H, int64_t N, int64_t S,
                    int64_t slice_stride_rows, uint32_t hpt, uint32_t rpt) {
  const uint64_t dims[4] = {uint64_t(cb), uint64_t(H), uint64_t(N), uint64_t(S)};
  const uint64_t str[3] = {uint64_t(cb), uint64_t(H) * cb, uint64_t(slice_stride_rows) * H * cb};
  const uint32_t box[4] = {128u, hpt, rpt, 1u};
  return Runtime::encode_4d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<uint8_t*>(base), dims,
                            str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BITS, int G, int ROT>
int quantize256_impl(const QuantCall& c) {
  using S = Shape256<BITS, G>;
  using Lay = BlockLayout256<BITS, G, true>;
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  if (c.n_rows > INT_MAX || c.n_slices > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  int64_t total = 0;
  const TileGeom g = make_geom(c.n_slices, c.n_rows, c.heads, &total);
  if (total > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  const uint32_t hpt = 1u << g.hpt_log2, rpt = uint32_t(kTileRows) >> g.hpt_log2;
  CUtensorMap tm_x, tm_c;
  if (encode_x256(&tm_x, c.x, c.heads, c.n_rows, c.n_slices, c.x_slice_stride_rows, hpt, rpt) != 0 ||
      encode_codes256(&tm_c, c.codes, S::CB, c.heads, c.n_rows, c.n_slices,
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

  constexpr auto K = quantize256_kernel<BITS, G, ROT, kMinBlocks256>;
  const int smem = Lay::kBytes + kSmemSlack;
  int bps = 0;
  const int rc = prepare_kernel<K>(smem, 64, &bps);
  if (rc != SRFTQ_OK) return rc;
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int grid = int(total < cap ? total : cap);
  K<<<grid, 64, smem, c.stream>>>(tm_x, tm_c, a);
  return finish_launch();
}

template <int BITS, int G, int ROT>
int dequantize256_impl(const DequantCall& c) {
  using S = Shape256<BITS, G>;
  using Lay = BlockLayout256<BITS, G, false>;
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  if (c.n_rows > INT_MAX || c.n_slices > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  int64_t total = 0;
  const TileGeom g = make_geom(c.n_slices, c.n_rows, c.heads, &total);
  if (total > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  const uint32_t hpt = 1u << g.hpt_log2, rpt = uint32_t(kTileRows) >> g.hpt_log2;
  CUtensorMap tm_c, tm_x;
  if (encode_codes256(&tm_c, c.codes, S::CB, c.heads, c.n_rows, c.n_slices,
                      c.in_slice_stride_rows, hpt, rpt) != 0 ||
      encode_x256(&tm_x, c.xhat, c.heads, c.n_rows, c.n_slices, c.out_slice_stride_rows, hpt,
                  rpt) != 0)
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

  constexpr auto K = dequantize256_kernel<BITS, G, ROT, kMinBlocks256>;
  const int smem = Lay::kBytes + kSmemSlack;
  int bps = 0;
  const int rc = prepare_kernel<K>(smem, 64, &bps);
  if (rc != SRFTQ_OK) return rc;
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int grid = int(total < cap ? total : cap);
  K<<<grid, 64, smem, c.stream>>>(tm_c, tm_x, a);
  return finish_launch();
}

}  // namespace

template <>
int launch_quantize<256>(const QuantCall& c) {
  return dispatch_config256(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto r_) {
    return quantize256_impl<decltype(b_)::value, decltype(g_)::value, decltype(r_)::value>(c);
  });
}

template <>
int launch_dequantize<256>(const DequantCall& c) {
  return dispatch_config256(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto r_) {
    return dequantize256_impl<decltype(b_)::value, decltype(g_)::value, decltype(r_)::value>(c);
  });
}

template <>
int launch_rotate<256>(const RotateCall& c) {
  const int64_t total = c.n_slices * c.n_rows * c.heads;
  if (total == 0) return SRFTQ_OK;
  RotateArgs a{c.n_slices, c.n_rows, c.x_slice_stride_rows, c.heads, c.x, c.signs, c.lambda, c.y};
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
  CalibArgs a{c.n_cal, c.x_slice_stride_rows, c.heads, c.x, c.signs, c.lambda_out};
  if (c.rotation == kSRFT)
    calibrate256_kernel<kSRFT><<<int(blocks), 128, 0, c.stream>>>(a);
  else
    calibrate256_kernel<kSRHT><<<int(blocks), 128, 0, c.stream>>>(a);
  return finish_launch();
}

}  // namespace srftq
