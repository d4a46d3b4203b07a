// Per-d launch implementation, included by one translation unit per head
// dimension (launch_d16.cu ... launch_d128.cu).
#pragma once

#include <atomic>
#include <climits>
#include <cstring>

#include "aux.cuh"
#include "codec.cuh"
#include "launch.cuh"
#include "rotated.cuh"

namespace srftq {

// Launch shapes: warps per block and the blocks per SM the register budget
// is sized for (their product is the resident warps per SM), and input
// stages per warp. Measured on B200: one warp per block (a block's only
// warp has index 0, so the tile walk and the TMA operands are warp-uniform
// and live in uniform registers); one input stage, refilled as soon as it is
// read, hides the load as well as two and leaves shared memory for the
// per-head tables; d = 128 runs 8 warps per SM with the full register
// budget (at 12 the transform spills), d <= 64 runs 12.
#ifndef SRFTQ_Q_WPC
#define SRFTQ_Q_WPC 1
#endif
#ifndef SRFTQ_Q_MINB
#define SRFTQ_Q_MINB 0   // 0: by head dimension (q_min_blocks)
#endif
#ifndef SRFTQ_D_WPC
#define SRFTQ_D_WPC 1
#endif
#ifndef SRFTQ_D_MINB
#define SRFTQ_D_MINB 0   // 0: by head dimension (q_min_blocks)
#endif
#ifndef SRFTQ_NST
#define SRFTQ_NST 1
#endif
constexpr int kQWPC = SRFTQ_Q_WPC;
constexpr int kDWPC = SRFTQ_D_WPC;
// Blocks per SM the register budget is sized for: d <= 64 keeps its vector
// in <= 168 registers without spills, so 12 one-warp blocks fit; d = 128
// needs the full 255 registers (8 blocks).
template <int D, int MINB>
constexpr int min_blocks() {
  return MINB > 0 ? MINB : (D <= 64 ? 12 : 8);
}
constexpr int kNST = SRFTQ_NST;

inline CUtensorMapSwizzle swizzle_mode(int span) {
  switch (span) {
    case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
    case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
    case 128: return CU_TENSOR_MAP_SWIZZLE_128B;
    default: return CU_TENSOR_MAP_SWIZZLE_NONE;
  }
}

// Sets the dynamic shared-memory limit of kernel K once per device and
// caches its occupancy (blocks per SM) for the block shape it is launched
// with.
template <auto K>
int prepare_kernel(int smem_bytes, int threads, int* blocks_per_sm) {
  static std::atomic<uint64_t> attr_done{0};
  static std::atomic<int> bps{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SRFTQ_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    if (smem_bytes > 48 * 1024 &&
        cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
            cudaSuccess)
      return SRFTQ_ERR_CUDA;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  int b = bps.load(std::memory_order_acquire);
  if (b == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, K, threads, smem_bytes) != cudaSuccess)
      return SRFTQ_ERR_CUDA;
    if (b < 1) return SRFTQ_ERR_CUDA;
    bps.store(b, std::memory_order_release);
  }
  *blocks_per_sm = b;
  return SRFTQ_OK;
}

// The dynamic shared-memory opt-in alone (for cluster kernels, whose
// occupancy is not a per-SM block count).
template <auto K>
int prepare_smem(int smem_bytes) {
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SRFTQ_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    if (smem_bytes > 48 * 1024 &&
        cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
            cudaSuccess)
      return SRFTQ_ERR_CUDA;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  return SRFTQ_OK;
}

// Calls f(Int<BITS>, Int<G>, Int<ROT>) for the run-time configuration.
template <int D, typename F>
int dispatch_config(int bits, int group, int rot, F&& f) {
  int rc = SRFTQ_ERR_UNSUPPORTED;
  static_for<0, 2>([&](auto b_) {
    constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
    static_for<3, ilog2(D) + 1>([&](auto lg_) {
      constexpr int G = 1 << decltype(lg_)::value;
      static_for<0, 2>([&](auto r_) {
        constexpr int ROT = decltype(r_)::value;
        if (bits == BITS && group == G && rot == ROT) rc = f(Int<BITS>{}, Int<G>{}, Int<ROT>{});
      });
    });
  });
  return rc;
}

inline int finish_launch() {
  return cudaGetLastError() == cudaSuccess ? SRFTQ_OK : SRFTQ_ERR_CUDA;
}

// Tile geometry for H heads: HPT = 2^hpt_log2 heads x (32 / HPT) rows.
inline TileGeom make_geom(int64_t n_slices, int64_t n_rows, int heads, int64_t* total) {
  const int lg = heads_per_tile_log2(heads);
  const int64_t rpt = kTileRows >> lg;
  const int64_t row_blocks = (n_rows + rpt - 1) / rpt;
  const int64_t head_blocks = heads >> lg;
  *total = n_slices * head_blocks * row_blocks;
  return TileGeom{heads, int32_t(row_blocks), int32_t(n_rows), int32_t(*total),
                  int32_t(n_slices), lg, int32_t(head_blocks)};
}

template <int D, int BITS, int G, int ROT>
int quantize_impl(const QuantCall& c) {
  using S = Shape<D, BITS, G>;
  using Lay = WarpLayout<D, BITS, G, kNST, true>;
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  if (c.n_rows > INT_MAX || c.n_slices > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  int64_t total = 0;
  const TileGeom g = make_geom(c.n_slices, c.n_rows, c.heads, &total);
  if (total > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  const uint32_t hpt = 1u << g.hpt_log2, rpt = uint32_t(kTileRows) >> g.hpt_log2;

  CUtensorMap tm_x, tm_c;
  std::memset(&tm_c, 0, sizeof(tm_c));
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(c.heads), uint64_t(c.n_rows),
                              uint64_t(c.n_slices)};
    const uint64_t str[3] = {uint64_t(S::XB), uint64_t(c.heads) * S::XB,
                             uint64_t(c.x_slice_stride_rows) * c.heads * S::XB};
    const uint32_t box[4] = {uint32_t(S::X_SPAN / 2), hpt, rpt, 1u};
    if (Runtime::encode_4d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT16, const_cast<uint16_t*>(c.x), dims,
                           str, box, swizzle_mode(S::X_SPAN)) != 0)
      return SRFTQ_ERR_CUDA;
  }
  if constexpr (S::CODES_TMA) {
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

  constexpr auto K = quantize_kernel<D, BITS, G, ROT, kQWPC, kNST, min_blocks<D, SRFTQ_Q_MINB>()>;
  const int smem = kQWPC * Lay::kWarpBytes + kSmemSlack;
  int bps = 0;
  int rc = prepare_kernel<K>(smem, kQWPC * 32, &bps);
  if (rc != SRFTQ_OK) return rc;
  const int64_t want = (total + kQWPC - 1) / kQWPC;
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int grid = int(want < cap ? want : cap);
  K<<<grid, kQWPC * 32, smem, c.stream>>>(tm_x, tm_c, a);
  return finish_launch();
}

template <int D, int BITS, int G, int ROT>
int dequantize_impl(const DequantCall& c) {
  using S = Shape<D, BITS, G>;
  using Lay = WarpLayout<D, BITS, G, kNST, false>;
  if (c.n_slices == 0 || c.n_rows == 0) return SRFTQ_OK;
  if (c.n_rows > INT_MAX || c.n_slices > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  int64_t total = 0;
  const TileGeom g = make_geom(c.n_slices, c.n_rows, c.heads, &total);
  if (total > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  const uint32_t hpt = 1u << g.hpt_log2, rpt = uint32_t(kTileRows) >> g.hpt_log2;

  CUtensorMap tm_c, tm_x;
  std::memset(&tm_c, 0, sizeof(tm_c));
  if constexpr (S::CODES_TMA) {
    const uint64_t dims[4] = {uint64_t(S::CB), uint64_t(c.heads), uint64_t(c.n_rows),
                              uint64_t(c.n_slices)};
    const uint64_t str[3] = {uint64_t(S::CB), uint64_t(c.heads) * S::CB,
                             uint64_t(c.in_slice_stride_rows) * c.heads * S::CB};
    const uint32_t box[4] = {uint32_t(S::C_SPAN), hpt, rpt, 1u};
    if (Runtime::encode_4d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<uint8_t*>(c.codes),
                           dims, str, box, swizzle_mode(S::C_SPAN)) != 0)
      return SRFTQ_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(c.heads), uint64_t(c.n_rows),
                              uint64_t(c.n_slices)};
    const uint64_t str[3] = {uint64_t(S::XB), uint64_t(c.heads) * S::XB,
                             uint64_t(c.out_slice_stride_rows) * c.heads * S::XB};
    const uint32_t box[4] = {uint32_t(S::X_SPAN / 2), hpt, rpt, 1u};
    if (Runtime::encode_4d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT16, c.xhat, dims, str, box,
                           swizzle_mode(S::X_SPAN)) != 0)
      return SRFTQ_ERR_CUDA;
  }
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

  constexpr auto K = dequantize_kernel<D, BITS, G, ROT, kDWPC, kNST, min_blocks<D, SRFTQ_D_MINB>()>;
  const int smem = kDWPC * Lay::kWarpBytes + kSmemSlack;
  int bps = 0;
  int rc = prepare_kernel<K>(smem, kDWPC * 32, &bps);
  if (rc != SRFTQ_OK) return rc;
  const int64_t want = (total + kDWPC - 1) / kDWPC;
  const int64_t cap = int64_t(Runtime::num_sms()) * bps;
  const int grid = int(want < cap ? want : cap);
  K<<<grid, kDWPC * 32, smem, c.stream>>>(tm_c, tm_x, a);
  return finish_launch();
}

template <int D>
int launch_quantize(const QuantCall& c) {
  return dispatch_config<D>(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto r_) {
    return quantize_impl<D, decltype(b_)::value, decltype(g_)::value, decltype(r_)::value>(c);
  });
}

template <int D>
int launch_dequantize(const DequantCall& c) {
  return dispatch_config<D>(c.bits, c.group, c.rotation, [&](auto b_, auto g_, auto r_) {
    return dequantize_impl<D, decltype(b_)::value, decltype(g_)::value, decltype(r_)::value>(c);
  });
}

template <int D>
int launch_rotate(const RotateCall& c) {
  const int64_t total = c.n_slices * c.n_rows * c.heads;
  if (total == 0) return SRFTQ_OK;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  RotateArgs a{c.n_slices, c.n_rows, c.x_slice_stride_rows, c.heads, c.x, c.signs, c.lambda, c.y,
               guard};
  const int64_t want = (total + 127) / 128;
  const int64_t cap = int64_t(Runtime::num_sms()) * 16;
  const int grid = int(want < cap ? want : cap);
  if (c.rotation == kSRFT)
    rotate_kernel<D, kSRFT><<<grid, 128, 0, c.stream>>>(a);
  else
    rotate_kernel<D, kSRHT><<<grid, 128, 0, c.stream>>>(a);
  return finish_launch();
}

template <int D>
int launch_calibrate(const CalibCall& c) {
  const int64_t blocks = c.n_slices * c.heads * kCalibCluster;   // one cluster per (slice, head)
  if (blocks == 0) return SRFTQ_OK;
  if (blocks > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  CalibArgs a{c.n_cal, c.x_slice_stride_rows, c.heads, c.x, c.signs, c.lambda_out, c.n_slices,
              guard};
  if (c.rotation == kSRFT)
    calibrate_kernel<D, kSRFT><<<int(blocks), kCalibRows, 0, c.stream>>>(a);
  else
    calibrate_kernel<D, kSRHT><<<int(blocks), kCalibRows, 0, c.stream>>>(a);
  return finish_launch();
}

template <int D>
int launch_dequantize_rotated(const RotDequantCall& c) {
  const int64_t per_slice = c.n_rows * c.heads * (D / 8);
  if (per_slice == 0 || c.n_slices == 0) return SRFTQ_OK;
  if (per_slice >= (int64_t(1) << 32)) return SRFTQ_ERR_UNSUPPORTED;   // 32-bit in-slice index
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  RotDequantArgs a{c.n_slices, c.n_rows, c.in_slice_stride_rows, c.out_slice_stride_rows,
                   c.heads, c.codes, c.scales, c.lambda, c.out, guard};
  // y walks the slices; x covers a slice, about 8 blocks of 256 per SM in all
  const int64_t gy = c.n_slices < 65535 ? c.n_slices : 65535;
  const int64_t cap_x = (int64_t(Runtime::num_sms()) * 8 + gy - 1) / gy;
  const int64_t want_x = (per_slice + 1023) / 1024;   // 4 chunks per thread and step
  const dim3 grid(unsigned(want_x < cap_x ? want_x : cap_x), unsigned(gy));
  int rc = SRFTQ_ERR_UNSUPPORTED;
  static_for<0, 2>([&](auto b_) {
    constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
    static_for<3, ilog2(D) + 1>([&](auto lg_) {
      constexpr int G = 1 << decltype(lg_)::value;
      if (c.bits == BITS && c.group == G) {
        dequantize_rotated_kernel<D, BITS, G><<<grid, 256, 0, c.stream>>>(a);
        rc = finish_launch();
      }
    });
  });
  return rc;
}

template <int D>
int launch_unrotate(const UnrotateCall& c) {
  const int64_t total = c.n_slices * c.n_rows * c.heads;
  if (total == 0) return SRFTQ_OK;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  UnrotateArgs a{c.n_slices, c.n_rows, c.y_slice_stride_rows, c.x_slice_stride_rows, c.heads,
                 c.y, c.signs, c.x, guard};
  const int64_t want = (total + 127) / 128;
  const int64_t cap = int64_t(Runtime::num_sms()) * 16;
  const int grid = int(want < cap ? want : cap);
  if (c.rotation == kSRFT)
    unrotate_kernel<D, kSRFT><<<grid, 128, 0, c.stream>>>(a);
  else
    unrotate_kernel<D, kSRHT><<<grid, 128, 0, c.stream>>>(a);
  return finish_launch();
}

}  // namespace srftq

#define SRFTQ_INSTANTIATE_D(D)                                        \
  template int srftq::launch_quantize<D>(const srftq::QuantCall&);     \
  template int srftq::launch_dequantize<D>(const srftq::DequantCall&); \
  template int srftq::launch_rotate<D>(const srftq::RotateCall&);      \
  template int srftq::launch_calibrate<D>(const srftq::CalibCall&);       \
  template int srftq::launch_dequantize_rotated<D>(const srftq::RotDequantCall&); \
  template int srftq::launch_unrotate<D>(const srftq::UnrotateCall&);
