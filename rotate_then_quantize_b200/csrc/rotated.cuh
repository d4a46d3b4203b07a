// Decode in the rotated domain. R is orthogonal ("When Quantization Is Free",
// Methodology 1), so q . x = (R q) . (R x): attention can score a rotated
// query against the cache without undoing the rotation of every key, and it
// can accumulate the values in the rotated domain and undo the rotation once
// per output. Two primitives serve that path:
//
//   dequantize_rotated_kernel  yhat'_j = lambda_j * sigma_g * q_j, fp16: the
//       cached vector's reconstruction R xhat in the rotated domain (no
//       inverse transform, no signs). One thread per 8 coordinates, plain
//       vector loads and stores; every byte is touched once.
//   unrotate_kernel            x = s * R^T y (float32 in and out), one thread
//       per vector (d <= 128) or two (d = 256), the inverse transforms of the
//       dequantisers.
#pragma once

#include <cuda_fp16.h>

#include <type_traits>

#include "aux256.cuh"

namespace srftq {

struct RotDequantArgs {
  int64_t n_slices, n_rows, in_slice_stride_rows, out_slice_stride_rows;
  int32_t heads;
  const uint8_t* codes;     // [S][T_in][H][d * bits / 8]
  const uint16_t* scales;   // [S][T_in][H][d / G] fp16
  const float* lambda;      // [S][H][d]
  uint16_t* out;            // [S][T_out][H][d] fp16
  unsigned* guard;          // debug-build index checks
};

// One thread per 8 coordinates (one 16-byte output chunk) of a slice; the
// grid's y dimension walks the slices, so the index arithmetic inside a
// slice is 32-bit (the launcher checks rows x heads x d/8 < 2^32). Codes
// become exact float32 q * sigma without int-to-float conversions: a pair of
// codes is spread into the fp16 pair 1024 + offset + code with one AND-XOR,
// and `fma.rn.f32.f16` multiplies it by the fp16 scale and subtracts the
// offset's product, rounding once (the product is exact).
template <int D, int BITS, int G>
__global__ void __launch_bounds__(256) dequantize_rotated_kernel(const RotDequantArgs a) {
  static_assert(G >= 8 && D % 8 == 0, "8 coordinates of one group per thread");
  constexpr int CPV = D / 8;   // chunks of 8 coordinates per vector
  constexpr int U = 4;         // chunks per thread and step, 256 apart: all loads first
  using CodeT = typename std::conditional<BITS == 4, uint32_t, uint2>::type;
  const uint32_t H = uint32_t(a.heads);
  const uint32_t per_slice = uint32_t(a.n_rows) * H * CPV;
  for (int64_t s = blockIdx.y; s < a.n_slices; s += gridDim.y) {
    const int64_t in_base = s * a.in_slice_stride_rows * H;     // vectors
    const int64_t out_base = s * a.out_slice_stride_rows * H;
    const float* lam_s = a.lambda + s * int64_t(H) * D;
    for (uint32_t base = blockIdx.x * (256u * U) + threadIdx.x; base < per_slice;
         base += gridDim.x * (256u * U)) {
      CodeT w[U];
      uint32_t sw[U];
      float4 l0[U], l1[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t c = base + 256u * u;
        if (c < per_slice) {
          const uint32_t k = c % CPV, vh = c / CPV;   // chunk, (row, head) of the slice
          int64_t vin = in_base + vh;
          if (!dbg_ok(vin < vec_limit(a.n_slices, a.in_slice_stride_rows, a.n_rows, H), a.guard))
            vin = 0;   // debug build: recorded, read vector 0 instead
          const int j0 = 8 * int(k);
          w[u] = *reinterpret_cast<const CodeT*>(a.codes + vin * (D * BITS / 8) + j0 * BITS / 8);
          sw[u] = a.scales[vin * (D / G) + j0 / G];
          const float4* lam = reinterpret_cast<const float4*>(lam_s + (vh % H) * D + j0);
          l0[u] = __ldg(lam);
          l1[u] = __ldg(lam + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t c = base + 256u * u;
        if (c >= per_slice) continue;
        float q[8];   // q_e * sigma, coordinates j0 .. j0 + 7
        if constexpr (BITS == 4) {
          // element 2k in the low nibble of byte k: w >> 4t holds codes t
          // and t + 4 in the low nibbles of its two 16-bit halves
          const float off = -1032.0f * __half2float(__ushort_as_half(uint16_t(sw[u])));
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint32_t hp = ((w[u] >> (4 * t)) & 0x000F000Fu) ^ 0x64086408u;   // 1032 + q
            q[t] = fma_f16<0, 0>(hp, sw[u], off);
            q[t + 4] = fma_f16<1, 0>(hp, sw[u], off);
          }
        } else {
          const float off = -1152.0f * __half2float(__ushort_as_half(uint16_t(sw[u])));
          const uint32_t ww[2] = {w[u].x, w[u].y};
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            // bytes 0, 2 and 1, 3 of each word into fp16 pairs 1152 + q
            const uint32_t h02 = (ww[t] & 0x00FF00FFu) ^ 0x64806480u;
            const uint32_t h13 = ((ww[t] >> 8) & 0x00FF00FFu) ^ 0x64806480u;
            q[4 * t + 0] = fma_f16<0, 0>(h02, sw[u], off);
            q[4 * t + 2] = fma_f16<1, 0>(h02, sw[u], off);
            q[4 * t + 1] = fma_f16<0, 0>(h13, sw[u], off);
            q[4 * t + 3] = fma_f16<1, 0>(h13, sw[u], off);
          }
        }
        const float lv[8] = {l0[u].x, l0[u].y, l0[u].z, l0[u].w,
                             l1[u].x, l1[u].y, l1[u].z, l1[u].w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_f16x2(q[2 * e] * lv[2 * e], q[2 * e + 1] * lv[2 * e + 1]);
        const int64_t vout = out_base + c / CPV;
        if (dbg_ok(vout < vec_limit(a.n_slices, a.out_slice_stride_rows, a.n_rows, H), a.guard))
          *reinterpret_cast<uint4*>(a.out + vout * D + 8 * (c % CPV)) =
              make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

struct UnrotateArgs {
  int64_t n_slices, n_rows, y_slice_stride_rows, x_slice_stride_rows;
  int32_t heads;
  const float* y;         // [S][T_y][H][d] float32, rotated-domain vectors
  const int8_t* signs;    // [S][H][d]
  float* x;               // [S][T_x][H][d] float32
  unsigned* guard;        // debug-build index checks
};

// x = s * R^T y for d <= 128, one thread per vector.
template <int D, int ROT>
__global__ void __launch_bounds__(128) unrotate_kernel(const UnrotateArgs a) {
  const int64_t total = a.n_slices * a.n_rows * a.heads;
  for (int64_t v_id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; v_id < total;
       v_id += int64_t(gridDim.x) * blockDim.x) {
    const int h = int(v_id % a.heads);
    const int64_t sr = v_id / a.heads;
    const int64_t r = sr % a.n_rows;
    const int64_t s = sr / a.n_rows;
    int64_t vy = (s * a.y_slice_stride_rows + r) * a.heads + h;
    if (!dbg_ok(vy < vec_limit(a.n_slices, a.y_slice_stride_rows, a.n_rows, a.heads), a.guard))
      vy = 0;   // debug build: recorded, read vector 0 instead
    const float* yv = a.y + vy * D;
    const int8_t* sg = a.signs + (s * a.heads + h) * D;
    float2 v[D / 2];
    // inverse input: coordinate gain times y (transform.cuh, rotate_inverse)
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 y4 = reinterpret_cast<const float4*>(yv)[ci];
      v[2 * ci] = make_float2(y4.x * gain_f<ROT, D>(4 * ci), y4.y * gain_f<ROT, D>(4 * ci + 1));
      v[2 * ci + 1] =
          make_float2(y4.z * gain_f<ROT, D>(4 * ci + 2), y4.w * gain_f<ROT, D>(4 * ci + 3));
    });
    rotate_inverse<ROT, D>(v);
    const int64_t vxo = (s * a.x_slice_stride_rows + r) * a.heads + h;
    if (!dbg_ok(vxo < vec_limit(a.n_slices, a.x_slice_stride_rows, a.n_rows, a.heads), a.guard))
      continue;
    float* xv = a.x + vxo * D;
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const char4 s4 = reinterpret_cast<const char4*>(sg)[ci];
      reinterpret_cast<float4*>(xv)[ci] =
          make_float4(s4.x < 0 ? -v[2 * ci].x : v[2 * ci].x, s4.y < 0 ? -v[2 * ci].y : v[2 * ci].y,
                      s4.z < 0 ? -v[2 * ci + 1].x : v[2 * ci + 1].x,
                      s4.w < 0 ? -v[2 * ci + 1].y : v[2 * ci + 1].y);
    });
  }
}

// x = s * R^T y for d = 256: two threads per vector (lanes 2i and 2i + 1),
// the lane-pair inverse transforms of transform256.cuh.
template <int ROT>
__global__ void __launch_bounds__(128) unrotate256_kernel(const UnrotateArgs a) {
  const int64_t total = a.n_slices * a.n_rows * a.heads;
  const bool p = threadIdx.x & 1;
  // whole warps iterate together (the lane pairs exchange with shuffles)
  for (int64_t base = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) / 2;;
       base += int64_t(gridDim.x) * blockDim.x / 2) {
    const int64_t warp_first = base - ((threadIdx.x & 31) >> 1);
    if (warp_first >= total) break;
    const bool valid = base < total;
    const int64_t v_id = valid ? base : total - 1;
    const int h = int(v_id % a.heads);
    const int64_t sr = v_id / a.heads;
    const int64_t r = sr % a.n_rows;
    const int64_t s = sr / a.n_rows;
    int64_t vy = (s * a.y_slice_stride_rows + r) * a.heads + h;
    if (!dbg_ok(vy < vec_limit(a.n_slices, a.y_slice_stride_rows, a.n_rows, a.heads), a.guard))
      vy = 0;   // debug build: recorded, read vector 0 instead
    const float* yv = a.y + vy * 256;
    const int8_t* sg = a.signs + (s * a.heads + h) * 256;
    float2 v[64];
    static_for<0, 64>([&](auto j_) {
      constexpr int j = decltype(j_)::value;
      const int pair = pair256<ROT>(j, p);
      const float g = igain256<ROT>(pair);
      const float2 y2 = reinterpret_cast<const float2*>(yv)[pair];
      v[j] = make_float2(y2.x * g, y2.y * g);
    });
    const int64_t vxo = (s * a.x_slice_stride_rows + r) * a.heads + h;
    const bool out_ok = valid && dbg_ok(vxo < vec_limit(a.n_slices, a.x_slice_stride_rows,
                                                        a.n_rows, a.heads),
                                        a.guard);
    float* xv = a.x + vxo * 256;
    auto put = [&](int n, float val) {   // element n, sign applied
      if (out_ok) xv[n] = sg[n] < 0 ? -val : val;
    };
    if constexpr (ROT == kSRFT) {
      float2 us[64];
      srft256_inverse(v, p, us);
      // lane 0 writes the fp16-word pairs 0..63 of the row, lane 1 64..127:
      // word 2k = (u_{4k'}, u_{4k'+1}) with u_even from lane 0, u_odd lane 1
      static_for<0, 32>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        const float2 recv = shfl1(sel2(p, us[k], us[32 + k]));
        const float2 own = sel2(p, us[32 + k], us[k]);
        const float2 ev = sel2(p, recv, own), od = sel2(p, own, recv);
        const int w = (p ? 64 : 0) + 2 * k;   // word w = elements 2w, 2w + 1
        put(2 * w, ev.x);
        put(2 * w + 1, od.x);
        put(2 * w + 2, ev.y);
        put(2 * w + 3, od.y);
      });
    } else {
      float2 lo[32], hi[32];
      srht256_inverse(v, p, lo, hi);
      static_for<0, 32>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        const int wl = (p ? 32 : 0) + k, wh = 64 + (p ? 32 : 0) + k;
        put(2 * wl, lo[k].x);
        put(2 * wl + 1, lo[k].y);
        put(2 * wh, hi[k].x);
        put(2 * wh + 1, hi[k].y);
      });
    }
  }
}

}  // namespace srftq
