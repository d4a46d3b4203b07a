// Rotation-only and calibration kernels for d = 256: two threads per vector
// (lanes 2i and 2i + 1), plain global loads, the lane-pair transforms of
// transform256.cuh. Neither is on the bandwidth-critical path.
#pragma once

#include "aux.cuh"
#include "transform256.cuh"

namespace srftq {

// Gain from a lane slot value to the packed coordinate (forward) for
// coordinate pair `pair` (SRFT: pair 0 of lane 0 holds 2 X_0 and 2 X_128).
template <int ROT>
__device__ __forceinline__ float gain256(int pair) {
  if constexpr (ROT == kSRHT) {
    return 0.0625f;
  } else {
    return pair == 0 ? 0.03125f : 0.04419417382415922f;   // 1/32, sqrt(2)/32
  }
}

// Inverse: from the packed coordinate to the lane slot value (SRFT: X / 256).
template <int ROT>
__device__ __forceinline__ float igain256(int pair) {
  if constexpr (ROT == kSRHT) {
    return 0.0625f;
  } else {
    return pair == 0 ? 0.0625f : 0.04419417382415922f;    // 1/16, 1/(16 sqrt(2))
  }
}

// Transform of vector xv (fp16, signs sgn) by lane half p (slot -> pair map
// of transform256.cuh).
template <int ROT>
__device__ __forceinline__ void rotate256_lane(const uint16_t* xv, const int8_t* sgn, bool p,
                                               float2 (&v)[64]) {
  const uint4* x4 = reinterpret_cast<const uint4*>(xv);
  if constexpr (ROT == kSRFT) {
    uint32_t xw[64], sgw[64];
    const uint32_t selp = p ? 0x7632u : 0x5410u;
    static_for<0, 32>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const uint4 w = x4[ci];
      xw[2 * ci] = __byte_perm(w.x, w.y, selp);
      xw[2 * ci + 1] = __byte_perm(w.z, w.w, selp);
    });
    static_for<0, 64>([&](auto m_) {
      constexpr int m = decltype(m_)::value;
      sgw[m] = sign_halves(sgn[4 * m + (p ? 1 : 0)], sgn[4 * m + 2 + (p ? 1 : 0)]);
    });
    srft256_forward(xw, sgw, p, v);
  } else {
    static_for<0, 16>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const uint4 wl = x4[ci], wh = x4[16 + ci];
      const uint32_t l[4] = {wl.x, wl.y, wl.z, wl.w}, hh[4] = {wh.x, wh.y, wh.z, wh.w};
      static_for<0, 4>([&](auto k_) {
        constexpr int m = 4 * ci + decltype(k_)::value;
        const uint32_t sl = sign_halves(sgn[2 * m], sgn[2 * m + 1]);
        uint32_t sh = sign_halves(sgn[128 + 2 * m], sgn[129 + 2 * m]);
        if (p) sh ^= 0x80008000u;
        v[m] = srht256_plane0(l[decltype(k_)::value], hh[decltype(k_)::value], sl, sh);
      });
    });
    wht_packed_planes<128>(v);
  }
}

template <int ROT>
__global__ void __launch_bounds__(128) rotate256_kernel(const RotateArgs a) {
  const int64_t total = a.n_slices * a.n_rows * a.heads;
  const bool p = threadIdx.x & 1;
  // whole warps iterate together (the lane pairs exchange with shuffles)
  for (int64_t base = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) / 2; ;
       base += int64_t(gridDim.x) * blockDim.x / 2) {
    const int64_t warp_first = base - ((threadIdx.x & 31) >> 1);
    if (warp_first >= total) break;
    const bool valid = base < total;
    const int64_t v_id = valid ? base : total - 1;
    const int h = int(v_id % a.heads);
    const int64_t sr = v_id / a.heads;
    const int64_t rr = sr % a.n_rows;
    const int64_t s = sr / a.n_rows;
    int64_t vx = (s * a.x_slice_stride_rows + rr) * a.heads + h;
    if (!dbg_ok(vx < vec_limit(a.n_slices, a.x_slice_stride_rows, a.n_rows, a.heads), a.guard))
      vx = 0;   // debug build: recorded, read vector 0 instead
    const uint16_t* xv = a.x + vx * 256;
    const int64_t tab = (s * a.heads + h) * 256;
    float2 v[64];
    rotate256_lane<ROT>(xv, a.signs + tab, p, v);
    if (valid && dbg_ok(v_id < total, a.guard)) {
      float* yv = a.y + v_id * 256;
      static_for<0, 64>([&](auto j_) {
        constexpr int j = decltype(j_)::value;
        const int pair = pair256<ROT>(j, p);
        const float g = gain256<ROT>(pair);
        const float m0 = a.lambda ? __fdiv_rn(g, a.lambda[tab + 2 * pair]) : g;
        const float m1 = a.lambda ? __fdiv_rn(g, a.lambda[tab + 2 * pair + 1]) : g;
        reinterpret_cast<float2*>(yv)[pair] = make_float2(v[j].x * m0, v[j].y * m1);
      });
    }
  }
}

// One cluster of kCalibCluster blocks per (slice, head), block r taking the
// batches of 64 rows starting at 64 (r + kCalibCluster b); two threads per
// row; rank 0 adds the blocks' float64 partial sums in rank order through
// distributed shared memory (as calibrate_kernel).
template <int ROT>
__global__ void __cluster_dims__(kCalibCluster, 1, 1) __launch_bounds__(128)
    calibrate256_kernel(const CalibArgs a) {
  __shared__ float sq[kCalibRows / 2][257];
  __shared__ double part[256];
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int shd = blockIdx.x / kCalibCluster;
  const int s = shd / a.heads;
  const int h = shd % a.heads;
  const int64_t tab = (int64_t(s) * a.heads + h) * 256;
  const bool p = threadIdx.x & 1;
  const int rl = threadIdx.x >> 1;   // row within a batch of 64 (two threads per row)
  double acc0 = 0.0, acc1 = 0.0;
  for (int64_t b = int64_t(kCalibRows) * rank; b < a.n_cal;
       b += int64_t(kCalibRows) * kCalibCluster) {
    const int64_t rr = b + rl;
    const bool valid = rr < a.n_cal;
    const int64_t rc = valid ? rr : 0;
    int64_t vx = (int64_t(s) * a.x_slice_stride_rows + rc) * a.heads + h;
    if (!dbg_ok(vx < vec_limit(a.n_slices, a.x_slice_stride_rows, a.n_cal, a.heads), a.guard))
      vx = 0;   // debug build: recorded, read vector 0 instead
    const uint16_t* xv = a.x + vx * 256;
    float2 v[64];
    rotate256_lane<ROT>(xv, a.signs + tab, p, v);
    // two passes of 32 rows each through a 32 x 256 shared tile
    for (int half = 0; half < 2; ++half) {
      if ((rl >> 5) == half) {
        static_for<0, 64>([&](auto j_) {
          constexpr int j = decltype(j_)::value;
          const int pair = pair256<ROT>(j, p);
          const float g = gain256<ROT>(pair);
          const float y0 = valid ? v[j].x * g : 0.0f, y1 = valid ? v[j].y * g : 0.0f;
          sq[rl & 31][2 * pair] = y0 * y0;
          sq[rl & 31][2 * pair + 1] = y1 * y1;
        });
      }
      __syncthreads();
      for (int i = 0; i < 32; ++i) {
        acc0 += double(sq[i][threadIdx.x]);
        acc1 += double(sq[i][threadIdx.x + 128]);
      }
      __syncthreads();
    }
  }
  part[threadIdx.x] = acc0;
  part[threadIdx.x + 128] = acc1;
  cluster.sync();
  if (rank == 0) {
    double t0 = 0.0, t1 = 0.0;
    for (int r = 0; r < kCalibCluster; ++r) {
      const double* q = cluster.map_shared_rank(part, r);
      t0 += q[threadIdx.x];
      t1 += q[threadIdx.x + 128];
    }
    if (dbg_ok(tab + threadIdx.x + 128 < a.n_slices * a.heads * 256, a.guard)) {
      a.lambda_out[tab + threadIdx.x] = t0 > 0.0 ? float(sqrt(t0 / double(a.n_cal))) : 1.0f;
      a.lambda_out[tab + threadIdx.x + 128] =
          t1 > 0.0 ? float(sqrt(t1 / double(a.n_cal))) : 1.0f;
    }
  }
  cluster.sync();   // the other blocks keep their shared memory until rank 0 is done
}

}  // namespace srftq
