// Rotation-only and calibration kernels. They use the same per-thread
// transforms as the codec kernels but plain global loads: neither is on the
// bandwidth-critical path (the rotation kernel exists for parity checks, the
// calibration reads n_cal rows per (slice, head) once).
#pragma once

#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "codec.cuh"

namespace srftq {

// Loads vector x (fp16, 16-byte aligned) as fp16 pairs and the fp16 +-1
// sign pairs of its (slice, head) row.
template <int D>
__device__ __forceinline__ void load_vector(const uint16_t* x, const int8_t* sgn,
                                            uint32_t (&xw)[D / 2], uint32_t (&sgw)[D / 2]) {
  static_for<0, D / 8>([&](auto c_) {
    constexpr int ci = decltype(c_)::value;
    const uint4 raw = reinterpret_cast<const uint4*>(x)[ci];
    xw[4 * ci + 0] = raw.x;
    xw[4 * ci + 1] = raw.y;
    xw[4 * ci + 2] = raw.z;
    xw[4 * ci + 3] = raw.w;
  });
  static_for<0, D / 2>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    sgw[m] = sign_halves(sgn[2 * m], sgn[2 * m + 1]);
  });
}

struct RotateArgs {
  int64_t n_slices, n_rows, x_slice_stride_rows;
  int32_t heads;
  const uint16_t* x;
  const int8_t* signs;
  const float* lambda;  // may be null
  float* y;
  unsigned* guard;      // debug-build index checks
};

// y = R (s * x) [/ lambda], one thread per vector, grid-stride.
template <int D, int ROT>
__global__ void __launch_bounds__(128) rotate_kernel(const RotateArgs a) {
  const int64_t total = a.n_slices * a.n_rows * a.heads;
  for (int64_t v_id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; v_id < total;
       v_id += int64_t(gridDim.x) * blockDim.x) {
    const int h = int(v_id % a.heads);
    const int64_t sr = v_id / a.heads;
    const int64_t r = sr % a.n_rows;
    const int64_t s = sr / a.n_rows;
    int64_t vx = (s * a.x_slice_stride_rows + r) * a.heads + h;
    if (!dbg_ok(vx < vec_limit(a.n_slices, a.x_slice_stride_rows, a.n_rows, a.heads), a.guard))
      vx = 0;   // debug build: recorded, read vector 0 instead
    const uint16_t* xv = a.x + vx * D;
    const int64_t tab = (s * a.heads + h) * D;
    uint32_t xw[D / 2], sgw[D / 2];
    load_vector<D>(xv, a.signs + tab, xw, sgw);
    float2 v[D / 2];
    rotate_forward<ROT, D>(xw, sgw, v);
    if (!dbg_ok(v_id < a.n_slices * a.n_rows * a.heads, a.guard)) continue;
    float* yv = a.y + v_id * D;
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      float m[4];
      static_for<0, 4>([&](auto k_) {
        constexpr int j = 4 * ci + decltype(k_)::value;
        const float g = gain_f<ROT, D>(j);
        m[decltype(k_)::value] = a.lambda ? __fdiv_rn(g, a.lambda[tab + j]) : g;
      });
      reinterpret_cast<float4*>(yv)[ci] = make_float4(v[2 * ci].x * m[0], v[2 * ci].y * m[1],
                                                      v[2 * ci + 1].x * m[2],
                                                      v[2 * ci + 1].y * m[3]);
    });
  }
}

struct CalibArgs {
  int64_t n_cal, x_slice_stride_rows;
  int32_t heads;
  const uint16_t* x;
  const int8_t* signs;
  float* lambda_out;
  int64_t n_slices;     // debug-build index checks
  unsigned* guard;
};

constexpr int kCalibRows = 64;     // rows rotated per batch
constexpr int kCalibCluster = 8;   // blocks (a thread-block cluster) per (slice, head)

// One cluster of kCalibCluster blocks per (slice, head); block r of the
// cluster takes the batches of 64 rows starting at 64 (r + kCalibCluster b),
// so n_cal = 512 is one batch per block. Each of the 64 threads rotates one
// row and writes y^2 to shared memory; thread t then adds columns t, t + 64,
// ... over the batch's rows, in row order, into float64 accumulators. Blocks
// of 64 threads let 4 blocks share an SM at the transform's register count. Rank 0 adds the
// blocks' partial sums in rank order, reading them from the other blocks'
// shared memory (distributed shared memory of the cluster). Every addition
// happens in a fixed order, so the result does not depend on scheduling.
template <int D, int ROT>
__global__ void __cluster_dims__(kCalibCluster, 1, 1) __launch_bounds__(kCalibRows)
    calibrate_kernel(const CalibArgs a) {
  constexpr int NC = (D + kCalibRows - 1) / kCalibRows;   // columns per thread
  __shared__ float sq[kCalibRows][D + 1];
  __shared__ double part[D];
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int sh = blockIdx.x / kCalibCluster;
  const int s = sh / a.heads;
  const int h = sh % a.heads;
  const int64_t tab = (int64_t(s) * a.heads + h) * D;
  double acc[NC];   // columns threadIdx.x + kCalibRows c
#pragma unroll
  for (int c = 0; c < NC; ++c) acc[c] = 0.0;
  for (int64_t base = int64_t(kCalibRows) * rank; base < a.n_cal;
       base += int64_t(kCalibRows) * kCalibCluster) {
    const int64_t r = base + threadIdx.x;   // one row per thread
    if (r < a.n_cal) {
      int64_t vx = (int64_t(s) * a.x_slice_stride_rows + r) * a.heads + h;
      if (!dbg_ok(vx < vec_limit(a.n_slices, a.x_slice_stride_rows, a.n_cal, a.heads), a.guard))
        vx = 0;   // debug build: recorded, read vector 0 instead
      const uint16_t* xv = a.x + vx * D;
      uint32_t xw[D / 2], sgw[D / 2];
      load_vector<D>(xv, a.signs + tab, xw, sgw);
      float2 v[D / 2];
      rotate_forward<ROT, D>(xw, sgw, v);
      static_for<0, D / 2>([&](auto j_) {
        constexpr int j = decltype(j_)::value;
        const float y0 = v[j].x * gain_f<ROT, D>(2 * j);
        const float y1 = v[j].y * gain_f<ROT, D>(2 * j + 1);
        sq[threadIdx.x][2 * j] = y0 * y0;
        sq[threadIdx.x][2 * j + 1] = y1 * y1;
      });
    } else {
      for (int j = 0; j < D; ++j) sq[threadIdx.x][j] = 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int j = threadIdx.x + kCalibRows * c;
      if (j < D)
        for (int i = 0; i < kCalibRows; ++i) acc[c] += double(sq[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int j = threadIdx.x + kCalibRows * c;
    if (j < D) part[j] = acc[c];
  }
  cluster.sync();
  if (rank == 0) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int j = threadIdx.x + kCalibRows * c;
      if (j < D) {
        double total = 0.0;
        for (int q = 0; q < kCalibCluster; ++q) total += cluster.map_shared_rank(part, q)[j];
        if (dbg_ok(tab + j < a.n_slices * a.heads * D, a.guard))
          a.lambda_out[tab + j] = total > 0.0 ? float(sqrt(total / double(a.n_cal))) : 1.0f;
      }
    }
  }
  cluster.sync();   // the other blocks keep their shared memory until rank 0 is done
}

}  // namespace srftq
