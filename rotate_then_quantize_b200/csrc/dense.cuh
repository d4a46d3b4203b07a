// The codec with a rotation given as a dense matrix: the Householder variant
// of "When Quantization Is Free" (Methodology 3, Householder rotations: k
// reflectors on top of the fixed SRFT base), or any orthogonal R.
//
//   householder_kernel     R = H(v_1) ... H(v_k) B, B the signed SRFT/SRHT
//                          matrix, one block per (slice, head)
//   operand_kernel         R (float32) -> fp16 pair (hi, lo), hi + lo = R to
//                          about 2^-22; the layout every dense kernel reads
//   dense_calibrate_kernel lambda = RMS of R x over the calibration rows, as
//                          a register-tiled float32 product of 64-vector
//                          tiles (CUDA cores)
//
// The quantiser and dequantiser run on the tensor cores (dense_mma.cuh,
// dense_mma_dequant.cuh).
//
// Operand layout: [S][H][2][d][d] fp16, part 0 = hi, part 1 = lo, row n of a
// part is output coordinate n (y_n = sum_k R[n][k] x_k).
#pragma once

#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "codec.cuh"

namespace srftq {

// ---------------------------------------------------------------------------
// Householder rotation and operand
// ---------------------------------------------------------------------------

struct HouseholderArgs {
  int32_t heads, n_reflectors;
  const float* reflectors;   // [S][H][k][d]
  const int8_t* signs;       // [S][H][d]
  float* rot;                // [S][H][d][d]
  int64_t n_slices;          // debug-build index checks
  unsigned* guard;
};

// Entry (n, j) of the unsigned base rotation, in double: SRFT rows
// [X_0, X_{d/2}, sqrt2 Re X_k, sqrt2 Im X_k] of the unitary DFT (kernel
// exp(-2 pi i k j / d)), SRHT (-1)^popcount(n & j) / sqrt(d).
template <int D, int ROT>
__device__ __forceinline__ double base_entry(int n, int j) {
  const double c = inv_sqrt_pow2(D);
  if constexpr (ROT == kSRHT) {
    return (__popc(n & j) & 1) ? -c : c;
  } else {
    if (n == 0) return c;
    if (n == 1) return (j & 1) ? -c : c;
    const int k = n >> 1;
    const int m = (k * j) & (D - 1);   // k j mod d: the angle 2 pi m / d is exact
    double sn, cs;
    sincospi(2.0 * double(m) / double(D), &sn, &cs);
    const double r2 = 1.4142135623730950488 * c;
    return (n & 1) ? -r2 * sn : r2 * cs;
  }
}

// One block of D threads per (slice, head); thread j owns column j of R,
// which lives in `rot` (each column is touched by its own thread only, so
// only the reflector staged in shared memory needs barriers). Reflectors are
// applied innermost first: R = H(v_1) (H(v_2) ( ... (H(v_k) B))). Dot
// products and updates run in double; a zero reflector is skipped.
template <int D, int ROT>
__global__ void __launch_bounds__(D) householder_kernel(const HouseholderArgs a) {
  __shared__ double v[D];
  const int sh = blockIdx.x;                 // s * H + h
  const int j = threadIdx.x;
  if (!dbg_ok(sh < a.n_slices * a.heads, a.guard)) return;   // block-uniform
  float* R = a.rot + size_t(sh) * D * D;
  const double sj = a.signs[size_t(sh) * D + j] < 0 ? -1.0 : 1.0;
  for (int n = 0; n < D; ++n) R[size_t(n) * D + j] = float(base_entry<D, ROT>(n, j) * sj);
  for (int i = a.n_reflectors - 1; i >= 0; --i) {
    __syncthreads();   // every thread is done with the previous reflector
    v[j] = double(a.reflectors[(size_t(sh) * a.n_reflectors + i) * D + j]);
    __syncthreads();
    double vv = 0.0, dot = 0.0;
    for (int n = 0; n < D; ++n) {
      vv = fma(v[n], v[n], vv);
      dot = fma(v[n], double(R[size_t(n) * D + j]), dot);
    }
    if (vv == 0.0) continue;
    const double f = 2.0 * dot / vv;
    for (int n = 0; n < D; ++n) {
      float* p = R + size_t(n) * D + j;
      *p = float(double(*p) - f * v[n]);
    }
  }
}

// hi = fp16_rn(r), lo = fp16_rn(r - hi) (the difference is exact in float32).
__global__ void __launch_bounds__(256) operand_kernel(const float* rot, uint16_t* op, int64_t mats,
                                                     int dd) {
  const int64_t total = mats * dd;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float r = rot[i];
    const __half hi = __float2half_rn(r);
    const __half lo = __float2half_rn(r - __half2float(hi));
    const int64_t m = i / dd, e = i - m * dd;
    op[(2 * m) * dd + e] = __half_as_ushort(hi);
    op[(2 * m + 1) * dd + e] = __half_as_ushort(lo);
  }
}

// ---------------------------------------------------------------------------
// Register-tiled float32 product of one 64-vector tile (CUDA cores)
// ---------------------------------------------------------------------------

constexpr int kDenseRows = 64;      // vectors per tile
constexpr int kDenseThreads = 256;
constexpr int kDenseKC = 32;        // K columns staged per step

template <int D>
struct DenseTile {
  static constexpr int NT = D / 8;                 // threads along the outputs
  static constexpr int TVG = kDenseThreads / NT;   // thread groups along the vectors
  static constexpr int TV = kDenseRows / TVG;      // vectors per thread
  static constexpr int AS = D + 4;                 // A / C row stride (floats)
  static constexpr int BS = D + 4;                 // B row stride (floats)
  static constexpr int kABytes = kDenseRows * AS * 4;
  static constexpr int kBBytes = kDenseKC * BS * 4;
  static constexpr int kBytes = kABytes + kBBytes;
  static_assert(TV >= 1 && TVG * TV == kDenseRows, "tile shape");
};

// acc[i][c] = sum_k A[v_i][k] * Bt[k][n_c] over all K (y = R x), where the
// staged chunk Bt[kk][n] = R[n][k0 + kk]. A is already in shared memory.
template <int D>
__device__ __forceinline__ void dense_product(const float* As, float* Bs, const uint16_t* hi,
                                              const uint16_t* lo, int tid,
                                              float (&acc)[DenseTile<D>::TV][8]) {
  using T = DenseTile<D>;
  const int tn = tid % T::NT, tv = tid / T::NT;
#pragma unroll
  for (int i = 0; i < T::TV; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.0f;
  for (int k0 = 0; k0 < D; k0 += kDenseKC) {
    // 16-byte loads of 8 consecutive K values of one row of hi and of lo,
    // all issued before any is used (each thread has D / 64 of them per
    // part), then R = hi + lo stored transposed
    constexpr int kPer = D * (kDenseKC / 8) / kDenseThreads;
    static_assert(kPer >= 1 && kPer * kDenseThreads == D * (kDenseKC / 8), "staging split");
    uint4 wh[kPer], wl[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int t = tid + u * kDenseThreads;
      const size_t off = size_t(t / (kDenseKC / 8)) * D + k0 + 8 * (t % (kDenseKC / 8));
      wh[u] = *reinterpret_cast<const uint4*>(hi + off);
      wl[u] = *reinterpret_cast<const uint4*>(lo + off);
    }
    __syncthreads();   // the previous chunk has been read
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int t = tid + u * kDenseThreads;
      const int n = t / (kDenseKC / 8), c = t % (kDenseKC / 8);
      const uint32_t hw[4] = {wh[u].x, wh[u].y, wh[u].z, wh[u].w};
      const uint32_t lw[4] = {wl[u].x, wl[u].y, wl[u].z, wl[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 h2 = __half22float2(*reinterpret_cast<const __half2*>(&hw[e]));
        const float2 l2 = __half22float2(*reinterpret_cast<const __half2*>(&lw[e]));
        Bs[(8 * c + 2 * e) * T::BS + n] = h2.x + l2.x;
        Bs[(8 * c + 2 * e + 1) * T::BS + n] = h2.y + l2.y;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kDenseKC; ++kk) {
      const float4 b0 = *reinterpret_cast<const float4*>(Bs + kk * T::BS + 8 * tn);
      const float4 b1 = *reinterpret_cast<const float4*>(Bs + kk * T::BS + 8 * tn + 4);
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < T::TV; ++i) {
        const float av = As[(tv * T::TV + i) * T::AS + k0 + kk];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = fmaf(av, b[c], acc[i][c]);
      }
    }
  }
}

// lambda[s][h][n] = sqrt(mean over the first n_cal rows of y_n^2), y = R x
// (1 where the sum is 0). One cluster of kDenseCalibCluster blocks per
// (slice, head); block r of the cluster takes the 64-row tiles r, r + 8, ...
// Each thread sums its own products in double in a fixed order, the vector
// groups of a block are then added in a fixed order, and rank 0 adds the
// blocks' partial sums in rank order, reading them from the other blocks'
// shared memory (distributed shared memory of the cluster): deterministic.
struct DenseCalibArgs {
  int64_t n_cal, x_stride_rows;
  int32_t heads;
  const uint16_t* x;
  const uint16_t* operand;
  float* lambda_out;
  int64_t n_slices;           // debug-build index checks
  unsigned* guard;
};

constexpr int kDenseCalibCluster = 8;

template <int D>
__global__ void __cluster_dims__(kDenseCalibCluster, 1, 1) __launch_bounds__(kDenseThreads)
    dense_calibrate_kernel(const DenseCalibArgs a) {
  using T = DenseTile<D>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ double part[D];   // this block's column sums
  float* As = reinterpret_cast<float*>(smem_raw);
  float* Bs = reinterpret_cast<float*>(smem_raw + T::kABytes);
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int64_t sh = blockIdx.x / kDenseCalibCluster;
  const int64_t s = sh / a.heads;
  const int h = int(sh % a.heads);
  const uint16_t* hi = a.operand + size_t(sh) * 2 * D * D;
  const uint16_t* lo = hi + size_t(D) * D;
  const int tn = tid % T::NT, tv = tid / T::NT;
  double ss[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int64_t r0 = int64_t(kDenseRows) * rank; r0 < a.n_cal;
       r0 += int64_t(kDenseRows) * kDenseCalibCluster) {
    __syncthreads();   // the previous tile's A has been read
#pragma unroll
    for (int idx = tid; idx < kDenseRows * (D / 8); idx += kDenseThreads) {
      const int v = idx / (D / 8), c8 = idx % (D / 8);
      const int64_t r = r0 + v;
      float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      const size_t vec = size_t((s * a.x_stride_rows + r) * a.heads + h);
      if (r < a.n_cal &&
          dbg_ok(int64_t(vec) < vec_limit(a.n_slices, a.x_stride_rows, a.n_cal, a.heads),
                 a.guard)) {
        const uint4 w = *reinterpret_cast<const uint4*>(a.x + vec * D + 8 * c8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&ww[e]));
          f[2 * e] = p.x;
          f[2 * e + 1] = p.y;
        }
      }
      float* dst = As + v * T::AS + 8 * c8;
      *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
    }
    float acc[T::TV][8];
    dense_product<D>(As, Bs, hi, lo, tid, acc);
#pragma unroll
    for (int i = 0; i < T::TV; ++i)
#pragma unroll
      for (int c = 0; c < 8; ++c) ss[c] = fma(double(acc[i][c]), double(acc[i][c]), ss[c]);
  }
  // fixed-order sum over the TVG vector groups (the B stage is free now)
  __syncthreads();
  double* red = reinterpret_cast<double*>(smem_raw);
#pragma unroll
  for (int c = 0; c < 8; ++c) red[tv * D + 8 * tn + c] = ss[c];
  __syncthreads();
  for (int n = tid; n < D; n += kDenseThreads) {
    double t = 0.0;
    for (int g = 0; g < T::TVG; ++g) t += red[g * D + n];
    part[n] = t;
  }
  cluster.sync();
  if (rank == 0) {
    for (int n = tid; n < D; n += kDenseThreads) {
      double t = 0.0;
      for (int q = 0; q < kDenseCalibCluster; ++q) t += cluster.map_shared_rank(part, q)[n];
      if (dbg_ok(sh < a.n_slices * a.heads, a.guard))
        a.lambda_out[size_t(sh) * D + n] = t == 0.0 ? 1.0f : float(sqrt(t / double(a.n_cal)));
    }
  }
  cluster.sync();   // the other blocks keep their shared memory until rank 0 is done
}

}  // namespace srftq
