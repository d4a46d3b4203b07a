// In-register rotations for one head-dim vector held by one thread.
//
// SRFT ("When Quantization Is Free", Methodology 1 and Methodology 2 steps
// 1-3): the d real inputs u are read as L = d/2 complex points
// z_m = u_{2m} + i u_{2m+1}; a radix-2 complex FFT of length L (log2(d/2)
// butterfly passes) gives Z; the Hermitian step turns Z into the d-point real
// DFT X and lays it out in the packed order
//   [X_0, X_{d/2}, Re X_1, Im X_1, ..., Re X_{d/2-1}, Im X_{d/2-1}].
// The kernels here produce that layout *unnormalised*; the normalisation
// (1/sqrt(d), the sqrt(2) of the pack, factors of 2 of the Hermitian step) is
// one per-coordinate constant folded with 1/lambda into a single multiplier
// table by the caller (see srft_coordinate_gain).
//
// The FFT is decimation in time on a bit-reversed view of the registers (the
// permutation is a compile-time renaming, the "Stockham" reordering of the
// paper's kernel costs nothing in registers). Twiddled butterflies use the
// FMA form a +- w*b = a +- c*(b + tau*(i b)) with c = Re w, tau = Im w / Re w
// (or the cotangent form when |Im w| > |Re w|): 6 FMAs instead of 4
// multiplies and 4 adds. Butterflies with w = 1 or w = +-i are pure adds.
//
// SRHT ("HyperQuant", Methodology 1): in-place Walsh-Hadamard butterflies
// (a+b, a-b) over log2(d) bit planes, natural (Sylvester) order.
#pragma once

#include "common.cuh"

namespace srftq {

// One radix-2 DIT butterfly: (a, b) <- (a + w b, a - w b) with
// w = exp(SIGN * i * pi * K / H).
template <int SIGN, int K, int H>
__device__ __forceinline__ void butterfly(float& ar, float& ai, float& br, float& bi) {
  if constexpr (K == 0) {
    const float tr = br, ti = bi;
    br = ar - tr;
    bi = ai - ti;
    ar = ar + tr;
    ai = ai + ti;
  } else if constexpr (2 * K == H) {
    // w = SIGN * i, so w b = (-SIGN bi, SIGN br)
    const float tr = (SIGN > 0) ? -bi : bi;
    const float ti = (SIGN > 0) ? br : -br;
    br = ar - tr;
    bi = ai - ti;
    ar = ar + tr;
    ai = ai + ti;
  } else {
    constexpr double wr = ct::cos2pi(K, 2 * H);
    constexpr double wi = SIGN * ct::sin2pi(K, 2 * H);
    if constexpr (ct::dabs(wr) >= ct::dabs(wi)) {
      // w b = wr * (br - tau bi, bi + tau br), tau = wi / wr
      constexpr float tau = float(wi / wr);
      constexpr float c = float(wr);
      const float p = fmaf(-tau, bi, br);
      const float q = fmaf(tau, br, bi);
      br = fmaf(-c, p, ar);
      bi = fmaf(-c, q, ai);
      ar = fmaf(c, p, ar);
      ai = fmaf(c, q, ai);
    } else {
      // w b = wi * (kap br - bi, kap bi + br), kap = wr / wi
      constexpr float kap = float(wr / wi);
      constexpr float c = float(wi);
      const float p = fmaf(kap, br, -bi);
      const float q = fmaf(kap, bi, br);
      br = fmaf(-c, p, ar);
      bi = fmaf(-c, q, ai);
      ar = fmaf(c, p, ar);
      ai = fmaf(c, q, ai);
    }
  }
}

// Unnormalised complex DFT of length L, in place, natural order in and out.
// SIGN = -1: Z_k = sum z_m exp(-2 pi i m k / L); SIGN = +1: the inverse
// kernel without the 1/L.
template <int L, int SIGN>
__device__ __forceinline__ void fft_dit(float (&re)[L], float (&im)[L]) {
  constexpr int LOG = ilog2(L);
  float ar[L], ai[L];
  static_for<0, L>([&](auto i_) {
    constexpr int i = decltype(i_)::value;
    constexpr int b = bitrev(i, LOG);
    ar[i] = re[b];
    ai[i] = im[b];
  });
  static_for<0, LOG>([&](auto s_) {
    constexpr int h = 1 << decltype(s_)::value;
    static_for<0, L / (2 * h)>([&](auto b_) {
      constexpr int j = decltype(b_)::value * 2 * h;
      static_for<0, h>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        butterfly<SIGN, k, h>(ar[j + k], ai[j + k], ar[j + k + h], ai[j + k + h]);
      });
    });
  });
  static_for<0, L>([&](auto i_) {
    constexpr int i = decltype(i_)::value;
    re[i] = ar[i];
    im[i] = ai[i];
  });
}

// Gain g_j such that the SRFT packed coordinate is y_j = g_j / sqrt(d) *
// (output j of srft_forward_raw); the inverse input scaling uses the same
// gains (see srft_inverse_raw).
__host__ __device__ constexpr double srft_coordinate_gain(int j, int d) {
  const int L = d / 2;
  if (j < 2) return 1.0;
  if (j == L) return 1.4142135623730950488;
  if (j == L + 1) return -1.4142135623730950488;
  return 0.70710678118654752440;
}

// Forward SRFT core: u (d reals, signs already applied) -> unnormalised
// packed spectrum. Output j holds X_0 (j=0), X_{L} (j=1), Re Z_{L/2} and
// Im Z_{L/2} (j = L, L+1) and 2 Re X_k / 2 Im X_k elsewhere.
template <int D>
__device__ __forceinline__ void srft_forward_raw(float (&v)[D]) {
  constexpr int L = D / 2;
  float re[L], im[L];
  static_for<0, L>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    re[m] = v[2 * m];
    im[m] = v[2 * m + 1];
  });
  fft_dit<L, -1>(re, im);
  v[0] = re[0] + im[0];
  v[1] = re[0] - im[0];
  // Hermitian step for the bin pair (k, L-k):
  //   E = Z_k + conj Z_{L-k}, O = Z_k - conj Z_{L-k},
  //   2 X_k = E - i W^k O, 2 X_{L-k} = conj(E + i W^k O) with W = exp(-2 pi i / d).
  static_for<1, L / 2>([&](auto k_) {
    constexpr int k = decltype(k_)::value;
    const float Er = re[k] + re[L - k];
    const float Ei = im[k] - im[L - k];
    const float Or = re[k] - re[L - k];
    const float Oi = im[k] + im[L - k];
    constexpr double cw = ct::cos2pi(k, D);
    constexpr double sw = ct::sin2pi(k, D);
    if constexpr (cw >= sw) {
      constexpr float t = float(sw / cw);
      constexpr float c = float(cw);
      const float P = fmaf(-t, Or, Oi);   // (cw Oi - sw Or) / cw
      const float Q = fmaf(t, Oi, Or);    // (sw Oi + cw Or) / cw
      v[2 * k] = fmaf(c, P, Er);
      v[2 * (L - k)] = fmaf(-c, P, Er);
      v[2 * k + 1] = fmaf(-c, Q, Ei);
      v[2 * (L - k) + 1] = fmaf(-c, Q, -Ei);
    } else {
      constexpr float t = float(cw / sw);
      constexpr float c = float(sw);
      const float P = fmaf(-t, Oi, Or);   // -(cw Oi - sw Or) / sw
      const float Q = fmaf(t, Or, Oi);    // (sw Oi + cw Or) / sw
      v[2 * k] = fmaf(-c, P, Er);
      v[2 * (L - k)] = fmaf(c, P, Er);
      v[2 * k + 1] = fmaf(-c, Q, Ei);
      v[2 * (L - k) + 1] = fmaf(-c, Q, -Ei);
    }
  });
  v[L] = re[L / 2];
  v[L + 1] = im[L / 2];
}

// Inverse SRFT core: input v_j = (g_j / sqrt(d)) * yhat_j (packed spectrum
// already scaled by the coordinate gains), output u = R^T yhat before signs.
template <int D>
__device__ __forceinline__ void srft_inverse_raw(float (&v)[D]) {
  constexpr int L = D / 2;
  float re[L], im[L];
  re[0] = v[0] + v[1];
  im[0] = v[0] - v[1];
  // Inverse Hermitian step for (k, L-k): with a = Y_k, b = Y_{L-k},
  //   E = a + conj b, O = a - conj b, B = O V^k (V = exp(2 pi i / d)),
  //   Z_k = E + i B, Z_{L-k} = conj E + i conj B.
  static_for<1, L / 2>([&](auto k_) {
    constexpr int k = decltype(k_)::value;
    const float ar = v[2 * k], ai = v[2 * k + 1];
    const float br = v[2 * (L - k)], bi = v[2 * (L - k) + 1];
    const float Er = ar + br;
    const float Ei = ai - bi;
    const float Or = ar - br;
    const float Oi = ai + bi;
    constexpr double cw = ct::cos2pi(k, D);
    constexpr double sw = ct::sin2pi(k, D);
    if constexpr (cw >= sw) {
      constexpr float t = float(sw / cw);
      constexpr float c = float(cw);
      const float P = fmaf(t, Or, Oi);    // Im B / cw
      const float Q = fmaf(-t, Oi, Or);   // Re B / cw
      re[k] = fmaf(-c, P, Er);
      re[L - k] = fmaf(c, P, Er);
      im[k] = fmaf(c, Q, Ei);
      im[L - k] = fmaf(c, Q, -Ei);
    } else {
      constexpr float t = float(cw / sw);
      constexpr float c = float(sw);
      const float P = fmaf(t, Oi, Or);    // Im B / sw
      const float Q = fmaf(-t, Or, Oi);   // -Re B / sw
      re[k] = fmaf(-c, P, Er);
      re[L - k] = fmaf(c, P, Er);
      im[k] = fmaf(-c, Q, Ei);
      im[L - k] = fmaf(-c, Q, -Ei);
    }
  });
  re[L / 2] = v[L];
  im[L / 2] = v[L + 1];
  fft_dit<L, +1>(re, im);
  static_for<0, L>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    v[2 * m] = re[m];
    v[2 * m + 1] = im[m];
  });
}

// Unnormalised Walsh-Hadamard transform in natural (Sylvester) order.
template <int D>
__device__ __forceinline__ void wht(float (&v)[D]) {
  static_for<0, ilog2(D)>([&](auto s_) {
    constexpr int h = 1 << decltype(s_)::value;
    static_for<0, D / (2 * h)>([&](auto b_) {
      constexpr int j = decltype(b_)::value * 2 * h;
      static_for<0, h>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        const float a = v[j + k], b = v[j + k + h];
        v[j + k] = a + b;
        v[j + k + h] = a - b;
      });
    });
  });
}

// Rotation kinds (match SRFTQ_ROT_* in srftq.h).
constexpr int kSRFT = 0;
constexpr int kSRHT = 1;

// 1/sqrt(d) for d a power of two, exact up to one rounding.
__host__ __device__ constexpr double inv_sqrt_pow2(int d) {
  const int k = ilog2(d);
  double r = 1.0;
  for (int i = 0; i < k / 2; ++i) r *= 0.5;
  return (k % 2) ? r * 0.70710678118654752440 : r;
}

// Gain of packed coordinate j: y_j = coordinate_gain(j) * raw_j, where raw
// is the output of rotate_forward_raw; the inverse takes
// v_j = coordinate_gain(j) * yhat_j as input of rotate_inverse_raw.
template <int ROT, int D>
__host__ __device__ constexpr double coordinate_gain(int j) {
  return (ROT == kSRFT ? srft_coordinate_gain(j, D) : 1.0) * inv_sqrt_pow2(D);
}

template <int ROT, int D>
__device__ __forceinline__ void rotate_forward_raw(float (&v)[D]) {
  if constexpr (ROT == kSRFT) {
    srft_forward_raw<D>(v);
  } else {
    wht<D>(v);
  }
}

template <int ROT, int D>
__device__ __forceinline__ void rotate_inverse_raw(float (&v)[D]) {
  if constexpr (ROT == kSRFT) {
    srft_inverse_raw<D>(v);
  } else {
    wht<D>(v);
  }
}

}  // namespace srftq
