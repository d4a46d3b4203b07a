// In-register rotations for one head-dim vector held by one thread.
//
// SRFT ("When Quantization Is Free", Methodology 1 and Methodology 2 steps
// 1-3): the d real inputs u = s * x are read as L = d/2 complex points
// z_m = u_{2m} + i u_{2m+1}; a radix-2 complex FFT of length L (log2(d/2)
// butterfly passes) gives Z; the Hermitian step turns Z into the d-point real
// DFT X in the packed order
//   [X_0, X_{d/2}, Re X_1, Im X_1, ..., Re X_{d/2-1}, Im X_{d/2-1}].
// The transforms here produce that layout *unnormalised*; the normalisation
// (1/sqrt(d), the sqrt(2) of the pack, the factors of 2 of the Hermitian
// step) is one per-coordinate gain that the callers fold, together with
// lambda, into a single multiplier table (coordinate_gain).
//
// Register layout. The FFT works on the decimation-in-time (bit-reversed)
// arrangement a_i = z_{bitrev(i)}, i < L, held as Q = L/2 pairs of packed
// float2 registers PR[i] = (Re a_i, Re a_{i+Q}), PI[i] = (Im a_i, Im a_{i+Q}).
// Every butterfly pass with span h < Q pairs index j with j + h inside each
// half, so the two lanes of a pair undergo the same butterfly with the same
// twiddle: one packed f32x2 instruction does the work of two. The last pass
// (span Q) combines the two lanes of a pair and runs as scalar FMAs. The
// bit-reversal itself is a compile-time choice of which register each value
// is written to (the "Stockham" reordering of the paper's kernel is free).
//
// Twiddled butterflies use the FMA form a +- w*b = a +- c*(b + tau*(i b))
// with c = Re w, tau = Im w / Re w (or the cotangent form when |Im w| >
// |Re w|): 6 FMAs instead of 4 multiplies and 4 adds. Butterflies with
// w = 1 or w = +-i are pure additions.
//
// The quantiser's first pass reads fp16 inputs directly: the signs are fp16
// +-1.0 and `fma.rn.f32.f16` multiplies an fp16 value by its sign and adds an
// fp32 value with a single rounding, so conversion, sign and the first
// butterfly pass cost three instructions per pair of inputs.
//
// SRHT ("HyperQuant", Methodology 1): Walsh-Hadamard butterflies (a+b, a-b)
// over log2(d) bit planes, natural (Sylvester) order; plane 0 is computed
// from fp16 the same way, the others on packed natural pairs (2j, 2j+1).
#pragma once

#include "common.cuh"

namespace srftq {

// ---------------------------------------------------------------------------
// Packed float2 arithmetic (sm_100 f32x2 instructions)
// ---------------------------------------------------------------------------

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 splat(float c) { return make_float2(c, c); }

// a * b + c with a, b the selected fp16 halves of two 32-bit words (HA, HB:
// 0 = low half, 1 = high half); product and sum are formed exactly and
// rounded once to fp32.
template <int HA, int HB>
__device__ __forceinline__ float fma_f16(uint32_t a, uint32_t b, float c) {
  float d;
  if constexpr (HA == 0 && HB == 0)
    asm("{ .reg .f16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a0, b0, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
  else if constexpr (HA == 1 && HB == 1)
    asm("{ .reg .f16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a1, b1, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
  else if constexpr (HA == 0 && HB == 1)
    asm("{ .reg .f16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a0, b1, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
  else
    asm("{ .reg .f16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a1, b0, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

// ---------------------------------------------------------------------------
// Butterflies
// ---------------------------------------------------------------------------

// Scalar radix-2 DIT butterfly: (a, b) <- (a + w b, a - w b),
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
      constexpr float tau = float(wi / wr);   // w b = wr (br - tau bi, bi + tau br)
      constexpr float c = float(wr);
      const float p = fmaf(-tau, bi, br);
      const float q = fmaf(tau, br, bi);
      br = fmaf(-c, p, ar);
      bi = fmaf(-c, q, ai);
      ar = fmaf(c, p, ar);
      ai = fmaf(c, q, ai);
    } else {
      constexpr float kap = float(wr / wi);   // w b = wi (kap br - bi, kap bi + br)
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

// Whether twiddled butterflies in the packed passes use f32x2 FMAs (their
// constants must then be materialised as register pairs) or two scalar
// butterflies with immediate constants.
#ifndef SRFTQ_PACKED_TWIDDLE
#define SRFTQ_PACKED_TWIDDLE 1
#endif

// The same butterfly on two independent lanes at once (packed f32x2).
template <int SIGN, int K, int H>
__device__ __forceinline__ void butterfly2(float2& ar, float2& ai, float2& br, float2& bi) {
  if constexpr (K != 0 && 2 * K != H && !SRFTQ_PACKED_TWIDDLE) {
    butterfly<SIGN, K, H>(ar.x, ai.x, br.x, bi.x);
    butterfly<SIGN, K, H>(ar.y, ai.y, br.y, bi.y);
  } else if constexpr (K == 0) {
    const float2 tr = br, ti = bi;
    br = sub2(ar, tr);
    bi = sub2(ai, ti);
    ar = add2(ar, tr);
    ai = add2(ai, ti);
  } else if constexpr (2 * K == H) {
    const float2 a_r = ar, a_i = ai, b_r = br, b_i = bi;
    if constexpr (SIGN < 0) {   // w b = (bi, -br)
      ar = add2(a_r, b_i);
      ai = sub2(a_i, b_r);
      br = sub2(a_r, b_i);
      bi = add2(a_i, b_r);
    } else {                    // w b = (-bi, br)
      ar = sub2(a_r, b_i);
      ai = add2(a_i, b_r);
      br = add2(a_r, b_i);
      bi = sub2(a_i, b_r);
    }
  } else {
    constexpr double wr = ct::cos2pi(K, 2 * H);
    constexpr double wi = SIGN * ct::sin2pi(K, 2 * H);
    if constexpr (ct::dabs(wr) >= ct::dabs(wi)) {
      constexpr float tau = float(wi / wr);
      constexpr float c = float(wr);
      const float2 p = fma2(splat(-tau), bi, br);
      const float2 q = fma2(splat(tau), br, bi);
      br = fma2(splat(-c), p, ar);
      bi = fma2(splat(-c), q, ai);
      ar = fma2(splat(c), p, ar);
      ai = fma2(splat(c), q, ai);
    } else {
      constexpr float kap = float(wr / wi);
      constexpr float c = float(wi);
      const float2 p = fma2(splat(kap), br, make_float2(-bi.x, -bi.y));
      const float2 q = fma2(splat(kap), bi, br);
      br = fma2(splat(-c), p, ar);
      bi = fma2(splat(-c), q, ai);
      ar = fma2(splat(c), p, ar);
      ai = fma2(splat(c), q, ai);
    }
  }
}

// Packed DIT passes with spans h = H0, 2*H0, ..., Q/2 on the pair arrays
// (index i pairs with i + Q in the two lanes; see the file comment).
template <int Q, int SIGN, int H0>
__device__ __forceinline__ void packed_passes(float2 (&PR)[Q], float2 (&PI)[Q]) {
  if constexpr (H0 < Q) {
    constexpr int h = H0;
    static_for<0, Q / (2 * h)>([&](auto b_) {
      constexpr int j = decltype(b_)::value * 2 * h;
      static_for<0, h>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        butterfly2<SIGN, k, h>(PR[j + k], PI[j + k], PR[j + k + h], PI[j + k + h]);
      });
    });
    packed_passes<Q, SIGN, 2 * H0>(PR, PI);
  }
}

// Final DIT pass (span Q): butterfly k combines the two lanes of pair k.
template <int Q, int SIGN>
__device__ __forceinline__ void last_pass(float2 (&PR)[Q], float2 (&PI)[Q]) {
  static_for<0, Q>([&](auto k_) {
    constexpr int k = decltype(k_)::value;
    butterfly<SIGN, k, Q>(PR[k].x, PI[k].x, PR[k].y, PI[k].y);
  });
}

// Register slot of a_i in the packed arrays: pair i % Q, lane x if i < Q.
template <int Q, int I>
__device__ __forceinline__ float& lane(float2 (&P)[Q]) {
  if constexpr (I < Q) {
    return P[I].x;
  } else {
    return P[I - Q].y;
  }
}

// ---------------------------------------------------------------------------
// SRFT
// ---------------------------------------------------------------------------

// Gain g_j such that the SRFT packed coordinate is y_j = g_j / sqrt(d) * raw_j.
__host__ __device__ constexpr double srft_coordinate_gain(int j, int d) {
  const int L = d / 2;
  if (j < 2) return 1.0;
  if (j == L) return 1.4142135623730950488;
  if (j == L + 1) return -1.4142135623730950488;
  return 0.70710678118654752440;
}

// Hermitian step of one bin K (0 < K < L, L = D/2) from E = Z_K + conj Z_{L-K}
// and O = Z_K - conj Z_{L-K}: with W = exp(-2 pi i / D),
//   xk = 2 X_K = E - i W^K O,   xm = conj(2 X_{L-K}) = E + i W^K O,
// stored as xk = (Re, Im) of 2 X_K and xm = (Re, Im) of 2 X_{L-K}. The
// twiddle enters as c (a + t b) with |t| <= 1, six FMAs for both bins.
template <int D, int K>
__device__ __forceinline__ void hermitian_out(float Er, float Ei, float Or, float Oi, float2& xk,
                                              float2& xm) {
  constexpr double cw = ct::cos2pi(K, D);
  constexpr double sw = ct::sin2pi(K, D);
  if constexpr (ct::dabs(cw) >= ct::dabs(sw)) {
    constexpr float t = float(sw / cw);
    constexpr float c = float(cw);
    const float P = fmaf(-t, Or, Oi);   // (cw Oi - sw Or) / cw
    const float Qv = fmaf(t, Oi, Or);   // (sw Oi + cw Or) / cw
    xk = make_float2(fmaf(c, P, Er), fmaf(-c, Qv, Ei));
    xm = make_float2(fmaf(-c, P, Er), fmaf(-c, Qv, -Ei));
  } else {
    constexpr float t = float(cw / sw);
    constexpr float c = float(sw);
    const float P = fmaf(-t, Oi, Or);   // -(cw Oi - sw Or) / sw
    const float Qv = fmaf(t, Or, Oi);   // (sw Oi + cw Or) / sw
    xk = make_float2(fmaf(-c, P, Er), fmaf(-c, Qv, Ei));
    xm = make_float2(fmaf(c, P, Er), fmaf(-c, Qv, -Ei));
  }
}

// Passes 2 .. log2(L) of the forward FFT, the last pass and the Hermitian
// step, from pass-1 output in the packed bit-reversed arrangement PR / PI
// (see the file comment) to the unnormalised packed spectrum v.
template <int D>
__device__ __forceinline__ void srft_forward_rest(float2 (&PR)[D / 4], float2 (&PI)[D / 4],
                                                  float2 (&v)[D / 2]) {
  constexpr int L = D / 2, Q = L / 2;
  packed_passes<Q, -1, 2>(PR, PI);

  // Last pass (span Q) fused with the Hermitian step. Butterfly k gives
  // (Z_k, Z_{k+Q}) in the lanes of PR[k] / PI[k]; butterfly Q-k gives
  // (Z_{Q-k}, Z_{L-k}), written here lane-swapped as (Z_{L-k}, Z_{Q-k}), so
  // that each lane of the pair holds a bin and its Hermitian partner: the
  // sums and differences E = Z_k + conj Z_{L-k}, O = Z_k - conj Z_{L-k} of
  // the bins k and k+Q then take four packed instructions.
  butterfly<-1, 0, Q>(PR[0].x, PI[0].x, PR[0].y, PI[0].y);   // Z_0, Z_Q
  v[0] = make_float2(PR[0].x + PI[0].x, PR[0].x - PI[0].x);
  v[Q] = make_float2(PR[0].y, PI[0].y);
  {
    constexpr int k = Q / 2;   // Z_{Q/2} and Z_{3Q/2} are each other's partner
    butterfly<-1, k, Q>(PR[k].x, PI[k].x, PR[k].y, PI[k].y);
    const float ar = PR[k].x, ai = PI[k].x, br = PR[k].y, bi = PI[k].y;
    hermitian_out<D, k>(ar + br, ai - bi, ar - br, ai + bi, v[k], v[L - k]);
  }
  static_for<1, Q / 2>([&](auto k_) {
    constexpr int k = decltype(k_)::value;
    butterfly<-1, k, Q>(PR[k].x, PI[k].x, PR[k].y, PI[k].y);
    float a_r = PR[Q - k].x, a_i = PI[Q - k].x, b_r = PR[Q - k].y, b_i = PI[Q - k].y;
    butterfly<-1, Q - k, Q>(a_r, a_i, b_r, b_i);   // a = Z_{Q-k}, b = Z_{L-k}
    const float2 Vr = make_float2(b_r, a_r), Vi = make_float2(b_i, a_i);
    const float2 Er = add2(PR[k], Vr), Ei = sub2(PI[k], Vi);
    const float2 Or = sub2(PR[k], Vr), Oi = add2(PI[k], Vi);
    hermitian_out<D, k>(Er.x, Ei.x, Or.x, Oi.x, v[k], v[L - k]);
    hermitian_out<D, k + Q>(Er.y, Ei.y, Or.y, Oi.y, v[k + Q], v[Q - k]);
  });
}

// Forward SRFT from fp16: xw[m] holds (x_{2m}, x_{2m+1}), sw[m] the fp16
// signs (s_{2m}, s_{2m+1}) as +-1.0. Output v[j] = (raw_{2j}, raw_{2j+1}),
// the unnormalised packed spectrum: raw_0 = X_0, raw_1 = X_L, raw_L / raw_{L+1}
// = Re / Im Z_{L/2}, and 2 Re X_k / 2 Im X_k elsewhere.
template <int D>
__device__ __forceinline__ void srft_forward(const uint32_t (&xw)[D / 2],
                                             const uint32_t (&sw)[D / 2], float2 (&v)[D / 2]) {
  constexpr int L = D / 2, Q = L / 2, LOG = ilog2(L);
  float2 PR[Q], PI[Q];
  // pass 1 (span 1) straight from fp16: a_i = z_m, a_{i+1} = z_{m+Q} with
  // m = bitrev(i), i even; (a_i, a_{i+1}) <- (a_i + a_{i+1}, a_i - a_{i+1}).
  static_for<0, Q>([&](auto p_) {
    constexpr int i = 2 * decltype(p_)::value;
    constexpr int m = bitrev(i, LOG);
    const uint32_t xa = xw[m], sa = sw[m], xb = xw[m + Q], sb = sw[m + Q];
    const float tr = fma_f16<0, 0>(xb, sb, 0.0f);
    const float ti = fma_f16<1, 1>(xb, sb, 0.0f);
    lane<Q, i>(PR) = fma_f16<0, 0>(xa, sa, tr);
    lane<Q, i + 1>(PR) = fma_f16<0, 0>(xa, sa, -tr);
    lane<Q, i>(PI) = fma_f16<1, 1>(xa, sa, ti);
    lane<Q, i + 1>(PI) = fma_f16<1, 1>(xa, sa, -ti);
  });
  srft_forward_rest<D>(PR, PI, v);
}

// Inverse SRFT: input v[j] = (c_{2j}, c_{2j+1}) with c_j = coordinate gain
// times yhat_j; output v[m] = (u_{2m}, u_{2m+1}) = R^T yhat before the signs.
template <int D>
__device__ __forceinline__ void srft_inverse(float2 (&v)[D / 2]) {
  constexpr int L = D / 2, Q = L / 2, LOG = ilog2(L);
  float2 PR[Q], PI[Q];
  // Inverse Hermitian step for (k, L-k): with a = Y_k, b = Y_{L-k},
  //   E = a + conj b, O = a - conj b, B = O V^k (V = exp(2 pi i / d)),
  //   Z_k = E + i B, Z_{L-k} = conj E + i conj B.
  // Z_k is written to the bit-reversed slot a_{bitrev(k)} for the DIT passes.
  lane<Q, 0>(PR) = v[0].x + v[0].y;
  lane<Q, 0>(PI) = v[0].x - v[0].y;
  const float2 pm = make_float2(1.0f, -1.0f), mp = make_float2(-1.0f, 1.0f);
  static_for<1, Q>([&](auto k_) {
    constexpr int k = decltype(k_)::value;
    constexpr int ik = bitrev(k, LOG), ilk = bitrev(L - k, LOG);
    const float2 E = fma2(v[L - k], pm, v[k]);   // (ar + br, ai - bi)
    const float2 O = fma2(v[L - k], mp, v[k]);   // (ar - br, ai + bi)
    const float Er = E.x, Ei = E.y, Or = O.x, Oi = O.y;
    constexpr double cw = ct::cos2pi(k, D);
    constexpr double sw_ = ct::sin2pi(k, D);
    if constexpr (cw >= sw_) {
      constexpr float t = float(sw_ / cw);
      constexpr float c = float(cw);
      const float P = fmaf(t, Or, Oi);    // Im B / cw
      const float Qv = fmaf(-t, Oi, Or);  // Re B / cw
      lane<Q, ik>(PR) = fmaf(-c, P, Er);
      lane<Q, ilk>(PR) = fmaf(c, P, Er);
      lane<Q, ik>(PI) = fmaf(c, Qv, Ei);
      lane<Q, ilk>(PI) = fmaf(c, Qv, -Ei);
    } else {
      constexpr float t = float(cw / sw_);
      constexpr float c = float(sw_);
      const float P = fmaf(t, Oi, Or);    // Im B / sw
      const float Qv = fmaf(-t, Or, Oi);  // -Re B / sw
      lane<Q, ik>(PR) = fmaf(-c, P, Er);
      lane<Q, ilk>(PR) = fmaf(c, P, Er);
      lane<Q, ik>(PI) = fmaf(-c, Qv, Ei);
      lane<Q, ilk>(PI) = fmaf(-c, Qv, -Ei);
    }
  });
  constexpr int iq = bitrev(Q, LOG);
  lane<Q, iq>(PR) = v[Q].x;
  lane<Q, iq>(PI) = v[Q].y;
  packed_passes<Q, +1, 1>(PR, PI);
  last_pass<Q, +1>(PR, PI);
  // PR[m] = (Re z_m, Re z_{m+Q}), z_m = u_{2m} + i u_{2m+1}
  static_for<0, Q>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    v[m] = make_float2(PR[m].x, PI[m].x);
    v[m + Q] = make_float2(PR[m].y, PI[m].y);
  });
}

// ---------------------------------------------------------------------------
// SRHT
// ---------------------------------------------------------------------------

// Walsh-Hadamard passes over bit planes 1 .. log2(d)-1 on packed natural
// pairs v[j] = (e_{2j}, e_{2j+1}) (plane 0 lives inside a pair).
template <int D>
__device__ __forceinline__ void wht_packed_planes(float2 (&v)[D / 2]) {
  constexpr int P = D / 2;
  static_for<0, ilog2(P)>([&](auto s_) {
    constexpr int h = 1 << decltype(s_)::value;
    static_for<0, P / (2 * h)>([&](auto b_) {
      constexpr int j = decltype(b_)::value * 2 * h;
      static_for<0, h>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        const float2 a = v[j + k], b = v[j + k + h];
        v[j + k] = add2(a, b);
        v[j + k + h] = sub2(a, b);
      });
    });
  });
}

// Forward SRHT from fp16 (same inputs as srft_forward); plane 0 from fp16.
template <int D>
__device__ __forceinline__ void srht_forward(const uint32_t (&xw)[D / 2],
                                             const uint32_t (&sw)[D / 2], float2 (&v)[D / 2]) {
  static_for<0, D / 2>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    const float t = fma_f16<1, 1>(xw[m], sw[m], 0.0f);
    v[m] = make_float2(fma_f16<0, 0>(xw[m], sw[m], t), fma_f16<0, 0>(xw[m], sw[m], -t));
  });
  wht_packed_planes<D>(v);
}

// Inverse SRHT on float pairs (the normalised Hadamard matrix is its own inverse).
template <int D>
__device__ __forceinline__ void srht_inverse(float2 (&v)[D / 2]) {
  static_for<0, D / 2>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    v[m] = make_float2(v[m].x + v[m].y, v[m].x - v[m].y);
  });
  wht_packed_planes<D>(v);
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
// is the output of rotate_forward; the inverse takes
// v_j = coordinate_gain(j) * yhat_j as input of rotate_inverse.
template <int ROT, int D>
__host__ __device__ constexpr double coordinate_gain(int j) {
  return (ROT == kSRFT ? srft_coordinate_gain(j, D) : 1.0) * inv_sqrt_pow2(D);
}

template <int ROT, int D>
__device__ __forceinline__ void rotate_forward(const uint32_t (&xw)[D / 2],
                                               const uint32_t (&sw)[D / 2], float2 (&v)[D / 2]) {
  if constexpr (ROT == kSRFT) {
    srft_forward<D>(xw, sw, v);
  } else {
    srht_forward<D>(xw, sw, v);
  }
}

template <int ROT, int D>
__device__ __forceinline__ void rotate_inverse(float2 (&v)[D / 2]) {
  if constexpr (ROT == kSRFT) {
    srft_inverse<D>(v);
  } else {
    srht_inverse<D>(v);
  }
}

}  // namespace srftq
