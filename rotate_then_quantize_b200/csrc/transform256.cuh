// d = 256: two threads per vector (lanes 2i and 2i+1; p = lane & 1).
//
// SRFT. The 256-point real DFT splits into two 128-point real DFTs of the
// even- and odd-indexed inputs, X_k = E_k + W^k O_k (W = exp(-2 pi i/256)),
// X_{128-k} = conj(E_k - W^k O_k). Lane p runs the d = 128 transform of
// transform.cuh on its sub-vector u_{2n+p} (p = 0 computes E, p = 1 computes
// O; identical code). Lane 0 then finishes bins k = i and lane 1 bins
// k = 32 + i, i = 0..32, after one exchange of half a spectrum with the
// partner lane; both lanes write their bins to the same register slots
// (bin k -> slot i, bin 128-k -> slot 64-i), so the code stays uniform.
// Slots map to packed coordinate pairs: lane 0 holds pairs 0..31 and 96..127
// (pair 0 holding X_0 and X_128), lane 1 pairs 32..95.
//
// SRHT. H_256 u = [H_128 (u_lo + u_hi); H_128 (u_lo - u_hi)] (Sylvester):
// lane 0 transforms u_lo + u_hi into pairs 0..63, lane 1 u_lo - u_hi into
// pairs 64..127 (the minus sign lives in lane 1's sign table).
//
// The inverses run the same steps backwards; their outputs are exchanged so
// that each lane writes one contiguous half of the fp16 row.
#pragma once

#include "transform.cuh"

namespace srftq {

__device__ __forceinline__ float shfl1(float v) { return __shfl_xor_sync(0xffffffffu, v, 1); }
__device__ __forceinline__ float2 shfl1(float2 v) { return make_float2(shfl1(v.x), shfl1(v.y)); }
__device__ __forceinline__ float2 sel2(bool p, float2 a, float2 b) {
  return make_float2(p ? a.x : b.x, p ? a.y : b.y);
}
__device__ __forceinline__ float2 cmul(float2 w, float2 z) {
  return make_float2(fmaf(w.x, z.x, -w.y * z.y), fmaf(w.x, z.y, w.y * z.x));
}
__device__ __forceinline__ float2 conj2(float2 z) { return make_float2(z.x, -z.y); }

// Packed coordinate pair held in slot j (j < 64) by lane p.
template <int ROT>
__host__ __device__ constexpr int pair256(int j, int p) {
  if (ROT == kSRHT) return p ? 64 + j : j;
  return p ? 32 + j : (j < 32 ? j : 64 + j);
}

// Forward SRFT, d = 256. xw[m] = (x_{4m+p}, x_{4m+2+p}) (this lane's
// sub-vector as fp16 pairs), sw the matching fp16 signs. Output slot j holds
// 2 X_k of bin k (real pair (2 X_0, 2 X_128) in lane 0's slot 0): packed
// coordinate y = out * sqrt(2) / 32 (1/32 for coordinates 0 and 1).
__device__ __forceinline__ void srft256_forward(const uint32_t (&xw)[64],
                                                const uint32_t (&sw)[64], bool p,
                                                float2 (&out)[64]) {
  float2 v[64];
  srft_forward<128>(xw, sw, v);   // v[0] = (F_0, F_64), v[32] = conj(F_32), v[j] = 2 F_j
  // bins 0, 32, 64, 96 (lane 0 finishes 0 / 128 / 96, lane 1 32 / 64)
  const float2 v0p = shfl1(v[0]), v32p = shfl1(v[32]);
  const float2 e0 = sel2(p, v0p, v[0]), o0 = sel2(p, v[0], v0p);
  const float2 e32 = sel2(p, v32p, v[32]), o32 = sel2(p, v[32], v32p);
  const float x0 = 2.0f * (e0.x + o0.x), x128 = 2.0f * (e0.x - o0.x);
  const float2 x64 = make_float2(2.0f * e0.y, -2.0f * o0.y);
  const float2 ge32 = make_float2(2.0f * e32.x, -2.0f * e32.y);
  const float2 go32 = make_float2(2.0f * o32.x, -2.0f * o32.y);
  constexpr float c8 = 0.70710678118654752440f;   // W^32 = (1 - i)/sqrt(2)
  const float2 t32 = make_float2(c8 * (go32.x + go32.y), c8 * (go32.y - go32.x));
  const float2 x32 = make_float2(ge32.x + t32.x, ge32.y + t32.y);
  const float2 x96 = make_float2(ge32.x - t32.x, t32.y - ge32.y);
  out[0] = sel2(p, x32, make_float2(x0, x128));
  out[32] = sel2(p, x64, x96);
  // general bins: lane 0 k = i, lane 1 k = 32 + i
  static_for<1, 32>([&](auto i_) {
    constexpr int i = decltype(i_)::value;
    const float2 recv = shfl1(sel2(p, v[i], v[32 + i]));
    const float2 e = sel2(p, recv, v[i]);
    const float2 o = sel2(p, v[32 + i], recv);
    constexpr float wa_r = float(ct::cos2pi(i, 256)), wa_i = float(-ct::sin2pi(i, 256));
    constexpr float wb_r = float(ct::cos2pi(32 + i, 256)), wb_i = float(-ct::sin2pi(32 + i, 256));
    const float2 w = make_float2(p ? wb_r : wa_r, p ? wb_i : wa_i);
    const float2 t = cmul(w, o);
    out[i] = make_float2(e.x + t.x, e.y + t.y);
    out[64 - i] = make_float2(e.x - t.x, t.y - e.y);
  });
}

// Inverse SRFT, d = 256. in slot j: X_k / 256 for this lane's bins (slot 0 of
// lane 0: the reals (X_0 / 256, X_128 / 256)). Output: this lane's sub-vector
// u_{2n+p} as pairs us[m] = (u_{4m+p}, u_{4m+2+p}) (before signs).
__device__ __forceinline__ void srft256_inverse(const float2 (&in)[64], bool p,
                                                float2 (&us)[64]) {
  // bins 0/128 (lane 0) and 64 (lane 1) are local; bin 32 needs X_32 (lane 1,
  // slot 0) and X_96 (lane 0, slot 32).
  const float2 in0p = shfl1(in[0]), in32p = shfl1(in[32]);
  const float2 x32 = sel2(p, in[0], in0p), x96 = sel2(p, in32p, in[32]);
  constexpr float c8 = 0.70710678118654752440f;   // conj(W^32) = (1 + i)/sqrt(2)
  const float2 e32 = make_float2(x32.x + x96.x, x32.y - x96.y);
  const float2 d32 = make_float2(x32.x - x96.x, x32.y + x96.y);
  const float2 o32 = make_float2(c8 * (d32.x - d32.y), c8 * (d32.x + d32.y));
  // lane 0: E0 = X0 + X128, O0 = X0 - X128 (from its slot 0); lane 1: E64 =
  // 2 Re X64, O64 = -2 Im X64 (from its slot 32). Each lane keeps what its own
  // spectrum needs and sends the partner the rest.
  const float e0 = in[0].x + in[0].y, o0 = in[0].x - in[0].y;       // valid in lane 0
  const float e64 = 2.0f * in[32].x, o64 = -2.0f * in[32].y;        // valid in lane 1
  // lane 0 needs E64 from lane 1; lane 1 needs O0 from lane 0
  const float xr = shfl1(p ? e64 : o0);
  float2 v[64];
  v[0] = p ? make_float2(xr, o64) : make_float2(e0, xr);
  const float2 f32 = sel2(p, o32, e32);
  v[32] = make_float2(2.0f * f32.x, -2.0f * f32.y);
  static_for<1, 32>([&](auto i_) {
    constexpr int i = decltype(i_)::value;
    const float2 xk = in[i], xm = in[64 - i];
    const float2 e = make_float2(xk.x + xm.x, xk.y - xm.y);
    const float2 d = make_float2(xk.x - xm.x, xk.y + xm.y);
    constexpr float wa_r = float(ct::cos2pi(i, 256)), wa_i = float(ct::sin2pi(i, 256));
    constexpr float wb_r = float(ct::cos2pi(32 + i, 256)), wb_i = float(ct::sin2pi(32 + i, 256));
    const float2 w = make_float2(p ? wb_r : wa_r, p ? wb_i : wa_i);   // conj(W^k)
    const float2 o = cmul(w, d);
    // lane 0 keeps E_i and receives E_{32+i}; lane 1 keeps O_{32+i}, receives O_i
    const float2 recv = shfl1(sel2(p, e, o));
    v[i] = sel2(p, recv, e);
    v[32 + i] = sel2(p, o, recv);
  });
  srft_inverse<128>(v);   // input convention: F_k / 128 (specials as above)
  static_for<0, 64>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    us[m] = v[m];
  });
}

// First step of the forward SRHT, d = 256, for one pair of fp16 words:
// xl = (x_{2m}, x_{2m+1}), xh = (x_{2m+128}, x_{2m+129}) with their fp16 sign
// pairs sl, sh (lane 1's sh negated). Returns bit plane 0 of u_lo +- u_hi:
// (a_0 + a_1, a_0 - a_1), each sum of two exact products rounded once.
__device__ __forceinline__ float2 srht256_plane0(uint32_t xl, uint32_t xh, uint32_t sl,
                                                 uint32_t sh) {
  const float a0 = fma_f16<0, 0>(xl, sl, fma_f16<0, 0>(xh, sh, 0.0f));
  const float a1 = fma_f16<1, 1>(xl, sl, fma_f16<1, 1>(xh, sh, 0.0f));
  return make_float2(a0 + a1, a0 - a1);
}

// The forward SRHT then runs the remaining planes of H_128 on the 64 pairs
// (wht_packed_planes<128>); output slot j = unnormalised pair, y = out / 16.

// Inverse SRHT, d = 256: in = this lane's half of yhat (scaled by 1/16);
// output pairs of x (before signs) for fp16 words [32p, 32p + 32) and
// [64 + 32p, 64 + 32p + 32) of the row: lo[k] -> word 32p + k,
// hi[k] -> word 64 + 32p + k.
__device__ __forceinline__ void srht256_inverse(float2 (&in)[64], bool p, float2 (&lo)[32],
                                                float2 (&hi)[32]) {
  static_for<0, 64>([&](auto m_) {
    constexpr int m = decltype(m_)::value;
    in[m] = make_float2(in[m].x + in[m].y, in[m].x - in[m].y);
  });
  wht_packed_planes<128>(in);
  // lane 0 combines its pairs k < 32 with lane 1's; lane 1 its pairs 32 + k
  static_for<0, 32>([&](auto k_) {
    constexpr int k = decltype(k_)::value;
    const float2 recv = shfl1(sel2(p, in[k], in[32 + k]));
    const float2 own = sel2(p, in[32 + k], in[k]);
    const float2 a = sel2(p, recv, own), b = sel2(p, own, recv);   // (H y_lo, H y_hi)
    lo[k] = make_float2(a.x + b.x, a.y + b.y);
    hi[k] = make_float2(a.x - b.x, a.y - b.y);
  });
}

}  // namespace srftq
