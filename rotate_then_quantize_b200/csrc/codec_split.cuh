// Fused quantise / dequantise kernels that split every vector over two
// warps, for d = 256. The code is written in terms of d; d = 128 keeps the
// one-thread kernels of codec.cuh, which measured faster there (the split's
// exchange, barriers and per-role bookkeeping cost more than its doubled
// resident warps gain).
//
// A block is two warps that share one tile of 32 vectors (the tile geometry,
// tile walk and early stage refill of codec.cuh); lane l of both warps holds
// vector l. The warps split every vector's transform by role R = warp index,
// so each role's code is compile-time (no per-lane selects or twiddle
// tables), and they meet at block barriers to swap half results through
// shared memory. Each thread holds d / 2 coordinates, which keeps the
// d = 256 transform in registers without spills.
//
// SRFT ("When Quantization Is Free", Methodology 1). The d-point real DFT of
// u = s x splits into the d/2-point real DFTs E and O of the even and odd
// samples: X_k = E_k + W^k O_k and X_{d/2-k} = conj(E_k - W^k O_k), with
// W = exp(-2 pi i / d). Warp R transforms the samples u_{2n+R} with the
// d/2 transform of transform.cuh, its first pass reading half R of the
// fp16 words straight from the staged tile. The warps swap half spectra.
// Warp 0 then forms the butterflies k = 0..d/8 and warp 1 k = d/8..d/4.
// Warp 0's d/4 output slots are the coordinate pairs 0..d/8-1 and
// 3d/8..d/2-1, slot 0 holding X_0 and X_{d/2}; warp 1's are the pairs
// d/8..3d/8-1.
//
// SRHT ("HyperQuant", Methodology 1). H_d u = [H_{d/2} (u_lo + u_hi);
// H_{d/2} (u_lo - u_hi)] in Sylvester order: warp 0 transforms the sum into
// pairs 0..d/4-1, warp 1 the difference into pairs d/4..d/2-1. There is no
// exchange.
//
// Every group of 8..d/4 coordinates lies inside one warp's slots, so each
// warp quantises its own groups. A group of d/2 or d coordinates spans both
// warps' slots (SRFT d/2: each warp holds half of both groups; d: each warp
// holds half of the one group) except SRHT d/2, where each warp holds one
// whole group: the warps then swap their partial group absmaxes through
// shared memory before the scales are formed, so both compute the same
// scales. The dequantiser runs the steps backwards.
// For SRFT it decodes one extra bin (X_{d/8}) in warp 0, so that both of its
// inverse butterflies are local. Its even/odd outputs are swapped once more,
// so that each warp writes whole fp16 words of one half of the row.
#pragma once

#include "codec.cuh"

namespace srftq {

template <int D, int BITS, int G>
struct SplitShape {
  static_assert(D == 256, "split head dimension");
  static_assert(G >= 8 && G <= D && (G & (G - 1)) == 0, "group (split kernels)");
  static_assert(BITS == 4 || BITS == 8, "bits");
  static constexpr int TR = kTileRows;                   // vectors per tile
  static constexpr int DH = D / 2;                       // coordinates per role
  static constexpr int NP = D / 4;                       // slots (pairs) per role
  static constexpr int NQ = D / 8;                       // butterflies per role
  static constexpr int XB = 2 * D, X_SPAN = 128, X_PIECES = XB / 128, X_TILE = TR * XB;
  static constexpr int XC = XB / 16;                     // 16-byte chunks per fp16 row
  static constexpr int CB = D * BITS / 8;                // code bytes per vector
  static constexpr int C_SPAN = CB < 128 ? CB : 128, C_PIECES = CB / C_SPAN, C_TILE = TR * CB;
  static constexpr int C_CPP = C_SPAN / 16;              // 16-byte chunks per code piece
  static constexpr int SPC = 64 / BITS;                  // slots (pairs) per 16-byte chunk
  static constexpr int KR = NP / SPC;                    // code chunks per role
  static constexpr int CWR = 4 * KR;                     // code words per role
  static constexpr int NG = D / G;                       // groups per vector
  static constexpr int NGR = G <= D / 4 ? DH / G : 1;    // groups per role (local groups)
  static constexpr int GS = G / 2;                       // slots per group
  static constexpr int QMAX = (1 << (BITS - 1)) - 1;
  // SRFT role 0's groups are the vector's first and last NGR / 2: scale
  // words (two consecutive groups) stay aligned when NGR / 2 is even
  static constexpr bool kScaleWords = NGR % 4 == 0;
};

// Groups of one role's NP slots. kLocal: every group lies inside one role
// (G <= d/4; NGR groups of G/2 slots, mapped by split_group). Otherwise the
// role's slots fall into LG local groups of LGS slots each: SRFT G = d/2,
// the two slot halves belong to global groups 0 and 1 (in both roles); SRHT
// G = d/2, all slots belong to global group R; G = d, all to group 0.
// kCross: a global group has slots in both roles.
template <int D, int G, int ROT>
struct SplitGroups {
  static constexpr int NP = D / 4;
  static constexpr bool kLocal = G <= D / 4;
  static constexpr int LGS = kLocal ? G / 2 : ((ROT == kSRFT && G == D / 2) ? NP / 2 : NP);
  static constexpr int LG = NP / LGS;
  static constexpr bool kCross = !kLocal && !(ROT == kSRHT && G == D / 2);
};

// Per-block shared-memory layout: the input stage (x tile for the quantiser,
// codes for the dequantiser), the output staging tile, one exchange row per
// lane and warp (d/8 + 2 float2; the stride keeps the 16-byte accesses of 8
// lanes on distinct banks), the per-head tables of up to kMaxHPT heads
// (multipliers of both roles' slots, d floats; sign words, up to 3d/4) and
// the barrier.
template <int D, int BITS, int G, bool QUANT>
struct SplitLayout {
  using S = SplitShape<D, BITS, G>;
  static constexpr int kInTile = QUANT ? S::X_TILE : S::C_TILE;
  static constexpr int kInBytes = align_up(kInTile, 1024);
  static constexpr int kOutTile = QUANT ? S::C_TILE : S::X_TILE;
  static constexpr int kOutOff = kInBytes;
  static constexpr int kXchLane = (S::NQ + 2) * 8, kXchWarp = 32 * kXchLane;
  static constexpr int kXchOff = kOutOff + align_up(kOutTile, 1024);
  static constexpr int kXch2Off = kXchOff + 2 * kXchWarp;   // end of the exchange rows
  static constexpr int kMultStride = D + 4;           // floats per head
  static constexpr int kSignStride = 3 * D / 4 + 4;   // words per head
  static constexpr int kTableOff = kXch2Off;
  static constexpr int kSignTabOff = kTableOff + 4 * kMaxHPT * kMultStride;
  static constexpr int kBarOff = align_up(kSignTabOff + 4 * kMaxHPT * kSignStride, 16);
  // partial group absmaxes of both roles (2 per lane), for groups wider than d/4
  static constexpr int kAmxOff = kBarOff + 16;
  static constexpr int kBytes = kAmxOff + (G > D / 4 ? 2 * 32 * 2 * 4 : 0);
};

// (role, slot) holding coordinate pair p, and whether the slot stores the
// conjugate of the bin (SRFT: warp 0's slots d/8..d/4-1, warp 1's
// d/8+1..d/4-1).
template <int D, int ROT>
__device__ __forceinline__ void split_pair_slot(int p, int& r, int& j, bool& conj) {
  constexpr int NP = D / 4, NQ = D / 8;
  if (ROT == kSRHT) {
    r = p >= NP ? 1 : 0;
    j = p & (NP - 1);
    conj = false;
  } else {
    r = (p >= NQ && p < 3 * NQ) ? 1 : 0;
    j = r ? p - NQ : (p < NQ ? p : p - 2 * NQ);
    conj = r ? j >= NQ + 1 : j >= NQ;
  }
}

// Block barrier of the two warps (named barrier 1).
__device__ __forceinline__ void bar_pair() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

__device__ __forceinline__ float2 u2f2(uint2 u) {
  return make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
}
__device__ __forceinline__ uint2 f22u(float2 f) {
  return make_uint2(__float_as_uint(f.x), __float_as_uint(f.y));
}

// Builds the tables of the HPT heads of (slice s, head block hb) with all 64
// threads. Multipliers, per slot of each role (lane x / lane y = the pair's
// even / odd coordinate), for the slot values of the transforms below:
//   quantiser, SRFT: a slot holds 2 X_k, so the gain is 1/sqrt(2d) (slot 0
//   of role 0, X_0 and X_{d/2}: 1/(2 sqrt(d))), the imaginary gain negated
//   in conjugate slots; SRHT: 1/sqrt(d); each divided by lambda;
//   dequantiser, SRFT: the inverse butterflies want X_k / d, so the gain is
//   1/sqrt(2d) (slot 0 of role 0: 1/sqrt(d)), the imaginary gain negated in
//   conjugate slots; SRHT: 1/sqrt(d); each times lambda (int4: / 16 at odd
//   coordinates, whose code sits in the high nibble).
// Sign words: SRFT, per role R word m = (s_{4m+R}, s_{4m+2+R}) at R d/4 + m;
// the dequantiser's role 1 words also flip the sign of their second sample
// (see dequantize_split_kernel); SRHT quantiser: (s_{2w}, s_{2w+1}) for the
// low half (w < d/4) at w, the high half at w for role 0 and negated at
// d/4 + w for role 1 (which transforms u_lo - u_hi); SRHT dequantiser: word
// w = (s_{2w}, s_{2w+1}), w < d/2. Quantiser words are fp16 +-1 pairs,
// dequantiser words sign-bit masks.
template <int D, int BITS, int ROT, bool QUANT, int MS, int SS>
__device__ __forceinline__ void build_split_tables(float* mult, uint32_t* stab,
                                                   const float* lambda, const int8_t* signs,
                                                   int s, int hb, int H, int hpt_log2, int tid) {
  constexpr int NP = D / 4, DH = D / 2;
  constexpr int kL4 = kMaxHPT * D / 4 / 64;    // float4 loads per thread, at most
  constexpr int kS16 = kMaxHPT * D / 16 / 64;  // 16-sign loads per thread, at most
  constexpr float kRoot = float(inv_sqrt_pow2(D));        // 1/sqrt(d)
  constexpr float kRoot2 = float(inv_sqrt_pow2(2 * D));   // 1/sqrt(2d)
  const int hpt = 1 << hpt_log2;
  const size_t h0 = static_cast<size_t>(s) * H + static_cast<size_t>(hb) * hpt;
  const float4* lam4 = reinterpret_cast<const float4*>(lambda + h0 * D);
  const uint4* sg16 = reinterpret_cast<const uint4*>(signs + h0 * D);
  const int n4 = hpt * (D / 4), n16 = hpt * (D / 16);
  float4 l[kL4];
  uint4 g[kS16];
#pragma unroll
  for (int k = 0; k < kL4; ++k) {
    const int i = tid + 64 * k;
    if (i < n4) l[k] = __ldg(lam4 + i);
  }
#pragma unroll
  for (int k = 0; k < kS16; ++k) {
    const int i = tid + 64 * k;
    if (i < n16) g[k] = __ldg(sg16 + i);
  }
  __syncthreads();   // every thread is done reading the old tables
#pragma unroll
  for (int k = 0; k < kL4; ++k) {
    const int i = tid + 64 * k;
    if (i < n4) {
      const int h = i / (D / 4), c0 = 4 * (i % (D / 4));   // head, first coordinate
      const float lv[4] = {l[k].x, l[k].y, l[k].z, l[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = c0 + e, p = c >> 1, odd = c & 1;
        int r, j;
        bool conj;
        split_pair_slot<D, ROT>(p, r, j, conj);
        float gain;
        if constexpr (ROT == kSRHT) {
          gain = kRoot;
        } else if constexpr (QUANT) {
          gain = (r == 0 && j == 0) ? 0.5f * kRoot : kRoot2;
        } else {
          gain = (r == 0 && j == 0) ? kRoot : kRoot2;
        }
        if (odd && conj) gain = -gain;
        float m;
        if constexpr (QUANT)
          m = gain * rcp_approx(lv[e]);
        else
          m = gain * lv[e] * ((BITS == 4 && odd) ? 0.0625f : 1.0f);
        mult[h * MS + r * DH + 2 * j + odd] = m;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kS16; ++k) {
    const int i = tid + 64 * k;
    if (i < n16) {
      const int h = i / (D / 16), c0 = 16 * (i % (D / 16));   // head, first sign of the chunk
      const uint32_t wd[4] = {g[k].x, g[k].y, g[k].z, g[k].w};
      auto sb = [&](int t) -> int8_t { return static_cast<int8_t>(wd[t >> 2] >> (8 * (t & 3))); };
      if constexpr (ROT == kSRHT) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int8_t s0 = sb(2 * e), s1 = sb(2 * e + 1);
          const int w = c0 / 2 + e;
          if constexpr (QUANT) {
            const uint32_t sw = sign_halves(s0, s1);
            if (w < NP) {
              stab[h * SS + w] = sw;
            } else {
              stab[h * SS + w] = sw;                       // role 0: + u_hi
              stab[h * SS + NP + w] = sw ^ 0x80008000u;    // role 1: - u_hi
            }
          } else {
            stab[h * SS + w] = sign_mask(s0, s1);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {   // samples 4m .. 4m + 3, m = c0 / 4 + e
          const int m = c0 / 4 + e;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int8_t s0 = sb(4 * e + r), s1 = sb(4 * e + 2 + r);
            // the dequantiser's role 1 inverts the spectrum shifted by d/4
            // bins, whose samples carry (-1)^n: the odd one of each pair is
            // negated
            stab[h * SS + r * NP + m] =
                QUANT ? sign_halves(s0, s1) : (sign_mask(s0, s1) ^ (r ? 0x80000000u : 0u));
          }
        }
      }
    }
  }
  __syncthreads();
}

// Address of 16-byte chunk ci of an fp16 row in a tile of 128-byte-swizzled
// pieces of 32 rows (xrow = swz_row<128>(tile, lane)).
__device__ __forceinline__ uint32_t row_chunk(uint32_t xrow, int ci) {
  return swz_chunk<128>(xrow, ci & 7) + (ci >> 3) * (kTileRows * 128);
}

// Address of 16-byte chunk cg of a code row (crow = swz_row<C_SPAN>(tile, lane)).
template <typename S>
__device__ __forceinline__ uint32_t code_chunk_addr(uint32_t crow, int cg) {
  return swz_chunk<S::C_SPAN>(crow, cg % S::C_CPP) + (cg / S::C_CPP) * (S::TR * S::C_SPAN);
}

// ---------------------------------------------------------------------------
// Transforms (one code path for both roles)
// ---------------------------------------------------------------------------

// SRFT: the d/2-point real DFT of u_{2n+R}, from the staged fp16 row. Its
// complex sample m is (u_{4m+R}, u_{4m+2+R}): half R of x words 2m and
// 2m + 1, gathered with one PRMT (sel = 0x5410 for R = 0, 0x7632 for R = 1);
// sgn = this role's sign words (lo half = real part's sign).
template <int D>
__device__ __forceinline__ void srft_split_forward(uint32_t xrow, uint32_t sel,
                                                   const uint32_t* sgn, float2 (&v)[D / 4]) {
  constexpr int Q = D / 8, LOG = ilog2(D / 4);
  float2 PR[Q], PI[Q];
  // pass 1: butterflies (z_m, z_{m+Q}) into the bit-reversed slots
  // i = bitrev(m), i + 1; two at a time from two 16-byte chunks each.
  static_for<0, Q / 2>([&](auto c_) {
    constexpr int c = decltype(c_)::value;
    const uint4 A = lds128(row_chunk(xrow, c));           // words 4c .. 4c+3: m = 2c, 2c+1
    const uint4 B = lds128(row_chunk(xrow, Q / 2 + c));   // m = 2c+Q, 2c+Q+1
    const uint2 sa = *reinterpret_cast<const uint2*>(sgn + 2 * c);
    const uint2 sbb = *reinterpret_cast<const uint2*>(sgn + Q + 2 * c);
    const uint32_t za[2] = {__byte_perm(A.x, A.y, sel), __byte_perm(A.z, A.w, sel)};
    const uint32_t zb[2] = {__byte_perm(B.x, B.y, sel), __byte_perm(B.z, B.w, sel)};
    const uint32_t sA[2] = {sa.x, sa.y}, sB[2] = {sbb.x, sbb.y};
    static_for<0, 2>([&](auto e_) {
      constexpr int e = decltype(e_)::value;
      constexpr int i = bitrev(2 * c + e, LOG);
      const float tr = fma_f16<0, 0>(zb[e], sB[e], 0.0f);
      const float ti = fma_f16<1, 1>(zb[e], sB[e], 0.0f);
      lane<Q, i>(PR) = fma_f16<0, 0>(za[e], sA[e], tr);
      lane<Q, i + 1>(PR) = fma_f16<0, 0>(za[e], sA[e], -tr);
      lane<Q, i>(PI) = fma_f16<1, 1>(za[e], sA[e], ti);
      lane<Q, i + 1>(PI) = fma_f16<1, 1>(za[e], sA[e], -ti);
    });
  });
  srft_forward_rest<D / 2>(PR, PI, v);
}

// SRHT: H_{d/2} of u_lo + u_hi (role 0) or u_lo - u_hi (role 1; the minus
// sign lives in that role's high-half sign words), unnormalised, natural
// pairs.
template <int D>
__device__ __forceinline__ void srht_split_forward(uint32_t xrow, const uint32_t* slo,
                                                   const uint32_t* shi, float2 (&v)[D / 4]) {
  constexpr int HC = D / 16;   // 16-byte chunks per half row
  static_for<0, HC>([&](auto c_) {
    constexpr int c = decltype(c_)::value;
    const uint4 wl = lds128(row_chunk(xrow, c)), wh = lds128(row_chunk(xrow, HC + c));
    const uint4 sl = *reinterpret_cast<const uint4*>(slo + 4 * c);
    const uint4 sh = *reinterpret_cast<const uint4*>(shi + 4 * c);
    const uint32_t l[4] = {wl.x, wl.y, wl.z, wl.w}, hh[4] = {wh.x, wh.y, wh.z, wh.w};
    const uint32_t ls[4] = {sl.x, sl.y, sl.z, sl.w}, hs[4] = {sh.x, sh.y, sh.z, sh.w};
    static_for<0, 4>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      const float a0 = fma_f16<0, 0>(l[k], ls[k], fma_f16<0, 0>(hh[k], hs[k], 0.0f));
      const float a1 = fma_f16<1, 1>(l[k], ls[k], fma_f16<1, 1>(hh[k], hs[k], 0.0f));
      v[4 * c + k] = make_float2(a0 + a1, a0 - a1);
    });
  });
  wht_packed_planes<D / 2>(v);
}

// S(k) = 2 F_k of a d/2-point forward output v (NP = d/4 pairs):
// v[0] = (F_0, F_{d/4}), v[d/8] = conj F_{d/8}, v[k] = 2 F_k otherwise.
template <int NP, int K>
__device__ __forceinline__ float2 spec2(const float2 (&v)[NP]) {
  if constexpr (K == 0) {
    return make_float2(2.0f * v[0].x, 0.0f);
  } else if constexpr (K == NP) {
    return make_float2(2.0f * v[0].y, 0.0f);
  } else if constexpr (2 * K == NP) {
    return make_float2(2.0f * v[K].x, -2.0f * v[K].y);
  } else {
    return v[K];
  }
}

// Writes S(k) for k = K0 .. K0 + NP/2 (NP/2 + 1 values) to this lane's
// exchange row.
template <int NP, int K0>
__device__ __forceinline__ void put_half_spectrum(uint32_t row, const float2 (&v)[NP]) {
  constexpr int NQ = NP / 2;
  static_for<0, NQ / 2>([&](auto j_) {
    constexpr int j = decltype(j_)::value;
    const float2 a = spec2<NP, K0 + 2 * j>(v), b = spec2<NP, K0 + 2 * j + 1>(v);
    sts128(row + 16 * j, make_uint4(__float_as_uint(a.x), __float_as_uint(a.y),
                                    __float_as_uint(b.x), __float_as_uint(b.y)));
  });
  sts64(row + 8 * NQ, f22u(spec2<NP, K0 + NQ>(v)));
}

// Forward combine of role R after the exchange: own = this role's d/2
// spectrum, rr = the partner's exchange row (S of the other sub-sequence,
// k = 0..d/8 for role 0, k = d/8..d/4 for role 1). out[j] = slot j.
template <int D, int R>
__device__ __forceinline__ void srft_split_combine(const float2 (&own)[D / 4], uint32_t rr,
                                                   float2 (&out)[D / 4]) {
  constexpr int NP = D / 4, NQ = D / 8;
  auto recv = [&](int j) -> float2 { return u2f2(lds64(rr + 8 * j)); };
  if constexpr (R == 0) {
    {   // k = 0: X_0 and X_{d/2} are real
      const float2 o = recv(0);
      const float e = spec2<NP, 0>(own).x;
      out[0] = make_float2(e + o.x, e - o.x);
    }
    static_for<1, NQ + 1>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      float2 a = spec2<NP, k>(own), b = recv(k);
      butterfly<-1, k, D / 2>(a.x, a.y, b.x, b.y);
      if constexpr (k < NQ) out[k] = a;
      out[NP - k] = b;
    });
  } else {
    static_for<NQ, NP>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      float2 a = recv(k - NQ), b = spec2<NP, k>(own);
      butterfly<-1, k, D / 2>(a.x, a.y, b.x, b.y);
      out[k - NQ] = a;
      if constexpr (k > NQ) out[3 * NQ - k] = b;
    });
    {   // k = d/4: X_{d/4} = E_{d/4} - i O_{d/4} (E_{d/4}, O_{d/4} real)
      const float2 e = recv(NQ);
      out[NQ] = make_float2(e.x, -spec2<NP, NP>(own).x);
    }
  }
}

// Global code chunk of a role's local chunk k (KR chunks of SPC slots).
template <int ROT, int KR>
__device__ __forceinline__ int split_code_chunk(int k, int role) {
  if constexpr (ROT == kSRHT) return k + role * KR;
  return k + (role ? KR / 2 : (k < KR / 2 ? 0 : KR));
}

// Global group of a role's local group g (NGR groups of G / 2 slots).
template <int ROT, int NGR>
__device__ __forceinline__ int split_group(int g, int role) {
  if constexpr (ROT == kSRHT) return g + role * NGR;
  return g + (role ? NGR / 2 : (g < NGR / 2 ? 0 : NGR));
}

// ---------------------------------------------------------------------------
// Quantiser
// ---------------------------------------------------------------------------

template <int D, int BITS, int G, int ROT, int MINB>
__global__ void __launch_bounds__(64, MINB)
    quantize_split_kernel(const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_codes, const QuantArgs a) {
  using S = SplitShape<D, BITS, G>;
  using Lay = SplitLayout<D, BITS, G, true>;
  using Grp = SplitGroups<D, G, ROT>;
  constexpr int NP = S::NP;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int tid = threadIdx.x;
  const int role = tid >> 5;
  const int lane = tid & 31;
  const bool leader = tid == 0;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(smem + Lay::kTableOff);
  uint32_t* stab = reinterpret_cast<uint32_t*>(smem + Lay::kSignTabOff);
  uint8_t* sb = smem;                       // x stage
  uint8_t* ob = smem + Lay::kOutOff;        // codes staging tile

  TileWalk cur;
  if (!cur.start(blockIdx.x, gridDim.x, a.g)) return;
  const int hpt_log2 = a.g.hpt_log2;
  const int hpt = 1 << hpt_log2;
  const int rpt = kTileRows >> hpt_log2;
  const int hl = lane & (hpt - 1);
  const int rl = lane >> hpt_log2;
  const float* mrow = mult + hl * Lay::kMultStride + role * S::DH;
  const uint32_t* srow = stab + hl * Lay::kSignStride;
  const uint32_t* s1 = srow + (ROT == kSRFT ? role * NP : 0);          // SRFT: role words
  const uint32_t* s2 = srow + NP + role * NP;                           // SRHT: high half
  const uint32_t psel = role ? 0x7632u : 0x5410u;
  const uint32_t xrow = swz_row<128>(smem_addr(sb), lane);
  const uint32_t crow = swz_row<S::C_SPAN>(smem_addr(ob), lane);
  const uint32_t xch = smem_addr(smem + Lay::kXchOff);
  const uint32_t my_row = xch + role * Lay::kXchWarp + lane * Lay::kXchLane;
  const uint32_t partner_row = xch + (1 - role) * Lay::kXchWarp + lane * Lay::kXchLane;

  if (leader) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_codes);
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](const TileWalk& c) {
    if (!dbg_ok(tile_in_range(c, a.g), a.guard)) {
      mbar_arrive(bar);   // debug build: no copy, the phase completes empty
      return;
    }
    mbar_arrive_expect_tx(bar, S::X_TILE);
#pragma unroll
    for (int pc = 0; pc < S::X_PIECES; ++pc)
      tma_load_4d(sb + pc * (S::TR * S::X_SPAN), &tm_x, bar, pc * 64, c.hb * hpt, c.rb * rpt,
                  c.s);
  };
  auto store_codes = [&](const TileWalk& c) {
    if (dbg_ok(tile_in_range(c, a.g), a.guard)) {
#pragma unroll
      for (int pc = 0; pc < S::C_PIECES; ++pc)
        tma_store_4d(&tm_codes, ob + pc * (S::TR * S::C_SPAN), pc * S::C_SPAN, c.hb * hpt,
                     c.rb * rpt, c.s);
    }
    bulk_commit();
  };

  TileWalk ahead = cur;
  if (leader) {
    issue(ahead);
    ahead.advance(a.g);
  }

  int it = 0;
  int table_key = -1;
  bool pending = false;
  TileWalk prev = cur;
  for (; cur.valid(); ++it) {
    const int key = cur.table_key(a.g);
    if (key != table_key) {
      build_split_tables<D, BITS, ROT, true, Lay::kMultStride, Lay::kSignStride>(
          mult, stab, a.lambda, a.signs, cur.s, cur.hb, a.g.heads, hpt_log2, tid);
      table_key = key;
    }
    const bool ok = __syncthreads_and(mbar_wait_bounded(bar, it & 1)) != 0;
    if (!ok) {
      if (leader) {
        atomicOr(a.guard, kGuardWaitTimeout);
        bulk_wait<0>();
      }
      return;
    }

    // (b) this role's transform, straight from the staged row
    float2 v[NP];
    if constexpr (ROT == kSRFT)
      srft_split_forward<D>(xrow, psel, s1, v);
    else
      srht_split_forward<D>(xrow, srow, s2, v);
    // Both warps have read the stage and staged + fenced the previous
    // tile's codes: store those and refill the stage with the next tile.
    bar_pair();
    if (leader) {
      if (pending) store_codes(prev);
      if (ahead.valid()) {
        issue(ahead);
        ahead.advance(a.g);
      }
    }
    pending = false;

    // (c) SRFT: swap half spectra, butterflies of (E_k, O_k). The leader
    // also confirms that the store it just issued has read the staging tile
    // before anyone writes it again.
    float2 y[NP];
    if constexpr (ROT == kSRFT) {
      if (role == 0)
        put_half_spectrum<NP, S::NQ>(my_row, v);
      else
        put_half_spectrum<NP, 0>(my_row, v);
      if (leader) bulk_wait_read<0>();
      bar_pair();
      if (role == 0)
        srft_split_combine<D, 0>(v, partner_row, y);
      else
        srft_split_combine<D, 1>(v, partner_row, y);
    } else {
      if (leader) bulk_wait_read<0>();
      bar_pair();
      static_for<0, NP>([&](auto j_) { y[decltype(j_)::value] = v[decltype(j_)::value]; });
    }

    // (d) multipliers, group absmax, scales, codes (as in codec.cuh)
    static_for<0, NP / 2>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = *reinterpret_cast<const float4*>(mrow + 4 * ci);
      y[2 * ci] = mul2(y[2 * ci], make_float2(m4.x, m4.y));
      y[2 * ci + 1] = mul2(y[2 * ci + 1], make_float2(m4.z, m4.w));
    });
    // local groups of LGS slots (every group of this role, or this role's
    // part of a group that spans both roles)
    constexpr int LG = Grp::kLocal ? S::NGR : Grp::LG;
    constexpr int LGS = Grp::kLocal ? S::GS : Grp::LGS;
    float am[LG];
    static_for<0, LG>([&](auto g_) {
      constexpr int g = decltype(g_)::value;
      constexpr int P0 = g * LGS;
      float m = absmax3(0.0f, y[P0].x, y[P0].y);
      static_for<1, LGS>([&](auto p_) {
        constexpr int p = P0 + decltype(p_)::value;
        m = absmax3(m, y[p].x, y[p].y);
      });
      am[g] = m;
    });
    if constexpr (Grp::kCross) {
      // both roles hold part of every group: swap the partial absmaxes (the
      // slots of this exchange were last read before this tile's first barrier)
      float* amx = reinterpret_cast<float*>(smem + Lay::kAmxOff);
      static_for<0, LG>([&](auto g_) {
        constexpr int g = decltype(g_)::value;
        amx[(role * 32 + lane) * 2 + g] = am[g];
      });
      bar_pair();
      static_for<0, LG>([&](auto g_) {
        constexpr int g = decltype(g_)::value;
        am[g] = fmaxf(am[g], amx[((1 - role) * 32 + lane) * 2 + g]);
      });
    }
    float a_hi, a_lo;
    range_of(am, a_hi, a_lo);
    constexpr float kHi = 65504.0f * float(S::QMAX);
    constexpr float kLo = 6.103515625e-05f * float(S::QMAX);
    uint32_t sw[(LG + 1) / 2];
    uint32_t qb[2 * NP];
    if (a_hi <= kHi && a_lo >= kLo) {
      float invs[LG];
      group_scales<LG, S::QMAX, true>(am, sw, invs);
      static_for<0, NP>([&](auto p_) {
        constexpr int p = decltype(p_)::value;
        const float2 r = fma2(y[p], splat(invs[p / LGS]), splat(kMagic));
        qb[2 * p] = __float_as_uint(r.x);
        qb[2 * p + 1] = __float_as_uint(r.y);
      });
    } else {
      float invs[LG];
      group_scales<LG, S::QMAX, false>(am, sw, invs);
      static_for<0, NP>([&](auto p_) {
        constexpr int p = decltype(p_)::value;
        const float inv = invs[p / LGS];
        const float q0 = fminf(fmaxf(y[p].x * inv, -float(S::QMAX)), float(S::QMAX));
        const float q1 = fminf(fmaxf(y[p].y * inv, -float(S::QMAX)), float(S::QMAX));
        qb[2 * p] = __float_as_uint(q0 + kMagic);
        qb[2 * p + 1] = __float_as_uint(q1 + kMagic);
      });
    }
    uint32_t words[S::CWR];
    if constexpr (BITS == 4) {
      static_for<0, NP / 4>([&](auto m_) {
        constexpr int m = decltype(m_)::value;
        const uint32_t ev = __byte_perm(__byte_perm(qb[8 * m + 0], qb[8 * m + 2], 0x0040),
                                        __byte_perm(qb[8 * m + 4], qb[8 * m + 6], 0x0040), 0x5410);
        const uint32_t od = __byte_perm(__byte_perm(qb[8 * m + 1], qb[8 * m + 3], 0x0040),
                                        __byte_perm(qb[8 * m + 5], qb[8 * m + 7], 0x0040), 0x5410);
        words[m] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
      });
    } else {
      static_for<0, NP / 2>([&](auto m_) {
        constexpr int m = decltype(m_)::value;
        words[m] = __byte_perm(__byte_perm(qb[4 * m], qb[4 * m + 1], 0x0040),
                               __byte_perm(qb[4 * m + 2], qb[4 * m + 3], 0x0040), 0x5410);
      });
    }

    // (e) this role's code chunks into the staging tile
    static_for<0, S::KR>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      const int cg = split_code_chunk<ROT, S::KR>(k, role);   // chunk in the row
      sts128(code_chunk_addr<S>(crow, cg),
             make_uint4(words[4 * k], words[4 * k + 1], words[4 * k + 2], words[4 * k + 3]));
    });
    fence_proxy_async_smem();
    pending = true;
    prev = cur;

    // (f) this role's scales; consecutive global groups go out as words
    const int row = cur.rb * rpt + rl;
    const size_t svec = (static_cast<size_t>(cur.s) * a.out_slice_stride_rows + row) *
                            a.g.heads + cur.hb * hpt + hl;
    if (row < a.g.n_rows &&
        dbg_ok(int64_t(svec) < vec_limit(a.g.n_slices, a.out_slice_stride_rows, a.g.n_rows,
                                         a.g.heads),
               a.guard)) {
      uint16_t* dst = a.scales + svec * S::NG;
      if constexpr (Grp::kLocal) {
        constexpr bool kWords = ROT == kSRHT || S::kScaleWords;
        static_for<0, S::NGR / 2>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          const int g0 = split_group<ROT, S::NGR>(2 * k, role);
          if constexpr (kWords) {
            *reinterpret_cast<uint32_t*>(dst + g0) = sw[k];
          } else {
            dst[g0] = static_cast<uint16_t>(sw[k] & 0xFFFFu);
            dst[split_group<ROT, S::NGR>(2 * k + 1, role)] = static_cast<uint16_t>(sw[k] >> 16);
          }
        });
      } else if constexpr (Grp::kCross) {
        // both roles hold every scale of the vector (NG = 1 or 2); role 0 stores them
        if (role == 0) {
          if constexpr (S::NG == 2)
            *reinterpret_cast<uint32_t*>(dst) = sw[0];
          else
            dst[0] = static_cast<uint16_t>(sw[0] & 0xFFFFu);
        }
      } else {
        dst[role] = static_cast<uint16_t>(sw[0] & 0xFFFFu);   // SRHT, G = d/2: group R
      }
    }
    cur.advance(a.g);
  }
  __syncthreads();
  if (leader) {
    if (pending) store_codes(prev);
    bulk_wait<0>();
  }
}

// ---------------------------------------------------------------------------
// Dequantiser
// ---------------------------------------------------------------------------

// Decodes the 4 (int4: one word = 4 slots) or 2 (int8) slots of code word w
// of group scale half HS of word sgw into out.
template <int BITS, int HS>
__device__ __forceinline__ void decode_split_word(uint32_t w, uint32_t sgw, float2* out) {
  const float sgf = __half2float(__ushort_as_half(
      static_cast<unsigned short>((sgw >> (16 * HS)) & 0xFFFFu)));
  const float c_even = BITS == 4 ? -1032.0f * sgf : -1152.0f * sgf;
  const float c_odd = -1152.0f * sgf;
  unpack_word<BITS, HS>(w, sgw, c_even, c_odd, out);
}

// DIF butterfly for bin K: (a, b) <- (a + b, conj(W^K) (a - b)), W = exp(-2 pi i / d).
template <int D, int K>
__device__ __forceinline__ void split_dif(float2& a, float2& b) {
  const float2 s = add2(a, b), d = sub2(a, b);
  a = s;
  if constexpr (K == 0) {
    b = d;
  } else if constexpr (4 * K == D) {
    b = make_float2(-d.y, d.x);   // times i
  } else {
    constexpr double cw = ct::cos2pi(K, D), sn = ct::sin2pi(K, D);
    constexpr float c = float(cw), t = float(sn / cw);   // conj(W^K) = cw + i sn
    b = make_float2(c * fmaf(-t, d.y, d.x), c * fmaf(t, d.x, d.y));
  }
}

template <int D, int BITS, int G, int ROT, int MINB>
__global__ void __launch_bounds__(64, MINB)
    dequantize_split_kernel(const __grid_constant__ CUtensorMap tm_codes,
                            const __grid_constant__ CUtensorMap tm_xhat, const DequantArgs a) {
  using S = SplitShape<D, BITS, G>;
  using Lay = SplitLayout<D, BITS, G, false>;
  constexpr int NP = S::NP, NQ = S::NQ;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int tid = threadIdx.x;
  const int role = tid >> 5;
  const int lane = tid & 31;
  const bool leader = tid == 0;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(smem + Lay::kTableOff);
  uint32_t* mtab = reinterpret_cast<uint32_t*>(smem + Lay::kSignTabOff);
  uint8_t* sb = smem;                       // codes stage
  uint8_t* ob = smem + Lay::kOutOff;        // fp16 staging tile

  TileWalk cur;
  if (!cur.start(blockIdx.x, gridDim.x, a.g)) return;
  const int hpt_log2 = a.g.hpt_log2;
  const int hpt = 1 << hpt_log2;
  const int rpt = kTileRows >> hpt_log2;
  const int hl = lane & (hpt - 1);
  const int rl = lane >> hpt_log2;
  const float* mbase = mult + hl * Lay::kMultStride;
  const float* mrow = mbase + role * S::DH;
  const uint32_t* mkrow = mtab + hl * Lay::kSignStride;
  const uint32_t* mk = mkrow + (ROT == kSRFT ? role * NP : 0);
  const uint32_t crow = swz_row<S::C_SPAN>(smem_addr(sb), lane);
  const uint32_t xrow = swz_row<128>(smem_addr(ob), lane);
  const uint32_t xch = smem_addr(smem + Lay::kXchOff);
  const uint32_t my_row = xch + role * Lay::kXchWarp + lane * Lay::kXchLane;
  const uint32_t partner_row = xch + (1 - role) * Lay::kXchWarp + lane * Lay::kXchLane;

  if (leader) {
    prefetch_tensormap(&tm_codes);
    prefetch_tensormap(&tm_xhat);
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](const TileWalk& c) {
    if (!dbg_ok(tile_in_range(c, a.g), a.guard)) {
      mbar_arrive(bar);   // debug build: no copy, the phase completes empty
      return;
    }
    mbar_arrive_expect_tx(bar, S::C_TILE);
#pragma unroll
    for (int pc = 0; pc < S::C_PIECES; ++pc)
      tma_load_4d(sb + pc * (S::TR * S::C_SPAN), &tm_codes, bar, pc * S::C_SPAN, c.hb * hpt,
                  c.rb * rpt, c.s);
  };
  auto store_xhat = [&](const TileWalk& c) {
    if (dbg_ok(tile_in_range(c, a.g), a.guard)) {
#pragma unroll
      for (int pc = 0; pc < S::X_PIECES; ++pc)
        tma_store_4d(&tm_xhat, ob + pc * (S::TR * S::X_SPAN), pc * 64, c.hb * hpt, c.rb * rpt,
                     c.s);
    }
    bulk_commit();
  };

  TileWalk ahead = cur;
  if (leader) {
    issue(ahead);
    ahead.advance(a.g);
  }

  // The next tile's scales of this role's groups (as words: local groups 2k
  // and 2k + 1) and of the group of pair d/8 (SRFT: the extra bin), loaded
  // one tile ahead. Groups wider than a role: word 0 holds the scales of the
  // role's LG local groups (see SplitGroups).
  using Grp = SplitGroups<D, G, ROT>;
  constexpr int NSW = Grp::kLocal ? S::NGR / 2 : 1;
  constexpr int LGS = Grp::kLocal ? S::GS : Grp::LGS;
  constexpr bool kWords = ROT == kSRHT || S::kScaleWords;
  auto load_scales = [&](const TileWalk& c, uint32_t (&rs)[NSW], uint32_t& ex) {
    const int row = c.rb * rpt + rl;
    const size_t svec = (static_cast<size_t>(c.s) * a.in_slice_stride_rows + row) * a.g.heads +
                        c.hb * hpt + hl;
    if (row < a.g.n_rows &&
        dbg_ok(int64_t(svec) < vec_limit(a.g.n_slices, a.in_slice_stride_rows, a.g.n_rows,
                                         a.g.heads),
               a.guard)) {
      const uint16_t* src = a.scales + svec * S::NG;
      if constexpr (Grp::kLocal) {
        static_for<0, NSW>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          const int g0 = split_group<ROT, S::NGR>(2 * k, role);
          if constexpr (kWords) {
            rs[k] = *reinterpret_cast<const uint32_t*>(src + g0);
          } else {
            rs[k] = uint32_t(src[g0]) |
                    (uint32_t(src[split_group<ROT, S::NGR>(2 * k + 1, role)]) << 16);
          }
        });
      } else if constexpr (S::NG == 2) {
        // SRFT: local halves 0 / 1 are global groups 0 / 1; SRHT: group R
        const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
        rs[0] = ROT == kSRFT ? w : (role ? (w >> 16) : (w & 0xFFFFu));
      } else {
        rs[0] = src[0];
      }
      if constexpr (ROT == kSRFT) ex = src[(D / 4) / G];
    } else {
      static_for<0, NSW>([&](auto k_) { rs[decltype(k_)::value] = 0u; });
      ex = 0u;
    }
  };
  uint32_t rs_next[NSW], ex_next = 0u;
  load_scales(cur, rs_next, ex_next);

  int it = 0;
  int table_key = -1;
  bool pending = false;
  TileWalk prev = cur;
  for (; cur.valid(); ++it) {
    uint32_t rs[NSW];
    static_for<0, NSW>([&](auto k_) { rs[decltype(k_)::value] = rs_next[decltype(k_)::value]; });
    const uint32_t ex = ex_next;
    TileWalk nxt = cur;
    nxt.advance(a.g);
    if (nxt.valid()) load_scales(nxt, rs_next, ex_next);

    const int key = cur.table_key(a.g);
    if (key != table_key) {
      build_split_tables<D, BITS, ROT, false, Lay::kMultStride, Lay::kSignStride>(
          mult, mtab, a.lambda, a.signs, cur.s, cur.hb, a.g.heads, hpt_log2, tid);
      table_key = key;
    }
    const bool ok = __syncthreads_and(mbar_wait_bounded(bar, it & 1)) != 0;
    if (!ok) {
      if (leader) {
        atomicOr(a.guard, kGuardWaitTimeout);
        bulk_wait<0>();
      }
      return;
    }

    // (a) this role's slots, times the multipliers
    float2 y[NP];
    static_for<0, S::KR>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      const int cg = split_code_chunk<ROT, S::KR>(k, role);
      const uint4 u = lds128(code_chunk_addr<S>(crow, cg));
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
      static_for<0, 4>([&](auto q_) {
        constexpr int q = decltype(q_)::value;
        constexpr int j0 = k * S::SPC + q * (S::SPC / 4);   // first slot of the word
        constexpr int lg = j0 / LGS;                        // local group
        decode_split_word<BITS, lg & 1>(wd[q], rs[lg / 2], &y[j0]);
      });
    });
    static_for<0, NP / 2>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = *reinterpret_cast<const float4*>(mrow + 4 * ci);
      y[2 * ci] = mul2(y[2 * ci], make_float2(m4.x, m4.y));
      y[2 * ci + 1] = mul2(y[2 * ci + 1], make_float2(m4.z, m4.w));
    });
    float2 extra = make_float2(0.0f, 0.0f);   // SRFT: X_{d/8} (role 1's slot 0), used by role 0
    if constexpr (ROT == kSRFT) {
      constexpr int cg = NQ / S::SPC;
      const uint32_t w = lds128(code_chunk_addr<S>(crow, cg)).x;
      float2 t[4];
      decode_split_word<BITS, 0>(w, ex, t);
      extra = mul2(t[0], *reinterpret_cast<const float2*>(mbase + S::DH));
    }
    // Both warps have read the stage and staged + fenced the previous
    // tile's output: store it and refill the stage with the next tile.
    bar_pair();
    if (leader) {
      if (pending) store_xhat(prev);
      if (ahead.valid()) {
        issue(ahead);
        ahead.advance(a.g);
      }
    }
    pending = false;

    if constexpr (ROT == kSRFT) {
      // (b) inverse butterflies: role 0 k = 0..d/8 (keeps E, sends O), role 1
      // k = d/8+1..d/4 (keeps O, sends E); the slot values carry X_k / d, so
      // the sums and differences are E_k / (d/2) and O_k / (d/2). Role 1
      // inverts R_k = conj(O_{d/4-k}) = O_{k+d/4} instead of O: its samples
      // are then (-1)^n u_{2n+1} (the sign lives in its mask table), and
      // both roles fill their d/2 spectrum the same way: entries 0..d/8-1
      // (and d/8 for role 0) from their own butterflies, the rest from the
      // partner, whose exchange row holds the values in the receiver's order.
      float2 mine[NQ + 1];
      if (role == 0) {
        {   // k = 0: X_0 and X_{d/2} real
          const float s0 = y[0].x + y[0].y, d0 = y[0].x - y[0].y;
          mine[0] = make_float2(s0, 0.0f);
          sts64(my_row + 8 * NQ, f22u(make_float2(d0, 0.0f)));   // R_{d/4} = O_0
        }
        static_for<1, NQ>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          float2 p = y[k], q = y[NP - k];
          split_dif<D, k>(p, q);
          mine[k] = p;
          sts64(my_row + 8 * (NQ - k), f22u(make_float2(q.x, -q.y)));   // R_{d/4-k}
        });
        {
          float2 p = extra, q = y[NQ];
          split_dif<D, NQ>(p, q);
          mine[NQ] = p;
          sts64(my_row, f22u(make_float2(q.x, -q.y)));   // R_{d/8} = conj O_{d/8}
        }
      } else {
        static_for<NQ + 1, NP>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          float2 p = y[k - NQ], q = y[3 * NQ - k];
          split_dif<D, k>(p, q);
          sts64(my_row + 8 * (k - NQ), f22u(p));      // E_k at entry k - d/8
          mine[NP - k] = make_float2(q.x, -q.y);      // R_{d/4-k}
        });
        // k = d/4: y[d/8] = 2 X_{d/4} / d, X_{d/4} = E_{d/4} - i O_{d/4}
        sts64(my_row + 8 * NQ, f22u(make_float2(2.0f * y[NQ].x, 0.0f)));
        mine[0] = make_float2(-2.0f * y[NQ].y, 0.0f);   // R_0 = O_{d/4}
        mine[NQ] = make_float2(0.0f, 0.0f);
      }
      bar_pair();
      // (c) this role's d/2 spectrum (F = E for role 0, R for role 1):
      // v[0] = (F_0, F_{d/4}), v[d/8] = 2 conj F_{d/8} / (d/2), v[k] = F_k / (d/2)
      float2 v[NP];
      v[0] = make_float2(mine[0].x, u2f2(lds64(partner_row + 8 * NQ)).x);
      static_for<1, NQ>([&](auto k_) { v[decltype(k_)::value] = mine[decltype(k_)::value]; });
      {
        const float2 fq = role ? u2f2(lds64(partner_row)) : mine[NQ];
        v[NQ] = make_float2(2.0f * fq.x, -2.0f * fq.y);
      }
      static_for<NQ + 1, NP>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        v[k] = u2f2(lds64(partner_row + 8 * (k - NQ)));
      });
      srft_inverse<D / 2>(v);
      // (d) signs, fp16 pairs P_m = (x_{4m+R}, x_{4m+2+R}). Role 0 writes the
      // first half of the row's words (m < d/8), role 1 the second half: each
      // keeps its d/8 pairs K and sends the other d/8 through the partner's
      // exchange row (which this warp has finished reading).
      uint32_t K[NQ];
      auto pairs = [&](auto base_, auto keep_) {
        constexpr int B = decltype(base_)::value;
        static_for<0, NQ / 4>([&](auto c_) {
          constexpr int c = decltype(c_)::value;
          const uint4 m4 = *reinterpret_cast<const uint4*>(mk + B + 4 * c);
          const uint32_t w4[4] = {pack_f16x2(v[B + 4 * c].x, v[B + 4 * c].y) ^ m4.x,
                                  pack_f16x2(v[B + 4 * c + 1].x, v[B + 4 * c + 1].y) ^ m4.y,
                                  pack_f16x2(v[B + 4 * c + 2].x, v[B + 4 * c + 2].y) ^ m4.z,
                                  pack_f16x2(v[B + 4 * c + 3].x, v[B + 4 * c + 3].y) ^ m4.w};
          if constexpr (decltype(keep_)::value) {
            static_for<0, 4>([&](auto t_) { K[4 * c + decltype(t_)::value] = w4[decltype(t_)::value]; });
          } else {
            sts128(partner_row + 16 * c, make_uint4(w4[0], w4[1], w4[2], w4[3]));
          }
        });
      };
      if (role == 0) {
        pairs(Int<NQ>{}, std::false_type{});
        pairs(Int<0>{}, std::true_type{});
      } else {
        pairs(Int<0>{}, std::false_type{});
        pairs(Int<NQ>{}, std::true_type{});
      }
      if (leader) bulk_wait_read<0>();
      bar_pair();
      // word 2m = (x_{4m}, x_{4m+1}), 2m + 1 = (x_{4m+2}, x_{4m+3}): role 0's
      // own pair holds the even samples, role 1's the odd ones
      const uint32_t sel_lo = role ? 0x1054u : 0x5410u, sel_hi = role ? 0x3276u : 0x7632u;
      static_for<0, NQ / 4>([&](auto j_) {
        constexpr int j = decltype(j_)::value;
        const uint4 q4 = lds128(my_row + 16 * j);
        const uint32_t qq[4] = {q4.x, q4.y, q4.z, q4.w};
        uint32_t o[8];
        static_for<0, 4>([&](auto t_) {
          constexpr int t = decltype(t_)::value;
          o[2 * t] = __byte_perm(K[4 * j + t], qq[t], sel_lo);
          o[2 * t + 1] = __byte_perm(K[4 * j + t], qq[t], sel_hi);
        });
        const int ci = (S::XC / 2) * role + 2 * j;   // words 2m: chunks ci, ci + 1
        sts128(row_chunk(xrow, ci), make_uint4(o[0], o[1], o[2], o[3]));
        sts128(row_chunk(xrow, ci + 1), make_uint4(o[4], o[5], o[6], o[7]));
      });
    } else {
      // SRHT: A_R = H_{d/2} (this role's half), u_n = A_0 + A_1, u_{n+d/2} =
      // A_0 - A_1 (1/sqrt(d) in the multipliers). Role 0 writes n < d/4,
      // role 1 n >= d/4: each sends the partner the half it needs.
      srht_inverse<D / 2>(y);
      if (role == 0) {
        static_for<0, NQ / 2>([&](auto j_) {
          constexpr int j = decltype(j_)::value;
          sts128(my_row + 16 * j,
                 make_uint4(__float_as_uint(y[NQ + 2 * j].x), __float_as_uint(y[NQ + 2 * j].y),
                            __float_as_uint(y[NQ + 2 * j + 1].x),
                            __float_as_uint(y[NQ + 2 * j + 1].y)));
        });
      } else {
        static_for<0, NQ / 2>([&](auto j_) {
          constexpr int j = decltype(j_)::value;
          sts128(my_row + 16 * j,
                 make_uint4(__float_as_uint(y[2 * j].x), __float_as_uint(y[2 * j].y),
                            __float_as_uint(y[2 * j + 1].x), __float_as_uint(y[2 * j + 1].y)));
        });
      }
      if (leader) bulk_wait_read<0>();
      bar_pair();
      auto out_words = [&](auto r_) {
        constexpr int R = decltype(r_)::value;
        static_for<0, NQ / 4>([&](auto c_) {
          constexpr int c = decltype(c_)::value;   // 4 words = 8 samples per chunk
          uint32_t lo[4], hi[4];
          static_for<0, 2>([&](auto h_) {
            constexpr int hh = decltype(h_)::value;
            const uint4 q4 = lds128(partner_row + 32 * c + 16 * hh);
            const float2 r2[2] = {make_float2(__uint_as_float(q4.x), __uint_as_float(q4.y)),
                                  make_float2(__uint_as_float(q4.z), __uint_as_float(q4.w))};
            static_for<0, 2>([&](auto t_) {
              constexpr int t = decltype(t_)::value;
              constexpr int w = NQ * R + 4 * c + 2 * hh + t;   // word of x_lo: (u_{2w}, u_{2w+1})
              const float2 mine = y[w];
              const float2 a0 = R == 0 ? mine : r2[t];
              const float2 a1 = R == 0 ? r2[t] : mine;
              lo[2 * hh + t] = pack_f16x2(a0.x + a1.x, a0.y + a1.y) ^ mkrow[w];
              hi[2 * hh + t] = pack_f16x2(a0.x - a1.x, a0.y - a1.y) ^ mkrow[NP + w];
            });
          });
          constexpr int ci = (NQ / 4) * R + c;   // chunk of word NQ R + 4 c
          sts128(row_chunk(xrow, ci), make_uint4(lo[0], lo[1], lo[2], lo[3]));
          sts128(row_chunk(xrow, S::XC / 2 + ci), make_uint4(hi[0], hi[1], hi[2], hi[3]));
        });
      };
      if (role == 0)
        out_words(Int<0>{});
      else
        out_words(Int<1>{});
    }
    fence_proxy_async_smem();
    pending = true;
    prev = cur;
    cur = nxt;
  }
  __syncthreads();
  if (leader) {
    if (pending) store_xhat(prev);
    bulk_wait<0>();
  }
}

}  // namespace srftq
