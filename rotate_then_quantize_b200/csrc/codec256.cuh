// Fused quantise / dequantise kernels for d = 256.
//
// A block is two warps that share one tile of 32 vectors (the tile geometry,
// tile walk and early stage refill of codec.cuh); lane l of both warps holds
// vector l. The warps split every vector's transform by role R = warp index,
// so each role's code is compile-time (no per-lane selects or twiddle
// tables), and they meet at block barriers to swap half results through
// shared memory.
//
// SRFT ("When Quantization Is Free", Methodology 1). The 256-point real DFT
// of u = s x splits into the 128-point real DFTs E and O of the even and odd
// samples: X_k = E_k + W^k O_k and X_{128-k} = conj(E_k - W^k O_k), with
// W = exp(-2 pi i / 256). Warp R transforms the samples u_{2n+R} with the
// d = 128 transform of transform.cuh, its first pass reading half R of the
// fp16 words straight from the staged tile. The warps swap half spectra.
// Warp 0 then forms the butterflies k = 0..32 and warp 1 k = 32..64. Warp 0's
// 64 output slots are the coordinate pairs 0..31 and 96..127, slot 0
// holding X_0 and X_128; warp 1's are pairs 32..95.
//
// SRHT ("HyperQuant", Methodology 1). H_256 u = [H_128 (u_lo + u_hi);
// H_128 (u_lo - u_hi)] in Sylvester order: warp 0 transforms the sum into
// pairs 0..63, warp 1 the difference into pairs 64..127. There is no
// exchange.
//
// Every group of 8..64 coordinates lies inside one warp's slots, so each
// warp quantises its own groups. The dequantiser runs the steps backwards.
// For SRFT it decodes one extra bin (X_32) in warp 0, so that both of its
// inverse butterflies are local. Its even/odd outputs are swapped once more,
// so that each warp writes whole fp16 words of one half of the row.
#pragma once

#include "codec.cuh"

namespace srftq {

template <int BITS, int G>
struct Shape256 {
  static_assert(G >= 8 && G <= 64 && (G & (G - 1)) == 0, "group (d = 256)");
  static_assert(BITS == 4 || BITS == 8, "bits");
  static constexpr int TR = kTileRows;                   // vectors per tile
  static constexpr int XB = 512, X_SPAN = 128, X_PIECES = 4, X_TILE = TR * XB;
  static constexpr int CB = 256 * BITS / 8;              // 128 or 256 bytes / vector
  static constexpr int C_SPAN = 128, C_PIECES = CB / 128, C_TILE = TR * CB;
  static constexpr int SPC = 64 / BITS;                  // slots (pairs) per 16-byte chunk
  static constexpr int KR = 64 / SPC;                    // code chunks per role
  static constexpr int CWR = 4 * KR;                     // code words per role
  static constexpr int NG = 256 / G, NGR = 128 / G;      // groups per vector / per role
  static constexpr int GS = G / 2;                       // slots per group
  static constexpr int SW = NG / 2;                      // scale words per vector
  static constexpr int QMAX = (1 << (BITS - 1)) - 1;
};

// Per-block shared-memory layout: the input stage (x tile for the quantiser,
// codes for the dequantiser), the output staging tile, one exchange row per
// lane and warp (34 float2; the stride keeps lanes on distinct banks), the per-head tables of up to kMaxHPT heads (multipliers
// of both roles' slots, 2 x 128 floats; sign words, up to 192) and the
// barrier.
template <int BITS, int G, bool QUANT>
struct BlockLayout256 {
  using S = Shape256<BITS, G>;
  static constexpr int kInTile = QUANT ? S::X_TILE : S::C_TILE;
  static constexpr int kInBytes = align_up(kInTile, 1024);
  static constexpr int kOutTile = QUANT ? S::C_TILE : S::X_TILE;
  static constexpr int kOutOff = kInBytes;
  static constexpr int kXchLane = 34 * 8, kXchWarp = 32 * kXchLane;
  static constexpr int kXchOff = kOutOff + align_up(kOutTile, 1024);
  static constexpr int kXch2Off = kXchOff + 2 * kXchWarp;   // end of the exchange rows
  static constexpr int kMultStride = 2 * 128 + 4;     // floats per head
  static constexpr int kSignStride = 192 + 4;         // words per head
  static constexpr int kTableOff = kXch2Off;
  static constexpr int kSignTabOff = kTableOff + 4 * kMaxHPT * kMultStride;
  static constexpr int kBarOff = align_up(kSignTabOff + 4 * kMaxHPT * kSignStride, 16);
  static constexpr int kBytes = align_up(kBarOff + 8, 1024);
};

// Coordinate pair held in slot j of role R.
template <int ROT, int R>
__host__ __device__ constexpr int slot_pair256(int j) {
  if (ROT == kSRHT) return R ? 64 + j : j;
  return R ? 32 + j : (j < 32 ? j : 64 + j);
}

// (role, slot) holding coordinate pair p, and whether the slot stores the
// conjugate of the bin (SRFT: warp 0's slots 32..63, warp 1's 33..63).
template <int ROT>
__device__ __forceinline__ void pair_slot256(int p, int& r, int& j, bool& conj) {
  if (ROT == kSRHT) {
    r = p >> 6;
    j = p & 63;
    conj = false;
  } else {
    r = (p >= 32 && p < 96) ? 1 : 0;
    j = r ? p - 32 : (p < 32 ? p : p - 64);
    conj = r ? j >= 33 : j >= 32;
  }
}

// Block barrier of the two warps (named barrier 1).
__device__ __forceinline__ void bar_pair() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts64(uint32_t addr, uint2 v) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ float2 u2f2(uint2 u) {
  return make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
}
__device__ __forceinline__ uint2 f22u(float2 f) {
  return make_uint2(__float_as_uint(f.x), __float_as_uint(f.y));
}

// Builds the tables of the HPT heads of (slice s, head block hb) with all 64
// threads. Multipliers, per slot of each role (lane x / lane y = the pair's
// even / odd coordinate):
//   quantiser: gain / lambda, gain = sqrt(2)/32 (SRFT; slot 0 of role 0:
//   1/32; the imaginary gain negated in conjugate slots) or 1/16 (SRHT);
//   dequantiser: gain' * lambda (int4: / 16 at odd coordinates), gain' =
//   1/(16 sqrt(2)) (SRFT, slot values scaled by 1/512 for the inverse;
//   slot 0 of role 0: 1/16; negated imaginary in conjugate slots) or 1/16
//   (SRHT).
// Sign words: SRFT, per role R word m = (s_{4m+R}, s_{4m+2+R}) at R * 64 + m;
// the dequantiser's role 1 words also flip the sign of their second sample
// (see dequantize256_kernel); SRHT quantiser: (s_{2w}, s_{2w+1}) for the low
// half (w < 64) at w, the high
// half at 64 + w for role 0 and negated at 128 + w for role 1 (which
// transforms u_lo - u_hi); SRHT dequantiser: word w = (s_{2w}, s_{2w+1}),
// w < 128. Quantiser words are fp16 +-1 pairs, dequantiser words sign-bit
// masks.
template <int BITS, int ROT, bool QUANT, int MS, int SS>
__device__ __forceinline__ void build_tables256(float* mult, uint32_t* stab, const float* lambda,
                                                const int8_t* signs, int s, int hb, int H,
                                                int hpt_log2, int tid) {
  constexpr int kL4 = kMaxHPT * 256 / 4 / 64;    // float4 loads per thread, at most
  constexpr int kS16 = kMaxHPT * 256 / 16 / 64;  // 16-sign loads per thread, at most
  const int hpt = 1 << hpt_log2;
  const size_t h0 = static_cast<size_t>(s) * H + static_cast<size_t>(hb) * hpt;
  const float4* lam4 = reinterpret_cast<const float4*>(lambda + h0 * 256);
  const uint4* sg16 = reinterpret_cast<const uint4*>(signs + h0 * 256);
  const int n4 = hpt * 64, n16 = hpt * 16;
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
      const int h = i >> 6, c0 = 4 * (i & 63);   // head, first coordinate
      const float lv[4] = {l[k].x, l[k].y, l[k].z, l[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = c0 + e, p = c >> 1, odd = c & 1;
        int r, j;
        bool conj;
        pair_slot256<ROT>(p, r, j, conj);
        float gain;
        if constexpr (ROT == kSRHT) {
          gain = 0.0625f;
        } else if constexpr (QUANT) {
          gain = (r == 0 && j == 0) ? 0.03125f : 0.04419417382415922f;
        } else {
          gain = (r == 0 && j == 0) ? 0.0625f : 0.04419417382415922f;
        }
        if (odd && conj) gain = -gain;
        float m;
        if constexpr (QUANT)
          m = gain * rcp_approx(lv[e]);
        else
          m = gain * lv[e] * ((BITS == 4 && odd) ? 0.0625f : 1.0f);
        mult[h * MS + r * 128 + 2 * j + odd] = m;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kS16; ++k) {
    const int i = tid + 64 * k;
    if (i < n16) {
      const int h = i >> 4, c0 = 16 * (i & 15);   // head, first sign of the chunk
      const uint32_t wd[4] = {g[k].x, g[k].y, g[k].z, g[k].w};
      auto sb = [&](int t) -> int8_t { return static_cast<int8_t>(wd[t >> 2] >> (8 * (t & 3))); };
      if constexpr (ROT == kSRHT) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int8_t s0 = sb(2 * e), s1 = sb(2 * e + 1);
          const int w = c0 / 2 + e;
          if constexpr (QUANT) {
            const uint32_t sw = sign_halves(s0, s1);
            if (w < 64) {
              stab[h * SS + w] = sw;
            } else {
              stab[h * SS + w] = sw;                       // role 0: + u_hi
              stab[h * SS + 64 + w] = sw ^ 0x80008000u;    // role 1: - u_hi
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
            // the dequantiser's role 1 inverts the spectrum shifted by 64 bins,
            // whose samples carry (-1)^n: the odd one of each pair is negated
            stab[h * SS + r * 64 + m] =
                QUANT ? sign_halves(s0, s1) : (sign_mask(s0, s1) ^ (r ? 0x80000000u : 0u));
          }
        }
      }
    }
  }
  __syncthreads();
}

// Address of 16-byte chunk ci (0..31) of a 512-byte row in a tile of four
// 128-byte-swizzled pieces of 32 rows (xrow = swz_row<128>(tile, lane)).
__device__ __forceinline__ uint32_t row_chunk256(uint32_t xrow, int ci) {
  return swz_chunk<128>(xrow, ci & 7) + (ci >> 3) * (kTileRows * 128);
}

// ---------------------------------------------------------------------------
// Transforms (one code path for both roles)
// ---------------------------------------------------------------------------

// SRFT: the 128-point real DFT of u_{2n+R}, from the staged fp16 row. Its
// complex sample m is (u_{4m+R}, u_{4m+2+R}): half R of x words 2m and
// 2m + 1, gathered with one PRMT (sel = 0x5410 for R = 0, 0x7632 for R = 1);
// sgn = this role's sign words (lo half = real part's sign).
__device__ __forceinline__ void srft256_forward(uint32_t xrow, uint32_t sel, const uint32_t* sgn,
                                                float2 (&v)[64]) {
  constexpr int Q = 32, LOG = 6;
  float2 PR[Q], PI[Q];
  // pass 1: butterflies (z_m, z_{m+32}) into the bit-reversed slots
  // i = bitrev(m), i + 1; two at a time from two 16-byte chunks each.
  static_for<0, 16>([&](auto c_) {
    constexpr int c = decltype(c_)::value;
    const uint4 A = lds128(row_chunk256(xrow, c));        // words 4c .. 4c+3: m = 2c, 2c+1
    const uint4 B = lds128(row_chunk256(xrow, 16 + c));   // m = 2c+32, 2c+33
    const uint2 sa = *reinterpret_cast<const uint2*>(sgn + 2 * c);
    const uint2 sbb = *reinterpret_cast<const uint2*>(sgn + 32 + 2 * c);
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
  srft_forward_rest<128>(PR, PI, v);
}

// SRHT: H_128 of u_lo + u_hi (role 0) or u_lo - u_hi (role 1; the minus sign
// lives in that role's high-half sign words), unnormalised, natural pairs.
__device__ __forceinline__ void srht256_forward(uint32_t xrow, const uint32_t* slo,
                                                const uint32_t* shi, float2 (&v)[64]) {
  static_for<0, 16>([&](auto c_) {
    constexpr int c = decltype(c_)::value;
    const uint4 wl = lds128(row_chunk256(xrow, c)), wh = lds128(row_chunk256(xrow, 16 + c));
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
  wht_packed_planes<128>(v);
}

// S(k) = 2 F_k of a d = 128 forward output v: v[0] = (F_0, F_64),
// v[32] = conj F_32, v[k] = 2 F_k otherwise.
template <int K>
__device__ __forceinline__ float2 spec2(const float2 (&v)[64]) {
  if constexpr (K == 0) {
    return make_float2(2.0f * v[0].x, 0.0f);
  } else if constexpr (K == 64) {
    return make_float2(2.0f * v[0].y, 0.0f);
  } else if constexpr (K == 32) {
    return make_float2(2.0f * v[32].x, -2.0f * v[32].y);
  } else {
    return v[K];
  }
}

// Writes S(k) for k = K0 .. K0 + 32 (33 values) to this lane's exchange row.
template <int K0>
__device__ __forceinline__ void put_half_spectrum(uint32_t row, const float2 (&v)[64]) {
  static_for<0, 16>([&](auto j_) {
    constexpr int j = decltype(j_)::value;
    const float2 a = spec2<K0 + 2 * j>(v), b = spec2<K0 + 2 * j + 1>(v);
    sts128(row + 16 * j, make_uint4(__float_as_uint(a.x), __float_as_uint(a.y),
                                    __float_as_uint(b.x), __float_as_uint(b.y)));
  });
  sts64(row + 256, f22u(spec2<K0 + 32>(v)));
}

// Forward combine of role R after the exchange: own = this role's d = 128
// spectrum, rr = the partner's exchange row (S of the other sub-sequence,
// k = 0..32 for role 0, k = 32..64 for role 1). out[j] = slot j.
template <int R>
__device__ __forceinline__ void srft256_combine(const float2 (&own)[64], uint32_t rr,
                                                float2 (&out)[64]) {
  auto recv = [&](int j) -> float2 { return u2f2(lds64(rr + 8 * j)); };
  if constexpr (R == 0) {
    {   // k = 0: X_0 and X_128 are real
      const float2 o = recv(0);
      const float e = spec2<0>(own).x;
      out[0] = make_float2(e + o.x, e - o.x);
    }
    static_for<1, 33>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      float2 a = spec2<k>(own), b = recv(k);
      butterfly<-1, k, 128>(a.x, a.y, b.x, b.y);
      if constexpr (k < 32) out[k] = a;
      out[64 - k] = b;
    });
  } else {
    static_for<32, 64>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      float2 a = recv(k - 32), b = spec2<k>(own);
      butterfly<-1, k, 128>(a.x, a.y, b.x, b.y);
      out[k - 32] = a;
      if constexpr (k > 32) out[96 - k] = b;
    });
    {   // k = 64: X_64 = E_64 - i O_64 (E_64, O_64 real)
      const float2 e = recv(32);
      out[32] = make_float2(e.x, -spec2<64>(own).x);
    }
  }
}

// Global code chunk of a role's local chunk k (KR chunks of SPC slots).
template <int ROT, int KR>
__device__ __forceinline__ int code_chunk256(int k, int role) {
  if constexpr (ROT == kSRHT) return k + role * KR;
  return k + (role ? KR / 2 : (k < KR / 2 ? 0 : KR));
}

// Global group of a role's local group g (NGR groups of G / 2 slots).
template <int ROT, int NGR>
__device__ __forceinline__ int group256(int g, int role) {
  if constexpr (ROT == kSRHT) return g + role * NGR;
  return g + (role ? NGR / 2 : (g < NGR / 2 ? 0 : NGR));
}

// ---------------------------------------------------------------------------
// Quantiser, d = 256
// ---------------------------------------------------------------------------

template <int BITS, int G, int ROT, int MINB>
__global__ void __launch_bounds__(64, MINB)
    quantize256_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_codes, const QuantArgs a) {
  using S = Shape256<BITS, G>;
  using Lay = BlockLayout256<BITS, G, true>;
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
  const float* mrow = mult + hl * Lay::kMultStride + role * 128;
  const uint32_t* srow = stab + hl * Lay::kSignStride;
  const uint32_t* s1 = srow + (ROT == kSRFT ? role * 64 : 0);          // SRFT: role words
  const uint32_t* s2 = srow + 64 + role * 64;                           // SRHT: high half
  const uint32_t psel = role ? 0x7632u : 0x5410u;
  const uint32_t xrow = swz_row<128>(smem_addr(sb), lane);
  const uint32_t crow = swz_row<128>(smem_addr(ob), lane);
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
    mbar_arrive_expect_tx(bar, S::X_TILE);
#pragma unroll
    for (int pc = 0; pc < S::X_PIECES; ++pc)
      tma_load_4d(sb + pc * (S::TR * S::X_SPAN), &tm_x, bar, pc * 64, c.hb * hpt, c.rb * rpt,
                  c.s);
  };
  auto store_codes = [&](const TileWalk& c) {
#pragma unroll
    for (int pc = 0; pc < S::C_PIECES; ++pc)
      tma_store_4d(&tm_codes, ob + pc * (S::TR * S::C_SPAN), pc * S::C_SPAN, c.hb * hpt,
                   c.rb * rpt, c.s);
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
      build_tables256<BITS, ROT, true, Lay::kMultStride, Lay::kSignStride>(
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
    float2 v[64];
    if constexpr (ROT == kSRFT)
      srft256_forward(xrow, psel, s1, v);
    else
      srht256_forward(xrow, srow, s2, v);
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
    float2 y[64];
    if constexpr (ROT == kSRFT) {
      if (role == 0)
        put_half_spectrum<32>(my_row, v);
      else
        put_half_spectrum<0>(my_row, v);
      if (leader) bulk_wait_read<0>();
      bar_pair();
      if (role == 0)
        srft256_combine<0>(v, partner_row, y);
      else
        srft256_combine<1>(v, partner_row, y);
    } else {
      if (leader) bulk_wait_read<0>();
      bar_pair();
      static_for<0, 64>([&](auto j_) { y[decltype(j_)::value] = v[decltype(j_)::value]; });
    }

    // (d) multipliers, group absmax, scales, codes (as in codec.cuh)
    static_for<0, 32>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = *reinterpret_cast<const float4*>(mrow + 4 * ci);
      y[2 * ci] = mul2(y[2 * ci], make_float2(m4.x, m4.y));
      y[2 * ci + 1] = mul2(y[2 * ci + 1], make_float2(m4.z, m4.w));
    });
    float am[S::NGR];
    static_for<0, S::NGR>([&](auto g_) {
      constexpr int g = decltype(g_)::value;
      constexpr int P0 = g * S::GS;
      float m = absmax3(0.0f, y[P0].x, y[P0].y);
      static_for<1, S::GS>([&](auto p_) {
        constexpr int p = P0 + decltype(p_)::value;
        m = absmax3(m, y[p].x, y[p].y);
      });
      am[g] = m;
    });
    float a_hi, a_lo;
    range_of(am, a_hi, a_lo);
    constexpr float kHi = 65504.0f * float(S::QMAX);
    constexpr float kLo = 6.103515625e-05f * float(S::QMAX);
    uint32_t sw[(S::NGR + 1) / 2];
    uint32_t qb[128];
    if (a_hi <= kHi && a_lo >= kLo) {
      float invs[S::NGR];
      group_scales<S::NGR, S::QMAX, true>(am, sw, invs);
      static_for<0, 64>([&](auto p_) {
        constexpr int p = decltype(p_)::value;
        const float2 r = fma2(y[p], splat(invs[p / S::GS]), splat(kMagic));
        qb[2 * p] = __float_as_uint(r.x);
        qb[2 * p + 1] = __float_as_uint(r.y);
      });
    } else {
      float invs[S::NGR];
      group_scales<S::NGR, S::QMAX, false>(am, sw, invs);
      static_for<0, 64>([&](auto p_) {
        constexpr int p = decltype(p_)::value;
        const float inv = invs[p / S::GS];
        const float q0 = fminf(fmaxf(y[p].x * inv, -float(S::QMAX)), float(S::QMAX));
        const float q1 = fminf(fmaxf(y[p].y * inv, -float(S::QMAX)), float(S::QMAX));
        qb[2 * p] = __float_as_uint(q0 + kMagic);
        qb[2 * p + 1] = __float_as_uint(q1 + kMagic);
      });
    }
    uint32_t words[S::CWR];
    if constexpr (BITS == 4) {
      static_for<0, 16>([&](auto m_) {
        constexpr int m = decltype(m_)::value;
        const uint32_t ev = __byte_perm(__byte_perm(qb[8 * m + 0], qb[8 * m + 2], 0x0040),
                                        __byte_perm(qb[8 * m + 4], qb[8 * m + 6], 0x0040), 0x5410);
        const uint32_t od = __byte_perm(__byte_perm(qb[8 * m + 1], qb[8 * m + 3], 0x0040),
                                        __byte_perm(qb[8 * m + 5], qb[8 * m + 7], 0x0040), 0x5410);
        words[m] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
      });
    } else {
      static_for<0, 32>([&](auto m_) {
        constexpr int m = decltype(m_)::value;
        words[m] = __byte_perm(__byte_perm(qb[4 * m], qb[4 * m + 1], 0x0040),
                               __byte_perm(qb[4 * m + 2], qb[4 * m + 3], 0x0040), 0x5410);
      });
    }

    // (e) this role's code chunks into the staging tile
    static_for<0, S::KR>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      const int cg = code_chunk256<ROT, S::KR>(k, role);   // chunk in the row
      sts128(swz_chunk<128>(crow, cg & 7) + (cg >> 3) * (S::TR * S::C_SPAN),
             make_uint4(words[4 * k], words[4 * k + 1], words[4 * k + 2], words[4 * k + 3]));
    });
    fence_proxy_async_smem();
    pending = true;
    prev = cur;

    // (f) this role's scales; consecutive global groups go out as words
    const int row = cur.rb * rpt + rl;
    if (row < a.g.n_rows) {
      uint16_t* dst = a.scales +
          ((static_cast<size_t>(cur.s) * a.out_slice_stride_rows + row) * a.g.heads +
           cur.hb * hpt + hl) * S::NG;
      constexpr bool kWords = ROT == kSRHT || G <= 32;   // runs of even length and start
      static_for<0, S::NGR / 2>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        const int g0 = group256<ROT, S::NGR>(2 * k, role);
        if constexpr (kWords) {
          *reinterpret_cast<uint32_t*>(dst + g0) = sw[k];
        } else {
          dst[g0] = static_cast<uint16_t>(sw[k] & 0xFFFFu);
          dst[group256<ROT, S::NGR>(2 * k + 1, role)] = static_cast<uint16_t>(sw[k] >> 16);
        }
      });
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
// Dequantiser, d = 256
// ---------------------------------------------------------------------------

// Decodes the 4 (int4: one word = 4 slots) or 2 (int8) slots of code word w
// of group scale half HS of word sgw into out.
template <int BITS, int HS>
__device__ __forceinline__ void decode_word256(uint32_t w, uint32_t sgw, float2* out) {
  const float sgf = __half2float(__ushort_as_half(
      static_cast<unsigned short>((sgw >> (16 * HS)) & 0xFFFFu)));
  const float c_even = BITS == 4 ? -1032.0f * sgf : -1152.0f * sgf;
  const float c_odd = -1152.0f * sgf;
  unpack_word<BITS, HS>(w, sgw, c_even, c_odd, out);
}

// DIF butterfly for bin K: (a, b) <- (a + b, conj(W^K) (a - b)).
template <int K>
__device__ __forceinline__ void dif256(float2& a, float2& b) {
  const float2 s = add2(a, b), d = sub2(a, b);
  a = s;
  if constexpr (K == 0) {
    b = d;
  } else if constexpr (K == 64) {
    b = make_float2(-d.y, d.x);   // times i
  } else {
    constexpr double cw = ct::cos2pi(K, 256), sn = ct::sin2pi(K, 256);
    constexpr float c = float(cw), t = float(sn / cw);   // conj(W^K) = cw + i sn
    b = make_float2(c * fmaf(-t, d.y, d.x), c * fmaf(t, d.x, d.y));
  }
}

template <int BITS, int G, int ROT, int MINB>
__global__ void __launch_bounds__(64, MINB)
    dequantize256_kernel(const __grid_constant__ CUtensorMap tm_codes,
                         const __grid_constant__ CUtensorMap tm_xhat, const DequantArgs a) {
  using S = Shape256<BITS, G>;
  using Lay = BlockLayout256<BITS, G, false>;
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
  const float* mrow = mbase + role * 128;
  const uint32_t* mkrow = mtab + hl * Lay::kSignStride;
  const uint32_t* mk = mkrow + (ROT == kSRFT ? role * 64 : 0);
  const uint32_t crow = swz_row<128>(smem_addr(sb), lane);
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
    mbar_arrive_expect_tx(bar, S::C_TILE);
#pragma unroll
    for (int pc = 0; pc < S::C_PIECES; ++pc)
      tma_load_4d(sb + pc * (S::TR * S::C_SPAN), &tm_codes, bar, pc * S::C_SPAN, c.hb * hpt,
                  c.rb * rpt, c.s);
  };
  auto store_xhat = [&](const TileWalk& c) {
#pragma unroll
    for (int pc = 0; pc < S::X_PIECES; ++pc)
      tma_store_4d(&tm_xhat, ob + pc * (S::TR * S::X_SPAN), pc * 64, c.hb * hpt, c.rb * rpt,
                   c.s);
    bulk_commit();
  };

  TileWalk ahead = cur;
  if (leader) {
    issue(ahead);
    ahead.advance(a.g);
  }

  // The next tile's scales of this role's groups (as words: local groups 2k
  // and 2k + 1) and of the group of pair 32 (SRFT: the extra bin), loaded one
  // tile ahead.
  constexpr int NSW = S::NGR / 2;
  constexpr bool kWords = ROT == kSRHT || G <= 32;
  auto load_scales = [&](const TileWalk& c, uint32_t (&rs)[NSW], uint32_t& ex) {
    const int row = c.rb * rpt + rl;
    if (row < a.g.n_rows) {
      const uint16_t* src = a.scales +
          ((static_cast<size_t>(c.s) * a.in_slice_stride_rows + row) * a.g.heads + c.hb * hpt +
           hl) * S::NG;
      static_for<0, NSW>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        const int g0 = group256<ROT, S::NGR>(2 * k, role);
        if constexpr (kWords) {
          rs[k] = *reinterpret_cast<const uint32_t*>(src + g0);
        } else {
          rs[k] = uint32_t(src[g0]) | (uint32_t(src[group256<ROT, S::NGR>(2 * k + 1, role)]) << 16);
        }
      });
      if constexpr (ROT == kSRFT) ex = src[64 / G];
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
      build_tables256<BITS, ROT, false, Lay::kMultStride, Lay::kSignStride>(
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
    float2 y[64];
    static_for<0, S::KR>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      const int cg = code_chunk256<ROT, S::KR>(k, role);
      const uint4 u = lds128(swz_chunk<128>(crow, cg & 7) + (cg >> 3) * (S::TR * S::C_SPAN));
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
      static_for<0, 4>([&](auto q_) {
        constexpr int q = decltype(q_)::value;
        constexpr int j0 = k * S::SPC + q * (S::SPC / 4);   // first slot of the word
        constexpr int lg = j0 / S::GS;                      // local group
        decode_word256<BITS, lg & 1>(wd[q], rs[lg / 2], &y[j0]);
      });
    });
    static_for<0, 32>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = *reinterpret_cast<const float4*>(mrow + 4 * ci);
      y[2 * ci] = mul2(y[2 * ci], make_float2(m4.x, m4.y));
      y[2 * ci + 1] = mul2(y[2 * ci + 1], make_float2(m4.z, m4.w));
    });
    float2 extra = make_float2(0.0f, 0.0f);   // SRFT: X_32 (role 1's slot 0), used by role 0
    if constexpr (ROT == kSRFT) {
      constexpr int cg = 32 / S::SPC;
      const uint32_t w = lds128(swz_chunk<128>(crow, cg & 7) + (cg >> 3) * (S::TR * S::C_SPAN)).x;
      float2 t[4];
      decode_word256<BITS, 0>(w, ex, t);
      extra = mul2(t[0], *reinterpret_cast<const float2*>(mbase + 128));
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
      // (b) inverse butterflies: role 0 k = 0..32 (keeps E, sends O), role 1
      // k = 33..64 (keeps O, sends E); the slot values carry 1/512, so the
      // sums and differences are E_k / 128 and O_k / 128. Role 1 inverts
      // R_k = conj(O_{64-k}) = O_{k+64} instead of O: its samples are then
      // (-1)^n u_{2n+1} (the sign lives in its mask table), and both roles
      // fill their d = 128 spectrum the same way: entries 0..31 (and 32 for
      // role 0) from their own butterflies, the rest from the partner, whose
      // exchange row holds the values in the receiver's order.
      float2 mine[33];
      if (role == 0) {
        {   // k = 0: X_0 and X_128 real
          const float s0 = y[0].x + y[0].y, d0 = y[0].x - y[0].y;
          mine[0] = make_float2(s0, 0.0f);
          sts64(my_row + 8 * 32, f22u(make_float2(d0, 0.0f)));   // R_64 = O_0
        }
        static_for<1, 32>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          float2 p = y[k], q = y[64 - k];
          dif256<k>(p, q);
          mine[k] = p;
          sts64(my_row + 8 * (32 - k), f22u(make_float2(q.x, -q.y)));   // R_{64-k}
        });
        {
          float2 p = extra, q = y[32];
          dif256<32>(p, q);
          mine[32] = p;
          sts64(my_row, f22u(make_float2(q.x, -q.y)));   // R_32 = conj O_32
        }
      } else {
        static_for<33, 64>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          float2 p = y[k - 32], q = y[96 - k];
          dif256<k>(p, q);
          sts64(my_row + 8 * (k - 32), f22u(p));      // E_k at entry k - 32
          mine[64 - k] = make_float2(q.x, -q.y);      // R_{64-k}
        });
        // k = 64: y[32] = 2 X_64 / 512, X_64 = E_64 - i O_64
        sts64(my_row + 8 * 32, f22u(make_float2(2.0f * y[32].x, 0.0f)));
        mine[0] = make_float2(-2.0f * y[32].y, 0.0f);   // R_0 = O_64
        mine[32] = make_float2(0.0f, 0.0f);
      }
      bar_pair();
      // (c) this role's d = 128 spectrum (F = E for role 0, R for role 1):
      // v[0] = (F_0, F_64), v[32] = conj F_32 / 64 * 128, v[k] = F_k / 128
      float2 v[64];
      v[0] = make_float2(mine[0].x, u2f2(lds64(partner_row + 8 * 32)).x);
      static_for<1, 32>([&](auto k_) { v[decltype(k_)::value] = mine[decltype(k_)::value]; });
      {
        const float2 f32 = role ? u2f2(lds64(partner_row)) : mine[32];
        v[32] = make_float2(2.0f * f32.x, -2.0f * f32.y);
      }
      static_for<33, 64>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        v[k] = u2f2(lds64(partner_row + 8 * (k - 32)));
      });
      srft_inverse<128>(v);
      // (d) signs, fp16 pairs P_m = (x_{4m+R}, x_{4m+2+R}). Role 0 writes the
      // words 0..63 of the row (m < 32), role 1 the words 64..127 (m >= 32):
      // each keeps its 32 pairs K and sends the other 32 through the
      // partner's exchange row (which this warp has finished reading).
      uint32_t K[32];
      auto pairs = [&](auto base_, auto keep_) {
        constexpr int B = decltype(base_)::value;
        static_for<0, 8>([&](auto c_) {
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
        pairs(Int<32>{}, std::false_type{});
        pairs(Int<0>{}, std::true_type{});
      } else {
        pairs(Int<0>{}, std::false_type{});
        pairs(Int<32>{}, std::true_type{});
      }
      if (leader) bulk_wait_read<0>();
      bar_pair();
      // word 2m = (x_{4m}, x_{4m+1}), 2m + 1 = (x_{4m+2}, x_{4m+3}): role 0's
      // own pair holds the even samples, role 1's the odd ones
      const uint32_t sel_lo = role ? 0x1054u : 0x5410u, sel_hi = role ? 0x3276u : 0x7632u;
      static_for<0, 8>([&](auto j_) {
        constexpr int j = decltype(j_)::value;
        const uint4 q4 = lds128(my_row + 16 * j);
        const uint32_t qq[4] = {q4.x, q4.y, q4.z, q4.w};
        uint32_t o[8];
        static_for<0, 4>([&](auto t_) {
          constexpr int t = decltype(t_)::value;
          o[2 * t] = __byte_perm(K[4 * j + t], qq[t], sel_lo);
          o[2 * t + 1] = __byte_perm(K[4 * j + t], qq[t], sel_hi);
        });
        const int ci = 16 * role + 2 * j;   // words 2m: chunks 16 R + 2 j, + 1
        sts128(row_chunk256(xrow, ci), make_uint4(o[0], o[1], o[2], o[3]));
        sts128(row_chunk256(xrow, ci + 1), make_uint4(o[4], o[5], o[6], o[7]));
      });
    } else {
      // SRHT: A_R = H_128 (this role's half), u_n = A_0 + A_1, u_{n+128} =
      // A_0 - A_1 (1/16 in the multipliers). Role 0 writes n < 64, role 1
      // n >= 64: each sends the partner the half it needs.
      srht_inverse<128>(y);
      if (role == 0) {
        static_for<0, 16>([&](auto j_) {
          constexpr int j = decltype(j_)::value;
          sts128(my_row + 16 * j, make_uint4(__float_as_uint(y[32 + 2 * j].x), __float_as_uint(y[32 + 2 * j].y),
                                             __float_as_uint(y[33 + 2 * j].x), __float_as_uint(y[33 + 2 * j].y)));
        });
      } else {
        static_for<0, 16>([&](auto j_) {
          constexpr int j = decltype(j_)::value;
          sts128(my_row + 16 * j, make_uint4(__float_as_uint(y[2 * j].x), __float_as_uint(y[2 * j].y),
                                             __float_as_uint(y[2 * j + 1].x), __float_as_uint(y[2 * j + 1].y)));
        });
      }
      if (leader) bulk_wait_read<0>();
      bar_pair();
      auto out_words = [&](auto r_) {
        constexpr int R = decltype(r_)::value;
        static_for<0, 8>([&](auto c_) {
          constexpr int c = decltype(c_)::value;   // 4 words = 8 samples per chunk
          uint32_t lo[4], hi[4];
          static_for<0, 2>([&](auto h_) {
            constexpr int hh = decltype(h_)::value;
            const uint4 q4 = lds128(partner_row + 32 * c + 16 * hh);
            const float2 r2[2] = {make_float2(__uint_as_float(q4.x), __uint_as_float(q4.y)),
                                  make_float2(__uint_as_float(q4.z), __uint_as_float(q4.w))};
            static_for<0, 2>([&](auto t_) {
              constexpr int t = decltype(t_)::value;
              constexpr int w = 32 * R + 4 * c + 2 * hh + t;   // word of x_lo: (u_{2w}, u_{2w+1})
              const float2 mine = y[w];
              const float2 a0 = R == 0 ? mine : r2[t];
              const float2 a1 = R == 0 ? r2[t] : mine;
              lo[2 * hh + t] = pack_f16x2(a0.x + a1.x, a0.y + a1.y) ^ mkrow[w];
              hi[2 * hh + t] = pack_f16x2(a0.x - a1.x, a0.y - a1.y) ^ mkrow[64 + w];
            });
          });
          constexpr int ci = 8 * R + c;   // chunk of word 32 R + 4 c
          sts128(row_chunk256(xrow, ci), make_uint4(lo[0], lo[1], lo[2], lo[3]));
          sts128(row_chunk256(xrow, 16 + ci), make_uint4(hi[0], hi[1], hi[2], hi[3]));
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
