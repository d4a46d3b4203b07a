// Fused quantise / dequantise kernels (one thread per head-dim vector).
//
// Work decomposition. A *tile* is the 32 vectors of HPT consecutive heads
// (HPT = the largest power of two <= 8 dividing H) of 32 / HPT consecutive
// rows of one slice: a contiguous block of memory when HPT = H. Lane l holds
// head l % HPT of row l / HPT. Tiles are numbered (s, head block, row block)
// with the row block fastest, and warp w of the grid takes one contiguous
// range of tile numbers, so each warp streams consecutive memory and its
// (slice, head block) -- and with it the per-head multiplier and sign tables
// -- changes only at the ends of a range. A warp owns NST input stages in
// shared memory; lane 0 issues the TMA box loads of a tile (128-byte
// swizzled rows, so each lane reading its own row hits distinct banks), all
// completing on one mbarrier. The lanes pull their vector into registers and
// compute; the results (codes, or the dequantised fp16 vectors) are written
// to a swizzled staging tile and fenced for the async proxy. Nothing on this
// path waits for the TMA engine: as soon as the lanes have read a stage into
// registers (where the warp converges anyway), lane 0 issues the refill of
// that stage with the tile NST ahead and the TMA store of the previously
// staged tile, so every copy overlaps a whole tile of compute.
// The quantiser stores scales straight from registers; the dequantiser loads
// them one tile ahead into registers.
//
// Quantiser stages follow "When Quantization Is Free", Methodology 2:
// (1) load and sign multiply (fused into the first butterfly pass, see
// transform.cuh), (2) the radix-2 FFT passes, (3) the Hermitian pack,
// (4) per-channel lambda, group absmax and rounding to signed int4/int8,
// (5) nibble packing. The dequantiser runs the same stages backwards.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"
#include "transform.cuh"

namespace srftq {

constexpr int kTileRows = 32;

struct TileGeom {
  int32_t heads;       // H
  int32_t row_blocks;  // ceil(N / rows per tile)
  int32_t n_rows;      // N
  int32_t total_tiles; // S * head_blocks * row_blocks
  int32_t n_slices;    // S
  int32_t hpt_log2;    // log2(heads per tile); heads x rows per tile = 32
  int32_t head_blocks; // H / heads per tile
};

// Heads per tile for H heads: the largest power of two <= kMaxHPT dividing H.
constexpr int kMaxHPT = 8;
__host__ __device__ constexpr int heads_per_tile_log2(int H) {
  int l = 0;
  while ((2 << l) <= kMaxHPT && H % (2 << l) == 0) ++l;
  return l;
}

struct TileCoord {
  int s, r0, h;
};

__device__ __forceinline__ TileCoord decode_tile(int t, const TileGeom& g) {
  const int h = t % g.heads;
  const int q = t / g.heads;
  const int rb = q % g.row_blocks;
  return {q / g.row_blocks, rb * kTileRows, h};
}

// A warp's current tile as digits (s, hb, rb) of t = (s * head_blocks + hb)
// * row_blocks + rb, and the number of tiles left in its range. Stepping
// carries rb into hb into s: no division inside the loop.
struct TileWalk {
  int s, hb, rb, left;

  // First tile of warp w of nw (balanced contiguous ranges); false if the
  // warp has none.
  __device__ __forceinline__ bool start(int w, int nw, const TileGeom& g) {
    const int T = g.total_tiles;
    const int base = T / nw, rem = T % nw;
    const int t0 = w * base + (w < rem ? w : rem);
    left = base + (w < rem ? 1 : 0);
    rb = t0 % g.row_blocks;
    const int q = t0 / g.row_blocks;
    hb = q % g.head_blocks;
    s = q / g.head_blocks;
    return left > 0;
  }
  __device__ __forceinline__ void advance(const TileGeom& g) {
    const int r = rb + 1;
    int c = r >= g.row_blocks;
    rb = c ? 0 : r;
    const int h = hb + c;
    c = h >= g.head_blocks;
    hb = c ? 0 : h;
    s += c;
    --left;
  }
  __device__ __forceinline__ bool valid() const { return left > 0; }
  // identity of the (slice, head block) the tables belong to
  __device__ __forceinline__ int table_key(const TileGeom& g) const {
    return s * g.head_blocks + hb;
  }
};

// The 1024-byte aligned start of dynamic shared memory, kept as a pointer
// into the shared window so that every access derived from it compiles to
// 32-bit shared loads and stores.
__device__ __forceinline__ uint8_t* smem_base_1024(uint8_t* raw) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(raw));
  return raw + ((0u - a) & 1023u);
}

// Number of vector slots rows 0..N-1 of S slices with a stride of `stride`
// rows span: the bound of every vector index a call may touch (debug checks).
__device__ __forceinline__ int64_t vec_limit(int64_t S, int64_t stride, int64_t N, int64_t H) {
  return ((S - 1) * stride + N) * H;
}

// The tile a TMA copy addresses lies inside the call's extents (debug checks).
__device__ __forceinline__ bool tile_in_range(const TileWalk& c, const TileGeom& g) {
  return c.s >= 0 && c.s < g.n_slices && c.hb >= 0 && c.hb < g.head_blocks && c.rb >= 0 &&
         c.rb < g.row_blocks;
}

struct QuantArgs {
  TileGeom g;
  const int8_t* signs;    // [S][H][d]
  const float* lambda;    // [S][H][d]
  uint8_t* codes;         // direct path only (code bytes per vector < 16)
  uint16_t* scales;       // [S][T_out][H][d/G]
  int64_t out_slice_stride_rows;
  unsigned* guard;
};

struct DequantArgs {
  TileGeom g;
  const int8_t* signs;
  const float* lambda;
  const uint8_t* codes;   // direct path only (code bytes per vector < 16)
  const uint16_t* scales; // [S][T_in][H][d/G]
  int64_t in_slice_stride_rows;
  uint16_t* xhat;         // [S][T_out][H][d]
  int64_t out_slice_stride_rows;
  unsigned* guard;
};


// Static shape of one codec configuration.
template <int D, int BITS, int G>
struct Shape {
  static_assert(D >= 16 && D <= 128 && (D & (D - 1)) == 0, "d");
  static_assert(G >= 8 && G <= D && (G & (G - 1)) == 0, "group");
  static_assert(BITS == 4 || BITS == 8, "bits");
  static constexpr int TR = kTileRows;
  static constexpr int XB = 2 * D;                      // fp16 bytes / vector
  static constexpr int X_SPAN = XB < 128 ? XB : 128;    // bytes per box row
  static constexpr int X_PIECES = XB / X_SPAN;
  static constexpr int X_TILE = TR * XB;
  static constexpr int CB = D * BITS / 8;               // code bytes / vector
  static constexpr bool CODES_TMA = CB >= 16;
  static constexpr int C_SPAN = CB < 128 ? CB : 128;
  static constexpr int C_PIECES = CB / C_SPAN;
  static constexpr int C_TILE = TR * CB;
  static constexpr int CW = (CB + 3) / 4;               // code words / vector
  static constexpr int NG = D / G;                      // groups / vector
  static constexpr int SW = (NG + 1) / 2;               // scale words / vector
  static constexpr int QMAX = (1 << (BITS - 1)) - 1;
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Per-warp shared-memory layout: NST input tiles (x for the quantiser, codes
// for the dequantiser; 1024-byte aligned for the swizzled TMA boxes), one
// output staging tile (codes, or the dequantised fp16 vectors), the per-head
// multiplier tables (d floats each) and sign tables (d/2 words each) of up to
// kMaxHPT heads, and the barriers. Each head's table is padded by 16 bytes so
// that the lanes of different heads reading the same column hit distinct
// banks.
template <int D, int BITS, int G, int NST, bool QUANT>
struct WarpLayout {
  using S = Shape<D, BITS, G>;
  static constexpr int kInTile = QUANT ? S::X_TILE : (S::CODES_TMA ? S::C_TILE : 0);
  static constexpr int kInBytes = align_up(kInTile, 1024);
  static constexpr int kOutTile = QUANT ? (S::CODES_TMA ? S::C_TILE : 0) : S::X_TILE;
  static constexpr int kOutBytes = align_up(kOutTile, 1024);
  static constexpr int kOutOff = NST * kInBytes;
  static constexpr int kStageTx = kInTile;
  static constexpr int kMultStride = D + 4;          // floats per head
  static constexpr int kSignStride = D / 2 + 4;      // words per head
  static constexpr int kTableOff = kOutOff + kOutBytes;
  static constexpr int kSignTabOff = kTableOff + 4 * kMaxHPT * kMultStride;
  static constexpr int kBarOff = align_up(kSignTabOff + 4 * kMaxHPT * kSignStride, 16);
  static constexpr int kWarpBytes = align_up(kBarOff + 8 * NST, 1024);
};

// The launch reserves 1 KB of slack so the swizzled TMA boxes can start on a
// 1024-byte boundary whatever the base of dynamic shared memory is.
constexpr int kSmemSlack = 1024;

__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Gain of packed coordinate j as a float (see coordinate_gain).
template <int ROT, int D>
__device__ __forceinline__ float gain_f(int j) {
  constexpr float g01 = float(coordinate_gain<ROT, D>(0));
  if constexpr (ROT == kSRHT) {
    return g01;
  } else {
    constexpr float gL = float(coordinate_gain<ROT, D>(D / 2));
    constexpr float gL1 = float(coordinate_gain<ROT, D>(D / 2 + 1));
    constexpr float gk = float(coordinate_gain<ROT, D>(2));
    return j < 2 ? g01 : (j == D / 2 ? gL : (j == D / 2 + 1 ? gL1 : gk));
  }
}

// fp16 +-1.0 pair for int8 signs s0, s1 (negative means -1).
__device__ __forceinline__ uint32_t sign_halves(int8_t s0, int8_t s1) {
  return (s0 < 0 ? 0xBC00u : 0x3C00u) | ((s1 < 0 ? 0xBC00u : 0x3C00u) << 16);
}

// XOR mask flipping the fp16 sign bits of a pair where the sign is negative.
__device__ __forceinline__ uint32_t sign_mask(int8_t s0, int8_t s1) {
  return (s0 < 0 ? 0x00008000u : 0u) | (s1 < 0 ? 0x80000000u : 0u);
}

// max(|a|, |b|, |c|) in one instruction.
__device__ __forceinline__ float absmax3(float a, float b, float c) {
  float r;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Correctly rounded a / Q for the constant Q: q0 = a * RN(1/Q) is within an
// ulp, the FMA remainder a - q0 Q is exact, and one correction step gives the
// rounded quotient (Markstein's theorem on division by a reciprocal).
template <int Q>
__device__ __forceinline__ float div_by_const(float a) {
  constexpr float inv = float(1.0 / double(Q));
  const float q0 = a * inv;
  const float r = fmaf(-q0, float(Q), a);
  return fmaf(r, inv, q0);
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Whether the rounding step uses f32x2 FMAs (constant pairs in registers)
// or scalar FMAs with an immediate.
#ifndef SRFTQ_PACKED_ROUND
#define SRFTQ_PACKED_ROUND 1
#endif

// 1.5 * 2^23: adding it to |v| < 2^22 rounds v to an integer (ties to even)
// whose two's complement lands in the low bits of the float's encoding.
constexpr float kMagic = 12582912.0f;

// ---------------------------------------------------------------------------
// Quantiser
// ---------------------------------------------------------------------------

// Three-input max / min (one instruction each on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Largest and smallest of the n group absmaxes.
template <int N>
__device__ __forceinline__ void range_of(const float (&a)[N], float& hi, float& lo) {
  if constexpr (N == 1) {
    hi = lo = a[0];
  } else {
    hi = fmaxf(a[0], a[1]);
    lo = fminf(a[0], a[1]);
    static_for<2, N>([&](auto i_) {
      constexpr int i = decltype(i_)::value;
      if constexpr (i % 2 == 0 && i + 1 < N) {
        hi = max3f(hi, a[i], a[i + 1]);
        lo = min3f(lo, a[i], a[i + 1]);
      } else if constexpr (i % 2 == 0) {
        hi = fmaxf(hi, a[i]);
        lo = fminf(lo, a[i]);
      }
    });
  }
}

// Packed form of div_by_const: two correctly rounded quotients a / Q.
template <int Q>
__device__ __forceinline__ float2 div_by_const2(float2 a) {
  constexpr float inv = float(1.0 / double(Q));
  const float2 q0 = mul2(a, splat(inv));
  const float2 r = fma2(q0, splat(-float(Q)), a);
  return fma2(r, splat(inv), q0);
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t h) {
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Scales and reciprocals of all groups of one vector from the group absmax
// a_g: sigma_g = fp16_rn(a_g / QMAX), written as packed fp16 words (low half
// = even group), inv_g = 1 / sigma_g. FAST: every sigma_g is a normal fp16
// and a_g / QMAX does not exceed 65504 (checked by the caller); otherwise
// saturation at 65504, sigma = 0 (inv = 0, all codes 0) and subnormal scales
// are handled, and CLAMP reports that the codes need clamping.
template <int NG, int QMAX, bool FAST>
__device__ __forceinline__ void group_scales(const float (&am)[NG], uint32_t (&sw)[(NG + 1) / 2],
                                             float (&inv)[NG]) {
  if constexpr (NG == 1) {
    float sf = div_by_const<QMAX>(am[0]);
    if constexpr (!FAST) sf = fminf(sf, 65504.0f);
    const __half hs = __float2half_rn(sf);
    sw[0] = __half_as_ushort(hs);
    const float sg = __half2float(hs);
    inv[0] = FAST ? rcp_approx(sg) : (sg > 0.0f ? rcp_approx(sg) : 0.0f);
  } else {
    static_for<0, NG / 2>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      float2 sf = div_by_const2<QMAX>(make_float2(am[2 * k], am[2 * k + 1]));
      if constexpr (!FAST) sf = make_float2(fminf(sf.x, 65504.0f), fminf(sf.y, 65504.0f));
      const uint32_t h2 = pack_f16x2(sf.x, sf.y);
      sw[k] = h2;
      const float2 sg = unpack_f16x2(h2);
      if constexpr (FAST) {
        inv[2 * k] = rcp_approx(sg.x);
        inv[2 * k + 1] = rcp_approx(sg.y);
      } else {
        inv[2 * k] = sg.x > 0.0f ? rcp_approx(sg.x) : 0.0f;
        inv[2 * k + 1] = sg.y > 0.0f ? rcp_approx(sg.y) : 0.0f;
      }
    });
  }
}

// Builds the tables of the HPT heads of (slice s, head block hb) from global
// memory (all lanes; rare: a warp's head block changes only at the ends of
// its tile range). QUANT: multiplier gain_j / lambda_j and fp16 +-1 sign
// pairs; otherwise multiplier gain_j * lambda_j (int4: / 16 at odd j,
// matching the x16 of the odd codes' unpacking) and fp16 sign-bit masks.
template <int D, int BITS, int ROT, bool QUANT, int MS, int SS>
__device__ __forceinline__ void build_tables(float* mult, uint32_t* stab, const float* lambda,
                                             const int8_t* signs, int s, int hb, int H,
                                             int hpt_log2, int lane) {
  // The HPT heads' lambda rows (HPT * D floats) and sign rows (HPT * D
  // bytes) are contiguous; every lane issues all of its 16-byte loads before
  // using any, so a rebuild costs one memory round trip.
  constexpr int kL4 = (kMaxHPT * D / 4 + 31) / 32;    // float4 loads per lane, at most
  constexpr int kS16 = (kMaxHPT * D / 16 + 31) / 32;  // 16-sign loads per lane, at most
  const int hpt = 1 << hpt_log2;
  const size_t h0 = static_cast<size_t>(s) * H + static_cast<size_t>(hb) * hpt;
  const float4* lam4 = reinterpret_cast<const float4*>(lambda + h0 * D);
  const uint4* sg16 = reinterpret_cast<const uint4*>(signs + h0 * D);
  const int n4 = (hpt * D) / 4, n16 = (hpt * D) / 16;
  float4 l[kL4];
  uint4 g[kS16];
#pragma unroll
  for (int k = 0; k < kL4; ++k) {
    const int i = lane + 32 * k;
    if (i < n4) l[k] = __ldg(lam4 + i);
  }
#pragma unroll
  for (int k = 0; k < kS16; ++k) {
    const int i = lane + 32 * k;
    if (i < n16) g[k] = __ldg(sg16 + i);
  }
  __syncwarp();   // every lane is done reading the old tables
#pragma unroll
  for (int k = 0; k < kL4; ++k) {
    const int i = lane + 32 * k;
    if (i < n4) {
      const int h = (4 * i) / D, j = (4 * i) % D;
      const float lv[4] = {l[k].x, l[k].y, l[k].z, l[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float m;
        if constexpr (QUANT)
          m = gain_f<ROT, D>(j + e) * rcp_approx(lv[e]);
        else
          m = gain_f<ROT, D>(j + e) * lv[e] * ((BITS == 4 && ((j + e) & 1)) ? 0.0625f : 1.0f);
        mult[h * MS + j + e] = m;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kS16; ++k) {
    const int i = lane + 32 * k;
    if (i < n16) {
      const int h = (16 * i) / D, w0 = ((16 * i) % D) / 2;
      const uint32_t wd[4] = {g[k].x, g[k].y, g[k].z, g[k].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int8_t s0 = static_cast<int8_t>(wd[e / 2] >> (16 * (e & 1)));
        const int8_t s1 = static_cast<int8_t>(wd[e / 2] >> (16 * (e & 1) + 8));
        stab[h * SS + w0 + e] = QUANT ? sign_halves(s0, s1) : sign_mask(s0, s1);
      }
    }
  }
  __syncwarp();
}

// Group absmax -> fp16 scales -> codes of one vector w (pairs v[p] =
// (w_{2p}, w_{2p+1}), already divided by lambda): sw = the packed fp16 scale
// pairs, words = the packed codes (int4: byte k = code 2k in the low nibble,
// code 2k+1 in the high nibble; int8: one byte per code).
template <int D, int BITS, int G>
__device__ __forceinline__ void quantize_codes(const float2 (&v)[D / 2],
                                               uint32_t (&sw)[Shape<D, BITS, G>::SW],
                                               uint32_t (&words)[Shape<D, BITS, G>::CW]) {
  using S = Shape<D, BITS, G>;
  // Group absmax -> fp16 scale -> codes as float-encoded integers.
  // When every group's scale is a normal fp16 and no a_g / qmax exceeds
  // 65504, |w / sigma| <= qmax * (1 + 2^-10) up to rounding, which rounds
  // inside the range: that common case (decided once per vector from the
  // largest and smallest absmax) runs without clamps; a vector with a zero,
  // subnormal-scale or saturating group takes the clamped block.
  float am[S::NG];
  static_for<0, S::NG>([&](auto g_) {
    constexpr int g = decltype(g_)::value;
    constexpr int P0 = g * G / 2;   // first pair of the group
    float m = absmax3(0.0f, v[P0].x, v[P0].y);
    static_for<1, G / 2>([&](auto p_) {
      constexpr int p = P0 + decltype(p_)::value;
      m = absmax3(m, v[p].x, v[p].y);
    });
    am[g] = m;
  });
  float a_hi, a_lo;
  range_of(am, a_hi, a_lo);
  constexpr float kHi = 65504.0f * float(S::QMAX);            // no saturation
  constexpr float kLo = 6.103515625e-05f * float(S::QMAX);    // sigma >= 2^-14
  uint32_t qb[D];
  if (a_hi <= kHi && a_lo >= kLo) {
    float invs[S::NG];
    group_scales<S::NG, S::QMAX, true>(am, sw, invs);
    static_for<0, D / 2>([&](auto p_) {
      constexpr int p = decltype(p_)::value;
      const float2 r = fma2(v[p], splat(invs[(2 * p) / G]), splat(kMagic));
      qb[2 * p] = __float_as_uint(r.x);
      qb[2 * p + 1] = __float_as_uint(r.y);
    });
  } else {
    float invs[S::NG];
    group_scales<S::NG, S::QMAX, false>(am, sw, invs);
    static_for<0, D / 2>([&](auto p_) {
      constexpr int p = decltype(p_)::value;
      const float inv = invs[(2 * p) / G];
      const float q0 = fminf(fmaxf(v[p].x * inv, -float(S::QMAX)), float(S::QMAX));
      const float q1 = fminf(fmaxf(v[p].y * inv, -float(S::QMAX)), float(S::QMAX));
      qb[2 * p] = __float_as_uint(q0 + kMagic);
      qb[2 * p + 1] = __float_as_uint(q1 + kMagic);
    });
  }

  // Pack. The low byte of every qb is its code in two's complement.
  // int4: byte k = code 2k in the low nibble | code 2k+1 in the high nibble;
  // gather the even and the odd codes' bytes, then merge the nibbles.
  if constexpr (BITS == 4) {
    static_for<0, D / 8>([&](auto m_) {
      constexpr int m = decltype(m_)::value;
      const uint32_t ev = __byte_perm(__byte_perm(qb[8 * m + 0], qb[8 * m + 2], 0x0040),
                                      __byte_perm(qb[8 * m + 4], qb[8 * m + 6], 0x0040), 0x5410);
      const uint32_t od = __byte_perm(__byte_perm(qb[8 * m + 1], qb[8 * m + 3], 0x0040),
                                      __byte_perm(qb[8 * m + 5], qb[8 * m + 7], 0x0040), 0x5410);
      words[m] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
    });
  } else {
    static_for<0, D / 4>([&](auto m_) {
      constexpr int m = decltype(m_)::value;
      words[m] = __byte_perm(__byte_perm(qb[4 * m], qb[4 * m + 1], 0x0040),
                             __byte_perm(qb[4 * m + 2], qb[4 * m + 3], 0x0040), 0x5410);
    });
  }
}

template <int D, int BITS, int G, int ROT, int WPC, int NST, int MINB>
__global__ void __launch_bounds__(WPC * 32, MINB)
    quantize_kernel(const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_codes, const QuantArgs a) {
  using S = Shape<D, BITS, G>;
  using Lay = WarpLayout<D, BITS, G, NST, true>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int warp = WPC == 1 ? 0 : int(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  uint8_t* ws = smem + warp * Lay::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ws + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(ws + Lay::kTableOff);
  uint32_t* stab = reinterpret_cast<uint32_t*>(ws + Lay::kSignTabOff);
  uint8_t* ob = ws + Lay::kOutOff;   // codes staging tile

  TileWalk cur;
  if (!cur.start(blockIdx.x * WPC + warp, gridDim.x * WPC, a.g)) return;
  const int hpt_log2 = a.g.hpt_log2;
  const int hpt = 1 << hpt_log2;
  const int rpt = kTileRows >> hpt_log2;
  const int hl = lane & (hpt - 1);         // this lane's head inside the tile
  const int rl = lane >> hpt_log2;         // and its row
  const float* mrow = mult + hl * Lay::kMultStride;
  const uint32_t* srow = stab + hl * Lay::kSignStride;

  if (lane == 0) {
    prefetch_tensormap(&tm_x);
    if constexpr (S::CODES_TMA) prefetch_tensormap(&tm_codes);
    for (int s = 0; s < NST; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto issue = [&](const TileWalk& c, int st) {
    uint8_t* sb = ws + st * Lay::kInBytes;
    if (!dbg_ok(tile_in_range(c, a.g), a.guard)) {
      mbar_arrive(&bars[st]);   // debug build: no copy, the phase completes empty
      return;
    }
    mbar_arrive_expect_tx(&bars[st], Lay::kStageTx);
#pragma unroll
    for (int p = 0; p < S::X_PIECES; ++p)
      tma_load_4d(sb + p * (S::TR * S::X_SPAN), &tm_x, &bars[st], p * (S::X_SPAN / 2),
                  c.hb * hpt, c.rb * rpt, c.s);
  };
  auto store_codes = [&](const TileWalk& c) {
    if (dbg_ok(tile_in_range(c, a.g), a.guard)) {
#pragma unroll
      for (int p = 0; p < S::C_PIECES; ++p)
        tma_store_4d(&tm_codes, ob + p * (S::TR * S::C_SPAN), p * S::C_SPAN, c.hb * hpt,
                     c.rb * rpt, c.s);
    }
    bulk_commit();
  };

  // Lane 0 issues the first NST tiles; `ahead` is then the next tile to
  // issue and `issued` counts the tiles issued so far.
  TileWalk ahead = cur;
  int issued = 0;
  if (lane == 0) {
    for (int k = 0; k < NST && ahead.valid(); ++k) {
      issue(ahead, k);
      ++issued;
      ahead.advance(a.g);
    }
  }

  int it = 0;
  int table_key = -1;         // (slice, head block) the tables were built for
  bool pending = false;       // a staged codes tile awaits its TMA store
  TileWalk prev = cur;
  for (; cur.valid(); ++it) {
    const int st = it % NST;
    const uint32_t parity = (it / NST) & 1;
    const uint8_t* sb = ws + st * Lay::kInBytes;

    // (a) per-head tables, rebuilt only when the (slice, head block) changes
    const int key = cur.table_key(a.g);
    if (key != table_key) {
      build_tables<D, BITS, ROT, true, Lay::kMultStride, Lay::kSignStride>(
          mult, stab, a.lambda, a.signs, cur.s, cur.hb, a.g.heads, hpt_log2, lane);
      table_key = key;
    }

    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], parity));
    if (!ok) {
      if (lane == 0) {
        atomicOr(a.guard, kGuardWaitTimeout);
        // give the other issued stages' copies (again boundedly) a chance to land
        for (int k = it + 1; k < issued; ++k)
          (void)mbar_wait_bounded(&bars[k % NST], (k / NST) & 1);
        bulk_wait<0>();
      }
      __syncwarp();
      return;
    }
    // (b) this lane's vector (swizzled 16-byte chunks) and the sign words
    uint32_t xw[D / 2], sgw[D / 2];
    const uint32_t xrow = swz_row<S::X_SPAN>(smem_addr(sb), lane);
    static_for<0, D / 8>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      constexpr int piece = (ci * 16) / S::X_SPAN;
      constexpr int cc = ((ci * 16) % S::X_SPAN) / 16;
      const uint4 raw = lds128(swz_chunk<S::X_SPAN>(xrow, cc) + piece * (S::TR * S::X_SPAN));
      const uint4 sg = *reinterpret_cast<const uint4*>(srow + 4 * ci);
      xw[4 * ci + 0] = raw.x;
      xw[4 * ci + 1] = raw.y;
      xw[4 * ci + 2] = raw.z;
      xw[4 * ci + 3] = raw.w;
      sgw[4 * ci + 0] = sg.x;
      sgw[4 * ci + 1] = sg.y;
      sgw[4 * ci + 2] = sg.z;
      sgw[4 * ci + 3] = sg.w;
    });
    // Converged: every lane has read this stage and has staged and fenced
    // the previous tile's codes. Store those, and refill this stage with the
    // tile NST ahead right away, so the copy overlaps all of this tile's work.
    __syncwarp();
    if (lane == 0) {
      if (pending) store_codes(prev);
      if (ahead.valid()) {
        issue(ahead, st);
        ++issued;
        ahead.advance(a.g);
      }
    }
    pending = false;

    // (c) rotation, then w_j = y_j / lambda_j through the multiplier table
    float2 v[D / 2];
    rotate_forward<ROT, D>(xw, sgw, v);
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = *reinterpret_cast<const float4*>(mrow + 4 * ci);
      v[2 * ci] = mul2(v[2 * ci], make_float2(m4.x, m4.y));
      v[2 * ci + 1] = mul2(v[2 * ci + 1], make_float2(m4.z, m4.w));
    });

    // (d), (e) scales and packed codes
    uint32_t sw[S::SW];
    uint32_t words[S::CW];
    quantize_codes<D, BITS, G>(v, sw, words);

    const int row = cur.rb * rpt + rl;
    const size_t vec = (static_cast<size_t>(cur.s) * a.out_slice_stride_rows + row) * a.g.heads +
                       cur.hb * hpt + hl;
    const bool valid =
        row < a.g.n_rows &&
        dbg_ok(int64_t(vec) < vec_limit(a.g.n_slices, a.out_slice_stride_rows, a.g.n_rows,
                                        a.g.heads),
               a.guard);

    // (f) codes: swizzled staging tile, stored by TMA at the next convergence
    // (rows past N are clipped by TMA). The store issued at this tile's start
    // read the staging tile long ago; the wait only confirms it.
    if constexpr (S::CODES_TMA) {
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      const uint32_t crow = swz_row<S::C_SPAN>(smem_addr(ob), lane);
      static_for<0, S::CB / 16>([&](auto c_) {
        constexpr int ci = decltype(c_)::value;
        constexpr int piece = (ci * 16) / S::C_SPAN;
        constexpr int cc = ((ci * 16) % S::C_SPAN) / 16;
        sts128(swz_chunk<S::C_SPAN>(crow, cc) + piece * (S::TR * S::C_SPAN),
               make_uint4(words[4 * ci], words[4 * ci + 1], words[4 * ci + 2], words[4 * ci + 3]));
      });
      fence_proxy_async_smem();
      pending = true;
      prev = cur;
    } else {
      static_assert(S::CODES_TMA || S::CB == 8, "direct code path covers d=16 int4 only");
      if (valid) *reinterpret_cast<uint2*>(a.codes + vec * S::CB) = make_uint2(words[0], words[1]);
    }

    // (g) scales straight from registers (packed fp16 words)
    if (valid) {
      uint16_t* dst = a.scales + vec * S::NG;
      if constexpr (S::NG == 1) {
        dst[0] = static_cast<uint16_t>(sw[0]);
      } else if constexpr (S::NG == 2) {
        *reinterpret_cast<uint32_t*>(dst) = sw[0];
      } else if constexpr (S::NG == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(sw[0], sw[1]);
      } else {
        static_for<0, S::NG / 8>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          reinterpret_cast<uint4*>(dst)[k] =
              make_uint4(sw[4 * k], sw[4 * k + 1], sw[4 * k + 2], sw[4 * k + 3]);
        });
      }
    }
    cur.advance(a.g);
  }
  __syncwarp();
  if (lane == 0) {
    if (pending) store_codes(prev);
    bulk_wait<0>();
  }
}

// ---------------------------------------------------------------------------
// Dequantiser
// ---------------------------------------------------------------------------

// Codes of one 32-bit word to exact fp32 values q * sigma (int8: 4 codes;
// int4: 8 codes, odd positions scaled by 16). The codes are spread into fp16
// pairs 1024 + offset + code (one AND-XOR each), then `fma.rn.f32.f16`
// multiplies by the fp16 scale and subtracts the offset's product exactly.
template <int BITS, int HS>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t sgw, float c_even, float c_odd,
                                            float2* out) {
  const uint32_t w8 = w >> 8;
  if constexpr (BITS == 4) {
    const uint32_t h04 = (w & 0x000F000Fu) ^ 0x64086408u;   // 1024 + 8 + q
    const uint32_t h15 = (w & 0x00F000F0u) ^ 0x64806480u;   // 1024 + 16 (8 + q)
    const uint32_t h26 = (w8 & 0x000F000Fu) ^ 0x64086408u;
    const uint32_t h37 = (w8 & 0x00F000F0u) ^ 0x64806480u;
    out[0] = make_float2(fma_f16<0, HS>(h04, sgw, c_even), fma_f16<0, HS>(h15, sgw, c_odd));
    out[1] = make_float2(fma_f16<0, HS>(h26, sgw, c_even), fma_f16<0, HS>(h37, sgw, c_odd));
    out[2] = make_float2(fma_f16<1, HS>(h04, sgw, c_even), fma_f16<1, HS>(h15, sgw, c_odd));
    out[3] = make_float2(fma_f16<1, HS>(h26, sgw, c_even), fma_f16<1, HS>(h37, sgw, c_odd));
  } else {
    const uint32_t h02 = (w & 0x00FF00FFu) ^ 0x64806480u;   // 1024 + 128 + q
    const uint32_t h13 = (w8 & 0x00FF00FFu) ^ 0x64806480u;
    out[0] = make_float2(fma_f16<0, HS>(h02, sgw, c_even), fma_f16<0, HS>(h13, sgw, c_even));
    out[1] = make_float2(fma_f16<1, HS>(h02, sgw, c_even), fma_f16<1, HS>(h13, sgw, c_even));
  }
}

template <int D, int BITS, int G, int ROT, int WPC, int NST, int MINB>
__global__ void __launch_bounds__(WPC * 32, MINB)
    dequantize_kernel(const __grid_constant__ CUtensorMap tm_codes,
                      const __grid_constant__ CUtensorMap tm_xhat, const DequantArgs a) {
  using S = Shape<D, BITS, G>;
  using Lay = WarpLayout<D, BITS, G, NST, false>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int warp = WPC == 1 ? 0 : int(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  uint8_t* ws = smem + warp * Lay::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ws + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(ws + Lay::kTableOff);
  uint32_t* mtab = reinterpret_cast<uint32_t*>(ws + Lay::kSignTabOff);
  uint8_t* ob = ws + Lay::kOutOff;   // fp16 staging tile

  TileWalk cur;
  if (!cur.start(blockIdx.x * WPC + warp, gridDim.x * WPC, a.g)) return;
  const int hpt_log2 = a.g.hpt_log2;
  const int hpt = 1 << hpt_log2;
  const int rpt = kTileRows >> hpt_log2;
  const int hl = lane & (hpt - 1);
  const int rl = lane >> hpt_log2;
  const float* mrow = mult + hl * Lay::kMultStride;
  const uint32_t* mkrow = mtab + hl * Lay::kSignStride;

  if (lane == 0) {
    if constexpr (S::CODES_TMA) prefetch_tensormap(&tm_codes);
    prefetch_tensormap(&tm_xhat);
    for (int s = 0; s < NST; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto issue = [&](const TileWalk& c, int st) {
    uint8_t* sb = ws + st * Lay::kInBytes;
    if (!dbg_ok(tile_in_range(c, a.g), a.guard)) {
      mbar_arrive(&bars[st]);   // debug build: no copy, the phase completes empty
      return;
    }
    if constexpr (S::CODES_TMA) {
      mbar_arrive_expect_tx(&bars[st], Lay::kStageTx);
#pragma unroll
      for (int p = 0; p < S::C_PIECES; ++p)
        tma_load_4d(sb + p * (S::TR * S::C_SPAN), &tm_codes, &bars[st], p * S::C_SPAN,
                    c.hb * hpt, c.rb * rpt, c.s);
    } else {
      mbar_arrive(&bars[st]);   // no asynchronous input: the phase completes at once
    }
  };
  auto store_xhat = [&](const TileWalk& c) {
    if (dbg_ok(tile_in_range(c, a.g), a.guard)) {
#pragma unroll
      for (int p = 0; p < S::X_PIECES; ++p)
        tma_store_4d(&tm_xhat, ob + p * (S::TR * S::X_SPAN), p * (S::X_SPAN / 2), c.hb * hpt,
                     c.rb * rpt, c.s);
    }
    bulk_commit();
  };

  TileWalk ahead = cur;
  int issued = 0;
  if (lane == 0) {
    for (int k = 0; k < NST && ahead.valid(); ++k) {
      issue(ahead, k);
      ++issued;
      ahead.advance(a.g);
    }
  }

  // the next tile's scales are loaded one tile ahead, into registers
  auto load_scales = [&](const TileWalk& c, uint32_t (&sw)[S::SW]) {
    const int row = c.rb * rpt + rl;
    const size_t vec = (static_cast<size_t>(c.s) * a.in_slice_stride_rows + row) * a.g.heads +
                       c.hb * hpt + hl;
    if (row < a.g.n_rows &&
        dbg_ok(int64_t(vec) < vec_limit(a.g.n_slices, a.in_slice_stride_rows, a.g.n_rows,
                                        a.g.heads),
               a.guard)) {
      const uint16_t* src = a.scales + vec * S::NG;
      if constexpr (S::NG == 1) {
        sw[0] = src[0];
      } else if constexpr (S::NG == 2) {
        sw[0] = *reinterpret_cast<const uint32_t*>(src);
      } else if constexpr (S::NG == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(src);
        sw[0] = u.x;
        sw[1] = u.y;
      } else {
        static_for<0, S::NG / 8>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          const uint4 u = reinterpret_cast<const uint4*>(src)[k];
          sw[4 * k] = u.x;
          sw[4 * k + 1] = u.y;
          sw[4 * k + 2] = u.z;
          sw[4 * k + 3] = u.w;
        });
      }
    } else {
      static_for<0, S::SW>([&](auto k_) { sw[decltype(k_)::value] = 0u; });
    }
  };
  uint32_t sw_next[S::SW];
  load_scales(cur, sw_next);

  int it = 0;
  int table_key = -1;         // (slice, head block) the tables were built for
  bool pending = false;       // a staged fp16 tile awaits its TMA store
  TileWalk prev = cur;
  for (; cur.valid(); ++it) {
    const int st = it % NST;
    const uint32_t parity = (it / NST) & 1;
    const uint8_t* sb = ws + st * Lay::kInBytes;
    const int row = cur.rb * rpt + rl;
    const bool valid =
        row < a.g.n_rows &&
        dbg_ok(int64_t((static_cast<size_t>(cur.s) * a.in_slice_stride_rows + row) * a.g.heads +
                       cur.hb * hpt + hl) <
                   vec_limit(a.g.n_slices, a.in_slice_stride_rows, a.g.n_rows, a.g.heads),
               a.guard);

    uint32_t sw[S::SW];
    static_for<0, S::SW>([&](auto k_) { sw[decltype(k_)::value] = sw_next[decltype(k_)::value]; });
    TileWalk nxt = cur;
    nxt.advance(a.g);
    if (nxt.valid()) load_scales(nxt, sw_next);

    uint32_t words[S::CW];
    if constexpr (!S::CODES_TMA) {
      if (valid) {
        const size_t vec = (static_cast<size_t>(cur.s) * a.in_slice_stride_rows + row) *
                               a.g.heads + cur.hb * hpt + hl;
        const uint2 u = *reinterpret_cast<const uint2*>(a.codes + vec * S::CB);
        words[0] = u.x;
        words[1] = u.y;
      } else {
        words[0] = words[1] = 0u;
      }
    }

    // (a) per-head tables, rebuilt only when the (slice, head block) changes
    const int key = cur.table_key(a.g);
    if (key != table_key) {
      build_tables<D, BITS, ROT, false, Lay::kMultStride, Lay::kSignStride>(
          mult, mtab, a.lambda, a.signs, cur.s, cur.hb, a.g.heads, hpt_log2, lane);
      table_key = key;
    }

    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], parity));
    if (!ok) {
      if (lane == 0) {
        atomicOr(a.guard, kGuardWaitTimeout);
        for (int k = it + 1; k < issued; ++k)
          (void)mbar_wait_bounded(&bars[k % NST], (k / NST) & 1);
        bulk_wait<0>();
      }
      __syncwarp();
      return;
    }
    // (b) codes of this lane's vector
    if constexpr (S::CODES_TMA) {
      const uint32_t crow = swz_row<S::C_SPAN>(smem_addr(sb), lane);
      static_for<0, S::CB / 16>([&](auto c_) {
        constexpr int ci = decltype(c_)::value;
        constexpr int piece = (ci * 16) / S::C_SPAN;
        constexpr int cc = ((ci * 16) % S::C_SPAN) / 16;
        const uint4 u = lds128(swz_chunk<S::C_SPAN>(crow, cc) + piece * (S::TR * S::C_SPAN));
        words[4 * ci] = u.x;
        words[4 * ci + 1] = u.y;
        words[4 * ci + 2] = u.z;
        words[4 * ci + 3] = u.w;
      });
    }
    // Converged: every lane has read this stage and has staged and fenced
    // the previous tile's output. Store that, and refill this stage with the
    // tile NST ahead right away.
    __syncwarp();
    if (lane == 0) {
      if (pending) store_xhat(prev);
      if (ahead.valid()) {
        issue(ahead, st);
        ++issued;
        ahead.advance(a.g);
      }
    }
    pending = false;

    // (c) yhat_j = q_j * sigma_g * lambda_j * gain_j
    float2 v[D / 2];
    constexpr int CPW = 32 / BITS;   // codes per word
    static_for<0, S::CW>([&](auto m_) {
      constexpr int m = decltype(m_)::value;
      constexpr int g = (m * CPW) / G;
      const float sgf = __half2float(__ushort_as_half(
          static_cast<unsigned short>((sw[g / 2] >> (16 * (g & 1))) & 0xFFFFu)));
      const float c_even = BITS == 4 ? -1032.0f * sgf : -1152.0f * sgf;
      const float c_odd = -1152.0f * sgf;
      unpack_word<BITS, g & 1>(words[m], sw[g / 2], c_even, c_odd, &v[m * CPW / 2]);
    });
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = *reinterpret_cast<const float4*>(mrow + 4 * ci);
      v[2 * ci] = mul2(v[2 * ci], make_float2(m4.x, m4.y));
      v[2 * ci + 1] = mul2(v[2 * ci + 1], make_float2(m4.z, m4.w));
    });

    // (d) inverse rotation
    rotate_inverse<ROT, D>(v);

    // (e) signs + fp16 into the swizzled staging tile, stored by TMA at the
    // next convergence. The store issued at this tile's start read the
    // staging tile long ago; the wait only confirms it.
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
    const uint32_t xrow = swz_row<S::X_SPAN>(smem_addr(ob), lane);
    static_for<0, D / 8>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      constexpr int piece = (ci * 16) / S::X_SPAN;
      constexpr int cc = ((ci * 16) % S::X_SPAN) / 16;
      const uint4 mk = *reinterpret_cast<const uint4*>(mkrow + 4 * ci);
      uint4 o;
      o.x = pack_f16x2(v[4 * ci + 0].x, v[4 * ci + 0].y) ^ mk.x;
      o.y = pack_f16x2(v[4 * ci + 1].x, v[4 * ci + 1].y) ^ mk.y;
      o.z = pack_f16x2(v[4 * ci + 2].x, v[4 * ci + 2].y) ^ mk.z;
      o.w = pack_f16x2(v[4 * ci + 3].x, v[4 * ci + 3].y) ^ mk.w;
      sts128(swz_chunk<S::X_SPAN>(xrow, cc) + piece * (S::TR * S::X_SPAN), o);
    });
    fence_proxy_async_smem();
    pending = true;
    prev = cur;
    cur = nxt;
  }
  __syncwarp();
  if (lane == 0) {
    if (pending) store_xhat(prev);
    bulk_wait<0>();
  }
}

}  // namespace srftq
