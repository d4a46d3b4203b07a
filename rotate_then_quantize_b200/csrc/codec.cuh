// Fused quantise / dequantise kernels (one thread per head-dim vector).
//
// Work decomposition. A *tile* is 32 consecutive rows of one (slice, head):
// vectors (s, r0..r0+31, h). Tiles are numbered with the head fastest, then
// the row block, then the slice, so consecutive tile numbers cover adjacent
// memory. Every warp is an independent persistent pipeline: warp w of the
// grid handles tiles w, w + W, w + 2W, ... (W = warps in the grid). A warp
// owns NST input stages in shared memory; lane 0 issues, per stage, the TMA
// box loads of the tile (32 rows x d fp16, 128-byte swizzled so that each
// lane reading its own row hits distinct banks) plus 1-D bulk copies of that
// (slice, head)'s lambda row and sign row, all completing on one mbarrier.
// The lanes then build the per-tile multiplier and sign-mask tables, pull
// their vector into registers, hand the stage back to the TMA engine, and
// compute. Codes leave through a swizzled shared staging buffer and a TMA
// tensor store; scales are stored straight from registers.
//
// Quantiser stages follow "When Quantization Is Free", Methodology 2:
// (1) load and sign multiply (an XOR of the fp16 sign bit in registers),
// (2) the radix-2 FFT passes, (3) the Hermitian pack, (4) per-channel
// lambda, group absmax and rounding to signed int4/int8, (5) nibble packing.
// The dequantiser runs the same stages backwards.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"
#include "transform.cuh"

namespace srftq {

constexpr int kTileRows = 32;

struct TileGeom {
  int32_t heads;       // H
  int32_t row_blocks;  // ceil(N / 32)
  int32_t n_rows;      // N
  int32_t total_tiles; // S * row_blocks * H
};

struct TileCoord {
  int s, r0, h;
};

__device__ __forceinline__ TileCoord decode_tile(int t, const TileGeom& g) {
  const int h = t % g.heads;
  const int q = t / g.heads;
  const int rb = q % g.row_blocks;
  return {q / g.row_blocks, rb * kTileRows, h};
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
  static constexpr int QMAX = (1 << (BITS - 1)) - 1;
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Per-warp shared-memory layout. Stage s: [x or codes tile][lambda row][sign row].
template <int D, int BITS, int G, int NST, int NOUT, bool QUANT>
struct WarpLayout {
  using S = Shape<D, BITS, G>;
  static constexpr int kInTile = QUANT ? S::X_TILE : (S::CODES_TMA ? S::C_TILE : 0);
  static constexpr int kLamOff = align_up(kInTile, 16);
  static constexpr int kSgnOff = kLamOff + 4 * D;
  static constexpr int kStageTx = kInTile + 4 * D + D;
  static constexpr int kStageBytes = align_up(kSgnOff + D, 1024);
  static constexpr int kOutTile = QUANT ? (S::CODES_TMA ? S::C_TILE : 0) : S::X_TILE;
  static constexpr int kOutBytes = align_up(kOutTile, 1024);
  static constexpr int kOutOff = NST * kStageBytes;
  static constexpr int kTableOff = kOutOff + NOUT * kOutBytes;
  static constexpr int kMaskOff = kTableOff + 4 * D;
  static constexpr int kBarOff = align_up(kMaskOff + 2 * D, 16);
  static constexpr int kWarpBytes = align_up(kBarOff + 8 * NST, 1024);
};

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

// Builds the sign-mask table (one 32-bit XOR mask per fp16 pair: bit 15 and
// bit 31 set where the sign is negative) from a raw int8 sign row.
template <int D>
__device__ __forceinline__ void build_masks(const int8_t* sgn, uint32_t* mask, int lane) {
  for (int w = lane; w < D / 2; w += 32) {
    const uint32_t lo = sgn[2 * w] < 0 ? 0x00008000u : 0u;
    const uint32_t hi = sgn[2 * w + 1] < 0 ? 0x80000000u : 0u;
    mask[w] = lo | hi;
  }
}

__device__ __forceinline__ __half2 u32_as_half2(uint32_t u) {
  __half2 h;
  *reinterpret_cast<uint32_t*>(&h) = u;
  return h;
}

__device__ __forceinline__ uint32_t half2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}

// 1.5 * 2^23: adding it to |v| < 2^22 rounds v to an integer (ties to even)
// whose two's complement lands in the low bits of the float's encoding.
constexpr float kMagic0 = 12582912.0f;

// The launch reserves 1 KB of slack so the swizzled TMA boxes can start on a
// 1024-byte boundary whatever the base of dynamic shared memory is.
constexpr int kSmemSlack = 1024;

__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ---------------------------------------------------------------------------
// Quantiser
// ---------------------------------------------------------------------------

template <int D, int BITS, int G, int ROT, int WPC, int NST, int NOUT>
__global__ void __launch_bounds__(WPC * 32)
    quantize_kernel(const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_codes, const QuantArgs a) {
  using S = Shape<D, BITS, G>;
  using Lay = WarpLayout<D, BITS, G, NST, NOUT, true>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* ws = smem + warp * Lay::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ws + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(ws + Lay::kTableOff);
  uint32_t* mask = reinterpret_cast<uint32_t*>(ws + Lay::kMaskOff);

  const int total = a.g.total_tiles;
  const int nw = gridDim.x * WPC;
  const int first = blockIdx.x * WPC + warp;
  if (first >= total) return;

  if (lane == 0) {
    prefetch_tensormap(&tm_x);
    if constexpr (S::CODES_TMA) prefetch_tensormap(&tm_codes);
    for (int s = 0; s < NST; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto issue = [&](int t, int st) {
    const TileCoord c = decode_tile(t, a.g);
    uint8_t* sb = ws + st * Lay::kStageBytes;
    mbar_arrive_expect_tx(&bars[st], Lay::kStageTx);
#pragma unroll
    for (int p = 0; p < S::X_PIECES; ++p)
      tma_load_4d(sb + p * (S::TR * S::X_SPAN), &tm_x, &bars[st], p * (S::X_SPAN / 2), c.h, c.r0,
                  c.s);
    const size_t row = static_cast<size_t>(c.s) * a.g.heads + c.h;
    bulk_load(sb + Lay::kLamOff, a.lambda + row * D, 4 * D, &bars[st]);
    bulk_load(sb + Lay::kSgnOff, a.signs + row * D, D, &bars[st]);
  };

  if (lane == 0) {
    for (int k = 0; k < NST; ++k) {
      const int t = first + k * nw;
      if (t < total) issue(t, k);
    }
  }

  int it = 0;
  for (int t = first; t < total; t += nw, ++it) {
    const int st = it % NST;
    const uint32_t parity = (it / NST) & 1;
    const TileCoord c = decode_tile(t, a.g);
    uint8_t* sb = ws + st * Lay::kStageBytes;

    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], parity));
    if (!ok) {
      if (lane == 0) {
        atomicOr(a.guard, kGuardWaitTimeout);
        // give the other stages' copies (again boundedly) a chance to land
        for (int k = 1; k < NST; ++k) {
          const int tk = t + k * nw;
          if (tk < total) (void)mbar_wait_bounded(&bars[(it + k) % NST], ((it + k) / NST) & 1);
        }
        bulk_wait<0>();
      }
      __syncwarp();
      return;
    }

    // (a) per-(slice, head) tables: multiplier gain_j / lambda_j and sign masks
    const float* lam_raw = reinterpret_cast<const float*>(sb + Lay::kLamOff);
    const int8_t* sgn_raw = reinterpret_cast<const int8_t*>(sb + Lay::kSgnOff);
    __syncwarp();
    for (int j = lane; j < D; j += 32) mult[j] = __fdiv_rn(gain_f<ROT, D>(j), lam_raw[j]);
    build_masks<D>(sgn_raw, mask, lane);
    __syncwarp();

    // (b) this lane's vector: swizzled 16-byte chunks, sign XOR, fp16 -> fp32
    float v[D];
    static_for<0, D / 8>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      constexpr int piece = (ci * 16) / S::X_SPAN;
      constexpr int cc = ((ci * 16) % S::X_SPAN) / 16;
      const uint32_t off =
          piece * (S::TR * S::X_SPAN) + swizzle<S::X_SPAN>(lane * S::X_SPAN + cc * 16);
      uint4 raw = *reinterpret_cast<const uint4*>(sb + off);
      const uint4 m = *reinterpret_cast<const uint4*>(mask + 4 * ci);
      raw.x ^= m.x;
      raw.y ^= m.y;
      raw.z ^= m.z;
      raw.w ^= m.w;
      const float2 f0 = __half22float2(u32_as_half2(raw.x));
      const float2 f1 = __half22float2(u32_as_half2(raw.y));
      const float2 f2 = __half22float2(u32_as_half2(raw.z));
      const float2 f3 = __half22float2(u32_as_half2(raw.w));
      v[8 * ci + 0] = f0.x;
      v[8 * ci + 1] = f0.y;
      v[8 * ci + 2] = f1.x;
      v[8 * ci + 3] = f1.y;
      v[8 * ci + 4] = f2.x;
      v[8 * ci + 5] = f2.y;
      v[8 * ci + 6] = f3.x;
      v[8 * ci + 7] = f3.y;
    });
    __syncwarp();
    if (lane == 0) {
      const int tn = t + NST * nw;
      if (tn < total) issue(tn, st);
    }

    // (c) rotation, then w_j = y_j / lambda_j through the multiplier table
    rotate_forward_raw<ROT, D>(v);
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = *reinterpret_cast<const float4*>(mult + 4 * ci);
      v[4 * ci + 0] *= m4.x;
      v[4 * ci + 1] *= m4.y;
      v[4 * ci + 2] *= m4.z;
      v[4 * ci + 3] *= m4.w;
    });

    // (d) group absmax -> fp16 scale -> rounded codes (float-encoded integers)
    uint32_t qb[D];
    uint16_t sig[S::NG];
    static_for<0, S::NG>([&](auto g_) {
      constexpr int g = decltype(g_)::value;
      float amax = 0.0f;
      static_for<0, G>([&](auto j_) {
        amax = fmaxf(amax, fabsf(v[g * G + decltype(j_)::value]));
      });
      const float sf = __fdiv_rn(amax, float(S::QMAX));
      const __half hs = __float2half_rn(fminf(sf, 65504.0f));
      sig[g] = __half_as_ushort(hs);
      const float sg = __half2float(hs);
      // With a normal, unsaturated scale |w/sigma| <= qmax * (1 + 2^-10), which
      // rounds inside the range: no clamp needed.
      if (sg >= 6.103515625e-05f && sf <= 65504.0f) {
        const float inv = __frcp_rn(sg);
        static_for<0, G>([&](auto j_) {
          constexpr int j = g * G + decltype(j_)::value;
          qb[j] = __float_as_uint(fmaf(v[j], inv, kMagic0));
        });
      } else {
        const float inv = sg > 0.0f ? __frcp_rn(sg) : 0.0f;
        static_for<0, G>([&](auto j_) {
          constexpr int j = g * G + decltype(j_)::value;
          const float q = fminf(fmaxf(v[j] * inv, -float(S::QMAX)), float(S::QMAX));
          qb[j] = __float_as_uint(q + kMagic0);
        });
      }
    });

    // (e) pack. The low byte of every qb is its code in two's complement.
    // int4: byte k = code 2k in the low nibble | code 2k+1 in the high nibble;
    // gather the even and the odd codes' bytes, then merge the nibbles.
    uint32_t words[S::CW];
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

    const int row = c.r0 + lane;
    const bool valid = row < a.g.n_rows;
    const size_t vec = (static_cast<size_t>(c.s) * a.out_slice_stride_rows + row) * a.g.heads + c.h;

    // (f) codes: swizzled staging + TMA store (rows past N are clipped by TMA)
    if constexpr (S::CODES_TMA) {
      uint8_t* ob = ws + Lay::kOutOff + (it % NOUT) * Lay::kOutBytes;
      if (lane == 0) bulk_wait_read<NOUT - 1>();
      __syncwarp();
      static_for<0, S::CB / 16>([&](auto c_) {
        constexpr int ci = decltype(c_)::value;
        constexpr int piece = (ci * 16) / S::C_SPAN;
        constexpr int cc = ((ci * 16) % S::C_SPAN) / 16;
        const uint32_t off =
            piece * (S::TR * S::C_SPAN) + swizzle<S::C_SPAN>(lane * S::C_SPAN + cc * 16);
        *reinterpret_cast<uint4*>(ob + off) =
            make_uint4(words[4 * ci], words[4 * ci + 1], words[4 * ci + 2], words[4 * ci + 3]);
      });
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int p = 0; p < S::C_PIECES; ++p)
          tma_store_4d(&tm_codes, ob + p * (S::TR * S::C_SPAN), p * S::C_SPAN, c.h, c.r0, c.s);
        bulk_commit();
      }
    } else {
      if (valid) {
        uint8_t* dst = a.codes + vec * S::CB;
        if constexpr (S::CB == 8) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
        } else {
          static_assert(S::CB == 8, "direct code path covers d=16 int4 only");
        }
      }
    }

    // (g) scales straight from registers
    if (valid) {
      uint16_t* dst = a.scales + vec * S::NG;
      if constexpr (S::NG == 1) {
        dst[0] = sig[0];
      } else {
        uint32_t sw[S::NG / 2];
        static_for<0, S::NG / 2>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          sw[k] = uint32_t(sig[2 * k]) | (uint32_t(sig[2 * k + 1]) << 16);
        });
        if constexpr (S::NG == 2) {
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
    }
  }
  if constexpr (S::CODES_TMA) {
    if (lane == 0) bulk_wait<0>();
  }
}

// ---------------------------------------------------------------------------
// Dequantiser
// ---------------------------------------------------------------------------

template <int D, int BITS, int G, int ROT, int WPC, int NST, int NOUT>
__global__ void __launch_bounds__(WPC * 32)
    dequantize_kernel(const __grid_constant__ CUtensorMap tm_codes,
                      const __grid_constant__ CUtensorMap tm_xhat, const DequantArgs a) {
  using S = Shape<D, BITS, G>;
  using Lay = WarpLayout<D, BITS, G, NST, NOUT, false>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* ws = smem + warp * Lay::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ws + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(ws + Lay::kTableOff);
  uint32_t* mask = reinterpret_cast<uint32_t*>(ws + Lay::kMaskOff);

  const int total = a.g.total_tiles;
  const int nw = gridDim.x * WPC;
  const int first = blockIdx.x * WPC + warp;
  if (first >= total) return;

  if (lane == 0) {
    if constexpr (S::CODES_TMA) prefetch_tensormap(&tm_codes);
    prefetch_tensormap(&tm_xhat);
    for (int s = 0; s < NST; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto issue = [&](int t, int st) {
    const TileCoord c = decode_tile(t, a.g);
    uint8_t* sb = ws + st * Lay::kStageBytes;
    mbar_arrive_expect_tx(&bars[st], Lay::kStageTx);
    if constexpr (S::CODES_TMA) {
#pragma unroll
      for (int p = 0; p < S::C_PIECES; ++p)
        tma_load_4d(sb + p * (S::TR * S::C_SPAN), &tm_codes, &bars[st], p * S::C_SPAN, c.h, c.r0,
                    c.s);
    }
    const size_t row = static_cast<size_t>(c.s) * a.g.heads + c.h;
    bulk_load(sb + Lay::kLamOff, a.lambda + row * D, 4 * D, &bars[st]);
    bulk_load(sb + Lay::kSgnOff, a.signs + row * D, D, &bars[st]);
  };

  if (lane == 0) {
    for (int k = 0; k < NST; ++k) {
      const int t = first + k * nw;
      if (t < total) issue(t, k);
    }
  }

  int it = 0;
  for (int t = first; t < total; t += nw, ++it) {
    const int st = it % NST;
    const uint32_t parity = (it / NST) & 1;
    const TileCoord c = decode_tile(t, a.g);
    uint8_t* sb = ws + st * Lay::kStageBytes;
    const int row = c.r0 + lane;
    const bool valid = row < a.g.n_rows;
    const size_t vec = (static_cast<size_t>(c.s) * a.in_slice_stride_rows + row) * a.g.heads + c.h;

    // scales for this lane's vector (plain loads; rows past N read as zero)
    uint32_t sw[(S::NG + 1) / 2];
    if (valid) {
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
      static_for<0, (S::NG + 1) / 2>([&](auto k_) { sw[decltype(k_)::value] = 0u; });
    }
    uint32_t words[S::CW];
    if constexpr (!S::CODES_TMA) {
      if (valid) {
        const uint2 u = *reinterpret_cast<const uint2*>(a.codes + vec * S::CB);
        words[0] = u.x;
        words[1] = u.y;
      } else {
        words[0] = words[1] = 0u;
      }
    }

    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], parity));
    if (!ok) {
      if (lane == 0) {
        atomicOr(a.guard, kGuardWaitTimeout);
        for (int k = 1; k < NST; ++k) {
          const int tk = t + k * nw;
          if (tk < total) (void)mbar_wait_bounded(&bars[(it + k) % NST], ((it + k) / NST) & 1);
        }
        bulk_wait<0>();
      }
      __syncwarp();
      return;
    }

    // (a) tables: multiplier gain_j * lambda_j and sign masks
    const float* lam_raw = reinterpret_cast<const float*>(sb + Lay::kLamOff);
    const int8_t* sgn_raw = reinterpret_cast<const int8_t*>(sb + Lay::kSgnOff);
    __syncwarp();
    for (int j = lane; j < D; j += 32) mult[j] = gain_f<ROT, D>(j) * lam_raw[j];
    build_masks<D>(sgn_raw, mask, lane);
    __syncwarp();

    // (b) codes of this lane's vector
    if constexpr (S::CODES_TMA) {
      static_for<0, S::CB / 16>([&](auto c_) {
        constexpr int ci = decltype(c_)::value;
        constexpr int piece = (ci * 16) / S::C_SPAN;
        constexpr int cc = ((ci * 16) % S::C_SPAN) / 16;
        const uint32_t off =
            piece * (S::TR * S::C_SPAN) + swizzle<S::C_SPAN>(lane * S::C_SPAN + cc * 16);
        const uint4 u = *reinterpret_cast<const uint4*>(sb + off);
        words[4 * ci] = u.x;
        words[4 * ci + 1] = u.y;
        words[4 * ci + 2] = u.z;
        words[4 * ci + 3] = u.w;
      });
    }
    __syncwarp();
    if (lane == 0) {
      const int tn = t + NST * nw;
      if (tn < total) issue(tn, st);
    }

    // (c) yhat_j = q_j * sigma_g * lambda_j * gain_j
    float v[D];
    static_for<0, S::NG>([&](auto g_) {
      constexpr int g = decltype(g_)::value;
      const uint32_t sbits = (sw[g / 2] >> (16 * (g & 1))) & 0xFFFFu;
      const float sg = __half2float(__ushort_as_half(static_cast<unsigned short>(sbits)));
      static_for<0, G>([&](auto j_) {
        constexpr int j = g * G + decltype(j_)::value;
        float q;
        if constexpr (BITS == 4) {
          const uint32_t nib = (words[j / 8] >> (4 * (j % 8))) & 0xFu;
          q = __uint_as_float(0x4B400000u | (nib ^ 0x8u)) - (kMagic0 + 8.0f);
        } else {
          const uint32_t byte = (words[j / 4] >> (8 * (j % 4))) & 0xFFu;
          q = __uint_as_float(0x4B400000u | (byte ^ 0x80u)) - (kMagic0 + 128.0f);
        }
        v[j] = q * (sg * mult[j]);
      });
    });

    // (d) inverse rotation
    rotate_inverse_raw<ROT, D>(v);

    // (e) signs + fp16, swizzled staging, TMA store
    uint8_t* ob = ws + Lay::kOutOff + (it % NOUT) * Lay::kOutBytes;
    if (lane == 0) bulk_wait_read<NOUT - 1>();
    __syncwarp();
    static_for<0, D / 8>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      constexpr int piece = (ci * 16) / S::X_SPAN;
      constexpr int cc = ((ci * 16) % S::X_SPAN) / 16;
      const uint4 m = *reinterpret_cast<const uint4*>(mask + 4 * ci);
      uint4 o;
      o.x = half2_as_u32(__floats2half2_rn(v[8 * ci + 0], v[8 * ci + 1])) ^ m.x;
      o.y = half2_as_u32(__floats2half2_rn(v[8 * ci + 2], v[8 * ci + 3])) ^ m.y;
      o.z = half2_as_u32(__floats2half2_rn(v[8 * ci + 4], v[8 * ci + 5])) ^ m.z;
      o.w = half2_as_u32(__floats2half2_rn(v[8 * ci + 6], v[8 * ci + 7])) ^ m.w;
      const uint32_t off =
          piece * (S::TR * S::X_SPAN) + swizzle<S::X_SPAN>(lane * S::X_SPAN + cc * 16);
      *reinterpret_cast<uint4*>(ob + off) = o;
    });
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int p = 0; p < S::X_PIECES; ++p)
        tma_store_4d(&tm_xhat, ob + p * (S::TR * S::X_SPAN), p * (S::X_SPAN / 2), c.h, c.r0, c.s);
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait<0>();
}

}  // namespace srftq
