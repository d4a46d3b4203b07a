// Fused quantise / dequantise kernels for d = 256 (two threads per vector).
//
// Same pipeline as codec.cuh (persistent warps, head-uniform tiles, TMA
// stages with deferred store/refill issue), with 16 vectors per warp tile:
// lanes 2r and 2r + 1 share row r. Each lane holds 128 of the vector's 256
// coordinates in its 64 slots (transform256.cuh gives the slot -> coordinate
// map), quantises the groups those coordinates form (group sizes 8..64 keep
// every group inside one lane), and writes its own code chunks and scales.
#pragma once

#include "aux.cuh"
#include "codec.cuh"
#include "transform256.cuh"

namespace srftq {

constexpr int kTileRows256 = 16;

template <int BITS, int G>
struct Shape256 {
  static_assert(G >= 8 && G <= 64 && (G & (G - 1)) == 0, "group (d = 256)");
  static_assert(BITS == 4 || BITS == 8, "bits");
  static constexpr int D = 256;
  static constexpr int TR = kTileRows256;
  static constexpr int XB = 512, X_SPAN = 128, X_PIECES = 4, X_TILE = TR * XB;
  static constexpr int CB = D * BITS / 8;              // 128 or 256 bytes / vector
  static constexpr int C_SPAN = 128, C_PIECES = CB / 128, C_TILE = TR * CB;
  static constexpr int CBL = CB / 2;                   // code bytes per lane
  static constexpr int KL = CBL / 16;                  // code chunks per lane
  static constexpr int CWL = CBL / 4;                  // code words per lane
  static constexpr int NG = D / G, NGL = 128 / G;      // groups per vector / lane
  static constexpr int SW = NG / 2;                    // scale words per vector
  static constexpr int QMAX = (1 << (BITS - 1)) - 1;
};

template <int BITS, int G, int NST, bool QUANT>
struct WarpLayout256 {
  using S = Shape256<BITS, G>;
  static constexpr int kInTile = QUANT ? S::X_TILE : S::C_TILE;
  static constexpr int kInBytes = align_up(kInTile, 1024);
  static constexpr int kOutTile = QUANT ? S::C_TILE : S::X_TILE;
  static constexpr int kOutBytes = align_up(kOutTile, 1024);
  static constexpr int kOutOff = NST * kInBytes;
  static constexpr int kRowBytes = 4 * 256 + 256;
  static constexpr int kRowsOff = kOutOff + kOutBytes;
  static constexpr int kStageTx = kInTile + kRowBytes;
  static constexpr int kTableOff = kRowsOff + NST * kRowBytes;   // 256 floats
  static constexpr int kSignTabOff = kTableOff + 4 * 256;        // up to 192 words
  static constexpr int kBarOff = align_up(kSignTabOff + 4 * 192, 16);
  static constexpr int kWarpBytes = align_up(kBarOff + 8 * NST, 1024);
};

// Global code chunk of this lane's chunk k (K chunks per lane).
template <int ROT, int K>
__device__ __forceinline__ int code_chunk256(int k, bool p) {
  if constexpr (ROT == kSRHT) {
    return p ? K + k : k;
  } else {
    return p ? K / 2 + k : (k < K / 2 ? k : k + K);
  }
}

// Global group of this lane's local group lg (groups of G coordinates).
template <int ROT, int G>
__host__ __device__ constexpr int group256(int lg, int p) {
  return 2 * pair256<ROT>(lg * (G / 2), p) / G;
}

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

__device__ __forceinline__ TileCoord decode_tile256(int t, const TileGeom& g) {
  const int h = t % g.heads;
  const int q = t / g.heads;
  const int rb = q % g.row_blocks;
  return {q / g.row_blocks, rb * kTileRows256, h};
}

// ---------------------------------------------------------------------------
// Quantiser, d = 256
// ---------------------------------------------------------------------------

template <int BITS, int G, int ROT, int WPC, int NST, int MINB>
__global__ void __launch_bounds__(WPC * 32, MINB)
    quantize256_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_codes, const QuantArgs a) {
  using S = Shape256<BITS, G>;
  using Lay = WarpLayout256<BITS, G, NST, true>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 1;
  const bool p = lane & 1;
  uint8_t* ws = smem + warp * Lay::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ws + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(ws + Lay::kTableOff);
  uint32_t* stab = reinterpret_cast<uint32_t*>(ws + Lay::kSignTabOff);
  uint8_t* ob = ws + Lay::kOutOff;

  const int total = a.g.total_tiles;
  const int nw = gridDim.x * WPC;
  const int first = blockIdx.x * WPC + warp;
  if (first >= total) return;

  if (lane == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_codes);
    for (int s = 0; s < NST; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto issue = [&](int t, int st) {
    const TileCoord c = decode_tile256(t, a.g);
    uint8_t* sb = ws + st * Lay::kInBytes;
    uint8_t* rb = ws + Lay::kRowsOff + st * Lay::kRowBytes;
    mbar_arrive_expect_tx(&bars[st], Lay::kStageTx);
#pragma unroll
    for (int pc = 0; pc < S::X_PIECES; ++pc)
      tma_load_4d(sb + pc * (S::TR * S::X_SPAN), &tm_x, &bars[st], pc * 64, c.h, c.r0, c.s);
    const size_t row = static_cast<size_t>(c.s) * a.g.heads + c.h;
    bulk_load(rb, a.lambda + row * 256, 4 * 256, &bars[st]);
    bulk_load(rb + 4 * 256, a.signs + row * 256, 256, &bars[st]);
  };
  auto store_codes = [&](const TileCoord& c) {
#pragma unroll
    for (int pc = 0; pc < S::C_PIECES; ++pc)
      tma_store_4d(&tm_codes, ob + pc * (S::TR * S::C_SPAN), pc * S::C_SPAN, c.h, c.r0, c.s);
    bulk_commit();
  };

  if (lane == 0) {
    for (int k = 0; k < NST; ++k) {
      const int t = first + k * nw;
      if (t < total) issue(t, k);
    }
  }

  int it = 0;
  int table_sh = -1;
  bool pending = false;
  TileCoord prev{0, 0, 0};
  for (int t = first; t < total; t += nw, ++it) {
    const int st = it % NST;
    const uint32_t parity = (it / NST) & 1;
    const TileCoord c = decode_tile256(t, a.g);
    const uint8_t* sb = ws + st * Lay::kInBytes;
    const uint8_t* rb = ws + Lay::kRowsOff + st * Lay::kRowBytes;

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
    __syncwarp();
    if (lane == 0) {
      if (pending) store_codes(prev);
      const int tn = t + (NST - 1) * nw;
      if (it > 0 && tn < total) issue(tn, (it - 1) % NST);
    }
    pending = false;

    // (a) tables: mult[256] = per-lane-half multipliers in slot order, sign words
    const int sh = c.s * a.g.heads + c.h;
    if (sh != table_sh) {
      const float* lam_raw = reinterpret_cast<const float*>(rb);
      const int8_t* sgn_raw = reinterpret_cast<const int8_t*>(rb + 4 * 256);
      for (int e = lane; e < 256; e += 32) {
        const int hp = e >> 7, sl = e & 127;          // half, slot coordinate
        const int pair = pair256<ROT>(sl >> 1, hp);
        mult[e] = gain256<ROT>(pair) * rcp_approx(lam_raw[2 * pair + (sl & 1)]);
      }
      if constexpr (ROT == kSRFT) {
        for (int w = lane; w < 128; w += 32) {       // [half][m]: (s_{4m+p}, s_{4m+2+p})
          const int hp = w >> 6, m = w & 63;
          stab[w] = sign_halves(sgn_raw[4 * m + hp], sgn_raw[4 * m + 2 + hp]);
        }
      } else {
        for (int w = lane; w < 192; w += 32) {       // lo[64], hi+[64], hi-[64]
          const int part = w >> 6, m = w & 63;
          const int base = part == 0 ? 2 * m : 128 + 2 * m;
          const uint32_t sgw = sign_halves(sgn_raw[base], sgn_raw[base + 1]);
          stab[w] = part == 2 ? (sgw ^ 0x80008000u) : sgw;
        }
      }
      __syncwarp();
      table_sh = sh;
    }

    // (b)+(c) this lane's half of the vector, transform, multipliers
    float2 v[64];
    auto chunk = [&](int ci) -> uint4 {
      const uint32_t off = (ci >> 3) * (S::TR * S::X_SPAN) + swizzle<128>(r * 128 + (ci & 7) * 16);
      return *reinterpret_cast<const uint4*>(sb + off);
    };
    if constexpr (ROT == kSRFT) {
      uint32_t xw[64], sgw[64];
      const uint32_t selp = p ? 0x7632u : 0x5410u;
      static_for<0, 32>([&](auto c_) {
        constexpr int ci = decltype(c_)::value;
        const uint4 w = chunk(ci);
        xw[2 * ci] = __byte_perm(w.x, w.y, selp);
        xw[2 * ci + 1] = __byte_perm(w.z, w.w, selp);
      });
      static_for<0, 16>([&](auto c_) {
        constexpr int ci = decltype(c_)::value;
        const uint4 sg = reinterpret_cast<const uint4*>(stab + (p ? 64 : 0))[ci];
        sgw[4 * ci] = sg.x;
        sgw[4 * ci + 1] = sg.y;
        sgw[4 * ci + 2] = sg.z;
        sgw[4 * ci + 3] = sg.w;
      });
      srft256_forward(xw, sgw, p, v);
    } else {
      static_for<0, 16>([&](auto c_) {
        constexpr int ci = decltype(c_)::value;
        const uint4 wl = chunk(ci), wh = chunk(16 + ci);
        const uint4 sl = reinterpret_cast<const uint4*>(stab)[ci];
        const uint4 sh4 = reinterpret_cast<const uint4*>(stab + (p ? 128 : 64))[ci];
        v[4 * ci] = srht256_plane0(wl.x, wh.x, sl.x, sh4.x);
        v[4 * ci + 1] = srht256_plane0(wl.y, wh.y, sl.y, sh4.y);
        v[4 * ci + 2] = srht256_plane0(wl.z, wh.z, sl.z, sh4.z);
        v[4 * ci + 3] = srht256_plane0(wl.w, wh.w, sl.w, sh4.w);
      });
      wht_packed_planes<128>(v);
    }
    const float* mh = mult + (p ? 128 : 0);
    static_for<0, 32>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = reinterpret_cast<const float4*>(mh)[ci];
      v[2 * ci] = mul2(v[2 * ci], make_float2(m4.x, m4.y));
      v[2 * ci + 1] = mul2(v[2 * ci + 1], make_float2(m4.z, m4.w));
    });

    // (d) local groups -> scales -> codes (as in codec.cuh)
    uint16_t sig[S::NGL];
    float invs[S::NGL];
    bool clamp = false;
    static_for<0, S::NGL>([&](auto g_) {
      constexpr int g = decltype(g_)::value;
      float amax = 0.0f;
      static_for<0, G / 2>([&](auto q_) {
        constexpr int q = g * G / 2 + decltype(q_)::value;
        amax = absmax3(amax, v[q].x, v[q].y);
      });
      const float sf = div_by_const<S::QMAX>(amax);
      const __half hs = __float2half_rn(fminf(sf, 65504.0f));
      sig[g] = __half_as_ushort(hs);
      const float sg = __half2float(hs);
      invs[g] = sg > 0.0f ? rcp_approx(sg) : 0.0f;
      clamp |= sg > 0.0f && !(sg >= 6.103515625e-05f && sf <= 65504.0f);
    });
    uint32_t qb[128];
    if (!clamp) {
      static_for<0, 64>([&](auto q_) {
        constexpr int q = decltype(q_)::value;
        const float2 rr = fma2(v[q], splat(invs[(2 * q) / G]), splat(kMagic));
        qb[2 * q] = __float_as_uint(rr.x);
        qb[2 * q + 1] = __float_as_uint(rr.y);
      });
    } else {
      static_for<0, 64>([&](auto q_) {
        constexpr int q = decltype(q_)::value;
        const float inv = invs[(2 * q) / G];
        const float q0 = fminf(fmaxf(v[q].x * inv, -float(S::QMAX)), float(S::QMAX));
        const float q1 = fminf(fmaxf(v[q].y * inv, -float(S::QMAX)), float(S::QMAX));
        qb[2 * q] = __float_as_uint(q0 + kMagic);
        qb[2 * q + 1] = __float_as_uint(q1 + kMagic);
      });
    }
    uint32_t words[S::CWL];
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

    // (f) codes into the staging tile at this lane's chunks
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
    static_for<0, S::KL>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      const int cg = code_chunk256<ROT, S::KL>(k, p);      // global chunk in the row
      const uint32_t off =
          (cg >> 3) * (S::TR * S::C_SPAN) + swizzle<128>(r * 128 + (cg & 7) * 16);
      *reinterpret_cast<uint4*>(ob + off) =
          make_uint4(words[4 * k], words[4 * k + 1], words[4 * k + 2], words[4 * k + 3]);
    });
    fence_proxy_async_smem();
    pending = true;
    prev = c;

    // (g) this lane's scales
    const int row = c.r0 + r;
    if (row < a.g.n_rows) {
      uint16_t* dst = a.scales +
          ((static_cast<size_t>(c.s) * a.out_slice_stride_rows + row) * a.g.heads + c.h) * S::NG;
      static_for<0, S::NGL>([&](auto g_) {
        constexpr int g = decltype(g_)::value;
        dst[p ? group256<ROT, G>(g, 1) : group256<ROT, G>(g, 0)] = sig[g];
      });
    }
  }
  __syncwarp();
  if (lane == 0) {
    if (pending) store_codes(prev);
    bulk_wait<0>();
  }
}

// ---------------------------------------------------------------------------
// Dequantiser, d = 256
// ---------------------------------------------------------------------------

template <int BITS, int G, int ROT, int WPC, int NST, int MINB>
__global__ void __launch_bounds__(WPC * 32, MINB)
    dequantize256_kernel(const __grid_constant__ CUtensorMap tm_codes,
                         const __grid_constant__ CUtensorMap tm_xhat, const DequantArgs a) {
  using S = Shape256<BITS, G>;
  using Lay = WarpLayout256<BITS, G, NST, false>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 1;
  const bool p = lane & 1;
  uint8_t* ws = smem + warp * Lay::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ws + Lay::kBarOff);
  float* mult = reinterpret_cast<float*>(ws + Lay::kTableOff);
  uint32_t* mtab = reinterpret_cast<uint32_t*>(ws + Lay::kSignTabOff);
  uint8_t* ob = ws + Lay::kOutOff;

  const int total = a.g.total_tiles;
  const int nw = gridDim.x * WPC;
  const int first = blockIdx.x * WPC + warp;
  if (first >= total) return;

  if (lane == 0) {
    prefetch_tensormap(&tm_codes);
    prefetch_tensormap(&tm_xhat);
    for (int s = 0; s < NST; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto issue = [&](int t, int st) {
    const TileCoord c = decode_tile256(t, a.g);
    uint8_t* sb = ws + st * Lay::kInBytes;
    uint8_t* rb = ws + Lay::kRowsOff + st * Lay::kRowBytes;
    mbar_arrive_expect_tx(&bars[st], Lay::kStageTx);
#pragma unroll
    for (int pc = 0; pc < S::C_PIECES; ++pc)
      tma_load_4d(sb + pc * (S::TR * S::C_SPAN), &tm_codes, &bars[st], pc * S::C_SPAN, c.h, c.r0,
                  c.s);
    const size_t row = static_cast<size_t>(c.s) * a.g.heads + c.h;
    bulk_load(rb, a.lambda + row * 256, 4 * 256, &bars[st]);
    bulk_load(rb + 4 * 256, a.signs + row * 256, 256, &bars[st]);
  };
  auto store_xhat = [&](const TileCoord& c) {
#pragma unroll
    for (int pc = 0; pc < S::X_PIECES; ++pc)
      tma_store_4d(&tm_xhat, ob + pc * (S::TR * S::X_SPAN), pc * 64, c.h, c.r0, c.s);
    bulk_commit();
  };

  if (lane == 0) {
    for (int k = 0; k < NST; ++k) {
      const int t = first + k * nw;
      if (t < total) issue(t, k);
    }
  }

  auto load_scales = [&](int t, uint32_t (&sw)[S::SW]) {
    const TileCoord c = decode_tile256(t, a.g);
    const int row = c.r0 + r;
    if (row < a.g.n_rows) {
      const uint16_t* src = a.scales +
          ((static_cast<size_t>(c.s) * a.in_slice_stride_rows + row) * a.g.heads + c.h) * S::NG;
      if constexpr (S::SW == 2) {
        const uint2 u = *reinterpret_cast<const uint2*>(src);
        sw[0] = u.x;
        sw[1] = u.y;
      } else {
        static_for<0, S::SW / 4>([&](auto k_) {
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
  load_scales(first, sw_next);

  int it = 0;
  int table_sh = -1;
  bool pending = false;
  TileCoord prev{0, 0, 0};
  for (int t = first; t < total; t += nw, ++it) {
    const int st = it % NST;
    const uint32_t parity = (it / NST) & 1;
    const TileCoord c = decode_tile256(t, a.g);
    const uint8_t* sb = ws + st * Lay::kInBytes;
    const uint8_t* rb = ws + Lay::kRowsOff + st * Lay::kRowBytes;

    uint32_t sw[S::SW];
    static_for<0, S::SW>([&](auto k_) { sw[decltype(k_)::value] = sw_next[decltype(k_)::value]; });
    if (t + nw < total) load_scales(t + nw, sw_next);

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
    __syncwarp();
    if (lane == 0) {
      if (pending) store_xhat(prev);
      const int tn = t + (NST - 1) * nw;
      if (it > 0 && tn < total) issue(tn, (it - 1) % NST);
    }
    pending = false;

    // (a) tables: mult[256] (per-lane-half, slot order; int4 odd slots /16)
    // and the row's 128 output sign masks
    const int sh = c.s * a.g.heads + c.h;
    if (sh != table_sh) {
      const float* lam_raw = reinterpret_cast<const float*>(rb);
      const int8_t* sgn_raw = reinterpret_cast<const int8_t*>(rb + 4 * 256);
      for (int e = lane; e < 256; e += 32) {
        const int hp = e >> 7, sl = e & 127;
        const int pair = pair256<ROT>(sl >> 1, hp);
        mult[e] = igain256<ROT>(pair) * lam_raw[2 * pair + (sl & 1)] *
                  ((BITS == 4 && (sl & 1)) ? 0.0625f : 1.0f);
      }
      for (int w = lane; w < 128; w += 32) mtab[w] = sign_mask(sgn_raw[2 * w], sgn_raw[2 * w + 1]);
      __syncwarp();
      table_sh = sh;
    }

    // (b) this lane's code chunks
    uint32_t words[S::CWL];
    static_for<0, S::KL>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      const int cg = code_chunk256<ROT, S::KL>(k, p);
      const uint32_t off =
          (cg >> 3) * (S::TR * S::C_SPAN) + swizzle<128>(r * 128 + (cg & 7) * 16);
      const uint4 u = *reinterpret_cast<const uint4*>(sb + off);
      words[4 * k] = u.x;
      words[4 * k + 1] = u.y;
      words[4 * k + 2] = u.z;
      words[4 * k + 3] = u.w;
    });

    // (c) this lane's scales (fp16 pairs in words; local group g -> global)
    uint32_t lsw[(S::NGL + 1) / 2];
    static_for<0, (S::NGL + 1) / 2>([&](auto w_) {
      constexpr int w = decltype(w_)::value;
      auto half_of = [&](int gg) -> uint32_t { return (sw[gg >> 1] >> (16 * (gg & 1))) & 0xFFFFu; };
      constexpr int a0 = group256<ROT, G>(2 * w, 0), b0 = group256<ROT, G>(2 * w, 1);
      uint32_t lo = p ? half_of(b0) : half_of(a0);
      uint32_t hi = 0;
      if constexpr (2 * w + 1 < S::NGL) {
        constexpr int a1 = group256<ROT, G>(2 * w + 1, 0), b1 = group256<ROT, G>(2 * w + 1, 1);
        hi = p ? half_of(b1) : half_of(a1);
      }
      lsw[w] = lo | (hi << 16);
    });
    float2 v[64];
    constexpr int CPW = 32 / BITS;
    static_for<0, S::CWL>([&](auto m_) {
      constexpr int m = decltype(m_)::value;
      constexpr int g = (m * CPW) / G;
      const float sgf = __half2float(__ushort_as_half(
          static_cast<unsigned short>((lsw[g / 2] >> (16 * (g & 1))) & 0xFFFFu)));
      const float c_even = BITS == 4 ? -1032.0f * sgf : -1152.0f * sgf;
      const float c_odd = -1152.0f * sgf;
      unpack_word<BITS, g & 1>(words[m], lsw[g / 2], c_even, c_odd, &v[m * CPW / 2]);
    });
    const float* mh = mult + (p ? 128 : 0);
    static_for<0, 32>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 m4 = reinterpret_cast<const float4*>(mh)[ci];
      v[2 * ci] = mul2(v[2 * ci], make_float2(m4.x, m4.y));
      v[2 * ci + 1] = mul2(v[2 * ci + 1], make_float2(m4.z, m4.w));
    });

    // (d)+(e) inverse rotation, this lane's 64 fp16 output words, staging
    uint32_t outw[64];
    if constexpr (ROT == kSRFT) {
      float2 us[64];
      srft256_inverse(v, p, us);
      // lane 0 writes words 0..63 = (u_even[n], u_odd[n]), lane 1 words 64..127
      static_for<0, 32>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        const float2 recv = shfl1(sel2(p, us[k], us[32 + k]));
        const float2 own = sel2(p, us[32 + k], us[k]);
        const float2 ev = sel2(p, recv, own), od = sel2(p, own, recv);
        outw[2 * k] = pack_f16x2(ev.x, od.x);
        outw[2 * k + 1] = pack_f16x2(ev.y, od.y);
      });
    } else {
      float2 lo[32], hi[32];
      srht256_inverse(v, p, lo, hi);
      static_for<0, 32>([&](auto k_) {
        constexpr int k = decltype(k_)::value;
        outw[k] = pack_f16x2(lo[k].x, lo[k].y);
        outw[32 + k] = pack_f16x2(hi[k].x, hi[k].y);
      });
    }
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
    static_for<0, 16>([&](auto k_) {
      constexpr int k = decltype(k_)::value;
      // global fp16 chunk (8 halves) of this lane's chunk k
      int cg;
      if constexpr (ROT == kSRFT) {
        cg = (p ? 16 : 0) + k;
      } else {
        cg = (k < 8 ? 0 : 8) + (p ? 8 : 0) + k;
      }
      const uint4 mk = reinterpret_cast<const uint4*>(mtab)[cg];
      const uint4 o = make_uint4(outw[4 * k] ^ mk.x, outw[4 * k + 1] ^ mk.y,
                                 outw[4 * k + 2] ^ mk.z, outw[4 * k + 3] ^ mk.w);
      const uint32_t off =
          (cg >> 3) * (S::TR * S::X_SPAN) + swizzle<128>(r * 128 + (cg & 7) * 16);
      *reinterpret_cast<uint4*>(ob + off) = o;
    });
    fence_proxy_async_smem();
    pending = true;
    prev = c;
  }
  __syncwarp();
  if (lane == 0) {
    if (pending) store_xhat(prev);
    bulk_wait<0>();
  }
}

// ---------------------------------------------------------------------------
// Rotation and calibration, d = 256 (plain loads; two threads per vector)
// ---------------------------------------------------------------------------

// Transform of vector xv (fp16, signs sgn) by lane half p; out slots as above.
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
    const uint16_t* xv = a.x + ((s * a.x_slice_stride_rows + rr) * a.heads + h) * 256;
    const int64_t tab = (s * a.heads + h) * 256;
    float2 v[64];
    rotate256_lane<ROT>(xv, a.signs + tab, p, v);
    if (valid) {
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

// One block per (slice, head): 64 rows per batch, two threads per row.
template <int ROT>
__global__ void __launch_bounds__(128) calibrate256_kernel(const CalibArgs a) {
  __shared__ float sq[kCalibRows / 2][257];
  const int s = blockIdx.x / a.heads;
  const int h = blockIdx.x % a.heads;
  const int64_t tab = (int64_t(s) * a.heads + h) * 256;
  const bool p = threadIdx.x & 1;
  const int rl = threadIdx.x >> 1;   // row within a batch of 64 (two threads per row)
  double acc0 = 0.0, acc1 = 0.0;
  for (int64_t b = 0; b < a.n_cal; b += 64) {
    const int64_t rr = b + rl;
    const bool valid = rr < a.n_cal;
    const int64_t rc = valid ? rr : 0;
    const uint16_t* xv = a.x + ((int64_t(s) * a.x_slice_stride_rows + rc) * a.heads + h) * 256;
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
  a.lambda_out[tab + threadIdx.x] =
      acc0 > 0.0 ? float(sqrt(acc0 / double(a.n_cal))) : 1.0f;
  a.lambda_out[tab + threadIdx.x + 128] =
      acc1 > 0.0 ? float(sqrt(acc1 / double(a.n_cal))) : 1.0f;
}

}  // namespace srftq
