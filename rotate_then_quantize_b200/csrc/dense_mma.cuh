// Tensor-core quantiser of the dense-rotation codec (tcgen05, TMA, tensor
// memory): y = R x for 128 vectors at a time as one fp16 product with a
// float32 accumulator, then the codec's lambda rescale, group absmax, fp16
// scale, rounding and packing ("When Quantization Is Free", Methodology 2,
// step 4-5; Methodology 3, Householder rotations: R = H(v_1)...H(v_k) B).
//
// The operand of R is split into fp16 halves R = hi + lo (dense.cuh), and x
// is exact in fp16, so Y = X hi^T + X lo^T: two chains of MMAs into the same
// float32 accumulator give y to about 2^-22 of R's magnitude, summed over d
// products per coordinate.
//
// A *block* is 128 consecutive rows of one (slice, head): the MMA's M = 128
// rows are 128 vectors, N = d outputs, K = d inputs (16 per instruction).
// CTA c (one per SM) serves head c % H, and the CTAs of one head split that
// head's (slice, row block) sequence into contiguous ranges: the operand
// changes only at slice boundaries, and the CTAs of all H heads walk the same
// rows at about the same time, so every row of H heads that a DRAM page holds
// is read while the page is open (one block reads only its head's d elements
// of each row).
//
// Warp roles (128 + 128 E threads, E = 2):
//   warp 0      A producer: TMA loads of x tiles (128-byte swizzled K-major
//               rows, rows past N zero-filled): whole 128-row blocks in NST
//               stages for d <= 128, 64-wide K pieces through a ring of
//               NST piece slots for d = 256
//   warp 1      tensor-memory allocation and the MMA issue (one lane)
//   warp 2      B producer: TMA loads of the operand. d <= 128: the whole
//               operand (hi and lo) stays resident and is reloaded when the
//               (slice, head) changes, after the MMAs that read the old one
//               have completed. d = 256 (256 KB of operand): streamed from
//               L2 in chunks of one 64-wide K piece of hi or lo, through a
//               ring of five slots, in the order the MMAs read them (piece
//               by piece, hi then lo).
//   warp 3      idle
//   warps 4..   epilogue, E groups of four warps; group g takes the blocks
//               g, g + E, ... of the range; warp 4 + 4g + q reads TMEM lanes
//               32q .. 32q + 31 (rows of the block), 64 columns at a time,
//               with its own copy of the 1 / lambda row (no barrier across
//               warps), and stores codes and scales from registers.
// Every wait is bounded. A wait that gives up raises the guard word and a
// shared abort flag that ends every role's loop; the roles drain what they
// have in flight (boundedly) before tensor memory is released.
#pragma once

#include "codec.cuh"
#include "tc.cuh"

namespace srftq {

template <int D, int EPI>
struct DenseMma {
  static constexpr bool kStreamB = D > 128;
  static constexpr int kPieces = D / 64;                    // 128-byte K pieces
  static constexpr int kAPiece = 128 * 128;                 // 128 rows x 128 B
  static constexpr int kABytes = kPieces * kAPiece;         // one A stage
  // A stages: whole blocks (d <= 128), or single K pieces of a block when
  // the operand is streamed (d = 256), which leaves room for a deeper ring
  static constexpr int kNST = kStreamB ? 3 : (D == 128 ? 3 : 4);
  static constexpr int kAStage = kStreamB ? kAPiece : kABytes;
  static constexpr int kBPiece = D * 128;                   // d rows x 128 B
  static constexpr int kBChunks = 2 * kPieces;              // (part, piece) chunks
  static constexpr int kBSlots = kStreamB ? 5 : kBChunks;
  static constexpr int kBBytes = kBSlots * kBPiece;
  static constexpr int kAcc = D == 256 ? 2 : 4;             // TMEM accumulators
  static constexpr uint32_t kTmemCols = kAcc * D <= 256 ? 256u : 512u;
  static constexpr int kEpi = EPI;
  static constexpr int kThreads = 128 + 128 * EPI;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kNST * kAStage;
  static constexpr int kTabOff = kBOff + kBBytes;           // 1 / lambda, per epilogue warp
  static constexpr int kBarOff = kTabOff + 4 * EPI * D * 4;
  // full, empty per A stage; bfull, bempty per B slot; tfull, tempty per
  // accumulator; the MMA role's final drain
  static constexpr int kNumBars = 2 * kNST + 2 * kBSlots + 2 * kAcc + 1;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;   // TMEM base, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr uint32_t kIdesc = f16_idesc<128, D>();
  static constexpr int kMmaPerBlock = 2 * D / 16;
  static_assert(kBytes + kSmemSlack <= 227 * 1024, "shared memory");
  static_assert((kBOff % 1024) == 0 && (kBPiece % 1024) == 0, "swizzled tiles");
};

struct DenseMmaArgs {
  int64_t n_rows, row_blocks, n_slices;
  int32_t heads;
  uint8_t* codes;         // [S][T_out][H][d*bits/8]
  uint16_t* scales;       // [S][T_out][H][d/G]
  int64_t out_stride_rows;
  const float* lambda;    // [S][H][d]
  unsigned* guard;
};

// Codes of 64 coordinates from float-encoded integers (low byte of each
// qb = the code in two's complement): int4 8 words, int8 16 words.
template <int BITS>
__device__ __forceinline__ void pack64(const uint32_t (&qb)[64], uint32_t (&words)[BITS * 2]) {
  if constexpr (BITS == 4) {
    static_for<0, 8>([&](auto m_) {
      constexpr int m = decltype(m_)::value;
      const uint32_t ev = __byte_perm(__byte_perm(qb[8 * m + 0], qb[8 * m + 2], 0x0040),
                                      __byte_perm(qb[8 * m + 4], qb[8 * m + 6], 0x0040), 0x5410);
      const uint32_t od = __byte_perm(__byte_perm(qb[8 * m + 1], qb[8 * m + 3], 0x0040),
                                      __byte_perm(qb[8 * m + 5], qb[8 * m + 7], 0x0040), 0x5410);
      words[m] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
    });
  } else {
    static_for<0, 16>([&](auto m_) {
      constexpr int m = decltype(m_)::value;
      words[m] = __byte_perm(__byte_perm(qb[4 * m], qb[4 * m + 1], 0x0040),
                             __byte_perm(qb[4 * m + 2], qb[4 * m + 3], 0x0040), 0x5410);
    });
  }
}

// 64 columns c0 .. c0 + 63 of this thread's TMEM lane, times 1 / lambda.
__device__ __forceinline__ void load_w64(uint32_t taddr, const float* rl, float2 (&v)[32]) {
  uint32_t r0[32], r1[32];
  tmem_ld32(taddr, r0);
  tmem_ld32(taddr + 32u, r1);
  tmem_wait_ld(r0, r1);
  static_for<0, 16>([&](auto i_) {
    constexpr int i = decltype(i_)::value;
    const float2 m0 = *reinterpret_cast<const float2*>(rl + 2 * i);
    const float2 m1 = *reinterpret_cast<const float2*>(rl + 32 + 2 * i);
    v[i] = mul2(make_float2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1])), m0);
    v[16 + i] = mul2(make_float2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1])),
                     m1);
  });
}

template <int D, int BITS, int G, int EPI>
__global__ void __launch_bounds__(DenseMma<D, EPI>::kThreads, 1)
    quantize_dense_mma_kernel(const __grid_constant__ CUtensorMap tm_x,
                              const __grid_constant__ CUtensorMap tm_op, const DenseMmaArgs a) {
  using L = DenseMma<D, EPI>;
  constexpr int QMAX = (1 << (BITS - 1)) - 1;
  constexpr int CB = D * BITS / 8, NG = D / G;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + L::kNST;
  uint64_t* bfull = bars + 2 * L::kNST;
  uint64_t* bempty = bfull + L::kBSlots;
  uint64_t* tfull = bempty + L::kBSlots;
  uint64_t* tempty = tfull + L::kAcc;
  uint64_t* drain = tempty + L::kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  // this CTA's head and contiguous range of (slice, row block) steps
  const int hh = int(blockIdx.x % a.heads);
  const int64_t j = blockIdx.x / a.heads, per_head = gridDim.x / a.heads;
  const int64_t T = a.n_slices * a.row_blocks;
  const int64_t per = T / per_head, rem = T % per_head;
  const int64_t u0 = j * per + (j < rem ? j : rem);
  const int n = int(per + (j < rem ? 1 : 0));
  if (n == 0) return;
  const BlockWalk w0(u0, a.row_blocks, a.heads, hh);

  if (tid == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_op);
    for (int i = 0; i < L::kNST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < L::kBSlots; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 1);
    }
    for (int i = 0; i < L::kAcc; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);   // the four warps of one epilogue group
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  uint8_t* As = smem + L::kAOff;
  uint8_t* Bs = smem + L::kBOff;

  if (warp == 0) {
    // ---------------- A producer ----------------
    if (lane == 0) {
      // stage u = block u (whole blocks) or piece u of the CTA's sequence
      int u = 0;
      bool ok = true;
      BlockWalk w = w0;
      for (int i = 0; i < n && ok; ++i, w.next()) {
        const int r0 = int(w.rb * 128);
        const int s = int(w.s), h = hh;
        const bool in = dbg_ok(s < a.n_slices && r0 < a.n_rows, a.guard);
        for (int p0 = 0; p0 < L::kPieces; p0 += L::kStreamB ? 1 : L::kPieces) {
          const int st = u % L::kNST;
          if (u >= L::kNST &&
              !wait_or_abort(&empty[st], ((u / L::kNST) & 1) ^ 1, abort_flag, a.guard)) {
            ok = false;
            break;
          }
          ++u;
          if (!in) {
            mbar_arrive(&full[st]);   // debug build: no copy, the phase completes empty
            continue;
          }
          mbar_arrive_expect_tx(&full[st], L::kAStage);
          if constexpr (L::kStreamB) {
            tma_load_4d(As + st * L::kAStage, &tm_x, &full[st], 64 * p0, h, r0, s);
          } else {
#pragma unroll
            for (int p = 0; p < L::kPieces; ++p)
              tma_load_4d(As + st * L::kAStage + p * L::kAPiece, &tm_x, &full[st], 64 * p, h,
                          r0, s);
          }
        }
      }
      // drain: every issued stage lands before the CTA can exit
      for (int k = (u > L::kNST ? u - L::kNST : 0); k < u; ++k)
        (void)mbar_wait_bounded(&full[k % L::kNST], (k / L::kNST) & 1);
    }
  } else if (warp == 2) {
    // ---------------- B producer ----------------
    if (lane == 0) {
      if constexpr (!L::kStreamB) {
        int run = -1;
        int64_t prev = -1;
        BlockWalk w = w0;
        for (int i = 0; i < n; ++i, w.next()) {
          const int64_t sh = w.sh();
          if (sh == prev) continue;
          if (run >= 0 && !wait_or_abort(&bempty[0], run & 1, abort_flag, a.guard)) break;
          ++run;
          prev = sh;
          mbar_arrive_expect_tx(&bfull[0], L::kBChunks * L::kBPiece);
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int p = 0; p < L::kPieces; ++p)
              tma_load_4d(Bs + (q * L::kPieces + p) * L::kBPiece, &tm_op, &bfull[0], 64 * p,
                          int((sh * 2 + q) * D), 0, 0);
        }
        if (run >= 0) (void)mbar_wait_bounded(&bfull[0], run & 1);
      } else {
        int c = 0;
        bool ok = true;
        BlockWalk w = w0;
        for (int i = 0; i < n && ok; ++i, w.next()) {
          const int64_t sh = w.sh();
          for (int p = 0; p < L::kPieces && ok; ++p)
            for (int q = 0; q < 2; ++q) {
              const int slot = c % L::kBSlots;
              if (c >= L::kBSlots &&
                  !wait_or_abort(&bempty[slot], ((c / L::kBSlots) & 1) ^ 1, abort_flag,
                                 a.guard)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&bfull[slot], L::kBPiece);
              tma_load_4d(Bs + slot * L::kBPiece, &tm_op, &bfull[slot], 64 * p,
                          int((sh * 2 + q) * D), 0, 0);
              ++c;
            }
        }
        for (int k = (c > L::kBSlots ? c - L::kBSlots : 0); k < c; ++k)
          (void)mbar_wait_bounded(&bfull[k % L::kBSlots], (k / L::kBSlots) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int run = -1, c = 0, i = 0, u = 0;
      int64_t prev = -1;
      bool ok = true;
      BlockWalk w = w0;
      for (; i < n && ok; ++i, w.next()) {
        const int acc = i % L::kAcc;
        const int64_t sh = w.sh();
        if (i >= L::kAcc &&
            !wait_or_abort(&tempty[acc], ((i / L::kAcc) & 1) ^ 1, abort_flag, a.guard))
          break;
        const uint32_t d = tmem_base + uint32_t(acc) * uint32_t(D);
        if constexpr (L::kStreamB) {
          // piece by piece: A piece p with the hi and lo chunks of piece p
          int k = 0;
          for (int p = 0; p < L::kPieces && ok; ++p) {
            const int st = u % L::kNST;
            if (!wait_or_abort(&full[st], (u / L::kNST) & 1, abort_flag, a.guard)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_addr(As + st * L::kAStage);
            for (int q = 0; q < 2; ++q) {
              const int slot = c % L::kBSlots;
              if (!wait_or_abort(&bfull[slot], (c / L::kBSlots) & 1, abort_flag, a.guard)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t sb = smem_addr(Bs + slot * L::kBPiece);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                tc_mma_f16(d, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), L::kIdesc,
                           k > 0 ? 1u : 0u);
                ++k;
              }
              tc_commit(&bempty[slot]);
              ++c;
            }
            if (!ok) break;
            tc_commit(&empty[st]);
            ++u;
          }
          if (!ok) break;
          tc_commit(&tfull[acc]);
          continue;
        }
        const int st = i % L::kNST;
        if (!wait_or_abort(&full[st], (i / L::kNST) & 1, abort_flag, a.guard)) break;
        if constexpr (!L::kStreamB) {
          if (sh != prev) {
            ++run;
            prev = sh;
            if (!wait_or_abort(&bfull[0], run & 1, abort_flag, a.guard)) break;
          }
        }
        tc_fence_after();
        const uint32_t sa = smem_addr(As + st * L::kAStage);
        int k = 0;
        for (int q = 0; q < 2; ++q)
          for (int p = 0; p < L::kPieces; ++p) {
            const uint32_t sb = smem_addr(Bs + (q * L::kPieces + p) * L::kBPiece);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t ad = sw128_desc(sa + p * L::kAPiece + 32 * j);
              const uint64_t bd = sw128_desc(sb + 32 * j);
              tc_mma_f16(d, ad, bd, L::kIdesc, k > 0 ? 1u : 0u);
              ++k;
            }
          }
        tc_commit(&empty[st]);
        tc_commit(&tfull[acc]);
        if (i + 1 == n || w.last_of_slice()) tc_commit(&bempty[0]);
      }
      // drain: every MMA issued (a block cut short by an abort included)
      // completes before TMEM is freed
      tc_commit(drain);
      (void)mbar_wait_bounded(drain, 0);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue ----------------
    const int grp = (warp - 4) >> 2;
    const int q = warp & 3;             // TMEM lane quarter
    // this warp's own 1 / lambda table (no barrier across warps)
    float* rl = reinterpret_cast<float*>(smem + L::kTabOff) + (warp - 4) * D;
    int64_t tab_sh = -1;
    BlockWalk w = w0;
    for (int k = 0; k < grp; ++k) w.next();
    for (int i = grp; i < n; i += L::kEpi) {
      const int acc = i % L::kAcc;
      const int64_t sh = w.sh();
      if (sh != tab_sh) {
        __syncwarp();   // every lane is done reading the old table
        for (int j = lane; j < D; j += 32) rl[j] = __frcp_rn(a.lambda[sh * D + j]);
        __syncwarp();
        tab_sh = sh;
      }
      // warp-uniform outcome: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, wait_or_abort(&tfull[acc], (i / L::kAcc) & 1, abort_flag,
                                                 a.guard)))
        break;
      tc_fence_after();
      const int64_t row = int64_t(w.rb) * 128 + 32 * q + lane;
      const int64_t s = w.s, h = hh;
      for (int k = 0; k < L::kEpi; ++k) w.next();   // this group's next block
      const size_t vec = size_t((s * a.out_stride_rows + row) * a.heads + h);
      const bool valid =
          row < a.n_rows &&
          dbg_ok(int64_t(vec) < vec_limit(a.n_slices, a.out_stride_rows, a.n_rows, a.heads),
                 a.guard);
      const uint32_t taddr = tmem_base + (uint32_t(32 * q) << 16) + uint32_t(acc) * uint32_t(D);
      if constexpr (G <= 64) {
        // every group lies inside one 64-column chunk
        using SP = Shape<64, BITS, G>;
        static_for<0, D / 64>([&](auto c_) {
          constexpr int cc = decltype(c_)::value;
          float2 v[32];
          load_w64(taddr + uint32_t(64 * cc), rl + 64 * cc, v);
          if constexpr (cc == D / 64 - 1) {
            tc_fence_before();   // this warp is done with the accumulator
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
          }
          uint32_t sw[SP::SW];
          uint32_t words[SP::CW];
          quantize_codes<64, BITS, G>(v, sw, words);
          if (valid) {
            uint4* cdst = reinterpret_cast<uint4*>(a.codes + vec * CB + cc * SP::CB);
            static_for<0, SP::CB / 16>([&](auto k_) {
              constexpr int k = decltype(k_)::value;
              cdst[k] = make_uint4(words[4 * k], words[4 * k + 1], words[4 * k + 2],
                                   words[4 * k + 3]);
            });
            uint16_t* dst = a.scales + vec * NG + cc * SP::NG;
            if constexpr (SP::NG == 1) {
              dst[0] = static_cast<uint16_t>(sw[0]);
            } else if constexpr (SP::NG == 2) {
              *reinterpret_cast<uint32_t*>(dst) = sw[0];
            } else if constexpr (SP::NG == 4) {
              *reinterpret_cast<uint2*>(dst) = make_uint2(sw[0], sw[1]);
            } else {
              *reinterpret_cast<uint4*>(dst) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
            }
          }
        });
      } else {
        // groups of 128 or 256 coordinates: absmax over the chunks first,
        // then the codes from a second read of the accumulator
        float am[NG];
        static_for<0, NG>([&](auto g_) { am[decltype(g_)::value] = 0.0f; });
        static_for<0, D / 64>([&](auto c_) {
          constexpr int cc = decltype(c_)::value;
          float2 v[32];
          load_w64(taddr + uint32_t(64 * cc), rl + 64 * cc, v);
          float m = 0.0f;
          static_for<0, 32>([&](auto p_) {
            constexpr int p = decltype(p_)::value;
            m = absmax3(m, v[p].x, v[p].y);
          });
          am[(64 * cc) / G] = fmaxf(am[(64 * cc) / G], m);
        });
        float inv[NG];
        uint16_t sg16[NG];
        static_for<0, NG>([&](auto g_) {
          constexpr int g = decltype(g_)::value;
          const float sf = fminf(div_by_const<QMAX>(am[g]), 65504.0f);
          const __half hs = __float2half_rn(sf);
          sg16[g] = __half_as_ushort(hs);
          const float sg = __half2float(hs);
          inv[g] = sg > 0.0f ? rcp_approx(sg) : 0.0f;
        });
        static_for<0, D / 64>([&](auto c_) {
          constexpr int cc = decltype(c_)::value;
          float2 v[32];
          load_w64(taddr + uint32_t(64 * cc), rl + 64 * cc, v);
          if constexpr (cc == D / 64 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
          }
          const float iv = inv[(64 * cc) / G];
          uint32_t qb[64];
          static_for<0, 32>([&](auto p_) {
            constexpr int p = decltype(p_)::value;
            const float q0 = fminf(fmaxf(v[p].x * iv, -float(QMAX)), float(QMAX));
            const float q1 = fminf(fmaxf(v[p].y * iv, -float(QMAX)), float(QMAX));
            qb[2 * p] = __float_as_uint(q0 + kMagic);
            qb[2 * p + 1] = __float_as_uint(q1 + kMagic);
          });
          uint32_t words[BITS * 2];
          pack64<BITS>(qb, words);
          if (valid) {
            uint4* cdst = reinterpret_cast<uint4*>(a.codes + vec * CB + cc * (8 * BITS));
            static_for<0, BITS / 2>([&](auto k_) {
              constexpr int k = decltype(k_)::value;
              cdst[k] = make_uint4(words[4 * k], words[4 * k + 1], words[4 * k + 2],
                                   words[4 * k + 3]);
            });
          }
        });
        if (valid) {
          if constexpr (NG == 2)
            *reinterpret_cast<uint32_t*>(a.scales + vec * NG) =
                uint32_t(sg16[0]) | (uint32_t(sg16[1]) << 16);
          else
            a.scales[vec * NG] = sg16[0];
        }
      }
    }
  }

  // Every role has finished (or aborted and drained): free tensor memory.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace srftq
