// Tensor-core dequantiser of the dense-rotation codec (tcgen05, TMA, tensor
// memory): xhat = R^T (lambda * sigma * q) for 128 vectors at a time, rounded
// to fp16 ("When Quantization Is Free", Methodology 2, step 6, with the
// Householder rotation of Methodology 3).
//
// The contraction runs over the rotated coordinate j:
//     xhat_i = sum_j R[j][i] a_j,    a_j = lambda_j sigma_g(j) q_j.
// MMA shape: M = 128 vectors, N = d outputs i, K = d coordinates j (16 per
// instruction). B[n = i][k = j] = R[j][i]: the operand matrix read MN-major
// (i is the contiguous index of R's rows), so the quantiser's operand buffer
// (R = hi + lo, fp16) serves unchanged.
//
// Precision. a_j is not exact in fp16 (q has up to 7 bits, sigma 11, lambda
// 24), so A is split like B: a = a_hi + a_lo, a_hi = fp16(a), a_lo =
// fp16(a - a_hi) (the residual a - a_hi is exact in float32). The product
// sums a_hi hi + a_lo hi + a_hi lo into one float32 accumulator; the dropped
// a_lo lo term is below 2^-24 of |a R|.
// Range. Each row (vector) is scaled by an exact power of two 2^-e before the
// split, so that |a_j 2^-e| < 2^15 stays inside fp16's normal range whatever
// the data's magnitude: e comes from the row's largest |sigma| and the
// (slice, head)'s largest |lambda|, and the epilogue multiplies the
// accumulator row by 2^e. The producers and the epilogue compute e with the
// same float32 operations.
//
// A *block* is 128 consecutive rows of one (slice, head); CTAs walk blocks as
// in the quantiser (CTA c serves head c % H, contiguous (slice, row block)
// ranges).
//
// Warp roles (512 threads):
//   warp 0      B producer: TMA loads of the operand in chunks of 64 rows of R
//               (64 values of j) x d columns, as boxes of 64 x 64 fp16 with
//               the 128-byte swizzle. d <= 128: the whole operand (hi and
//               lo) stays resident, reloaded when the (slice, head) changes;
//               d = 256: streamed through a ring of chunk slots in the order
//               the MMAs read them.
//   warp 1      tensor-memory allocation and the MMA issue (one lane)
//   warp 2      codes producer: one TMA load (two for 256-byte rows) of the
//               block's 128 x d*bits/8 code bytes per stage, swizzled
//   warp 3      idle
//   warps 4-11  A producers: warp 4 + w serves rows 32 (w % 4) .. + 31 and
//               half w / 4 of every 64-wide K piece; it turns codes, scales
//               and lambda into the hi / lo fp16 rows of A in the 128-byte
//               swizzled K-major layout, then hands the piece to the MMA
//   warps 12-15 epilogue: warp 12 + q reads TMEM lanes 32q .. 32q + 31 (rows),
//               scales by 2^e, rounds to fp16 and stores the row
// Every wait is bounded. A wait that gives up raises the guard word and a
// shared abort flag that ends every role's loop; the roles drain what they
// have in flight (boundedly) before tensor memory is released.
#pragma once

#include "codec.cuh"
#include "tc.cuh"

namespace srftq {

template <int D, int BITS>
struct DenseDeq {
  static constexpr int kPieces = D / 64;                // 64-wide K pieces
  static constexpr int kAPiece = 128 * 128;             // 128 rows x 64 fp16
  static constexpr int kASlot = 2 * kAPiece;            // hi, lo
  static constexpr int kASlots = D == 256 ? 2 : (D == 128 && BITS == 8 ? 3 : 4);
  static constexpr bool kStreamB = D > 128;
  static constexpr int kBBox = 64 * 128;                // 64 rows x 64 fp16
  static constexpr int kBChunk = D * 128;               // 64 rows of R x d columns
  static constexpr int kBSlots = kStreamB ? (BITS == 8 ? 2 : 3) : 2 * kPieces;
  static constexpr int kCB = D * BITS / 8;              // code bytes per vector
  static constexpr int kCSpan = kCB < 128 ? kCB : 128;  // bytes per TMA box row
  static constexpr int kCBoxes = kCB / kCSpan;
  static constexpr int kCTile = 128 * kCB;
  static constexpr int kCStages = 2;
  static constexpr int kAcc = D == 256 ? 2 : 4;         // TMEM accumulators
  static constexpr uint32_t kTmemCols = kAcc * D <= 256 ? 256u : 512u;
  static constexpr int kProdWarps = 8;
  static constexpr int kEpiWarp0 = 4 + kProdWarps;
  static constexpr int kThreads = 32 * kEpiWarp0 + 128;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + kASlots * kASlot;
  static constexpr int kCOff = kBOff + kBSlots * kBChunk;
  static constexpr int kBarOff = kCOff + kCStages * kCTile;
  // cfull, cempty per code stage; afull, aempty per A slot; bfull, bempty
  // per B slot; tfull, tempty per accumulator; the MMA role's final drain
  static constexpr int kNumBars = 2 * kCStages + 2 * kASlots + 2 * kBSlots + 2 * kAcc + 1;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;  // TMEM base, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  // kind::f16, float32 accumulator, fp16 A K-major, fp16 B MN-major (bit 16)
  static constexpr uint32_t kIdesc = f16_idesc<128, D>() | (1u << 16);
  static_assert(kBytes + kSmemSlack <= 227 * 1024, "shared memory");
  static_assert(kBOff % 1024 == 0 && kCOff % 1024 == 0 && kCTile % 1024 == 0,
                "swizzled tiles");
};

struct DenseDeqArgs {
  int64_t n_rows, row_blocks, n_slices;
  int32_t heads;
  const uint16_t* scales;  // [S][T_in][H][d/G]
  int64_t in_stride_rows;
  uint16_t* xhat;          // [S][T_out][H][d]
  int64_t out_stride_rows;
  const float* lambda;     // [S][H][d]
  unsigned* guard;
};

// Largest |lambda_j| of one (slice, head) row, on every lane of the warp.
template <int D>
__device__ __forceinline__ float dense_lambda_max(const float* lam, int lane) {
  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < D / 32; ++k) m = fmaxf(m, fabsf(__ldg(lam + lane + 32 * k)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// Largest |sigma| of a vector's NG fp16 scales, as fp16 bits (NaN and
// infinity order above every finite value).
template <int NG>
__device__ __forceinline__ uint32_t dense_sigma_max(const uint32_t (&sw)[(NG + 1) / 2]) {
  uint32_t m = 0u;
#pragma unroll
  for (int k = 0; k < (NG + 1) / 2; ++k) {
    m = max(m, sw[k] & 0x7FFFu);
    if (2 * k + 1 < NG) m = max(m, (sw[k] >> 16) & 0x7FFFu);
  }
  return m;
}

// Row exponent e: QMAX |sigma|max |lambda|max 2^-e lies in [2^14, 2^15) (e
// clamped to [-100, 100], so that 2^e and 2^-e are normal float32 numbers).
template <int QMAX>
__device__ __forceinline__ int dense_row_exponent(uint32_t smax_bits, float lmax) {
  const float bnd = (float(QMAX) * __half2float(__ushort_as_half(uint16_t(smax_bits)))) * lmax;
  const int e = int((__float_as_uint(bnd) >> 23) & 0xFFu) - 127 - 14;
  return min(max(e, -100), 100);
}

__device__ __forceinline__ float exp2_int(int e) {
  return __uint_as_float(uint32_t(127 + e) << 23);
}

// The NG fp16 scales of one vector as packed words (zero for rows past N).
template <int NG>
__device__ __forceinline__ void dense_load_scales(const uint16_t* src, bool valid,
                                                  uint32_t (&sw)[(NG + 1) / 2]) {
  if (!valid) {
#pragma unroll
    for (int k = 0; k < (NG + 1) / 2; ++k) sw[k] = 0u;
    return;
  }
  if constexpr (NG == 1) {
    sw[0] = src[0];
  } else if constexpr (NG == 2) {
    sw[0] = *reinterpret_cast<const uint32_t*>(src);
  } else if constexpr (NG == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    sw[0] = u.x;
    sw[1] = u.y;
  } else {
#pragma unroll
    for (int k = 0; k < NG / 8; ++k) {
      const uint4 u = reinterpret_cast<const uint4*>(src)[k];
      sw[4 * k] = u.x;
      sw[4 * k + 1] = u.y;
      sw[4 * k + 2] = u.z;
      sw[4 * k + 3] = u.w;
    }
  }
}

// Eight codes as exact floats plus the magic 2^23 + 2^(BITS-1): the biased
// code u = q + 2^(BITS-1) (the sign bit flipped) becomes the low mantissa
// byte of 2^23.
template <int BITS>
__device__ __forceinline__ void dense_codes8(const uint32_t* w, float (&f)[8]) {
  if constexpr (BITS == 4) {
    const uint32_t u = w[0] ^ 0x88888888u;
    const uint32_t t0 = u & 0x0F0F0F0Fu;           // codes 0, 2, 4, 6
    const uint32_t t1 = (u >> 4) & 0x0F0F0F0Fu;    // codes 1, 3, 5, 7
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      f[2 * m] = __uint_as_float(__byte_perm(t0, 0x4B000000u, 0x7540u + m));
      f[2 * m + 1] = __uint_as_float(__byte_perm(t1, 0x4B000000u, 0x7540u + m));
    }
  } else {
    const uint32_t u0 = w[0] ^ 0x80808080u, u1 = w[1] ^ 0x80808080u;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      f[m] = __uint_as_float(__byte_perm(u0, 0x4B000000u, 0x7540u + m));
      f[4 + m] = __uint_as_float(__byte_perm(u1, 0x4B000000u, 0x7540u + m));
    }
  }
}

template <int D, int BITS, int G>
__global__ void __launch_bounds__(DenseDeq<D, BITS>::kThreads, 1)
    dequantize_dense_mma_kernel(const __grid_constant__ CUtensorMap tm_c,
                                const __grid_constant__ CUtensorMap tm_op, const DenseDeqArgs a) {
  using L = DenseDeq<D, BITS>;
  constexpr int QMAX = (1 << (BITS - 1)) - 1;
  constexpr int NG = D / G;
  constexpr int SW = (NG + 1) / 2;
  constexpr float kBias = BITS == 4 ? 8388616.0f : 8388736.0f;   // 2^23 + 2^(BITS-1)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* cfull = bars;
  uint64_t* cempty = cfull + L::kCStages;
  uint64_t* afull = cempty + L::kCStages;
  uint64_t* aempty = afull + L::kASlots;
  uint64_t* bfull = aempty + L::kASlots;
  uint64_t* bempty = bfull + L::kBSlots;
  uint64_t* tfull = bempty + L::kBSlots;
  uint64_t* tempty = tfull + L::kAcc;
  uint64_t* drain = tempty + L::kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  // this CTA's head and contiguous range of (slice, row block) steps
  const int hh = int(blockIdx.x % a.heads);
  const int64_t jc = blockIdx.x / a.heads, per_head = gridDim.x / a.heads;
  const int64_t T = a.n_slices * a.row_blocks;
  const int64_t per = T / per_head, rem = T % per_head;
  const int64_t u0 = jc * per + (jc < rem ? jc : rem);
  const int n = int(per + (jc < rem ? 1 : 0));
  if (n == 0) return;
  auto sh_of = [&](int i) -> int64_t { return ((u0 + i) / a.row_blocks) * a.heads + hh; };
  auto rb_of = [&](int i) -> int64_t { return (u0 + i) % a.row_blocks; };

  if (tid == 0) {
    prefetch_tensormap(&tm_c);
    prefetch_tensormap(&tm_op);
    for (int i = 0; i < L::kCStages; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], L::kProdWarps);
    }
    for (int i = 0; i < L::kASlots; ++i) {
      mbar_init(&afull[i], L::kProdWarps);
      mbar_init(&aempty[i], 1);
    }
    for (int i = 0; i < L::kBSlots; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 1);
    }
    for (int i = 0; i < L::kAcc; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);   // the four epilogue warps
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
  uint8_t* Cs = smem + L::kCOff;

  if (warp == 0) {
    // ---------------- B producer ----------------
    // chunk (q, kc): rows 64 kc .. 64 kc + 63 of part q (hi, lo) of R, as
    // d / 64 boxes of 64 columns, box nb at nb * 8 KB
    if (lane == 0) {
      auto load_chunk = [&](uint8_t* dst, uint64_t* bar, int64_t sh, int q, int kc) {
        const int y = int((sh * 2 + q) * D + 64 * kc);
#pragma unroll
        for (int nb = 0; nb < L::kPieces; ++nb)
          tma_load_4d(dst + nb * L::kBBox, &tm_op, bar, 64 * nb, y, 0, 0);
      };
      if constexpr (!L::kStreamB) {
        int run = -1;
        int64_t prev = -1;
        for (int i = 0; i < n; ++i) {
          const int64_t sh = sh_of(i);
          if (sh == prev) continue;
          if (run >= 0 && !wait_or_abort(&bempty[0], run & 1, abort_flag, a.guard)) break;
          ++run;
          prev = sh;
          mbar_arrive_expect_tx(&bfull[0], 2 * L::kPieces * L::kBChunk);
          for (int q = 0; q < 2; ++q)
            for (int kc = 0; kc < L::kPieces; ++kc)
              load_chunk(Bs + (q * L::kPieces + kc) * L::kBChunk, &bfull[0], sh, q, kc);
        }
        if (run >= 0) (void)mbar_wait_bounded(&bfull[0], run & 1);
      } else {
        int c = 0;
        bool ok = true;
        for (int i = 0; i < n && ok; ++i) {
          const int64_t sh = sh_of(i);
          for (int kc = 0; kc < L::kPieces && ok; ++kc)
            for (int q = 0; q < 2; ++q) {
              const int slot = c % L::kBSlots;
              if (c >= L::kBSlots &&
                  !wait_or_abort(&bempty[slot], ((c / L::kBSlots) & 1) ^ 1, abort_flag,
                                 a.guard)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&bfull[slot], L::kBChunk);
              load_chunk(Bs + slot * L::kBChunk, &bfull[slot], sh, q, kc);
              ++c;
            }
        }
        for (int k = (c > L::kBSlots ? c - L::kBSlots : 0); k < c; ++k)
          (void)mbar_wait_bounded(&bfull[k % L::kBSlots], (k / L::kBSlots) & 1);
      }
    }
  } else if (warp == 2) {
    // ---------------- codes producer ----------------
    if (lane == 0) {
      int i = 0;
      for (; i < n; ++i) {
        const int st = i % L::kCStages;
        if (i >= L::kCStages &&
            !wait_or_abort(&cempty[st], ((i / L::kCStages) & 1) ^ 1, abort_flag, a.guard))
          break;
        const int64_t sh = sh_of(i);
        const int r0 = int(rb_of(i) * 128);
        const int s = int(sh / a.heads), h = int(sh % a.heads);
        if (!dbg_ok(s < a.n_slices && r0 < a.n_rows, a.guard)) {
          mbar_arrive(&cfull[st]);   // debug build: no copy, the phase completes empty
          continue;
        }
        mbar_arrive_expect_tx(&cfull[st], L::kCTile);
#pragma unroll
        for (int b = 0; b < L::kCBoxes; ++b)
          tma_load_4d(Cs + st * L::kCTile + b * 128 * L::kCSpan, &tm_c, &cfull[st],
                      b * L::kCSpan, h, r0, s);
      }
      for (int k = (i > L::kCStages ? i - L::kCStages : 0); k < i; ++k)
        (void)mbar_wait_bounded(&cfull[k % L::kCStages], (k / L::kCStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int run = -1, ca = 0, cb = 0;
      int64_t prev = -1;
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        const int acc = i % L::kAcc;
        const int64_t sh = sh_of(i);
        if (i >= L::kAcc &&
            !wait_or_abort(&tempty[acc], ((i / L::kAcc) & 1) ^ 1, abort_flag, a.guard))
          break;
        if constexpr (!L::kStreamB) {
          if (sh != prev) {
            ++run;
            prev = sh;
            if (!wait_or_abort(&bfull[0], run & 1, abort_flag, a.guard)) break;
          }
        }
        const uint32_t dt = tmem_base + uint32_t(acc) * uint32_t(D);
        for (int kc = 0; kc < L::kPieces && ok; ++kc) {
          const int as = ca % L::kASlots;
          if (!wait_or_abort(&afull[as], (ca / L::kASlots) & 1, abort_flag, a.guard)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(As + as * L::kASlot);
          for (int q = 0; q < 2; ++q) {
            uint32_t sb;
            int slot = 0;
            if constexpr (L::kStreamB) {
              slot = cb % L::kBSlots;
              if (!wait_or_abort(&bfull[slot], (cb / L::kBSlots) & 1, abort_flag, a.guard)) {
                ok = false;
                break;
              }
              tc_fence_after();
              sb = smem_addr(Bs + slot * L::kBChunk);
            } else {
              sb = smem_addr(Bs + (q * L::kPieces + kc) * L::kBChunk);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t bd = sw128_mn_desc(sb + 2048u * ks, L::kBBox);
              // a_hi x part q; a_lo x hi
              tc_mma_f16(dt, sw128_desc(sa + 32u * ks), bd, L::kIdesc,
                         (kc | ks | q) != 0 ? 1u : 0u);
              if (q == 0) tc_mma_f16(dt, sw128_desc(sa + L::kAPiece + 32u * ks), bd, L::kIdesc, 1u);
            }
            if constexpr (L::kStreamB) {
              tc_commit(&bempty[slot]);
              ++cb;
            }
          }
          if (!ok) break;
          tc_commit(&aempty[as]);
          ++ca;
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        if constexpr (!L::kStreamB) {
          if (i + 1 == n || sh_of(i + 1) != sh) tc_commit(&bempty[0]);
        }
      }
      // drain: every MMA issued (a block cut short by an abort included)
      // completes before TMEM is freed
      tc_commit(drain);
      (void)mbar_wait_bounded(drain, 0);
    }
  } else if (warp >= 4 && warp < L::kEpiWarp0) {
    // ---------------- A producers ----------------
    const int pw = warp - 4;
    const int r = 32 * (pw & 3) + lane;   // row of the block
    auto produce = [&](auto half_) {
      constexpr int HF = decltype(half_)::value;   // half of each 64-wide piece
      float lmax = 0.0f;
      int64_t lam_sh = -1;
      auto scales_of = [&](int i, uint32_t (&sw)[SW]) {
        const int64_t sh = sh_of(i);
        const int64_t row = rb_of(i) * 128 + r;
        const size_t vec =
            size_t(((sh / a.heads) * a.in_stride_rows + row) * a.heads + sh % a.heads);
        const bool valid =
            row < a.n_rows &&
            dbg_ok(int64_t(vec) < vec_limit(a.n_slices, a.in_stride_rows, a.n_rows, a.heads),
                   a.guard);
        dense_load_scales<NG>(a.scales + vec * NG, valid, sw);
      };
      uint32_t sw_next[SW];
      scales_of(0, sw_next);
      int ca = 0;
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        uint32_t sw[SW];
#pragma unroll
        for (int k = 0; k < SW; ++k) sw[k] = sw_next[k];
        if (i + 1 < n) scales_of(i + 1, sw_next);   // one block ahead
        const int64_t sh = sh_of(i);
        if (sh != lam_sh) {
          lmax = dense_lambda_max<D>(a.lambda + sh * D, lane);
          lam_sh = sh;
        }
        const float down = exp2_int(-dense_row_exponent<QMAX>(dense_sigma_max<NG>(sw), lmax));
        const float* lam = a.lambda + sh * D;
        const int st = i % L::kCStages;
        if (!__all_sync(0xffffffffu, wait_or_abort(&cfull[st], (i / L::kCStages) & 1,
                                                   abort_flag, a.guard))) {
          ok = false;
          break;
        }
        const uint32_t ctile = smem_addr(Cs + st * L::kCTile);
        static_for<0, L::kPieces>([&](auto p_) {
          constexpr int p = decltype(p_)::value;
          if (!ok) return;
          const int as = ca % L::kASlots;
          if (ca >= L::kASlots &&
              !__all_sync(0xffffffffu, wait_or_abort(&aempty[as], ((ca / L::kASlots) & 1) ^ 1,
                                                     abort_flag, a.guard))) {
            ok = false;
            return;
          }
          // this thread's 32 codes: elements 64 p + 32 HF .. + 31 of row r
          constexpr int kOff = (64 * p + 32 * HF) * BITS / 8;    // byte offset in the row
          constexpr int kBox = kOff / L::kCSpan;
          constexpr int kChunk = (kOff % L::kCSpan) / 16;
          const uint32_t rowa =
              swz_row<L::kCSpan>(ctile + uint32_t(kBox * 128 * L::kCSpan), uint32_t(r));
          uint32_t cw[BITS];
          {
            const uint4 v = lds128(swz_chunk<L::kCSpan>(rowa, kChunk));
            cw[0] = v.x;
            cw[1] = v.y;
            cw[2] = v.z;
            cw[3] = v.w;
          }
          if constexpr (BITS == 8) {
            const uint4 v = lds128(swz_chunk<L::kCSpan>(rowa, kChunk + 1));
            cw[4] = v.x;
            cw[5] = v.y;
            cw[6] = v.z;
            cw[7] = v.w;
          }
          const uint32_t arow = smem_addr(As + as * L::kASlot) + uint32_t(r) * 128u;
          static_for<0, 4>([&](auto k_) {
            constexpr int k = decltype(k_)::value;
            constexpr int j0 = 64 * p + 32 * HF + 8 * k;   // first coordinate
            constexpr int g = j0 / G;
            const float sg =
                __half2float(__ushort_as_half(uint16_t(sw[g / 2] >> (16 * (g % 2))))) * down;
            const float4 l0 = __ldg(reinterpret_cast<const float4*>(lam + j0));
            const float4 l1 = __ldg(reinterpret_cast<const float4*>(lam + j0 + 4));
            const float lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
            float f[8];
            dense_codes8<BITS>(cw + k * (BITS / 4), f);
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float2 qv = add2(make_float2(f[2 * m], f[2 * m + 1]), splat(-kBias));
              const float2 sv = mul2(splat(sg), make_float2(lv[2 * m], lv[2 * m + 1]));
              const float2 x = mul2(qv, sv);
              const __half2 hi = __floats2half2_rn(x.x, x.y);
              const float2 hf = __half22float2(hi);
              const __half2 lo = __floats2half2_rn(x.x - hf.x, x.y - hf.y);
              hw[m] = *reinterpret_cast<const uint32_t*>(&hi);
              lw[m] = *reinterpret_cast<const uint32_t*>(&lo);
            }
            const uint32_t pos = uint32_t(((4 * HF + k) ^ (r & 7)) << 4);
            sts128(arow + pos, make_uint4(hw[0], hw[1], hw[2], hw[3]));
            sts128(arow + uint32_t(L::kAPiece) + pos, make_uint4(lw[0], lw[1], lw[2], lw[3]));
          });
          fence_proxy_async_smem();   // generic writes -> the MMA's async-proxy reads
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[as]);
          ++ca;
        });
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[st]);   // this warp is done with the codes
      }
    };
    if (pw < 4)
      produce(Int<0>{});
    else
      produce(Int<1>{});
  } else if (warp >= L::kEpiWarp0) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;   // TMEM lane quarter
    float lmax = 0.0f;
    int64_t lam_sh = -1;
    for (int i = 0; i < n; ++i) {
      const int acc = i % L::kAcc;
      const int64_t sh = sh_of(i);
      if (sh != lam_sh) {
        lmax = dense_lambda_max<D>(a.lambda + sh * D, lane);
        lam_sh = sh;
      }
      const int64_t row = rb_of(i) * 128 + 32 * q + lane;
      const int64_t s = sh / a.heads, h = sh % a.heads;
      const size_t vin = size_t((s * a.in_stride_rows + row) * a.heads + h);
      const bool in_ok =
          row < a.n_rows &&
          dbg_ok(int64_t(vin) < vec_limit(a.n_slices, a.in_stride_rows, a.n_rows, a.heads),
                 a.guard);
      uint32_t sw[SW];
      dense_load_scales<NG>(a.scales + vin * NG, in_ok, sw);
      const float up = exp2_int(dense_row_exponent<QMAX>(dense_sigma_max<NG>(sw), lmax));
      // warp-uniform outcome: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, wait_or_abort(&tfull[acc], (i / L::kAcc) & 1, abort_flag,
                                                 a.guard)))
        break;
      tc_fence_after();
      const size_t vout = size_t((s * a.out_stride_rows + row) * a.heads + h);
      const bool valid =
          row < a.n_rows &&
          dbg_ok(int64_t(vout) < vec_limit(a.n_slices, a.out_stride_rows, a.n_rows, a.heads),
                 a.guard);
      const uint32_t taddr = tmem_base + (uint32_t(32 * q) << 16) + uint32_t(acc) * uint32_t(D);
      static_for<0, D / 64>([&](auto c_) {
        constexpr int cc = decltype(c_)::value;
        uint32_t r0[32], r1[32];
        tmem_ld32(taddr + uint32_t(64 * cc), r0);
        tmem_ld32(taddr + uint32_t(64 * cc + 32), r1);
        tmem_wait_ld(r0, r1);
        if constexpr (cc == D / 64 - 1) {
          tc_fence_before();   // this warp is done with the accumulator
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        uint32_t w[32];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float2 v0 = mul2(
              make_float2(__uint_as_float(r0[2 * m]), __uint_as_float(r0[2 * m + 1])), splat(up));
          const float2 v1 = mul2(
              make_float2(__uint_as_float(r1[2 * m]), __uint_as_float(r1[2 * m + 1])), splat(up));
          const __half2 h0 = __floats2half2_rn(v0.x, v0.y);
          const __half2 h1 = __floats2half2_rn(v1.x, v1.y);
          w[m] = *reinterpret_cast<const uint32_t*>(&h0);
          w[16 + m] = *reinterpret_cast<const uint32_t*>(&h1);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(a.xhat + vout * D + 64 * cc);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      });
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
