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
// 24), so A is split like B: a = a_hi + a_lo, a_hi = a with its low 13
// mantissa bits cleared (exact in fp16 inside its normal range), a_lo =
// fp16(a - a_hi) (the residual is exact in float32; |a_lo| < 2^-10 |a|).
// The product sums a_hi hi + a_lo hi + a_hi lo into one float32
// accumulator; the dropped a_lo lo term is below 2^-22 of |a R|. (The split
// by truncation costs two float-to-half conversions per pair of values
// instead of four for a rounded one.)
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
// Warp roles (768 threads):
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
//   warps 4-19  A producers: warp 4 + w serves rows 32 (w % 4) .. + 31 and
//               the 16 coordinates 16 (w / 4) .. + 15 of every 64-wide K
//               piece; it turns codes, scales and lambda (its columns'
//               values, kept in its own shared-memory table) into the hi / lo
//               fp16 rows of A in the 128-byte swizzled K-major layout, then
//               hands the piece to the MMA (sixteen warps, so that four per
//               scheduler hide each other's latency)
//   warps 20-23 epilogue: warp 20 + q reads TMEM lanes 32q .. 32q + 31 (rows),
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
  static constexpr int kParts = 4;                      // column parts of a piece
  static constexpr int kEW = 64 / kParts;               // coordinates per thread per piece
  static constexpr int kSub = kEW / 8;                  // 16-byte A chunks per thread
  static constexpr int kCW = kEW * BITS / 32;           // code words per thread per piece
  static constexpr int kProdWarps = 4 * kParts;
  static constexpr int kEpiWarp0 = 4 + kProdWarps;
  static constexpr int kThreads = 32 * kEpiWarp0 + 128;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + kASlots * kASlot;
  static constexpr int kCOff = kBOff + kBSlots * kBChunk;
  static constexpr int kLamOff = kCOff + kCStages * kCTile;   // lambda, per producer warp
  static constexpr int kLamWarp = kPieces * kEW;              // floats per producer warp
  static constexpr int kBarOff = kLamOff + kProdWarps * kLamWarp * 4;
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
  const BlockWalk w0(u0, a.row_blocks, a.heads, hh);

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
        BlockWalk w = w0;
        for (int i = 0; i < n; ++i, w.next()) {
          const int64_t sh = w.sh();
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
        BlockWalk w = w0;
        for (int i = 0; i < n && ok; ++i, w.next()) {
          const int64_t sh = w.sh();
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
      BlockWalk w = w0;
      for (; i < n; ++i, w.next()) {
        const int st = i % L::kCStages;
        if (i >= L::kCStages &&
            !wait_or_abort(&cempty[st], ((i / L::kCStages) & 1) ^ 1, abort_flag, a.guard))
          break;
        const int r0 = int(w.rb * 128);
        const int s = int(w.s), h = hh;
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
      BlockWalk w = w0;
      for (int i = 0; i < n && ok; ++i, w.next()) {
        const int acc = i % L::kAcc;
        const int64_t sh = w.sh();
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
          if (i + 1 == n || w.last_of_slice()) tc_commit(&bempty[0]);
        }
      }
      // drain: every MMA issued (a block cut short by an abort included)
      // completes before TMEM is freed
      tc_commit(drain);
      (void)mbar_wait_bounded(drain, 0);
    }
  } else if (warp >= 4 && warp < L::kEpiWarp0) {
    // ---------------- A producers ----------------
    constexpr int EW = L::kEW, SUB = L::kSub, CW = L::kCW;
    const int pw = warp - 4;
    const int r = 32 * (pw & 3) + lane;   // row of the block
    const int part = pw >> 2;             // coordinates EW part .. + EW - 1 of each piece
    // lambda_j of this warp's columns: ltab[EW p + c] = lambda[64 p + EW part + c]
    float* ltab = reinterpret_cast<float*>(smem + L::kLamOff) + pw * L::kLamWarp;
    float lmax = 0.0f;
    int64_t lam_sh = -1;
    auto scales_of = [&](const BlockWalk& ww, uint32_t (&sw)[SW]) {
      const int64_t row = int64_t(ww.rb) * 128 + r;
      const size_t vec = size_t((ww.s * a.in_stride_rows + row) * a.heads + hh);
      const bool valid =
          row < a.n_rows &&
          dbg_ok(int64_t(vec) < vec_limit(a.n_slices, a.in_stride_rows, a.n_rows, a.heads),
                 a.guard);
      dense_load_scales<NG>(a.scales + vec * NG, valid, sw);
    };
    BlockWalk w = w0, wn = w0;
    uint32_t sw_next[SW];
    scales_of(wn, sw_next);
    wn.next();
    int ca = 0;
    bool ok = true;
    for (int i = 0; i < n && ok; ++i, w.next()) {
      uint32_t sw[SW];
#pragma unroll
      for (int k = 0; k < SW; ++k) sw[k] = sw_next[k];
      if (i + 1 < n) {   // one block ahead
        scales_of(wn, sw_next);
        wn.next();
      }
      const int64_t sh = w.sh();
      if (sh != lam_sh) {
        lmax = dense_lambda_max<D>(a.lambda + sh * D, lane);
        __syncwarp();   // every lane is done reading the old table
        for (int t = lane; t < L::kLamWarp; t += 32)
          ltab[t] = __ldg(a.lambda + sh * D + 64 * (t / EW) + EW * part + t % EW);
        __syncwarp();
        lam_sh = sh;
      }
      const float down = exp2_int(-dense_row_exponent<QMAX>(dense_sigma_max<NG>(sw), lmax));
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
        // this thread's EW codes: coordinates 64 p + EW part .. of row r.
        // All loads first, then the arithmetic, then the stores (the stores
        // are ordered asm, so a load placed after one could not move ahead).
        const int off = (64 * p + EW * part) * BITS / 8;   // byte offset in the row
        const uint32_t rowa = swz_row<L::kCSpan>(
            ctile + uint32_t((off / L::kCSpan) * 128 * L::kCSpan), uint32_t(r));
        const uint32_t caddr =
            swz_chunk<L::kCSpan>(rowa, uint32_t((off % L::kCSpan) / 16)) + uint32_t(off % 16);
        uint32_t cw[CW];
        if constexpr (CW == 2) {
          const uint2 v = lds64(caddr);
          cw[0] = v.x;
          cw[1] = v.y;
        } else {
          static_for<0, CW / 4>([&](auto c_) {
            constexpr int c = decltype(c_)::value;
            const uint4 v = lds128(c == 0 ? caddr : swz_chunk<L::kCSpan>(rowa, uint32_t(
                                                        (off % L::kCSpan) / 16 + c)));
            cw[4 * c] = v.x;
            cw[4 * c + 1] = v.y;
            cw[4 * c + 2] = v.z;
            cw[4 * c + 3] = v.w;
          });
        }
        float2 lv[EW / 2];
        {
          const uint32_t lp = smem_addr(ltab + EW * p);
#pragma unroll
          for (int m = 0; m < EW / 4; ++m) {
            const uint4 t = lds128(lp + 16u * m);
            lv[2 * m] = make_float2(__uint_as_float(t.x), __uint_as_float(t.y));
            lv[2 * m + 1] = make_float2(__uint_as_float(t.z), __uint_as_float(t.w));
          }
        }
        uint32_t hw[EW / 2], lw[EW / 2];
        static_for<0, SUB>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          // sigma 2^-e of the group of this 8-coordinate chunk
          uint32_t hb = 0u;
          static_for<0, L::kParts>([&](auto t_) {
            constexpr int t = decltype(t_)::value;
            constexpr int g = (64 * p + EW * t + 8 * k) / G;
            if (part == t) hb = (sw[g / 2] >> (16 * (g % 2))) & 0xFFFFu;
          });
          const float2 s2 = splat(__half2float(__ushort_as_half(uint16_t(hb))) * down);
          float f[8];
          dense_codes8<BITS>(cw + k * (BITS / 4), f);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float2 x = mul2(add2(make_float2(f[2 * m], f[2 * m + 1]), splat(-kBias)),
                                  mul2(s2, lv[4 * k + m]));
            // a_hi: a with the low 13 mantissa bits cleared (exact in fp16);
            // a_lo: the exact float32 residual, rounded to fp16 once
            const float2 ht = make_float2(__uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u),
                                          __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u));
            const float2 res = add2(x, make_float2(-ht.x, -ht.y));
            const __half2 hi = __floats2half2_rn(ht.x, ht.y);
            const __half2 lo = __floats2half2_rn(res.x, res.y);
            hw[4 * k + m] = *reinterpret_cast<const uint32_t*>(&hi);
            lw[4 * k + m] = *reinterpret_cast<const uint32_t*>(&lo);
          }
        });
        const uint32_t arow = smem_addr(As + as * L::kASlot) + uint32_t(r) * 128u;
        static_for<0, SUB>([&](auto k_) {
          constexpr int k = decltype(k_)::value;
          const uint32_t pos = uint32_t(((SUB * part + k) ^ (r & 7)) << 4);
          sts128(arow + pos, make_uint4(hw[4 * k], hw[4 * k + 1], hw[4 * k + 2], hw[4 * k + 3]));
          sts128(arow + uint32_t(L::kAPiece) + pos,
                 make_uint4(lw[4 * k], lw[4 * k + 1], lw[4 * k + 2], lw[4 * k + 3]));
        });
        fence_proxy_async_smem();   // generic writes -> the MMA's async-proxy reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[as]);
        ++ca;
      });
      __syncwarp();
      if (lane == 0) mbar_arrive(&cempty[st]);   // this warp is done with the codes
    }
  } else if (warp >= L::kEpiWarp0) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;   // TMEM lane quarter
    float lmax = 0.0f;
    int64_t lam_sh = -1;
    auto scales_of = [&](const BlockWalk& ww, uint32_t (&sw)[SW]) {
      const int64_t row = int64_t(ww.rb) * 128 + 32 * q + lane;
      const size_t vin = size_t((ww.s * a.in_stride_rows + row) * a.heads + hh);
      const bool in_ok =
          row < a.n_rows &&
          dbg_ok(int64_t(vin) < vec_limit(a.n_slices, a.in_stride_rows, a.n_rows, a.heads),
                 a.guard);
      dense_load_scales<NG>(a.scales + vin * NG, in_ok, sw);
    };
    BlockWalk w = w0, wn = w0;
    uint32_t sw_next[SW];
    scales_of(wn, sw_next);
    wn.next();
    for (int i = 0; i < n; ++i, w.next()) {
      const int acc = i % L::kAcc;
      const int64_t sh = w.sh();
      if (sh != lam_sh) {
        lmax = dense_lambda_max<D>(a.lambda + sh * D, lane);
        lam_sh = sh;
      }
      const int64_t row = int64_t(w.rb) * 128 + 32 * q + lane;
      const int64_t s = w.s, h = hh;
      uint32_t sw[SW];
#pragma unroll
      for (int k = 0; k < SW; ++k) sw[k] = sw_next[k];
      if (i + 1 < n) {   // one block ahead
        scales_of(wn, sw_next);
        wn.next();
      }
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
      static_for<0, D / 32>([&](auto c_) {
        constexpr int cc = decltype(c_)::value;
        uint32_t r0[32];
        tmem_ld32(taddr + uint32_t(32 * cc), r0);
        tmem_wait_ld1(r0);
        if constexpr (cc == D / 32 - 1) {
          tc_fence_before();   // this warp is done with the accumulator
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        uint32_t wv[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float2 v = mul2(
              make_float2(__uint_as_float(r0[2 * m]), __uint_as_float(r0[2 * m + 1])), splat(up));
          const __half2 h2 = __floats2half2_rn(v.x, v.y);
          wv[m] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(a.xhat + vout * D + 32 * cc);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(wv[4 * k], wv[4 * k + 1], wv[4 * k + 2], wv[4 * k + 3]);
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
