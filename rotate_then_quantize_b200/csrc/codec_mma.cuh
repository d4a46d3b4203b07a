// Tensor-core SRFT quantiser for d = 128 (tcgen05, TMA, tensor memory).
//
// The SRFT of 128 vectors is one dense product. With U the sign-flipped fp16
// inputs (128 vectors x 128 samples, exact in fp16) and B the unnormalised
// packed real-DFT matrix, the raw outputs of transform.cuh's srft_forward are
// RAW = U B^T, where for n = 0..127 and k = 1..63, k != 32 ("When
// Quantization Is Free", Methodology 1; X_k = sum_n u_n e^{-2 pi i k n / 128}):
//   B[0][n] = 1                  raw_0 = X_0
//   B[1][n] = (-1)^n             raw_1 = X_64
//   B[2k][n] = 2 cos(2 pi k n / 128),  B[2k+1][n] = -2 sin(2 pi k n / 128)
//   B[64][n] = cos(pi n / 2),          B[65][n] = sin(pi n / 2)
// (2 Re X_k, 2 Im X_k; Re X_32 and -Im X_32). B is split into fp16 halves,
// B = B_hi + B_lo with B_lo the fp16 rounding of B - B_hi: two chains of MMAs
// (U B_hi^T, then U B_lo^T) accumulate into the same fp32 columns of tensor
// memory, with a relative error of about 2^-22 of the row norm, well inside
// the rotation tolerance. The epilogue then applies the coordinate gain /
// lambda and runs the same group absmax, scales and packing as the
// one-thread kernel (quantize_codes), on halves of 64 coordinates.
//
// Warp roles (EPI_GROUPS x 128 + 128 threads, one CTA per SM; an MMA block is
// 4 consecutive tiles of 32 vectors, 128 rows):
//   warp 0      TMA producer (one elected lane), NST stages of one block
//   warp 1      tensor-memory allocation (512 columns: four accumulators of
//               128 lanes x 128 fp32) and the MMA issue (one lane)
//   warps 2, 3  sign pass: warp 2 + h flips the fp16 sign bits of sub-tiles
//               2h and 2h + 1 in the staged block (u = s x), fenced for the
//               tensor core
//   warps 4..   epilogue, EPI_GROUPS groups of four that take blocks in turn:
//               warp w handles the blocks b with b % EPI_GROUPS == (w - 4) / 4, reads
//               TMEM lanes 32 (w % 4) .. +31 (sub-tile w % 4 of the block),
//               quantises its 32 vectors half by half and stores their codes
//               and scales straight from registers
// Every wait is bounded. A wait that gives up raises the guard word and a
// shared abort flag that ends every role's loop; the roles then drain what
// they have in flight (boundedly) before tensor memory is released.
#pragma once

#include "codec.cuh"

namespace srftq {

// ---------------------------------------------------------------------------
// tcgen05 wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives once on `bar` when every tcgen05 operation this thread issued
// before it has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}
// D[tmem] = A B^T (+ D if accumulate), fp16 operands from shared memory.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane. The values may
// be used only after tmem_wait_ld (which takes them as operands, so that no
// use is scheduled before it).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&a)[32], uint32_t (&b)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]),
        "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]),
        "+r"(a[13]), "+r"(a[14]), "+r"(a[15]), "+r"(a[16]), "+r"(a[17]), "+r"(a[18]),
        "+r"(a[19]), "+r"(a[20]), "+r"(a[21]), "+r"(a[22]), "+r"(a[23]), "+r"(a[24]),
        "+r"(a[25]), "+r"(a[26]), "+r"(a[27]), "+r"(a[28]), "+r"(a[29]), "+r"(a[30]),
        "+r"(a[31]), "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]),
        "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]),
        "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15]), "+r"(b[16]), "+r"(b[17]),
        "+r"(b[18]), "+r"(b[19]), "+r"(b[20]), "+r"(b[21]), "+r"(b[22]), "+r"(b[23]),
        "+r"(b[24]), "+r"(b[25]), "+r"(b[26]), "+r"(b[27]), "+r"(b[28]), "+r"(b[29]),
        "+r"(b[30]), "+r"(b[31])
      :
      : "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored as rows of 128
// bytes (64 fp16) with the 128-byte swizzle, 8-row groups 1024 bytes apart
// (the layout TMA writes for a box 128 bytes wide): start address >> 4 in
// bits 0-13, leading offset 1 (unused by this layout) in bits 16-29, stride
// offset 1024 >> 4 in bits 32-45, descriptor version 1 in bits 46-47, layout
// "128-byte swizzle" (2) in bits 61-63. Successive K steps of 16 elements
// advance the start address by 32 bytes inside the swizzle atom.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), fp16
// A and B (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 in
// bits 17-22, M >> 4 in bits 24-28.
template <int M, int N>
constexpr uint32_t f16_idesc() {
  static_assert(M == 128 && N % 16 == 0 && N >= 16 && N <= 256, "MMA shape");
  return (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------

template <int BITS, int G, int EPI_GROUPS>
struct MmaLayout {
  using S = Shape<128, BITS, G>;
  static constexpr int kSub = 4;                 // tiles of 32 vectors per MMA block
  static constexpr int kNST = 3;                 // input stages
  static constexpr int kSignWarps = 2;
  static constexpr int kEpiWarps = 4 * EPI_GROUPS;
  static constexpr int kAcc = 4;                 // TMEM accumulators of 128 columns
  static constexpr int kAPiece = 128 * 128;      // 128 rows x 64 fp16
  static constexpr int kABytes = 2 * kAPiece;    // one stage: 128 vectors x 256 bytes
  static constexpr int kBPiece = 256 * 128;      // 256 rows x 64 fp16
  static constexpr int kBBytes = 2 * kBPiece;
  static constexpr int kSubA = S::TR * 128;      // one sub-tile inside a piece
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + kNST * kABytes;
  static constexpr int kCOff = kBOff + kBBytes;                      // scratch at start
  static constexpr int kMultStride = 128 + 4;                        // floats per head
  static constexpr int kSignStride = 64 + 4;                         // words per head
  static constexpr int kMultBytes = 4 * kMaxHPT * kMultStride;
  static constexpr int kSignBytes = 4 * kMaxHPT * kSignStride;
  static constexpr int kMultOff = kCOff;
  static constexpr int kSignOff = kMultOff + kEpiWarps * kMultBytes;
  static constexpr int kBarOff = align_up(kSignOff + kSub * kSignBytes, 16);
  // full, signed, empty per stage; tfull, tempty per accumulator
  static constexpr int kNumBars = 3 * kNST + 2 * kAcc;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;            // TMEM base, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdesc = f16_idesc<128, 128>();
  static_assert(kBytes + kSmemSlack <= 227 * 1024, "shared memory");
};

// Builds B_hi (rows 0..127) and B_lo (rows 128..255) in the swizzled K-major
// layout: element (row r, column k) sits in piece k / 64 at row r, 16-byte
// chunk ((k % 64) / 8) XOR (r % 8). cosv[m] = cos(2 pi m / 128) rounded to
// fp32 (sin(2 pi m / 128) = cosv[(m - 32) mod 128]); every entry of B is a
// power of two times one of them, so B is exact to fp32 before the split.
__device__ __forceinline__ void build_dft_operand(uint8_t* bsm, const float* cosv, int tid,
                                                  int nthreads) {
  for (int idx = tid; idx < 256 * 16; idx += nthreads) {
    const int r = idx >> 4, ch = idx & 15;        // row, chunk of 8 columns
    const int p = ch >> 3, c = ch & 7;
    const int j = r & 127, k = j >> 1;
    const bool lo = r >= 128;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float val[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int n = 64 * p + 8 * c + e + t;
        const int m = (k * n) & 127;
        float f;
        if (j == 0)
          f = 1.0f;
        else if (j == 1)
          f = (n & 1) ? -1.0f : 1.0f;
        else if (k == 32)
          f = (j & 1) ? cosv[(m + 96) & 127] : cosv[m];
        else
          f = (j & 1) ? -2.0f * cosv[(m + 96) & 127] : 2.0f * cosv[m];
        const __half h = __float2half_rn(f);
        val[t] = lo ? f - __half2float(h) : __half2float(h);   // f - h is exact
      }
      const __half2 h2 = __floats2half2_rn(val[0], val[1]);
      w[e / 2] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    const uint32_t off = p * (256 * 128) + r * 128 + ((c ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(bsm + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, unsigned* guard) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 63u && *abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(guard, kGuardWaitTimeout);
  return false;
}

template <int BITS, int G, int EPI_GROUPS>
__global__ void __launch_bounds__(128 + 128 * EPI_GROUPS, 1)
    quantize_mma_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_codes, const QuantArgs a) {
  constexpr int D = 128;
  using S = Shape<D, BITS, G>;
  using L = MmaLayout<BITS, G, EPI_GROUPS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* signed_ = bars + L::kNST;
  uint64_t* empty = bars + 2 * L::kNST;
  uint64_t* tfull = bars + 3 * L::kNST;
  uint64_t* tempty = tfull + L::kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  // The CTA's contiguous range of tiles, in blocks of kSub.
  TileWalk first;
  const bool any = first.start(blockIdx.x, gridDim.x, a.g);
  const int n_tiles = any ? first.left : 0;
  const int n_blocks = (n_tiles + L::kSub - 1) / L::kSub;
  if (n_blocks == 0) return;
  const int hpt_log2 = a.g.hpt_log2;
  const int hpt = 1 << hpt_log2;
  const int rpt = kTileRows >> hpt_log2;

  if (tid == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_codes);
    for (int i = 0; i < L::kNST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&signed_[i], L::kSignWarps);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < L::kAcc; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], L::kSub);   // the four warps of one epilogue group
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  {
    // cos(2 pi m / 128) in fp32, staged in the (still unused) codes tiles
    float* cosv = reinterpret_cast<float*>(smem + L::kCOff);
    if (tid < 128) cosv[tid] = static_cast<float>(ct::cos_sin_2pi(tid, 128).c);
    __syncthreads();
    build_dft_operand(smem + L::kBOff, cosv, tid, L::kThreads);
    fence_proxy_async_smem();   // B is read by the tensor core (async proxy)
    __syncthreads();            // the codes tiles are free again
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      TileWalk t = first;
      int b = 0;
      for (; b < n_blocks; ++b) {
        const int st = b % L::kNST;
        if (b >= L::kNST &&
            !wait_or_abort(&empty[st], ((b / L::kNST) & 1) ^ 1, abort_flag, a.guard))
          break;
        const int nsub = min(L::kSub, n_tiles - b * L::kSub);
        uint8_t* sa = smem + L::kAOff + st * L::kABytes;
        mbar_arrive_expect_tx(&full[st], nsub * 2 * L::kSubA);
        for (int q = 0; q < nsub; ++q) {
#pragma unroll
          for (int p = 0; p < 2; ++p)
            tma_load_4d(sa + p * L::kAPiece + q * L::kSubA, &tm_x, &full[st], p * 64,
                        t.hb * hpt, t.rb * rpt, t.s);
          t.advance(a.g);
        }
      }
      // Drain: every issued stage must land before the CTA can exit.
      for (int k = (b > L::kNST ? b - L::kNST : 0); k < b; ++k)
        (void)mbar_wait_bounded(&full[k % L::kNST], (k / L::kNST) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int b = 0;
      for (; b < n_blocks; ++b) {
        const int st = b % L::kNST, acc = b % L::kAcc;
        if (!wait_or_abort(&signed_[st], (b / L::kNST) & 1, abort_flag, a.guard)) break;
        if (b >= L::kAcc &&
            !wait_or_abort(&tempty[acc], ((b / L::kAcc) & 1) ^ 1, abort_flag, a.guard))
          break;
        tc_fence_after();
        const uint32_t sa = smem_addr(smem + L::kAOff + st * L::kABytes);
        const uint32_t sb = smem_addr(smem + L::kBOff);
        const uint32_t d = tmem_base + uint32_t(acc) * 128u;
        // RAW = U B_hi^T, then += U B_lo^T (rows 128..255 of the B pieces)
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t kk = k & 7;
          const uint32_t koff = (kk & 3) * 32u;   // 16 fp16 per K step
          const uint32_t piece = kk >> 2;
          const uint64_t ad = sw128_desc(sa + piece * L::kAPiece + koff);
          const uint64_t bd =
              sw128_desc(sb + piece * L::kBPiece + (k >= 8 ? 128u * 128u : 0u) + koff);
          tc_mma_f16(d, ad, bd, L::kIdesc, k > 0 ? 1u : 0u);
        }
        tc_commit(&empty[st]);
        tc_commit(&tfull[acc]);
      }
      // Drain: the last issued block's MMAs complete before TMEM is freed.
      if (b > 0)
        (void)mbar_wait_bounded(&tfull[(b - 1) % L::kAcc], ((b - 1) / L::kAcc) & 1);
    }
  } else if (warp < 4) {
    // ---------------- sign pass (warps 2, 3) ----------------
    const int h2 = warp - 2;
    const int hl = lane & (hpt - 1);
    TileWalk t[2];
    int table_key[2] = {-1, -1};
    t[0] = first;
    for (int k = 0; k < 2 * h2 && t[0].valid(); ++k) t[0].advance(a.g);
    t[1] = t[0];
    if (t[1].valid()) t[1].advance(a.g);
    for (int b = 0; b < n_blocks; ++b) {
      const int st = b % L::kNST;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int q = 2 * h2 + e;
        uint32_t* stab = reinterpret_cast<uint32_t*>(smem + L::kSignOff + q * L::kSignBytes);
        if (b * L::kSub + q < n_tiles) {
          const int key = t[e].table_key(a.g);
          if (key != table_key[e]) {
            build_tables<D, BITS, kSRFT, true, L::kMultStride, L::kSignStride, false, true>(
                nullptr, stab, a.lambda, a.signs, t[e].s, t[e].hb, a.g.heads, hpt_log2, lane);
            table_key[e] = key;
          }
        }
      }
      if (!__all_sync(0xffffffffu, wait_or_abort(&full[st], (b / L::kNST) & 1, abort_flag,
                                                 a.guard)))
        break;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int q = 2 * h2 + e;
        if (b * L::kSub + q < n_tiles) {
          const uint32_t* srow = reinterpret_cast<const uint32_t*>(
                                     smem + L::kSignOff + q * L::kSignBytes) + hl * L::kSignStride;
          const uint32_t row = swz_row<128>(
              smem_addr(smem + L::kAOff + st * L::kABytes + q * L::kSubA), lane);
#pragma unroll
          for (int p = 0; p < 2; ++p) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t addr = swz_chunk<128>(row, c) + p * L::kAPiece;
              const uint4 x = lds128(addr);
              const uint4 s4 = *reinterpret_cast<const uint4*>(srow + 32 * p + 4 * c);
              // x ^ (s & sign bits): one LOP3 per word
              sts128(addr, make_uint4(x.x ^ (s4.x & 0x80008000u), x.y ^ (s4.y & 0x80008000u),
                                      x.z ^ (s4.z & 0x80008000u), x.w ^ (s4.w & 0x80008000u)));
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&signed_[st]);
#pragma unroll
      for (int e = 0; e < 2; ++e)
        for (int k = 0; k < L::kSub && t[e].valid(); ++k) t[e].advance(a.g);
    }
  } else {
    // ---------------- epilogue (warps 4..11) ----------------
    const int q = warp & 3;             // TMEM lane quarter = sub-tile
    const int grp = (warp - 4) >> 2;    // takes the blocks b with b % EPI_GROUPS == grp
    constexpr int DP = D / 2;           // coordinates per half
    using SP = Shape<DP, BITS, G>;
    static_assert(G <= DP, "groups of at most 64 coordinates");
    float* mult = reinterpret_cast<float*>(smem + L::kMultOff + (warp - 4) * L::kMultBytes);
    const int hl = lane & (hpt - 1);
    const int rl = lane >> hpt_log2;
    const float* mrow = mult + hl * L::kMultStride;
    TileWalk t = first;
    for (int k = 0; k < grp * L::kSub + q && t.valid(); ++k) t.advance(a.g);
    int table_key = -1;
    for (int b = grp; b < n_blocks; b += EPI_GROUPS) {
      const int acc = b % L::kAcc;
      const bool mine = b * L::kSub + q < n_tiles;
      if (mine) {
        const int key = t.table_key(a.g);
        if (key != table_key) {
          build_tables<D, BITS, kSRFT, true, L::kMultStride, L::kSignStride, true, false>(
              mult, nullptr, a.lambda, a.signs, t.s, t.hb, a.g.heads, hpt_log2, lane);
          table_key = key;
        }
      }
      // warp-uniform outcome: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, wait_or_abort(&tfull[acc], (b / L::kAcc) & 1, abort_flag,
                                                 a.guard)))
        break;
      tc_fence_after();
      const int row = t.rb * rpt + rl;
      const size_t vec = (static_cast<size_t>(t.s) * a.out_slice_stride_rows + row) *
                             a.g.heads + t.hb * hpt + hl;
      const bool valid = mine && row < a.g.n_rows;
      const uint32_t taddr = tmem_base + (uint32_t(32 * q) << 16) + uint32_t(acc) * 128u;
      static_for<0, 2>([&](auto h_) {
        constexpr int hh = decltype(h_)::value;   // half of the coordinates
        float2 v[DP / 2];
        if (mine) {
          uint32_t r0[32], r1[32];
          tmem_ld32(taddr + uint32_t(hh * DP), r0);
          tmem_ld32(taddr + uint32_t(hh * DP + 32), r1);
          tmem_wait_ld(r0, r1);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[i] = make_float2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
            v[16 + i] = make_float2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
          }
        }
        if constexpr (hh == 1) {
          // this warp is done with the accumulator
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (mine) {
          static_for<0, DP / 4>([&](auto c_) {
            constexpr int ci = decltype(c_)::value;
            const float4 m4 = *reinterpret_cast<const float4*>(mrow + hh * DP + 4 * ci);
            v[2 * ci] = mul2(v[2 * ci], make_float2(m4.x, m4.y));
            v[2 * ci + 1] = mul2(v[2 * ci + 1], make_float2(m4.z, m4.w));
          });
          uint32_t sw[SP::SW];
          uint32_t words[SP::CW];
          quantize_codes<DP, BITS, G>(v, sw, words);
          if (valid) {
            // this half's codes (contiguous bytes) and scales
            uint4* cdst = reinterpret_cast<uint4*>(a.codes + vec * S::CB + hh * SP::CB);
            static_for<0, SP::CB / 16>([&](auto c_) {
              constexpr int ci = decltype(c_)::value;
              cdst[ci] = make_uint4(words[4 * ci], words[4 * ci + 1], words[4 * ci + 2],
                                    words[4 * ci + 3]);
            });
            uint16_t* dst = a.scales + vec * S::NG + hh * SP::NG;
            if constexpr (SP::NG == 1) {
              dst[0] = static_cast<uint16_t>(sw[0]);
            } else if constexpr (SP::NG == 2) {
              *reinterpret_cast<uint32_t*>(dst) = sw[0];
            } else if constexpr (SP::NG == 4) {
              *reinterpret_cast<uint2*>(dst) = make_uint2(sw[0], sw[1]);
            } else {
              static_for<0, SP::NG / 8>([&](auto k_) {
                constexpr int k = decltype(k_)::value;
                reinterpret_cast<uint4*>(dst)[k] =
                    make_uint4(sw[4 * k], sw[4 * k + 1], sw[4 * k + 2], sw[4 * k + 3]);
              });
            }
          }
        }
      });
      for (int k = 0; k < EPI_GROUPS * L::kSub && t.valid(); ++k) t.advance(a.g);
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
