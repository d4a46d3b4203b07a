// Decode attention fused with dequantisation, in the rotated domain.
//
// For one decode step, every sequence b and KV head h attend with the
// q_per_kv query heads of that KV head over the n_ctx cached tokens:
//   score_t = scale * q . khat_t,  p = softmax(score),  out = sum_t p_t vhat_t,
// with khat, vhat the dequantised cache. R is orthogonal ("When Quantization
// Is Free", Methodology 1), so q . khat_t = (R_K q) . (lambda_K * sigma * c_t)
// and sum_t p_t vhat_t = s_V * R_V^T (lambda_V * sum_t p_t sigma c_t): the
// kernel rotates each query once, reads only codes and scales (never an fp16
// cache, never an inverse transform per token) and unrotates each output
// once. This is the form in which the pages' int4 cache is read with less
// traffic than fp16 (Key Results, decode latency).
//
// Three launches on the caller's stream:
//   attn_query_kernel     one thread per query: R_K (s_K q) * lambda_K * scale
//                         * log2 e, float32, written into `out` (scratch);
//   decode_attention_kernel  the attention, reading those queries and
//                         writing lambda_V * (sum_t p_t sigma c_t) / sum_t p_t
//                         (the rotated-domain output) back into `out`;
//   attn_unrotate_kernel  one thread per output: s_V * R_V^T, in place.
// The main kernel then carries no transform and stays small in registers.
// The second and third are programmatic launches: each may start while the
// grid before it finishes, and waits (griddepcontrol.wait) before it reads
// that grid's results. The attention CTAs issue their first chunk's copies
// before that wait, since those read only the caches.
//
// Main kernel: one cluster of kAttnSplit CTAs per (b, h); CTA r takes the
// r-th slice of the tokens and each of its warps every kAttnWarps-th chunk
// of 32 tokens. A warp streams its chunks through a kAttnStages-deep
// cp.async ring in shared memory (codes and scales of K and V), so data in
// flight holds no registers, and runs its own online softmax:
//   scores  int4 keys with one query per KV head and groups of 16 or more:
//           integer tensor-core products over 16 tokens at a time
//           (mma.m16n8k32, u8 codes x s8 query digits, see below), one
//           conversion per (token, 16-coordinate sub-group); otherwise
//           lane i takes token i, decodes its 128 key codes (fp16
//           magic-number decode, the scale applied by the same FMA) and
//           dots them with the staged queries in packed f32x2 FMAs;
//   softmax a warp-uniform running maximum and per-lane running sums;
//   values  lane (l, c) takes coordinates 8c .. 8c + 7 of the chunk's
//           tokens l, l + 2, ..., the weights shuffled from the scoring
//           lanes.
// The warps merge in order in shared memory, then rank 0 merges the CTAs'
// partial results in rank order through distributed shared memory
// (deterministic) and scales by lambda_V / sum.
#pragma once

#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "aux.cuh"

namespace srftq {

constexpr int kAttnSplit = 8;     // CTAs (one cluster) per (sequence, KV head)
constexpr int kAttnWarps = 4;     // warps per CTA, each with its own online softmax
// SRFTQ_ATTN_STAGES, SRFTQ_ATTN_MINB and SRFTQ_ATTN_VW can be set at build
// time (-D) for measurement sweeps. The defaults are the measured best on the
// decode-stream workload: 2 stages (3 took 0.457 against 0.407 ms per
// layer), 4 CTAs per SM (5, at 96 registers, took 0.375 against 0.364 ms),
// two value words per lane with one or two query heads (one took 0.365
// against 0.357 ms).
#ifndef SRFTQ_ATTN_STAGES
#define SRFTQ_ATTN_STAGES 2
#endif
#ifndef SRFTQ_ATTN_VW
#define SRFTQ_ATTN_VW 0   // 0: two words with one or two query heads, one with more
#endif
#ifndef SRFTQ_ATTN_PDL
#define SRFTQ_ATTN_PDL 1  // programmatic launches of the attention and unrotation grids
#endif
constexpr int kAttnStages = SRFTQ_ATTN_STAGES;   // 32-token chunks in flight per warp

struct AttnArgs {
  int64_t n_seq, n_ctx, tok_stride_rows, seq_stride_rows;
  int32_t heads, q_per_kv;
  float scale;
  const uint16_t* q;          // [n_seq][heads * q_per_kv][d] fp16
  const uint8_t* k_codes;     // rows [..][heads][d * bits / 8]
  const uint16_t* k_scales;   // rows [..][heads][d / G]
  const int8_t* k_signs;      // [heads][d]
  const float* k_lambda;      // [heads][d]
  const uint8_t* v_codes;
  const uint16_t* v_scales;
  const int8_t* v_signs;
  const float* v_lambda;
  float* out;                 // [n_seq][heads * q_per_kv][d] float32
  int64_t rows;               // rows the caches hold (debug-build index checks)
  unsigned* guard;
};

// sigma * code for the 8 codes of one code word (int4: one uint32; int8:
// two) whose fp16 scale is the low half of sw. out[e] = coordinate 8m + e,
// except that for int4 the odd coordinates come out as 16 * sigma * code:
// their nibbles are taken where they lie (bits 4..7 of each 16-bit half,
// the fp16 pair 1152 + 16 q), which saves the shifts, and the factor 16 is
// folded, exactly, into what they are multiplied with or summed into.
template <int BITS>
__device__ __forceinline__ void decode8(const uint32_t* w, uint32_t sw, float (&out)[8]) {
  if constexpr (BITS == 4) {
    const float sg = __half2float(__ushort_as_half(uint16_t(sw)));
    const float off_e = -1032.0f * sg, off_o = -1152.0f * sg;
    const uint32_t w8 = w[0] >> 8;   // codes 2, 3 and 6, 7 in the low bytes of the halves
    const uint32_t h0 = (w[0] & 0x000F000Fu) ^ 0x64086408u;   // 1032 + q, codes 0 and 4
    const uint32_t h1 = (w[0] & 0x00F000F0u) ^ 0x64806480u;   // 1152 + 16 q, codes 1 and 5
    const uint32_t h2 = (w8 & 0x000F000Fu) ^ 0x64086408u;     // codes 2 and 6
    const uint32_t h3 = (w8 & 0x00F000F0u) ^ 0x64806480u;     // codes 3 and 7
    out[0] = fma_f16<0, 0>(h0, sw, off_e);
    out[4] = fma_f16<1, 0>(h0, sw, off_e);
    out[1] = fma_f16<0, 0>(h1, sw, off_o);
    out[5] = fma_f16<1, 0>(h1, sw, off_o);
    out[2] = fma_f16<0, 0>(h2, sw, off_e);
    out[6] = fma_f16<1, 0>(h2, sw, off_e);
    out[3] = fma_f16<0, 0>(h3, sw, off_o);
    out[7] = fma_f16<1, 0>(h3, sw, off_o);
  } else {
    const float off = -1152.0f * __half2float(__ushort_as_half(uint16_t(sw)));
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t h02 = (w[t] & 0x00FF00FFu) ^ 0x64806480u;          // bytes 0, 2
      const uint32_t h13 = ((w[t] >> 8) & 0x00FF00FFu) ^ 0x64806480u;   // bytes 1, 3
      out[4 * t + 0] = fma_f16<0, 0>(h02, sw, off);
      out[4 * t + 2] = fma_f16<1, 0>(h02, sw, off);
      out[4 * t + 1] = fma_f16<0, 0>(h13, sw, off);
      out[4 * t + 3] = fma_f16<1, 0>(h13, sw, off);
    }
  }
}

// out[v] = R_K (s_K q[v]) * lambda_K * scale * log2 e for query vector v.
template <int ROT, int NQ>
__global__ void __launch_bounds__(128) attn_query_kernel(const AttnArgs a) {
  constexpr int D = 128;
  constexpr float kLog2e = 1.4426950408889634f;
  asm volatile("griddepcontrol.launch_dependents;");   // the attention grid waits for this one
  const int64_t total = a.n_seq * a.heads * NQ;
  for (int64_t v_id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; v_id < total;
       v_id += int64_t(gridDim.x) * blockDim.x) {
    const int h = int((v_id % (int64_t(a.heads) * NQ)) / NQ);
    uint32_t xw[D / 2], sgw[D / 2];
    load_vector<D>(a.q + v_id * D, a.k_signs + int64_t(h) * D, xw, sgw);
    float2 v[D / 2];
    rotate_forward<ROT, D>(xw, sgw, v);
    const float* lk = a.k_lambda + int64_t(h) * D;
    const float f = a.scale * kLog2e;
    float* ov = a.out + v_id * D;
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 l4 = reinterpret_cast<const float4*>(lk)[ci];
      reinterpret_cast<float4*>(ov)[ci] =
          make_float4(v[2 * ci].x * gain_f<ROT, D>(4 * ci) * l4.x * f,
                      v[2 * ci].y * gain_f<ROT, D>(4 * ci + 1) * l4.y * f,
                      v[2 * ci + 1].x * gain_f<ROT, D>(4 * ci + 2) * l4.z * f,
                      v[2 * ci + 1].y * gain_f<ROT, D>(4 * ci + 3) * l4.w * f);
    });
  }
}

// out[v] = s_V * R_V^T out[v], in place (out[v] holds packed rotated coordinates).
template <int ROT, int NQ>
__global__ void __launch_bounds__(128) attn_unrotate_kernel(const AttnArgs a) {
  constexpr int D = 128;
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the attention grid's outputs
  const int64_t total = a.n_seq * a.heads * NQ;
  for (int64_t v_id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; v_id < total;
       v_id += int64_t(gridDim.x) * blockDim.x) {
    const int h = int((v_id % (int64_t(a.heads) * NQ)) / NQ);
    float* ov = a.out + v_id * D;
    float2 v[D / 2];
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const float4 y4 = reinterpret_cast<const float4*>(ov)[ci];
      v[2 * ci] = make_float2(y4.x * gain_f<ROT, D>(4 * ci), y4.y * gain_f<ROT, D>(4 * ci + 1));
      v[2 * ci + 1] =
          make_float2(y4.z * gain_f<ROT, D>(4 * ci + 2), y4.w * gain_f<ROT, D>(4 * ci + 3));
    });
    rotate_inverse<ROT, D>(v);
    const int8_t* sv = a.v_signs + int64_t(h) * D;
    static_for<0, D / 4>([&](auto c_) {
      constexpr int ci = decltype(c_)::value;
      const char4 s4 = reinterpret_cast<const char4*>(sv)[ci];
      reinterpret_cast<float4*>(ov)[ci] =
          make_float4(s4.x < 0 ? -v[2 * ci].x : v[2 * ci].x, s4.y < 0 ? -v[2 * ci].y : v[2 * ci].y,
                      s4.z < 0 ? -v[2 * ci + 1].x : v[2 * ci + 1].x,
                      s4.w < 0 ? -v[2 * ci + 1].y : v[2 * ci + 1].y);
    });
  }
}

// cp.async of 16 (L2 only), 8 or 4 bytes into shared memory, and its groups.
template <int BYTES>
__device__ __forceinline__ void cp_async(uint32_t dst, const void* src) {
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(BYTES)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The maximum and the sum over the 32 lanes of a warp.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Shared memory of the attention kernel. Each warp owns kAttnStages stages
// of one 32-token chunk: key codes, value codes (32 rows of CB bytes, the
// 16-byte pieces of row r stored at piece ^ swz(r) so that a lane reading
// its own row and half-warps reading one row each are both conflict-free),
// then key and value scales (32 rows of SBS bytes).
template <int BITS, int G, int NQ>
struct AttnLayout {
  static constexpr int D = 128, CB = D * BITS / 8, NG = D / G;
  static constexpr int SB = 2 * NG;                 // scale bytes per vector
  static constexpr int SBS = SB >= 4 ? SB : 4;      // their row stride
  static constexpr int PPT = CB / 16;               // 16-byte code pieces per row
  static constexpr int KC = 0, VC = 32 * CB, KS = 64 * CB, VS = 64 * CB + 32 * SBS;
  static constexpr int kStage = 64 * CB + 64 * SBS;
  static constexpr int kQs = 0;                                     // float [NQ][D]
  static constexpr int kAcc = kQs + NQ * D * 4;                     // float [NQ][D]
  static constexpr int kMx = kAcc + NQ * D * 4;                     // float [NQ]
  static constexpr int kSm = kMx + 4 * NQ;                          // float [NQ]
  static constexpr int kWm = kSm + 4 * NQ;                          // float [NW][NQ]
  static constexpr int kWl = kWm + 4 * NQ * kAttnWarps;             // float [NW][NQ]
  static constexpr int kQe = kWl + 4 * NQ * kAttnWarps;             // int [8]: piece exponents
  static constexpr int kQm = kQe + 4 * 8;                           // float [8]: 2^-(E + 16)
  static constexpr int kQsum = kQm + 4 * 8;                         // int [3][8]: piece sums
  static constexpr int kBtab = (kQsum + 4 * 24 + 15) / 16 * 16;     // uint2 [4][3][32]: B fragments
  static constexpr int kStages = (kBtab + 8 * 4 * 3 * 32 + 127) / 128 * 128;
  static constexpr int kBytes = kStages + kAttnWarps * kAttnStages * kStage;
  static_assert(kStage >= NQ * D * 4, "a warp's partial sums fit in its first stage");
  __device__ static constexpr int swz(int r) { return (r * CB / 128) % PPT; }
};

// Integer tensor-core scores (int4 keys, one query per KV head, G >= 16).
//
// score_t = sum_j sigma_{t,g(j)} q_j c_{t,j} is a contraction over the 128
// coordinates, with sigma constant on each group. Each 16-coordinate
// sub-group m of the query gets its own exponent E_m (|q_j| 2^E_m < 64 on
// it) and the integer Q_j = rint(q_j 2^(E_m + 16)) = B0 2^16 + B1 2^8 + B2
// in balanced base-256 digits (each a signed byte). A warp-level
// mma.m16n8k32 (u8 x s8 -> s32) then gives, for 16 tokens at a time, the
// exact integers D_p[t][m] = sum_{j in m} c_{t,j} B_p[j]: the codes enter
// as offset-binary bytes u = c + 8 (one AND-XOR per four codes), and the
// accumulator starts at -8 sum_{j in m} B_p[j], which removes the offset
// exactly. Column m of n-tile p holds digit p on sub-group m only (a
// block-diagonal B), so every (token, sub-group) partial lands in one
// register of one lane. D_0 2^16 + D_1 2^8 + D_2 = sum c Q fits in int32
// (|c| <= 8, |B0| <= 65, |B1|, |B2| <= 128 over 16 coordinates), is
// converted once, and is scaled by sigma 2^-(E_m + 16). The query's
// representation error is at most 2^-22 of its sub-group maximum; the
// products and sums are exact until that one conversion.

// k-order of the fragments: for k-step ks, lane (row group g, thread t)
// holds word 4t + ks of its token rows; the low nibbles of the word's
// bytes (coordinates 8w + 2i) are k = 4t + i, the high nibbles
// (coordinates 8w + 2i + 1) are k = 4t + 16 + i.
__device__ __forceinline__ void imma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Q = rint(q 2^(e + 16)) split into balanced base-256 digits B0 2^16 + B1 2^8 + B2.
__device__ __forceinline__ void query_digits(float q, int e, int (&b)[3]) {
  const int Q = __float2int_rn(ldexpf(q, e + 16));
  b[2] = ((Q + 128) & 255) - 128;
  const int q1 = (Q - b[2]) >> 8;
  b[1] = ((q1 + 128) & 255) - 128;
  b[0] = (q1 - b[1]) >> 8;
}

#ifndef SRFTQ_ATTN_INT_SCORES
#define SRFTQ_ATTN_INT_SCORES 1   // 0: every case on the per-lane float32 scores
#endif
template <int BITS, int G, int NQ>
__host__ __device__ constexpr bool attn_int_scores() {
  return SRFTQ_ATTN_INT_SCORES && BITS == 4 && NQ == 1 && G >= 16;
}

// CTAs per SM the register budget is sized for (128, 168 or 255 registers).
#ifndef SRFTQ_ATTN_MINB
#define SRFTQ_ATTN_MINB 4
#endif
template <int NQ>
constexpr int attn_min_blocks() {
  return NQ <= 2 ? SRFTQ_ATTN_MINB : NQ == 4 ? 3 : 2;
}

template <int BITS, int G, int NQ>
__global__ void __cluster_dims__(kAttnSplit, 1, 1)
    __launch_bounds__(kAttnWarps * 32, attn_min_blocks<NQ>()) decode_attention_kernel(const AttnArgs a) {
  using L = AttnLayout<BITS, G, NQ>;
  constexpr int D = 128, CB = L::CB, NG = L::NG, SB = L::SB, SBS = L::SBS, PPT = L::PPT;
  constexpr int WB = BITS;                  // bytes per 8-code word (4 or 8)
  constexpr int NW = kAttnWarps, NS = kAttnStages;
  // value phase: each lane takes VW consecutive code words (8 VW
  // coordinates) of VT tokens; two words with one or two query heads (one
  // scale conversion per 16 codes), one with more (registers)
  constexpr int VW = SRFTQ_ATTN_VW > 0 ? SRFTQ_ATTN_VW : NQ <= 2 ? 2 : 1;
  constexpr int LPT = 16 / VW;              // lanes per token row
  constexpr int TPI = 32 / LPT;             // tokens per warp instruction
  constexpr int VT = 32 / TPI;              // value tokens per lane and chunk
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(128) uint8_t smem[];
  float* qs = reinterpret_cast<float*>(smem + L::kQs);
  float* acc_out = reinterpret_cast<float*>(smem + L::kAcc);
  float* mx = reinterpret_cast<float*>(smem + L::kMx);
  float* sm = reinterpret_cast<float*>(smem + L::kSm);
  float* wm = reinterpret_cast<float*>(smem + L::kWm);
  float* wl = reinterpret_cast<float*>(smem + L::kWl);
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = blockIdx.x / kAttnSplit;
  const int h = int(bh % a.heads);
  const int64_t b = bh / a.heads;
  float* qo = a.out + (b * a.heads * NQ + int64_t(h) * NQ) * D;   // queries in, result out
  uint8_t* wst = smem + L::kStages + warp * NS * L::kStage;        // this warp's stages
  const uint32_t wst_a = smem_addr(wst);
  const uint32_t qs_a = smem_addr(qs);

  // this CTA's tokens; warp w takes the 32-token chunks w, w + NW, ...
  const int64_t per = (a.n_ctx + kAttnSplit - 1) / kAttnSplit;
  const int64_t t_begin = rank * per;
  const int64_t t_end = t_begin + per < a.n_ctx ? t_begin + per : a.n_ctx;
  const int64_t bs = b * a.seq_stride_rows;
  auto vec_of = [&](int64_t t) { return (t * a.tok_stride_rows + bs) * a.heads + h; };
  const int64_t n_chunks =
      t_end > t_begin + 32 * warp ? (t_end - t_begin - 32 * warp + 32 * NW - 1) / (32 * NW) : 0;

  // Copies chunk c of this warp into stage c % NS (one cp.async group; an
  // empty group past the last chunk keeps the group count uniform).
  auto issue = [&](int64_t c) {
    if (c < n_chunks) {
      const int64_t t0 = t_begin + 32 * (warp + NW * c);
      const int nt = int(t_end - t0 < 32 ? t_end - t0 : 32);
      const uint32_t st = wst_a + uint32_t(c % NS) * L::kStage;
      const int pc = lane % PPT;
#pragma unroll
      for (int k = 0; k < PPT; ++k) {
        const int r = lane / PPT + (32 / PPT) * k;
        const int64_t vec = vec_of(t0 + r);
        if (r < nt && dbg_ok(vec < a.rows * a.heads, a.guard)) {
          const uint32_t o = uint32_t(r * CB + ((pc ^ L::swz(r)) * 16));
          cp_async<16>(st + L::KC + o, a.k_codes + vec * CB + pc * 16);
          cp_async<16>(st + L::VC + o, a.v_codes + vec * CB + pc * 16);
        }
      }
      const int64_t svec = vec_of(t0 + lane);
      if (lane < nt && dbg_ok(svec < a.rows * a.heads, a.guard)) {
        const int64_t vec = svec;
        const uint32_t o = uint32_t(lane * SBS);
        const uint16_t* ks = a.k_scales + vec * NG;
        const uint16_t* vs = a.v_scales + vec * NG;
        if constexpr (SB >= 16) {
#pragma unroll
          for (int q = 0; q < SB / 16; ++q) {
            cp_async<16>(st + L::KS + o + 16 * q, ks + 8 * q);
            cp_async<16>(st + L::VS + o + 16 * q, vs + 8 * q);
          }
        } else if constexpr (SB >= 4) {
          cp_async<SB>(st + L::KS + o, ks);
          cp_async<SB>(st + L::VS + o, vs);
        } else {
          // one scale per vector (2 bytes, below the smallest cp.async)
          *reinterpret_cast<uint16_t*>(wst + (c % NS) * L::kStage + L::KS + o) = ks[0];
          *reinterpret_cast<uint16_t*>(wst + (c % NS) * L::kStage + L::VS + o) = vs[0];
        }
      } else {
        // past the end: value scale 0, so the stale codes there decode to 0
        uint8_t* z = wst + (c % NS) * L::kStage + L::VS + lane * SBS;
#pragma unroll
        for (int q = 0; q < SBS / 4; ++q) reinterpret_cast<uint32_t*>(z)[q] = 0u;
      }
    }
    cp_async_commit();
  };

  // the first chunks' copies read only the caches, so they start before the
  // queries are ready; with a programmatic launch the queries come from the
  // grid launched just before, which this waits for (a no-op otherwise)
#pragma unroll
  for (int c = 0; c < NS - 1; ++c) issue(c);
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // int4 keys decode their odd coordinates 16 times too large (decode8);
  // the integer scores take the codes exactly
  constexpr bool kInt = attn_int_scores<BITS, G, NQ>();
  constexpr float kOdd = BITS == 4 ? 0.0625f : 1.0f;
  for (int i = tid; i < NQ * D; i += NW * 32) qs[i] = (!kInt && (i & 1)) ? qo[i] * kOdd : qo[i];
  __syncthreads();

  // integer scores: per sub-group exponent, multiplier and digit sums, then
  // the CTA's table of B fragments (one uint2 per k-step, digit and lane,
  // read back per chunk) and this lane's accumulator start -8 sum B_p for
  // its columns 2t, 2t + 1
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t btab_a = smem_addr(smem + L::kBtab) + 8u * uint32_t(lane);
  int cinit[3][2];
  float qmul[2];
  if constexpr (kInt) {
    int* qe = reinterpret_cast<int*>(smem + L::kQe);
    float* qm = reinterpret_cast<float*>(smem + L::kQm);
    int* qsum = reinterpret_cast<int*>(smem + L::kQsum);
    if (tid < 8) {
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(qs[16 * tid + j]));
      // a non-finite query gives NaN scores, as float32 arithmetic would
      const bool fin = amax <= 3.402823466e38f;
      const int e = (amax > 0.0f && fin) ? 5 - ilogbf(amax) : 0;
      int sum[3] = {0, 0, 0};
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        int b[3];
        query_digits(fin ? qs[16 * tid + j] : 0.0f, e, b);
        sum[0] += b[0];
        sum[1] += b[1];
        sum[2] += b[2];
      }
      qe[tid] = e;
      qm[tid] = fin ? ldexpf(1.0f, -(e + 16)) : __int_as_float(0x7fc00000);
#pragma unroll
      for (int p = 0; p < 3; ++p) qsum[8 * p + tid] = sum[p];
    }
    __syncthreads();
    // entry (ks, lane l, half hh): lane l = (row group g, thread t) holds, in
    // byte i, digit p of coordinate 8 w + 2 i + hh of word w = 4 t + ks when
    // column g is that word's sub-group w / 2, else 0
    uint32_t* btab = reinterpret_cast<uint32_t*>(smem + L::kBtab);
    for (int idx = tid; idx < 4 * 32 * 2; idx += NW * 32) {
      const int hh = idx & 1, l = (idx >> 1) & 31, ks = idx >> 6;
      const int w = 4 * (l & 3) + ks;
      const bool on = (w >> 1) == (l >> 2);
      const int e = qe[w >> 1];
      uint32_t r[3] = {0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int b[3];
        const float qv = qs[8 * w + 2 * i + hh];
        query_digits(on && qv == qv && fabsf(qv) <= 3.402823466e38f ? qv : 0.0f, e, b);
#pragma unroll
        for (int p = 0; p < 3; ++p) r[p] |= uint32_t(b[p] & 255) << (8 * i);
      }
#pragma unroll
      for (int p = 0; p < 3; ++p) btab[2 * (32 * (3 * ks + p) + l) + hh] = r[p];
    }
#pragma unroll
    for (int p = 0; p < 3; ++p)
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) cinit[p][jj] = -8 * qsum[8 * p + 2 * tq + jj];
    qmul[0] = qm[2 * tq];
    qmul[1] = qm[2 * tq + 1];
    __syncthreads();
  }

  float m[NQ], l[NQ];          // running max (warp-uniform) and this lane's sum
  float2 vacc[NQ][4 * VW];     // sum p sigma c, coordinates 8 VW vwi ..
#pragma unroll
  for (int g = 0; g < NQ; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
#pragma unroll
    for (int e = 0; e < 4 * VW; ++e) vacc[g][e] = make_float2(0.0f, 0.0f);
  }
  const int vwi = lane % LPT;  // value phase: words VW vwi .. of the row
  const int vt0 = lane / LPT;  // value phase: tokens vt0, vt0 + TPI, ... of the chunk

  for (int64_t c = 0; c < n_chunks; ++c) {
    issue(c + NS - 1);
    cp_async_wait<NS - 1>();   // chunk c has landed (this lane's copies) ...
    __syncwarp();              // ... and every lane's
    const int64_t t0 = t_begin + 32 * (warp + NW * c);
    const int nt = int(t_end - t0 < 32 ? t_end - t0 : 32);
    const uint8_t* st = wst + (c % NS) * L::kStage;

    // score of token t0 + lane (log2 units; -inf past the end); with integer
    // scores, of this lane's own token 16 (t >> 1) + 8 (t & 1) + g
    float s[NQ];
    if constexpr (kInt) {
      uint32_t bq[4][3][2];   // this lane's B fragments, held for the chunk's two tiles
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          const uint2 b = lds64(btab_a + uint32_t(256 * (3 * ks + p)));
          bq[ks][p][0] = b.x;
          bq[ks][p][1] = b.y;
        }
      float srow[2][2];   // [16-token tile][row g, row g + 8]
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        int acc[3][4];
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          acc[p][0] = cinit[p][0];
          acc[p][1] = cinit[p][1];
          acc[p][2] = cinit[p][0];
          acc[p][3] = cinit[p][1];
        }
        const int r0 = 16 * mt + gq, r1 = r0 + 8;
        const uint4 u0 =
            *reinterpret_cast<const uint4*>(st + L::KC + r0 * CB + ((tq ^ L::swz(r0)) * 16));
        const uint4 u1 =
            *reinterpret_cast<const uint4*>(st + L::KC + r1 * CB + ((tq ^ L::swz(r1)) * 16));
        const uint32_t w0[4] = {u0.x, u0.y, u0.z, u0.w}, w1[4] = {u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a0 = (w0[ks] & 0x0F0F0F0Fu) ^ 0x08080808u;
          const uint32_t a1 = (w1[ks] & 0x0F0F0F0Fu) ^ 0x08080808u;
          const uint32_t a2 = ((w0[ks] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
          const uint32_t a3 = ((w1[ks] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
#pragma unroll
          for (int p = 0; p < 3; ++p)
            imma_u8s8(acc[p], a0, a1, a2, a3, bq[ks][p][0], bq[ks][p][1]);
        }
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const uint8_t* ksr = st + L::KS + (r0 + 8 * hr) * SBS;
          float sa, sb;
          if constexpr (G == 16) {
            const uint32_t sp = *reinterpret_cast<const uint32_t*>(ksr + 4 * tq);
            sa = __half2float(__ushort_as_half(uint16_t(sp)));
            sb = __half2float(__ushort_as_half(uint16_t(sp >> 16)));
          } else {
            sa = sb = __half2float(*reinterpret_cast<const __half*>(ksr + 2 * ((32 * tq) / G)));
          }
          float f[2];
#pragma unroll
          for (int jj = 0; jj < 2; ++jj)
            f[jj] = float(acc[0][2 * hr + jj] * 65536 + acc[1][2 * hr + jj] * 256 +
                          acc[2][2 * hr + jj]) * qmul[jj];
          srow[mt][hr] = fmaf(sa, f[0], sb * f[1]);
        }
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          srow[mt][hr] += __shfl_xor_sync(0xffffffffu, srow[mt][hr], 1);
          srow[mt][hr] += __shfl_xor_sync(0xffffffffu, srow[mt][hr], 2);
        }
      const float own = (tq >> 1) ? ((tq & 1) ? srow[1][1] : srow[1][0])
                                  : ((tq & 1) ? srow[0][1] : srow[0][0]);
      s[0] = 16 * (tq >> 1) + 8 * (tq & 1) + gq < nt ? own : -INFINITY;
    } else if (lane < nt) {
      uint32_t sw[(NG + 1) / 2];
      const uint8_t* ksr = st + L::KS + lane * SBS;
      if constexpr (SB >= 16) {
#pragma unroll
        for (int q = 0; q < SB / 16; ++q) {
          const uint4 u = *reinterpret_cast<const uint4*>(ksr + 16 * q);
          sw[4 * q] = u.x;
          sw[4 * q + 1] = u.y;
          sw[4 * q + 2] = u.z;
          sw[4 * q + 3] = u.w;
        }
      } else if constexpr (SB == 8) {
        const uint2 u = *reinterpret_cast<const uint2*>(ksr);
        sw[0] = u.x;
        sw[1] = u.y;
      } else if constexpr (SB == 4) {
        sw[0] = *reinterpret_cast<const uint32_t*>(ksr);
      } else {
        sw[0] = *reinterpret_cast<const uint16_t*>(ksr);
      }
      float2 s2[NQ];
#pragma unroll
      for (int g = 0; g < NQ; ++g) s2[g] = make_float2(0.0f, 0.0f);
      const uint8_t* kr = st + L::KC + lane * CB;
#pragma unroll
      for (int pc = 0; pc < PPT; ++pc) {
        const uint4 u = *reinterpret_cast<const uint4*>(kr + ((pc ^ L::swz(lane)) * 16));
        const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 16 / WB; ++k) {
          const int w8 = pc * (16 / WB) + k;   // coordinates 8 w8 .. 8 w8 + 7
          const int g8 = (8 * w8) / G;
          float val[8];
          decode8<BITS>(&uw[k * WB / 4], (sw[g8 / 2] >> (16 * (g8 & 1))) & 0xFFFFu, val);
#pragma unroll
          for (int g = 0; g < NQ; ++g) {
            const uint4 q0 = lds128(qs_a + uint32_t(g * D + 8 * w8) * 4u);
            const uint4 q1 = lds128(qs_a + uint32_t(g * D + 8 * w8 + 4) * 4u);
            s2[g] = fma2(make_float2(val[0], val[1]),
                         make_float2(__uint_as_float(q0.x), __uint_as_float(q0.y)), s2[g]);
            s2[g] = fma2(make_float2(val[2], val[3]),
                         make_float2(__uint_as_float(q0.z), __uint_as_float(q0.w)), s2[g]);
            s2[g] = fma2(make_float2(val[4], val[5]),
                         make_float2(__uint_as_float(q1.x), __uint_as_float(q1.y)), s2[g]);
            s2[g] = fma2(make_float2(val[6], val[7]),
                         make_float2(__uint_as_float(q1.z), __uint_as_float(q1.w)), s2[g]);
          }
        }
      }
#pragma unroll
      for (int g = 0; g < NQ; ++g) s[g] = s2[g].x + s2[g].y;
    } else {
#pragma unroll
      for (int g = 0; g < NQ; ++g) s[g] = -INFINITY;
    }
    // online softmax over the chunk: lane 0 is always a token, so the new
    // maximum is finite; alpha is 0 on the first chunk (m = -inf)
    float p[NQ], alpha[NQ];
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
      const float mn = fmaxf(m[g], warp_max(s[g]));
      alpha[g] = exp2f(m[g] - mn);
      p[g] = exp2f(s[g] - mn);
      l[g] = fmaf(l[g], alpha[g], p[g]);
      m[g] = mn;
    }
    // integer scores: token i's weight moves to lane i, where the value
    // phase takes it from
    if constexpr (kInt) p[0] = __shfl_sync(0xffffffffu, p[0], 4 * (lane & 7) + (lane >> 3));
    // values: rescale, then p_i sigma c_i for tokens vt0, vt0 + TPI, ...
    // (a token past the end decodes with scale 0 and has p = 0)
#pragma unroll
    for (int g = 0; g < NQ; ++g)
#pragma unroll
      for (int e = 0; e < 4 * VW; ++e) vacc[g][e] = mul2(vacc[g][e], splat(alpha[g]));
#pragma unroll
    for (int u = 0; u < VT; ++u) {
      const int i = vt0 + TPI * u;
      const uint8_t* vr = st + L::VC + i * CB;
      // VW * WB bytes at byte VW * WB * vwi of the row (inside one 16-byte piece)
      constexpr int VB = VW * WB;
      const uint8_t* src = vr + ((((VB * vwi) >> 4) ^ L::swz(i)) * 16) + ((VB * vwi) & 15);
      uint32_t w[VB / 4];
      if constexpr (VB == 4) {
        w[0] = *reinterpret_cast<const uint32_t*>(src);
      } else if constexpr (VB == 8) {
        const uint2 u2 = *reinterpret_cast<const uint2*>(src);
        w[0] = u2.x;
        w[1] = u2.y;
      } else {
        const uint4 u4 = *reinterpret_cast<const uint4*>(src);
        w[0] = u4.x;
        w[1] = u4.y;
        w[2] = u4.z;
        w[3] = u4.w;
      }
      float pi[NQ];
#pragma unroll
      for (int g = 0; g < NQ; ++g) pi[g] = __shfl_sync(0xffffffffu, p[g], i);
#pragma unroll
      for (int k = 0; k < VW; ++k) {
        const int word = VW * vwi + k;   // coordinates 8 word .. 8 word + 7
        const uint32_t vsc =
            *reinterpret_cast<const uint16_t*>(st + L::VS + i * SBS + ((8 * word) / G) * 2);
        float val[8];
        decode8<BITS>(&w[k * WB / 4], vsc, val);
#pragma unroll
        for (int g = 0; g < NQ; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            vacc[g][4 * k + e] =
                fma2(splat(pi[g]), make_float2(val[2 * e], val[2 * e + 1]), vacc[g][4 * k + e]);
      }
    }
    __syncwarp();   // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
  __syncwarp();
  // the unrotation may be scheduled once every CTA is merging
  asm volatile("griddepcontrol.launch_dependents;");

  // warp totals: the lanes' sums, and the lanes vwi, vwi + LPT, ... (same
  // coordinates), into the warp's first stage
  float* wacc = reinterpret_cast<float*>(wst);
#pragma unroll
  for (int g = 0; g < NQ; ++g) {
    l[g] = warp_sum(l[g]);
#pragma unroll
    for (int e = 0; e < 4 * VW; ++e) {
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) {
        vacc[g][e].x += __shfl_xor_sync(0xffffffffu, vacc[g][e].x, o);
        vacc[g][e].y += __shfl_xor_sync(0xffffffffu, vacc[g][e].y, o);
      }
      vacc[g][e].y *= kOdd;   // int4: odd coordinates were summed 16 times too large
    }
    if (lane < LPT) {
      float4* dst = reinterpret_cast<float4*>(wacc + g * D + 8 * VW * vwi);
#pragma unroll
      for (int e = 0; e < 2 * VW; ++e)
        dst[e] = make_float4(vacc[g][2 * e].x, vacc[g][2 * e].y, vacc[g][2 * e + 1].x,
                             vacc[g][2 * e + 1].y);
    }
    if (lane == 0) {
      wm[warp * NQ + g] = m[g];
      wl[warp * NQ + g] = l[g];
    }
  }
  __syncthreads();
  // this CTA's (max, sum, accumulator), merging the warps in order
  for (int idx = tid; idx < NQ * D; idx += NW * 32) {
    const int g = idx / D;
    float mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mt = fmaxf(mt, wm[w * NQ + g]);
    float acc = 0.0f, lt = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = wm[w * NQ + g];
      const float cw = mw == -INFINITY ? 0.0f : exp2f(mw - mt);
      const float* wa = reinterpret_cast<const float*>(smem + L::kStages + w * NS * L::kStage);
      acc = fmaf(cw, wa[idx], acc);
      lt = fmaf(cw, wl[w * NQ + g], lt);
    }
    acc_out[idx] = acc;
    if (idx % D == 0) {
      mx[g] = mt;
      sm[g] = lt;
    }
  }
  cluster.sync();

  // rank 0 merges the partial results in rank order: the rotated-domain
  // output lambda_V * sum_t p_t sigma c_t / sum_t p_t, written over the
  // queries (the unrotation follows in attn_unrotate_kernel)
  if (rank == 0) {
    for (int idx = tid; idx < NQ * D; idx += NW * 32) {
      const int g = idx / D, j = idx % D;
      float m_tot = -INFINITY;
      for (int r = 0; r < kAttnSplit; ++r)
        m_tot = fmaxf(m_tot, cluster.map_shared_rank(&mx[g], r)[0]);
      float l_tot = 0.0f, sacc = 0.0f;
      for (int r = 0; r < kAttnSplit; ++r) {
        const float mr = cluster.map_shared_rank(&mx[g], r)[0];
        const float cr = mr == -INFINITY ? 0.0f : exp2f(mr - m_tot);
        l_tot += cr * cluster.map_shared_rank(&sm[g], r)[0];
        sacc += cr * cluster.map_shared_rank(&acc_out[idx], r)[0];
      }
      qo[idx] = sacc * a.v_lambda[int64_t(h) * D + j] / l_tot;
    }
  }
  cluster.sync();   // the other CTAs keep their shared memory until rank 0 is done
}

}  // namespace srftq
