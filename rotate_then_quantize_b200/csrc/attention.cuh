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
//
// Main kernel: one cluster of kAttnSplit CTAs per (b, h); CTA r takes the
// r-th slice of the tokens and each of its warps every kAttnWarps-th chunk
// of 32 tokens. A warp streams its chunks through a kAttnStages-deep
// cp.async ring in shared memory (codes and scales of K and V), so data in
// flight holds no registers, and runs its own online softmax:
//   scores  lane i takes token i: decodes its 128 key codes (fp16
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
  static constexpr int kStages = (kWl + 4 * NQ * kAttnWarps + 127) / 128 * 128;
  static constexpr int kBytes = kStages + kAttnWarps * kAttnStages * kStage;
  static_assert(kStage >= NQ * D * 4, "a warp's partial sums fit in its first stage");
  __device__ static constexpr int swz(int r) { return (r * CB / 128) % PPT; }
};

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

  // int4 keys decode their odd coordinates 16 times too large (decode8)
  constexpr float kOdd = BITS == 4 ? 0.0625f : 1.0f;
  for (int i = tid; i < NQ * D; i += NW * 32) qs[i] = (i & 1) ? qo[i] * kOdd : qo[i];
  __syncthreads();

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

#pragma unroll
  for (int c = 0; c < NS - 1; ++c) issue(c);
  for (int64_t c = 0; c < n_chunks; ++c) {
    issue(c + NS - 1);
    cp_async_wait<NS - 1>();   // chunk c has landed (this lane's copies) ...
    __syncwarp();              // ... and every lane's
    const int64_t t0 = t_begin + 32 * (warp + NW * c);
    const int nt = int(t_end - t0 < 32 ? t_end - t0 : 32);
    const uint8_t* st = wst + (c % NS) * L::kStage;

    // score of token t0 + lane (log2 units; -inf past the end)
    float s[NQ];
    if (lane < nt) {
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
