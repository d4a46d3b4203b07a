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
// Main kernel: one cluster of kSplit CTAs per (b, h); CTA r takes the r-th
// slice of the tokens. 128 threads per CTA, tokens in tiles of 128:
//   scores  thread i takes token i of the tile: decodes its 128 key codes
//           (fp16 magic-number decode, the scale applied by the same FMA)
//           and dots them with the rotated, lambda- and scale-weighted
//           queries held in shared memory;
//   softmax running maximum and sum per query head (online softmax);
//   values  thread (l, c) takes coordinates 8c .. 8c + 7 of the tile's
//           tokens l, l + 8, ... and accumulates p_t sigma c_t;
// then the 8 token lanes are summed, and rank 0 merges the kSplit partial
// results in rank order through distributed shared memory (deterministic)
// and scales by lambda_V / sum. Each tile's key codes are loaded during the
// previous tile, and each thread issues all its value-code loads of a tile
// before using any.
#pragma once

#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "aux.cuh"

namespace srftq {

constexpr int kAttnSplit = 8;     // CTAs (one cluster) per (sequence, KV head)
constexpr int kAttnTile = 128;    // tokens per tile
constexpr int kAttnMaxQ = 8;      // query heads per KV head, at most

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
};

// sigma * code for the 8 codes of one code word (int4: one uint32; int8:
// two) whose fp16 scale is the low half of sw. out[e] = coordinate 8m + e.
template <int BITS>
__device__ __forceinline__ void decode8(const uint32_t* w, uint32_t sw, float (&out)[8]) {
  if constexpr (BITS == 4) {
    // w >> 4t holds codes t and t + 4 in the low nibbles of its halves
    const float off = -1032.0f * __half2float(__ushort_as_half(uint16_t(sw)));
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t hp = ((w[0] >> (4 * t)) & 0x000F000Fu) ^ 0x64086408u;   // 1032 + q
      out[t] = fma_f16<0, 0>(hp, sw, off);
      out[t + 4] = fma_f16<1, 0>(hp, sw, off);
    }
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

// The key codes (CB bytes) and group scales (packed fp16 pairs) of one token.
template <int BITS, int G>
struct KeyRow {
  static constexpr int CB = 128 * BITS / 8, NG = 128 / G;
  uint32_t cw[CB / 4];
  uint32_t sc[(NG + 1) / 2];
  __device__ __forceinline__ void load(const uint8_t* codes, const uint16_t* scales,
                                       int64_t vec) {
    const uint4* cp = reinterpret_cast<const uint4*>(codes + vec * CB);
#pragma unroll
    for (int i = 0; i < CB / 16; ++i) {
      const uint4 u = cp[i];
      cw[4 * i] = u.x;
      cw[4 * i + 1] = u.y;
      cw[4 * i + 2] = u.z;
      cw[4 * i + 3] = u.w;
    }
    const uint16_t* sp = scales + vec * NG;
    if constexpr (NG >= 8) {
#pragma unroll
      for (int i = 0; i < NG / 8; ++i) {
        const uint4 u = reinterpret_cast<const uint4*>(sp)[i];
        sc[4 * i] = u.x;
        sc[4 * i + 1] = u.y;
        sc[4 * i + 2] = u.z;
        sc[4 * i + 3] = u.w;
      }
    } else if constexpr (NG == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(sp);
      sc[0] = u.x;
      sc[1] = u.y;
    } else if constexpr (NG == 2) {
      sc[0] = *reinterpret_cast<const uint32_t*>(sp);
    } else {
      sc[0] = sp[0];
    }
  }
};

template <int BITS, int G, int NQ>
__global__ void __cluster_dims__(kAttnSplit, 1, 1) __launch_bounds__(128)
    decode_attention_kernel(const AttnArgs a) {
  constexpr int D = 128;
  constexpr int CB = D * BITS / 8;            // code bytes per vector
  constexpr int NG = D / G;                   // scales per vector
  constexpr int WPV = D / 8;                  // 8-code words per vector (16)
  constexpr int WB = 8 * BITS / 8;            // bytes per 8-code word (4 or 8)
  constexpr int VU = kAttnTile / 8;           // value tokens per thread and tile (16)
  constexpr int VB = NQ >= 4 ? VU / 4 : VU;   // value loads in flight per batch
  constexpr int VNB = VU / VB;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.x / kAttnSplit;
  const int h = int(bh % a.heads);
  const int64_t b = bh / a.heads;
  float* qo = a.out + (b * a.heads * NQ + int64_t(h) * NQ) * D;   // queries in, result out

  __shared__ __align__(16) float qs[NQ][D];   // rotated queries * lambda_K * scale * log2 e
  __shared__ float ps[NQ][kAttnTile];         // scores, then weights, of the tile
  __shared__ float red[8][NQ][D];             // token-lane partial sums
  __shared__ float mx[NQ], sm[NQ];            // running max (log2 units) and sum
  __shared__ float wred[4][NQ];               // per-warp reductions
  __shared__ float acc_out[NQ][D];            // this CTA's accumulated sum p sigma c

  for (int i = tid; i < NQ * D; i += 128) qs[i / D][i % D] = qo[i];
  if (tid < NQ) {
    mx[tid] = -INFINITY;
    sm[tid] = 0.0f;
  }
  __syncthreads();

  // this CTA's tokens
  const int64_t per = (a.n_ctx + kAttnSplit - 1) / kAttnSplit;
  const int64_t t_begin = rank * per;
  const int64_t t_end = t_begin + per < a.n_ctx ? t_begin + per : a.n_ctx;
  const int lane_t = tid >> 4;       // value phase: token lane 0..7
  const int wc = tid & 15;           // value phase: code word (coordinates 8 wc ..)
  const int64_t bs = b * a.seq_stride_rows;
  auto vec_of = [&](int64_t t) { return (t * a.tok_stride_rows + bs) * a.heads + h; };
  float vacc[NQ][8];
#pragma unroll
  for (int g = 0; g < NQ; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) vacc[g][e] = 0.0f;

  // With one or two query heads the next tile's key is loaded while this
  // tile is scored; with more, the registers go to the accumulators.
  constexpr bool kPrefetch = NQ <= 2;
  KeyRow<BITS, G> kr;
  if (kPrefetch && t_begin + tid < t_end) kr.load(a.k_codes, a.k_scales, vec_of(t_begin + tid));
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kAttnTile) {
    const int nt = int(t_end - t0 < kAttnTile ? t_end - t0 : kAttnTile);
    KeyRow<BITS, G> kn;
    if constexpr (kPrefetch) {
      if (t0 + kAttnTile + tid < t_end)
        kn.load(a.k_codes, a.k_scales, vec_of(t0 + kAttnTile + tid));
    } else {
      if (tid < nt) kr.load(a.k_codes, a.k_scales, vec_of(t0 + tid));
    }
    // (2) scores of token t0 + tid
    if (tid < nt) {
      float s[NQ];
#pragma unroll
      for (int g = 0; g < NQ; ++g) s[g] = 0.0f;
#pragma unroll
      for (int m = 0; m < WPV; ++m) {
        float val[8];
        const int g8 = (8 * m) / G;
        decode8<BITS>(&kr.cw[m * WB / 4], (kr.sc[g8 / 2] >> (16 * (g8 & 1))) & 0xFFFFu, val);
#pragma unroll
        for (int g = 0; g < NQ; ++g) {
          const float4 q0 = *reinterpret_cast<const float4*>(&qs[g][8 * m]);
          const float4 q1 = *reinterpret_cast<const float4*>(&qs[g][8 * m + 4]);
          s[g] = fmaf(val[0], q0.x, s[g]);
          s[g] = fmaf(val[1], q0.y, s[g]);
          s[g] = fmaf(val[2], q0.z, s[g]);
          s[g] = fmaf(val[3], q0.w, s[g]);
          s[g] = fmaf(val[4], q1.x, s[g]);
          s[g] = fmaf(val[5], q1.y, s[g]);
          s[g] = fmaf(val[6], q1.z, s[g]);
          s[g] = fmaf(val[7], q1.w, s[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < NQ; ++g) ps[g][tid] = s[g];
    }
    // the value codes and scales of this thread's tokens, issued before use
    // (in VNB batches of VB tokens, the first one before the softmax)
    uint32_t vw[VB][WB / 4];
    uint32_t vsw[VB];
    auto load_values = [&](int ub) {
#pragma unroll
      for (int u = 0; u < VB; ++u) {
        const int i = lane_t + 8 * (ub * VB + u);
        if (i < nt) {
          const int64_t vec = vec_of(t0 + i);
          if constexpr (BITS == 4) {
            vw[u][0] = *reinterpret_cast<const uint32_t*>(a.v_codes + vec * CB + wc * WB);
          } else {
            const uint2 w2 = *reinterpret_cast<const uint2*>(a.v_codes + vec * CB + wc * WB);
            vw[u][0] = w2.x;
            vw[u][WB / 4 - 1] = w2.y;
          }
          vsw[u] = a.v_scales[vec * NG + (8 * wc) / G];
        }
      }
    };
    load_values(0);
    __syncthreads();

    // (3) online softmax: tile maximum per query head, then the weights
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
      float m = tid < nt ? ps[g][tid] : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if ((tid & 31) == 0) wred[tid >> 5][g] = m;
    }
    __syncthreads();
    float alpha[NQ], mnew[NQ], pown[NQ];
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
      const float tm = fmaxf(fmaxf(wred[0][g], wred[1][g]), fmaxf(wred[2][g], wred[3][g]));
      mnew[g] = fmaxf(mx[g], tm);
      alpha[g] = exp2f(mx[g] - mnew[g]);   // 0 on the first tile (mx = -inf)
      pown[g] = tid < nt ? exp2f(ps[g][tid] - mnew[g]) : 0.0f;
    }
    float psum[NQ];
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
      psum[g] = pown[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) psum[g] += __shfl_xor_sync(0xffffffffu, psum[g], o);
    }
    __syncthreads();   // everyone has read ps (scores), wred and mx
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
      ps[g][tid] = pown[g];
      if ((tid & 31) == 0) wred[tid >> 5][g] = psum[g];
    }
    __syncthreads();
    if (tid < NQ) {
      const int g = tid;
      sm[g] = sm[g] * alpha[g] + (wred[0][g] + wred[1][g] + wred[2][g] + wred[3][g]);
      mx[g] = mnew[g];
    }
    // (4) values: rescale, then tokens lane_t, lane_t + 8, ... of the tile
#pragma unroll
    for (int g = 0; g < NQ; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) vacc[g][e] *= alpha[g];
#pragma unroll
    for (int ub = 0; ub < VNB; ++ub) {
      if (ub > 0) load_values(ub);
#pragma unroll
      for (int u = 0; u < VB; ++u) {
        const int i = lane_t + 8 * (ub * VB + u);
        if (i < nt) {
          float val[8];
          decode8<BITS>(vw[u], vsw[u], val);
#pragma unroll
          for (int g = 0; g < NQ; ++g) {
            const float p = ps[g][i];
#pragma unroll
            for (int e = 0; e < 8; ++e) vacc[g][e] = fmaf(p, val[e], vacc[g][e]);
          }
        }
      }
    }
    if constexpr (kPrefetch) {
#pragma unroll
      for (int i = 0; i < CB / 4; ++i) kr.cw[i] = kn.cw[i];
#pragma unroll
      for (int i = 0; i < (NG + 1) / 2; ++i) kr.sc[i] = kn.sc[i];
    }
    __syncthreads();   // ps and mx are rewritten by the next tile
  }

  // (5) sum the 8 token lanes: acc_out[g][j]
#pragma unroll
  for (int g = 0; g < NQ; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) red[lane_t][g][8 * wc + e] = vacc[g][e];
  __syncthreads();
  for (int idx = tid; idx < NQ * D; idx += 128) {
    const int g = idx / D, j = idx % D;
    float sacc = 0.0f;
#pragma unroll
    for (int l = 0; l < 8; ++l) sacc += red[l][g][j];
    acc_out[g][j] = sacc;
  }
  cluster.sync();

  // (6) rank 0 merges the partial results in rank order: the rotated-domain
  // output lambda_V * sum_t p_t sigma c_t / sum_t p_t, written over the
  // queries (the unrotation follows in attn_unrotate_kernel)
  if (rank == 0) {
    for (int idx = tid; idx < NQ * D; idx += 128) {
      const int g = idx / D, j = idx % D;
      float m_tot = -INFINITY;
      for (int r = 0; r < kAttnSplit; ++r)
        m_tot = fmaxf(m_tot, cluster.map_shared_rank(&mx[g], r)[0]);
      float l_tot = 0.0f, sacc = 0.0f;
      for (int r = 0; r < kAttnSplit; ++r) {
        const float mr = cluster.map_shared_rank(&mx[g], r)[0];
        const float c = mr == -INFINITY ? 0.0f : exp2f(mr - m_tot);
        l_tot += c * cluster.map_shared_rank(&sm[g], r)[0];
        sacc += c * cluster.map_shared_rank(&acc_out[g][j], r)[0];
      }
      qo[idx] = sacc * a.v_lambda[int64_t(h) * D + j] / l_tot;
    }
  }
  cluster.sync();   // the other CTAs keep their shared memory until rank 0 is done
}

}  // namespace srftq
