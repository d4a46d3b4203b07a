// Launcher of the fused decode attention (d = 128; attention.cuh).
#include "attention.cuh"
#include "launch_impl.cuh"

namespace srftq {

int launch_decode_attention_d128(const AttnCall& c) {
  if (c.n_seq == 0) return SRFTQ_OK;
  const int64_t blocks = c.n_seq * c.heads * kAttnSplit;   // one cluster per (sequence, head)
  if (blocks > INT_MAX) return SRFTQ_ERR_UNSUPPORTED;
  unsigned* guard = Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  const int64_t rows = (c.n_ctx - 1) * c.tok_stride_rows + (c.n_seq - 1) * c.seq_stride_rows + 1;
  AttnArgs a{c.n_seq,   c.n_ctx,    c.tok_stride_rows, c.seq_stride_rows, c.heads,
             c.q_per_kv, c.scale,   c.q,               c.k_codes,         c.k_scales,
             c.k_signs, c.k_lambda, c.v_codes,         c.v_scales,        c.v_signs,
             c.v_lambda, c.out,     rows,              guard};
  int rc = SRFTQ_ERR_UNSUPPORTED;
  static_for<0, 2>([&](auto b_) {
    constexpr int BITS = decltype(b_)::value == 0 ? 4 : 8;
    static_for<3, 8>([&](auto lg_) {
      constexpr int G = 1 << decltype(lg_)::value;
      static_for<0, 2>([&](auto r_) {
        constexpr int ROT = decltype(r_)::value;
        static_for<0, 4>([&](auto n_) {
          constexpr int NQ = 1 << decltype(n_)::value;
          if (c.bits == BITS && c.group == G && c.rotation == ROT && c.q_per_kv == NQ) {
            // queries rotated into `out`, attention over the codes, outputs unrotated
            const int64_t nv = c.n_seq * c.heads * NQ;
            const int64_t cap = int64_t(Runtime::num_sms()) * 16;
            const int g1 = int((nv + 127) / 128 < cap ? (nv + 127) / 128 : cap);
            constexpr auto K = decode_attention_kernel<BITS, G, NQ>;
            constexpr int smem = AttnLayout<BITS, G, NQ>::kBytes;
            int bps = 0;
            rc = prepare_kernel<K>(smem, kAttnWarps * 32, &bps);
            if (rc != SRFTQ_OK) return;
            attn_query_kernel<ROT, NQ><<<g1, 128, 0, c.stream>>>(a);
            // the attention and unrotation grids are programmatic launches:
            // each may start while the grid before it finishes and waits for
            // its results with griddepcontrol.wait (attention.cuh)
            cudaLaunchAttribute pdl[1];
            pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            pdl[0].val.programmaticStreamSerializationAllowed = SRFTQ_ATTN_PDL;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(unsigned(blocks));
            cfg.blockDim = dim3(kAttnWarps * 32);
            cfg.dynamicSmemBytes = size_t(smem);
            cfg.stream = c.stream;
            cfg.attrs = pdl;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelEx(&cfg, K, a) != cudaSuccess) {
              (void)cudaGetLastError();
              rc = SRFTQ_ERR_CUDA;
              return;
            }
            cfg.gridDim = dim3(unsigned(g1));
            cfg.blockDim = dim3(128);
            cfg.dynamicSmemBytes = 0;
            if (cudaLaunchKernelEx(&cfg, attn_unrotate_kernel<ROT, NQ>, a) != cudaSuccess) {
              (void)cudaGetLastError();
              rc = SRFTQ_ERR_CUDA;
              return;
            }
            rc = finish_launch();
          }
        });
      });
    });
  });
  return rc;
}

}  // namespace srftq
