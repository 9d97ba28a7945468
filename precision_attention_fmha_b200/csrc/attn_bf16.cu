// BF16 Q/K/V instantiations of the attention kernel (D = 64, 128; contiguous and paged K/V).
#include "attn_kernel.cuh"

namespace fmha {
cudaError_t launch_attention_bf16(int D, bool paged, const AttnParams& p, const CUtensorMap& tq,
                                  const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                                  cudaStream_t s) {
  if (D == 128)
    return paged ? launch_attention_variants<128, QK_BF16, PV_BF16, true>(p, tq, tk, tv, to, s)
                 : launch_attention_variants<128, QK_BF16, PV_BF16, false>(p, tq, tk, tv, to, s);
  return paged ? launch_attention_variants<64, QK_BF16, PV_BF16, true>(p, tq, tk, tv, to, s)
               : launch_attention_variants<64, QK_BF16, PV_BF16, false>(p, tq, tk, tv, to, s);
}
}  // namespace fmha
