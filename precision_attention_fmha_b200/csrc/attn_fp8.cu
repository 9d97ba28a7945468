// All-E4M3 (Q, K, V) instantiations of the attention kernel (D = 128).
#include "attn_kernel.cuh"

namespace fmha {
cudaError_t launch_attention_fp8(int, bool paged, const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t s) {
  return paged ? launch_attention_variants<128, QK_E4M3, PV_E4M3, true>(p, tq, tk, tv, to, s)
               : launch_attention_variants<128, QK_E4M3, PV_E4M3, false>(p, tq, tk, tv, to, s);
}
}  // namespace fmha
