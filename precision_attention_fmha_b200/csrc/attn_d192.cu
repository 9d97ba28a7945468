// Instantiations of the attention kernel with a 192-wide QK head dim and a
// 128-wide V / O head dim (BF16 Q/K with BF16 or E4M3 V, and all-E4M3;
// contiguous and paged K/V). The case "FlashInfer FP8/BF16 mixed-precision
// attention for Blackwell" names in its reviewer notes as the one its
// shared-memory-P schedule gates off (QK head dim 128 only). With BF16 Q/K a
// CTA takes one 48 KB query tile (AttnCfg::NQ), with E4M3 Q/K two 24 KB tiles.
#include "attn_kernel.cuh"

namespace fmha {
template <int QK, int PV>
static cudaError_t launch_d192(bool paged, const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t s) {
  return paged ? launch_attention_t<AttnCfg<192, QK, PV, true, false, false, false, 128>>(p, tq, tk, tv, to, s)
               : launch_attention_t<AttnCfg<192, QK, PV, false, false, false, false, 128>>(p, tq, tk, tv, to, s);
}

cudaError_t launch_attention_d192(int qk, int pv, bool paged, const AttnParams& p, const CUtensorMap& tq,
                                  const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                                  cudaStream_t s) {
  if (qk == QK_BF16 && pv == PV_BF16) return launch_d192<QK_BF16, PV_BF16>(paged, p, tq, tk, tv, to, s);
  if (qk == QK_BF16 && pv == PV_E4M3) return launch_d192<QK_BF16, PV_E4M3>(paged, p, tq, tk, tv, to, s);
  if (qk == QK_E4M3 && pv == PV_E4M3) return launch_d192<QK_E4M3, PV_E4M3>(paged, p, tq, tk, tv, to, s);
  return cudaErrorInvalidValue;
}
}  // namespace fmha
