// Decode-shaped attention: GQA-packed query tiles (the query heads of one KV
// head share a 128-row tile, "FlashInfer block-sparse attention with PrimTS",
// section 1: the query tile is q_block_size x heads_q_per_kv) with split-KV
// ranges, and the merge of the splits' partial outputs by their log-sum-exp.
#include "attn_kernel.cuh"

namespace fmha {

cudaError_t launch_attention_packed(int qk, int pv, bool paged, const AttnParams& p, const CUtensorMap& tq,
                                    const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                                    cudaStream_t s) {
  if (qk == QK_BF16 && pv == PV_BF16)
    return paged ? launch_attention_t<AttnCfg<128, QK_BF16, PV_BF16, true, false, true>>(p, tq, tk, tv, to, s)
                 : launch_attention_t<AttnCfg<128, QK_BF16, PV_BF16, false, false, true>>(p, tq, tk, tv, to, s);
  if (qk == QK_BF16 && pv == PV_E4M3)
    return paged ? launch_attention_t<AttnCfg<128, QK_BF16, PV_E4M3, true, false, true>>(p, tq, tk, tv, to, s)
                 : launch_attention_t<AttnCfg<128, QK_BF16, PV_E4M3, false, false, true>>(p, tq, tk, tv, to, s);
  if (qk == QK_E4M3 && pv == PV_E4M3)
    return paged ? launch_attention_t<AttnCfg<128, QK_E4M3, PV_E4M3, true, false, true>>(p, tq, tk, tv, to, s)
                 : launch_attention_t<AttnCfg<128, QK_E4M3, PV_E4M3, false, false, true>>(p, tq, tk, tv, to, s);
  return cudaErrorInvalidValue;
}

namespace {

// One warp per output row (b, token, head): lane l owns d = 4l .. 4l+3.
// lse* = log sum_j exp(lse_j); O = sum_j exp(lse_j - lse*) O_j. Splits that
// saw no key carry lse_j = -inf and weigh nothing; if every split is empty the
// row is O = 0, lse = -inf.
__global__ void __launch_bounds__(128) split_merge_kernel(const MergeParams m) {
  // Launched as a programmatic dependent of the attention grid: wait here until
  // that grid has finished and its partials are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long rowid = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const long long rows = static_cast<long long>(m.B) * m.Sq * m.Hq;
  if (rowid >= rows) return;
  const int h = static_cast<int>(rowid % m.Hq);
  const int tok = static_cast<int>((rowid / m.Hq) % m.Sq);
  const int b = static_cast<int>(rowid / (static_cast<long long>(m.Hq) * m.Sq));
  const long long split_stride_lse = static_cast<long long>(m.B) * m.Hq * m.Sq;
  const long long lse_off = (static_cast<long long>(b) * m.Hq + h) * m.Sq + tok;
  float mx = -INFINITY;
  for (int j = lane; j < m.n_splits; j += 32) mx = fmaxf(mx, m.lse_part[j * split_stride_lse + lse_off]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (mx != -INFINITY) {
    const long long split_stride_o = static_cast<long long>(m.B) * m.Sq * m.Hq * m.D;
    const long long o_off = ((static_cast<long long>(b) * m.Sq + tok) * m.Hq + h) * m.D + 4 * lane;
    // Partials in groups of 8: all loads of a group are issued before any is
    // used, so the row pays about one memory latency per group, not per partial.
    for (int j0 = 0; j0 < m.n_splits; j0 += 8) {
      float lj[8];
      float4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int j = j0 + k;
        lj[k] = j < m.n_splits ? m.lse_part[j * split_stride_lse + lse_off] : -INFINITY;
        v[k] = (j < m.n_splits && 4 * lane < m.D)
                   ? *reinterpret_cast<const float4*>(m.o_part + j * split_stride_o + o_off)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (lj[k] == -INFINITY) continue;  // a split that saw no key
        const float wj = expf(lj[k] - mx);
        wsum += wj;
        acc[0] += wj * v[k].x;
        acc[1] += wj * v[k].y;
        acc[2] += wj * v[k].z;
        acc[3] += wj * v[k].w;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  if (4 * lane < m.D) {
    uint16_t* dst = m.o + b * m.o_sb + tok * m.o_ss + h * m.o_sh + 4 * lane;
    const uint32_t lo = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
    const uint32_t hi = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
  }
  if (m.lse != nullptr && lane == 0) m.lse[lse_off] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_split_merge(const MergeParams& m, cudaStream_t s) {
  const long long rows = static_cast<long long>(m.B) * m.Sq * m.Hq;
  const long long blocks = (rows + 3) / 4;
  if (blocks <= 0) return cudaSuccess;
  // Programmatic dependent launch: the merge grid is set up while the attention
  // grid (which allows it at its start) still runs, instead of after it.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, split_merge_kernel, m);
}

}  // namespace fmha
