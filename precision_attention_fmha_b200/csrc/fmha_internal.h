// fmha_internal.h -- structures shared by the host launchers and the kernels
// of libfmha.so. Not part of the public ABI (that is include/fmha.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fmha.h"  // include/ is on the include path

namespace fmha {

// Device error word bits (one word per device, see api.cu).
enum : uint32_t { kErrTimeout = 1u, kErrPageIndex = 2u };
// Bits 8..31 of the device error word: where the first wait that ran out was
// (set once): bits 8..19 = barrier address & 0xfff (shared-memory offset of the
// mbarrier), bit 20 = awaited parity, bits 24..28 = warp index + 1.
constexpr uint32_t kErrSiteShift = 8u;

// Default bound on one device-side wait (GPU clock cycles, ~1 s at 2 GHz).
constexpr uint64_t kDefaultWaitCycles = 2000000000ull;

// Operand kinds of the two tensor-core products.
enum QkKind : int { QK_BF16 = 0, QK_E4M3 = 1, QK_INT8 = 2 };
enum PvKind : int { PV_BF16 = 0, PV_E4M3 = 1 };

// How a CTA's two 128-row query tiles are chosen.
enum PairMode : int {
  PAIR_ROWS = 0,   // query blocks 2i and 2i+1 of one head
  PAIR_HEADS = 1,  // one query block of heads 2j and 2j+1 (same KV head)
  SINGLE = 2,      // one query block of one head (one query tile per CTA)
};

// Query tiles per attention CTA. Two share every K/V tile, except when the QK
// head dim makes a BF16 Q tile 48 KB (D = 192): two of them would leave room
// for only two 48 KB K/V slots, so such a CTA takes one query tile.
constexpr int query_tiles_per_cta(int qk_kind, int d_qk) { return (qk_kind == QK_BF16 && d_qk > 128) ? 1 : 2; }

struct AttnParams {
  int32_t B, Hq, Hkv, Sq, Skv, group;
  int32_t n_q_blocks;   // ceil(Sq / 128)
  int32_t n_kv_blocks;  // ceil(Skv / 128)
  int32_t pair_mode;  // PAIR_ROWS / PAIR_HEADS / SINGLE
  int32_t n_units;      // work items per (b, head unit): pairs of q blocks (PAIR_ROWS) or q blocks (PAIR_HEADS)
  int32_t causal;
  float scale_log2;     // softmax_scale * log2(e)
  // scale factors (dequantization multipliers), kinds from fmha_sf_kind
  const float* sf_q; int32_t sf_q_kind; int32_t sf_q_rpb; int32_t sf_q_nblk;
  const float* sf_k; int32_t sf_k_kind; int32_t sf_k_rpb; int32_t sf_k_nblk;
  const float* sf_v; int32_t sf_v_kind;
  const float* sf_p; int32_t sf_p_kind; int32_t sf_p_rpb; int32_t sf_p_nblk;
  float* lse;           // nullable [B, Hq, Sq]
  // block mask (nullable): byte (b, hkv, i, j) at mask[b*mask_sb + hkv*mask_sh + i*n_kv_blocks + j]
  const uint8_t* mask; int64_t mask_sb, mask_sh;
  // paged K/V (page_table == nullptr: contiguous)
  const int32_t* page_table; int32_t num_pages, page_size, max_pages_per_seq;
  int32_t p_terms;      // 1 or 2 E4M3 terms for P (E4M3 V only)
  int32_t o8;           // 1: O is written as E4M3(O / sf_o) (D = 128, not packed)
  const float* sf_o;    // nullable per-tensor output scale (1.0 when NULL)
  // GQA-packed query tiles (decode shapes): row r of a 128-row unit is query
  // token r >> group_shift of head (hkv * group + (r & (group - 1))); n_units
  // then counts pairs of 128-row units of the Sq * group packed rows.
  int32_t packed, group_shift, n_rows;
  int32_t narrow;  // packed, BF16 P, n_rows <= 16 in one tile: the 16-lane softmax pass
  // Split-KV (packed only): split j of a (b, kv head) takes the kept KV tiles
  // of ranks [j * per, (j + 1) * per), per = ceil(kept / n_splits). With several
  // partials each query tile writes O / l (fp32) and its lse to o_part / lse_part.
  // kv_interleave: all packed rows fit one 128-row tile, so the CTA's two query
  // tiles hold the same rows and take alternate kept KV tiles of the split;
  // each is then its own partial (n_parts = 2 * n_splits), else n_parts = n_splits.
  int32_t n_splits, split_tiles, kv_interleave, n_parts;
  float* o_part;   // [n_parts, B, Sq, Hq, D] when n_parts > 1
  float* lse_part; // [n_parts, B, Hq, Sq]
  uint32_t* err;        // device error word
  uint64_t wait_cycles; // bound on one wait
};

struct QuantParams {
  const uint16_t* src; int64_t s_sb, s_ss, s_sh;  // bf16 bits
  uint8_t* dst; int64_t d_sb, d_ss, d_sh;         // int8 / e4m3 bytes
  float* sf; int32_t kind; int32_t rpb; int32_t nblk;
  int32_t B, S, H, D;
  uint32_t* ws;          // amax accumulators (float bits) for the grid-wide kinds
  int32_t rows_per_cta;  // grid-wide kinds and the token mean: token rows per CTA
  const float* shift;    // nullable fp32 [B, H, D]: values quantized are x - shift
  // Token mean per channel (K smoothing): per-CTA fp64 partial sums, then the mean.
  double* partial;       // [B, H, n_chunks, D]
  float* mean;           // [B, H, D]
  int32_t n_chunks;
  uint32_t* err;         // device error word (a timed-out wait sets kErrTimeout)
  uint64_t wait_cycles;  // limit of one wait
};

// Launchers (defined in the .cu files). They return cudaSuccess or the launch error.
cudaError_t launch_attention(int qk_kind, int pv_kind, int D, bool paged, const AttnParams& p,
                             const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, cudaStream_t stream);
// tm_src (nullable): TMA map of the source as [D, H, S, B] with box [D, 1, rows_per_block, 1];
// token-block quantization then stages whole blocks in shared memory.
cudaError_t launch_quantize(bool to_e4m3, const QuantParams& p, const CUtensorMap* tm_src, cudaStream_t stream);
cudaError_t launch_channel_mean(const QuantParams& p, cudaStream_t stream);
// Decode path: attention over GQA-packed tiles (p.packed = 1), then, for
// n_splits > 1, the split merge into o (bf16, element strides) and lse.
cudaError_t launch_attention_packed(int qk_kind, int pv_kind, bool paged, const AttnParams& p,
                                    const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                    const CUtensorMap& to, cudaStream_t stream);
struct MergeParams {
  const float* o_part; const float* lse_part;
  uint16_t* o; int64_t o_sb, o_ss, o_sh;  // bf16 bits
  float* lse;                             // nullable [B, Hq, Sq]
  int32_t n_splits, B, Sq, Hq, D;
};
cudaError_t launch_split_merge(const MergeParams& m, cudaStream_t stream);

// Per-token NVFP4 quantization of a BF16 [rows, K] matrix (K % 16 == 0, K <= 16384).
struct Nvfp4Params {
  const uint16_t* src; int64_t src_rs;  // bf16 bits, row stride in elements
  int32_t rows, K;
  uint8_t* codes; int64_t codes_rs;     // [rows, K/2] packed E2M1, row stride in bytes
  uint8_t* sb; int64_t sb_rs;           // [rows, K/16] E4M3 block scales, row stride in bytes
  float* st;                            // [rows] token scales
  int32_t fast;                         // 1: x * (1 / e) instead of x / e
};
cudaError_t launch_nvfp4(const Nvfp4Params& p, cudaStream_t stream);

// Size of the built-in scratch used by fmha_quantize_blockwise_noalloc, in
// 32-bit words (one per scale group of the grid-wide granularities).
constexpr size_t kQuantNoallocScratchWords = 65536;
// Device address of that scratch on the current device (looked up once per
// device); nullptr and *err set on failure.
uint32_t* quant_noalloc_scratch(cudaError_t* err);

}  // namespace fmha
