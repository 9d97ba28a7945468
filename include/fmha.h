/*
 * fmha.h -- C ABI of libfmha.so: mixed-precision fused multi-head attention
 * forward for NVIDIA B200 (sm_100a), plus the block quantizer that produces
 * its 8-bit operands.
 *
 * Sources (page titles; sections):
 *  [DiT-Sage]  "FlashInfer DiT optimization: SageAttention and Int8/FP8
 *              mixed-precision kernels" (flashinfer PR #2711): section 1
 *              (kernel key over separate Q/K/V/O dtypes and the four
 *              SageAttention scale-factor granularities), section 2 (scale
 *              factors for Q, K, P and V passed to the kernel and applied
 *              after the Int8/FP8 BMM1 and BMM2), "Why" items 1-3.
 *  [BW-FP8]    "FlashInfer FP8/BF16 mixed-precision attention for Blackwell"
 *              (flashinfer PR #5900): introduction (dense context FMHA with
 *              QK-BF16/PV-FP8 and all-FP8), section 3 (lazy O correction,
 *              exp2 on MUFU and FMA).
 *  [PrimTS-BS] "FlashInfer block-sparse attention with PrimTS" (flashinfer
 *              PR #4474): section 2 (block-sparse attention over contiguous
 *              and paged K/V through a page table).
 *  [Cake-MLA]  "FlashInfer DeepSeek-V4 sparse-MLA: Cake backend" (flashinfer
 *              PR #5686): section 1 (output written through a TMA descriptor
 *              passed to the kernel as a grid constant).
 *
 * Conventions for every call
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    never allocates device memory for a call and keeps no state between
 *    calls except one device-global error word per device.
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream). The
 *    only host synchronisation is in fmha_get_device_error().
 *  - Argument errors are detected on the host and returned before anything
 *    is launched; nothing is written. fmha_last_error_message() then holds a
 *    one-line reason (thread-local).
 *  - A device-side wait that runs out (a lost signal inside a kernel) never
 *    traps or hangs: the kernel records FMHA_ERR_TIMEOUT in the device error
 *    word and returns; fmha_get_device_error() reports it.
 *  - Tensors are token-major "NHD": element (b, s, h, d) lives at
 *    ptr + b*stride_b + s*stride_s + h*stride_h + d (strides in ELEMENTS,
 *    d contiguous). Base pointers and strides must be 16-byte aligned
 *    (TMA requirement); otherwise FMHA_ERR_INVALID_ARG.
 *  - Indexing uses 64-bit offsets throughout.
 */
#ifndef FMHA_H_
#define FMHA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */

typedef enum {
  FMHA_OK = 0,
  FMHA_ERR_INVALID_ARG = 1, /* bad pointer, size, stride, alignment or scale layout */
  FMHA_ERR_UNSUPPORTED = 2, /* valid request this build does not implement (dtype tuple, D, page size) */
  FMHA_ERR_CUDA = 3,        /* a CUDA runtime / driver call failed (message has the CUDA error) */
  FMHA_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (reported by fmha_get_device_error) */
  FMHA_ERR_DEVICE_INDEX = 5 /* a kernel met an out-of-range page index (reported by fmha_get_device_error) */
} fmha_status;

/* Element types. BF16/FP16 are IEEE-style 16-bit floats, E4M3 is the OCP
 * 8-bit float (bias 7, max 448, no infinities), INT8 is two's complement. */
typedef enum { FMHA_BF16 = 0, FMHA_FP16 = 1, FMHA_FP32 = 2, FMHA_E4M3 = 3, FMHA_INT8 = 4 } fmha_dtype;

/* Scale-factor granularity ([DiT-Sage] sections 1-2). A scale factor is the
 * fp32 DEQUANTIZATION multiplier: real value = code * scale. Layouts (fp32,
 * contiguous), for a tensor of shape [B, S, H, D]:
 *   FMHA_SF_NONE            no scale (1.0); ptr may be NULL
 *   FMHA_SF_PER_TENSOR      [1]
 *   FMHA_SF_PER_HEAD        [B, H]
 *   FMHA_SF_PER_TOKEN_BLOCK [B, H, ceil(S / rows_per_block)]
 *   FMHA_SF_PER_CHANNEL     [B, H, D]                                      */
typedef enum {
  FMHA_SF_NONE = 0,
  FMHA_SF_PER_TENSOR = 1,
  FMHA_SF_PER_HEAD = 2,
  FMHA_SF_PER_TOKEN_BLOCK = 3,
  FMHA_SF_PER_CHANNEL = 4
} fmha_sf_kind;

typedef struct {
  void* ptr;        /* device pointer to element (0,0,0,0) */
  int32_t dtype;    /* fmha_dtype */
  int32_t reserved; /* must be 0 */
  int64_t stride_b, stride_s, stride_h; /* element strides; d is contiguous */
} fmha_tensor;

typedef struct {
  float* ptr;             /* device pointer, layout per `kind` */
  int32_t kind;           /* fmha_sf_kind */
  int32_t rows_per_block; /* tokens per block for FMHA_SF_PER_TOKEN_BLOCK, else ignored */
} fmha_sf;

/* Arguments of one attention call.
 *   q [B, Sq, Hq, D], k [B, Skv, Hkv, D], v [B, Skv, Hkv, Dv], o [B, Sq, Hq, Dv]
 *   (Dv = D except for the 192 / 128 head dims below).
 *   Query head h attends to KV head h / (Hq / Hkv) (grouped-query attention).
 *   O_i = sum_j softmax_j(softmax_scale * q_i . k_j) v_j over the visible keys
 *   j, where q, k, v are the DEQUANTIZED operands (code * scale).
 * Scale factors ([DiT-Sage] section 2): sf_q, sf_k, sf_v dequantize the
 * 8-bit operands; sf_q / sf_k are applied to QK^T before the softmax, sf_v to
 * the PV product in the epilogue. Allowed: sf_q PER_TENSOR / PER_HEAD /
 * PER_TOKEN_BLOCK (any rows_per_block >= 1); sf_k PER_TENSOR / PER_HEAD /
 * PER_TOKEN_BLOCK (rows_per_block a multiple of 32); sf_v PER_TENSOR /
 * PER_HEAD / PER_CHANNEL. For BF16 operands the kind must be FMHA_SF_NONE.
 * sf_p scales the softmax output P when P is cast to E4M3 for the PV product
 * (8-bit V only): P is stored as E4M3(p / sf_p) and the product is multiplied
 * back by sf_p. Allowed: NONE (= an internal power-of-two scale chosen for
 * precision), PER_TENSOR, or PER_TOKEN_BLOCK over query rows [B, Hq,
 * ceil(Sq / rows_per_block)] with rows_per_block a multiple of 128. Values
 * must be positive and finite.
 *   softmax_scale <= 0 selects 1/sqrt(D).
 *   causal != 0: key j is visible to query i iff j <= i + (Skv - Sq)
 *   (bottom-right aligned).
 *   lse (nullable): fp32 [B, Hq, Sq], natural-log log-sum-exp of the scaled
 *   scores; -inf for a row with no visible key (whose O row is 0). The sum
 *   runs over the exponentials before P is rounded to its BF16 or E4M3
 *   format (with one E4M3 term, plus the rounding error of each 128-key
 *   tile's largest weight, so that a dominant key's weight is exact, which
 *   moves lse by at most ln(1 + 2^-4) ~ 0.061); it is the normaliser O uses,
 *   so partial results merge exactly.
 * Supported (q, k, v, o) dtype tuples: (BF16, BF16, BF16, BF16),
 * (BF16, BF16, E4M3, BF16) ("QK-BF16/PV-FP8", [BW-FP8]),
 * (E4M3, E4M3, E4M3, BF16) ("all-FP8", [BW-FP8]), (INT8, INT8, E4M3, BF16)
 * ("SageAttention", [DiT-Sage]). D must be 64 or 128 (128 for 8-bit Q/K),
 * or D = 192 with Dv = 128 for the BF16, QK-BF16/PV-FP8 and all-FP8 tuples
 * with one-term P and a BF16 o, not through fmha_fwd_decode (with BF16 Q/K
 * also Skv <= 131072: a CTA deals its kept key blocks to two warpgroups
 * through a 1024-bit set; FMHA_ERR_UNSUPPORTED otherwise): the QK head dim
 * that [BW-FP8]'s reviewer notes name as the case their shared-memory-P
 * schedule was gated off for (shared-memory capacity).
 * Any of these may instead write an E4M3 o (D = 128, not fmha_fwd_decode):
 * o = E4M3(O / sf_o) rounded to nearest even and saturated to +-448. This is
 * the FP8 output that [BW-FP8]'s reviewer notes mention, where their shared-
 * memory-P schedule was limited to 16-bit outputs because of the TMA copy
 * granularity. Here an E4M3 row of 128 bytes is one TMA box.               */
typedef struct {
  fmha_tensor q, k, v, o;
  fmha_sf sf_q, sf_k, sf_v, sf_p;
  int32_t B, Hq, Hkv, Sq, Skv, D;
  float softmax_scale;
  int32_t causal;
  float* lse;
  int32_t p_terms; /* E4M3 P only: 0 or 1 = P cast to one E4M3 value (3 mantissa
                      bits); 2 = P split into two E4M3 terms hi + lo, each fed to
                      its own PV product (about 7 significant bits, twice the PV
                      tensor work). Must be 0 or 1 when V is BF16. */
  int32_t Dv;       /* head dim of V and O; 0 = D. Differs from D only for
                       D = 192 (QK) with Dv = 128 (V, O). */
  fmha_sf sf_o;     /* o of dtype E4M3 only: PER_TENSOR dequantization multiplier
                       of the output, O ~= code * sf_o[0], or NONE (= 1.0). Must
                       be NONE for a BF16 o. */
} fmha_args;

/* Block quantizer: amax -> scale = amax / R -> codes ([DiT-Sage] section 2,
 * "Why" item 2).
 *   src: BF16 [B, S, H, D]; dst: INT8 (R = 127) or E4M3 (R = 448), same shape.
 *   sf:  output scales, kind PER_TENSOR / PER_HEAD / PER_TOKEN_BLOCK /
 *        PER_CHANNEL (layouts above).
 * Per block: amax = max |x|; scale = fp32(amax) / fp32(R) (IEEE division;
 * 1.0 when amax == 0); code = RN(fp32(x) / scale) (IEEE division), INT8
 * rounded half-to-even and clamped to [-127, 127], E4M3 rounded to nearest
 * even with saturation to +-448. Inputs must be finite.
 * S == 0 writes no code; the grid-wide kinds then write scale 1.0 into every
 * group. H and B must be at most 65535 (FMHA_ERR_UNSUPPORTED otherwise).
 * PER_TOKEN_BLOCK needs no workspace. The other kinds reduce amax across the
 * whole grid and need `workspace`: a device buffer of at least
 * fmha_quantize_workspace_bytes(...) bytes, 4-byte aligned, owned by the
 * caller, not shared with a concurrent call; its contents on entry do not
 * matter. workspace may be NULL when that size is 0.                        */
fmha_status fmha_quantize_blockwise(const fmha_tensor* src, const fmha_tensor* dst, const fmha_sf* sf,
                                    int32_t B, int32_t S, int32_t H, int32_t D,
                                    void* workspace, size_t workspace_bytes, struct CUstream_st* stream);

/* Workspace bytes fmha_quantize_blockwise needs for this granularity and shape. */
size_t fmha_quantize_workspace_bytes(int32_t sf_kind, int32_t B, int32_t S, int32_t H, int32_t D);

/* The block quantizer for callers that cannot allocate device memory. (The
 * pages have no counterpart: this is an addition of this library.)
 * Some callers cannot allocate device memory for a call: a plugin inside an
 * engine that owns all device memory and exposes no allocator, or code on a
 * latency-critical path where cudaMalloc and the device synchronisation it
 * can imply are not allowed. This entry point takes the same arguments as
 * fmha_quantize_blockwise, minus the workspace, and allocates nothing: the
 * amax accumulators live in a device array built into the library, 256 KB
 * (65536 scale groups) that every GPU loading the library holds until the
 * process exits. Codes and scales are identical to fmha_quantize_blockwise.
 *  - Limit: at most 65536 scale groups (per tensor: 1; per head: B*H; per
 *    channel: B*H*D; per token block needs none). Larger requests return
 *    FMHA_ERR_INVALID_ARG with the sizes in fmha_last_error_message().
 *  - The first call on a device (that device current) looks up the array's
 *    device address with cudaGetSymbolAddress; make that first call before
 *    any stream capture. The address is kept for the life of the process:
 *    after cudaDeviceReset the library's module is loaded again and the kept
 *    address is stale, so do not call this entry point (nor any other that
 *    uses the device error word) after a device reset.
 *  - All calls share the one array. It keeps the last call's contents; each
 *    call clears the part it uses before use. Calls that overlap on the GPU
 *    (for example on two streams at once) race and give wrong scales: order
 *    them on one stream.                                                    */
fmha_status fmha_quantize_blockwise_noalloc(const fmha_tensor* src, const fmha_tensor* dst, const fmha_sf* sf,
                                            int32_t B, int32_t S, int32_t H, int32_t D,
                                            struct CUstream_st* stream);

/* K smoothing for the SageAttention path. (The pages name SageAttention and
 * its block scales, not this step; it follows the SageAttention paper, Zhang
 * et al. 2024: quantize K minus its mean over the tokens.) A shift that is
 * constant over the keys of one (b, h_kv) moves every score of a query row by
 * softmax_scale * q . shift. Softmax ignores that, so attention on the
 * smoothed keys gives the same O. The log-sum-exp (fmha_args.lse) is that of
 * the smoothed scores, lower by softmax_scale * q . shift. Smoothing removes
 * a per-channel bias from K before its blocks are scaled, which makes the
 * INT8 steps smaller.
 *
 * fmha_channel_mean: mean[b, h, d] = fp32(sum_s x[b, s, h, d] / S), for
 *   src BF16 [B, S, H, D] (element strides, D contiguous, 16-byte aligned
 *   rows) and mean fp32 [B, H, D] contiguous (device, caller-owned). The sum
 *   is taken in fp64 in a fixed order (per CTA, then over CTAs), divided by S
 *   in fp64 and rounded once to fp32. Results do not depend on timing. They
 *   equal any other summation order wherever the fp64 sum of the S values is
 *   exact, which holds for BF16 inputs whose magnitudes span at most about
 *   2^(45 - log2 S). S = 0 gives zeros. D must be a power of two in [8, 2048].
 *   workspace: device, 8-byte aligned, at least
 *   fmha_channel_mean_workspace_bytes(B, S, H, D) bytes (0 when S == 0). It
 *   must not be shared with a concurrent call.
 * fmha_quantize_blockwise_shifted: fmha_quantize_blockwise applied to
 *   x - shift, with shift fp32 [B, H, D] contiguous (device, 16-byte aligned,
 *   not NULL), normally the output of fmha_channel_mean. Each element is first
 *   reduced by one fp32 round-to-nearest subtraction, and the amax, scale and
 *   code rules apply to that difference. The codes dequantize to
 *   x - shift. Other arguments, the workspace rule and the errors are those
 *   of fmha_quantize_blockwise.                                              */
size_t fmha_channel_mean_workspace_bytes(int32_t B, int32_t S, int32_t H, int32_t D);
fmha_status fmha_channel_mean(const fmha_tensor* src, float* mean, int32_t B, int32_t S, int32_t H, int32_t D,
                              void* workspace, size_t workspace_bytes, struct CUstream_st* stream);
fmha_status fmha_quantize_blockwise_shifted(const fmha_tensor* src, const float* shift, const fmha_tensor* dst,
                                            const fmha_sf* sf, int32_t B, int32_t S, int32_t H, int32_t D,
                                            void* workspace, size_t workspace_bytes,
                                            struct CUstream_st* stream);

/* Dense attention (optionally causal) over contiguous K/V ([BW-FP8] intro). */
fmha_status fmha_fwd(const fmha_args* args, struct CUstream_st* stream);

/* Attention restricted by a 128x128 block mask ([PrimTS-BS] section 2).
 *   mask: uint8, element (b, h_kv, i, j) at mask[b*mask_stride_b +
 *   h_kv*mask_stride_h + i*ceil(Skv/128) + j], nonzero = the 128x128 block of
 *   query rows [128i, 128i+128) x keys [128j, 128j+128) is visible (ANDed with
 *   causal). Strides may be 0 to broadcast. Fully hidden rows give O = 0.
 *   Skv <= 131072 (1024 key blocks) when a mask is given: each CTA keeps its
 *   rows' kept key blocks as a 1024-bit set in shared memory.               */
fmha_status fmha_fwd_block_sparse(const fmha_args* args, const uint8_t* mask, int64_t mask_stride_b,
                                  int64_t mask_stride_h, struct CUstream_st* stream);

/* Attention over a paged K/V cache ([PrimTS-BS] section 2).
 *   args->k / args->v describe the page POOL: element (page, t, h, d) at
 *   ptr + page*stride_b + t*stride_s + h*stride_h + d, num_pages pages of
 *   page_size tokens. Token s of sequence b is row s % page_size of pool page
 *   page_table[b*max_pages_per_seq + s / page_size] (int32, device).
 *   page_size must be 16, 32, 64 or 128. Every sequence has Skv tokens.
 *   mask: optional block mask as in fmha_fwd_block_sparse (NULL = dense).
 *   A page index outside [0, num_pages) reads zeros and is reported as
 *   FMHA_ERR_DEVICE_INDEX by fmha_get_device_error().                       */
fmha_status fmha_fwd_paged(const fmha_args* args, const int32_t* page_table, int32_t num_pages,
                           int32_t page_size, int32_t max_pages_per_seq, const uint8_t* mask,
                           int64_t mask_stride_b, int64_t mask_stride_h, struct CUstream_st* stream);

/* Decode-shaped attention: few query tokens per sequence (Sq = 1 .. a few
 * dozen), GQA-packed query tiles and split-KV ("FlashInfer block-sparse
 * attention with PrimTS", section 1: the query tile is the query block times
 * the query heads per KV head).
 *   Computes exactly what fmha_fwd / fmha_fwd_paged compute (same args, same
 *   causal alignment, same optional block mask), but puts the query heads of
 *   one KV head into one 128-row tile (row = token * G + head in group,
 *   G = Hq / Hkv, a power of two <= 128) so every K/V tile is read once per
 *   KV head, and splits the KV range across CTAs.
 *   page_table: NULL = contiguous K/V [B, Skv, Hkv, D]; otherwise the paged
 *     pool as in fmha_fwd_paged (num_pages, page_size, max_pages_per_seq).
 *   num_splits: KV splits per (b, KV head, query-tile pair); <= 0 chooses
 *     about one CTA per SM. The count used is fmha_decode_num_splits().
 *   Split j takes the kept KV tiles (after causality and the block mask) of
 *     ranks [j*per, (j+1)*per), per = ceil(kept / splits). When all Sq * G
 *     rows fit one 128-row tile, the CTA's two query tiles take alternate
 *     kept tiles of the split, each as its own partial.
 *   workspace: device memory owned by the caller, 16-byte aligned, at least
 *     fmha_decode_workspace_bytes(args, num_splits) bytes (0 when there is a
 *     single partial: then workspace may be NULL). With several partials each
 *     writes O/l in fp32 and its log-sum-exp there, and a second kernel merges
 *     them: lse = log sum_j exp(lse_j), O = sum_j exp(lse_j - lse) O_j.
 *   Supported: D = 128, Skv <= 131072, Sq * Hq / Hkv < 2^31 packed rows
 *   (fmha_decode_num_splits and fmha_decode_workspace_bytes return 0 beyond
 *   it); Q/K/V BF16/BF16/BF16, BF16/BF16/E4M3
 *   or E4M3/E4M3/E4M3 with the scale kinds of fmha_fwd; p_terms 0 or 1.
 *   Errors: FMHA_ERR_UNSUPPORTED for other shapes/dtypes, FMHA_ERR_INVALID_ARG
 *   for a missing or short workspace; device errors as in fmha_fwd_paged.   */
fmha_status fmha_fwd_decode(const fmha_args* args, const int32_t* page_table, int32_t num_pages,
                            int32_t page_size, int32_t max_pages_per_seq, const uint8_t* mask,
                            int64_t mask_stride_b, int64_t mask_stride_h, int32_t num_splits, void* workspace,
                            size_t workspace_bytes, struct CUstream_st* stream);

/* Per-token NVFP4 quantization of a BF16 matrix [rows, K] ("FlashInfer
 * per-token NVFP4 quantization kernel"): E2M1 element codes, one E4M3 scale
 * per 16 consecutive elements and one fp32 scale per row (token):
 *   s_t  = amax_row / 2688  (448 * 6; 1 when the row is zero)
 *   sb   = E4M3((amax_block / s_t) / 6)      IEEE fp32 divisions, RN, satfinite
 *   e    = decode(sb) * s_t
 *   code = E2M1(x / e)  (fast_math != 0: E2M1(x * (1 / e))), 0 when e == 0;
 *   E2M1 rounds to nearest even and saturates to +-6.
 *   Dequantization: x ~= e2m1(code) * decode(sb) * s_t.
 * src: device BF16, 16-byte aligned, row stride in elements (multiple of 8).
 * codes: device uint8 [rows, K/2], element 2i in the low nibble of byte i,
 *   8-byte aligned, row stride in bytes (multiple of 8).
 * block_scales: device uint8 E4M3 [rows, K/16], row stride in bytes.
 * token_scales: device float [rows].
 * K: multiple of 16, at most 16384. The caller owns every buffer; nothing is
 * allocated. FMHA_ERR_UNSUPPORTED for other K, FMHA_ERR_INVALID_ARG for bad
 * pointers, alignment or strides.                                           */
fmha_status fmha_quantize_nvfp4(const void* src, int64_t src_row_stride, int32_t rows, int32_t K, uint8_t* codes,
                                int64_t codes_row_stride, uint8_t* block_scales, int64_t block_scales_row_stride,
                                float* token_scales, int32_t fast_math, struct CUstream_st* stream);

/* Workspace bytes fmha_fwd_decode needs for these args and num_splits
 * (0: a single split, or invalid sizes). Host only.                         */
size_t fmha_decode_workspace_bytes(const fmha_args* args, int32_t num_splits);

/* Number of KV splits fmha_fwd_decode uses for these args and num_splits
 * (0 for invalid sizes). Host only; queries the current device's SM count. */
int32_t fmha_decode_num_splits(const fmha_args* args, int32_t num_splits);

/* Synchronises `stream`, then returns and clears the current device's error
 * word: FMHA_OK, FMHA_ERR_TIMEOUT or FMHA_ERR_DEVICE_INDEX (or FMHA_ERR_CUDA if
 * the synchronisation itself failed). */
fmha_status fmha_get_device_error(struct CUstream_st* stream);

/* Static string naming a status code. */
const char* fmha_status_string(fmha_status status);

/* One-line reason for the last non-OK status returned on this host thread. */
const char* fmha_last_error_message(void);

/* Test hook: sets the bound on every device-side wait, in GPU clock cycles,
 * for launches made after the call (0 restores the default of about one
 * second). Lets a test make a wait run out quickly. Process-wide.          */
void fmha_set_wait_timeout_cycles(uint64_t cycles);

#ifdef __cplusplus
}
#endif

#endif /* FMHA_H_ */
