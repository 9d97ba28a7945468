// api.cu -- the C ABI of libfmha.so (include/fmha.h): argument validation,
// TMA descriptor construction, kernel selection and the device error word.
//
// The kernel key is the (Q, K, V, O) dtype tuple, the head dim and the K/V
// source, fixed at compile time ("FlashInfer DiT optimization: SageAttention
// and Int8/FP8 mixed-precision kernels", section 1: kernels are selected by
// separate Q/K/V/O dtypes plus the scale-factor granularities). TMA
// descriptors are built on the host per call and passed to the kernel as
// __grid_constant__ parameters ("FlashInfer DeepSeek-V4 sparse-MLA: Cake
// backend", section 1). An 8-bit operand is described to the TMA as plain
// bytes; only the tensor-core instruction gives the bytes a type ("FlashInfer
// DiT optimization ...", section 3).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fmha_internal.h"

namespace fmha {
cudaError_t launch_attention_bf16(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&,
                                  const CUtensorMap&, const CUtensorMap&, cudaStream_t);
cudaError_t launch_attention_pv8(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&,
                                 const CUtensorMap&, const CUtensorMap&, cudaStream_t);
cudaError_t launch_attention_fp8(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&,
                                 const CUtensorMap&, const CUtensorMap&, cudaStream_t);
cudaError_t launch_attention_sage(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&,
                                  const CUtensorMap&, const CUtensorMap&, cudaStream_t);
cudaError_t launch_attention_d192(int qk, int pv, bool paged, const AttnParams&, const CUtensorMap&,
                                  const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, cudaStream_t);

cudaError_t launch_attention(int qk_kind, int pv_kind, int D, bool paged, const AttnParams& p,
                             const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, cudaStream_t s) {
  if (qk_kind == QK_BF16 && pv_kind == PV_BF16) return launch_attention_bf16(D, paged, p, tq, tk, tv, to, s);
  if (qk_kind == QK_BF16 && pv_kind == PV_E4M3) return launch_attention_pv8(D, paged, p, tq, tk, tv, to, s);
  if (qk_kind == QK_E4M3 && pv_kind == PV_E4M3) return launch_attention_fp8(D, paged, p, tq, tk, tv, to, s);
  return launch_attention_sage(D, paged, p, tq, tk, tv, to, s);
}
}  // namespace fmha

namespace {

using namespace fmha;

// One error word per device: a file-scope device variable, so the library
// needs no allocation for it. Host code reaches it through its symbol address.
__device__ uint32_t g_device_error_word;

thread_local char g_msg[512] = "";
std::atomic<uint64_t> g_wait_cycles{0};

fmha_status fail(fmha_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

fmha_status ok_status() {
  g_msg[0] = '\0';
  return FMHA_OK;
}

uint32_t* device_error_word(cudaError_t* err) {
  constexpr int kMaxDevices = 64;
  static uint32_t* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_device_error_word);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint32_t*>(p);
  }
  return addr[dev];
}

// ------------------------------------------------------ TMA descriptors ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(cudaError_t* err) {
  static EncodeTiledFn fn = nullptr;
  static cudaError_t status = cudaSuccess;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    status = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (status == cudaSuccess && q != cudaDriverEntryPointSuccess) status = cudaErrorSymbolNotFound;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  *err = status;
  return fn;
}

// RANK-d map (dims innermost first, RANK = 4 or 5) with 128-byte swizzle.
// Strides in elements for dims 1..RANK-1. Size-1 dims get a packed stride so
// the descriptor stays valid whatever the caller's stride.
template <int RANK>
fmha_status make_map_n(CUtensorMap* map, void* base, int elem_bytes, const uint64_t (&dims)[RANK],
                       const int64_t (&strides_elems)[RANK - 1], const uint32_t (&box)[RANK], const char* what,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cudaError_t e;
  EncodeTiledFn fn = encode_fn(&e);
  if (fn == nullptr) return fail(FMHA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable: %s", cudaGetErrorString(e));
  cuuint64_t gdim[RANK];
  cuuint64_t gstride[RANK - 1];
  cuuint32_t ebox[RANK];
  cuuint32_t bdim[RANK];
  uint64_t packed = dims[0] * elem_bytes;
  for (int i = 0; i < RANK; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    ebox[i] = 1;
  }
  for (int i = 0; i < RANK - 1; ++i) {
    uint64_t s = static_cast<uint64_t>(strides_elems[i]) * elem_bytes;
    if (dims[i + 1] == 1) s = (packed + 15) / 16 * 16;
    gstride[i] = s;
    packed = s * dims[i + 1];
  }
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = fn(map, dt, RANK, base, gdim, gstride, bdim, ebox, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FMHA_ERR_INVALID_ARG, "TMA descriptor for %s rejected (CUresult %d)", what, (int)r);
  return FMHA_OK;
}
fmha_status make_map(CUtensorMap* map, void* base, int elem_bytes, const uint64_t (&dims)[4],
                     const int64_t (&strides_elems)[3], const uint32_t (&box)[4], const char* what) {
  return make_map_n<4>(map, base, elem_bytes, dims, strides_elems, box, what);
}

int elem_bytes(int dt) {
  switch (dt) {
    case FMHA_BF16:
    case FMHA_FP16: return 2;
    case FMHA_FP32: return 4;
    case FMHA_E4M3:
    case FMHA_INT8: return 1;
    default: return 0;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks a [B, S, H, D] operand: pointer, alignment, strides. Size-1 dims' strides are free.
fmha_status check_tensor(const fmha_tensor& t, const char* name, int B, int S, int H, int D) {
  if (t.reserved != 0) return fail(FMHA_ERR_INVALID_ARG, "%s.reserved must be 0", name);
  const int eb = elem_bytes(t.dtype);
  if (eb == 0) return fail(FMHA_ERR_INVALID_ARG, "%s has an unknown dtype %d", name, t.dtype);
  if (t.ptr == nullptr) return fail(FMHA_ERR_INVALID_ARG, "%s.ptr is NULL", name);
  if (!aligned16(t.ptr)) return fail(FMHA_ERR_INVALID_ARG, "%s.ptr is not 16-byte aligned", name);
  const int64_t st[3] = {t.stride_b, t.stride_s, t.stride_h};
  const int n[3] = {B, S, H};
  const char* nm[3] = {"stride_b", "stride_s", "stride_h"};
  for (int i = 0; i < 3; ++i) {
    if (n[i] <= 1) continue;
    if (st[i] <= 0) return fail(FMHA_ERR_INVALID_ARG, "%s.%s must be positive", name, nm[i]);
    if ((st[i] * eb) % 16 != 0) return fail(FMHA_ERR_INVALID_ARG, "%s.%s is not a multiple of 16 bytes", name, nm[i]);
    if (st[i] * eb >= (int64_t(1) << 40)) return fail(FMHA_ERR_INVALID_ARG, "%s.%s too large", name, nm[i]);
  }
  if (t.stride_h > 0 && H > 1 && t.stride_h < D)
    return fail(FMHA_ERR_INVALID_ARG, "%s.stride_h smaller than D (rows overlap)", name);
  return FMHA_OK;
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

fmha_status check_sf(const fmha_sf& sf, const char* name, bool allow_head, bool allow_tensor, bool allow_block,
                     int block_multiple, bool allow_channel) {
  switch (sf.kind) {
    case FMHA_SF_NONE: return FMHA_OK;
    case FMHA_SF_PER_TENSOR:
      if (!allow_tensor) return fail(FMHA_ERR_UNSUPPORTED, "%s: per-tensor scales not supported here", name);
      break;
    case FMHA_SF_PER_HEAD:
      if (!allow_head) return fail(FMHA_ERR_UNSUPPORTED, "%s: per-head scales not supported here", name);
      break;
    case FMHA_SF_PER_TOKEN_BLOCK:
      if (!allow_block) return fail(FMHA_ERR_UNSUPPORTED, "%s: token-block scales not supported here", name);
      if (sf.rows_per_block <= 0 || sf.rows_per_block % block_multiple != 0)
        return fail(FMHA_ERR_UNSUPPORTED, "%s.rows_per_block must be a positive multiple of %d", name,
                    block_multiple);
      break;
    case FMHA_SF_PER_CHANNEL:
      if (!allow_channel) return fail(FMHA_ERR_UNSUPPORTED, "%s: per-channel scales not supported here", name);
      break;
    default: return fail(FMHA_ERR_INVALID_ARG, "%s.kind %d unknown", name, sf.kind);
  }
  if (sf.ptr == nullptr) return fail(FMHA_ERR_INVALID_ARG, "%s.ptr is NULL", name);
  if ((reinterpret_cast<uintptr_t>(sf.ptr) & 3u) != 0) return fail(FMHA_ERR_INVALID_ARG, "%s.ptr misaligned", name);
  return FMHA_OK;
}

struct PagedArgs {
  const int32_t* page_table;
  int32_t num_pages, page_size, max_pages_per_seq;
};

struct DecodeArgs {
  int32_t num_splits;  // <= 0: chosen here
  void* workspace;
  size_t workspace_bytes;
};

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// The decode path packs Sq * (Hq / Hkv) query rows per KV head, counted in 32 bits.
bool packed_rows_fit(int Sq, int Hq, int Hkv) {
  return static_cast<int64_t>(Sq) * (Hq / Hkv) <= INT32_MAX;
}

// Split plan of the decode path: KV tiles per split and the split count
// (no trailing empty split). Automatic: about one CTA per SM, at least two KV
// tiles per split.
struct SplitPlan {
  int n_units, n_splits, split_tiles, interleave, n_parts;
  size_t workspace_bytes;
};
SplitPlan plan_splits(int B, int Hq, int Hkv, int Sq, int Skv, int D, int requested) {
  SplitPlan sp;
  const int group = Hq / Hkv;
  const int units = ceil_div(Sq * group, 128);
  // All rows in one 128-row tile: the CTA's second query tile takes the same
  // rows and alternate KV tiles (its own partial), so both softmax
  // warpgroups work.
  sp.interleave = units == 1 ? 1 : 0;
  sp.n_units = sp.interleave ? 1 : ceil_div(units, 2);
  const int n_kv = ceil_div(Skv, 128);
  int splits = requested;
  if (splits <= 0) {
    const long long base = static_cast<long long>(B) * Hkv * sp.n_units;
    splits = static_cast<int>(std::max<long long>(1, sm_count() / std::max<long long>(1, base)));
    splits = std::min(splits, std::max(1, n_kv / 2));
  }
  splits = std::max(1, std::min(splits, std::max(1, n_kv)));
  sp.split_tiles = std::max(1, ceil_div(n_kv, splits));
  sp.n_splits = std::max(1, ceil_div(n_kv, sp.split_tiles));
  sp.n_parts = sp.n_splits * (sp.interleave ? 2 : 1);
  sp.workspace_bytes = sp.n_parts > 1 ? static_cast<size_t>(sp.n_parts) * B * Sq * Hq * (size_t(D) + 1) * 4 + 16 : 0;
  return sp;
}

fmha_status run_attention(const fmha_args* a, const uint8_t* mask, int64_t msb, int64_t msh, const PagedArgs* pg,
                          cudaStream_t stream, const DecodeArgs* dec = nullptr) {
  if (a == nullptr) return fail(FMHA_ERR_INVALID_ARG, "args is NULL");
  const int B = a->B, Hq = a->Hq, Hkv = a->Hkv, Sq = a->Sq, Skv = a->Skv, D = a->D;
  if (B < 0 || Hq < 0 || Hkv < 0 || Sq < 0 || Skv < 0) return fail(FMHA_ERR_INVALID_ARG, "negative size");
  if (B == 0 || Hq == 0 || Sq == 0) return ok_status();  // nothing to compute
  if (Hkv == 0 || Hq % Hkv != 0) return fail(FMHA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (D != 64 && D != 128 && D != 192) return fail(FMHA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128, 192)", D);
  const int Dv = a->Dv == 0 ? D : a->Dv;  // head dim of V and O
  if (D == 192 ? Dv != 128 : Dv != D)
    return fail(FMHA_ERR_UNSUPPORTED, "V / O head dim %d with QK head dim %d (supported: equal, or 192 / 128)", Dv, D);

  // dtype tuple
  int qk, pv;
  const int dq = a->q.dtype, dk = a->k.dtype, dv = a->v.dtype, dout = a->o.dtype;
  if (dq == FMHA_BF16 && dk == FMHA_BF16) qk = QK_BF16;
  else if (dq == FMHA_E4M3 && dk == FMHA_E4M3) qk = QK_E4M3;
  else if (dq == FMHA_INT8 && dk == FMHA_INT8) qk = QK_INT8;
  else return fail(FMHA_ERR_UNSUPPORTED, "Q/K dtypes (%d, %d) unsupported", dq, dk);
  if (dv == FMHA_BF16) pv = PV_BF16;
  else if (dv == FMHA_E4M3) pv = PV_E4M3;
  else return fail(FMHA_ERR_UNSUPPORTED, "V dtype %d unsupported", dv);
  const bool tuple_ok = (qk == QK_BF16) || pv == PV_E4M3;
  if (!tuple_ok || (dout != FMHA_BF16 && dout != FMHA_E4M3))
    return fail(FMHA_ERR_UNSUPPORTED, "dtype tuple (q %d, k %d, v %d, o %d) unsupported", dq, dk, dv, dout);
  if (D == 64 && !(qk == QK_BF16 && pv == PV_BF16)) return fail(FMHA_ERR_UNSUPPORTED, "D=64 needs BF16 Q/K/V");
  if (D == 192 && (qk == QK_INT8 || dout != FMHA_BF16 || a->p_terms == 2 || dec != nullptr))
    return fail(FMHA_ERR_UNSUPPORTED, "D=192: BF16 or E4M3 Q/K, one-term P, BF16 O, not decode");
  // One query tile per CTA: its kept KV tiles are dealt to the two softmax
  // warpgroups through a 1024-bit keep set.
  if (query_tiles_per_cta(qk, D) == 1 && ceil_div(Skv, 128) > 1024)
    return fail(FMHA_ERR_UNSUPPORTED, "D=192 with BF16 Q/K: Skv %d > 131072", Skv);
  const bool packed = dec != nullptr;
  const bool o8 = dout == FMHA_E4M3;
  if (o8 && Dv != 128) return fail(FMHA_ERR_UNSUPPORTED, "E4M3 O needs D = 128");
  if (o8 && packed) return fail(FMHA_ERR_UNSUPPORTED, "decode: O must be BF16");
  const int group = Hq / Hkv;
  int group_shift = 0;
  if (packed) {
    while ((1 << group_shift) < group) ++group_shift;
    if ((1 << group_shift) != group || group > 128)
      return fail(FMHA_ERR_UNSUPPORTED, "decode: Hq / Hkv = %d must be a power of two <= 128", group);
    if (D != 128) return fail(FMHA_ERR_UNSUPPORTED, "decode: head dim %d (supported: 128)", D);
    if (qk == QK_INT8) return fail(FMHA_ERR_UNSUPPORTED, "decode: INT8 Q/K not supported");
    if (a->p_terms == 2) return fail(FMHA_ERR_UNSUPPORTED, "decode: p_terms = 2 not supported");
    if (ceil_div(Skv, 128) > 1024) return fail(FMHA_ERR_UNSUPPORTED, "decode: Skv %d > 131072", Skv);
    if (!packed_rows_fit(Sq, Hq, Hkv))
      return fail(FMHA_ERR_UNSUPPORTED, "decode: Sq * Hq / Hkv packed rows exceed 2^31 - 1");
  }

  // scale factors
  fmha_status st;
  const bool q8 = qk != QK_BF16, v8 = pv == PV_E4M3;
  if ((st = check_sf(a->sf_q, "sf_q", q8, q8, q8, 1, false)) != FMHA_OK) return st;
  if ((st = check_sf(a->sf_k, "sf_k", q8, q8, q8, 32, false)) != FMHA_OK) return st;
  if ((st = check_sf(a->sf_v, "sf_v", v8, v8, false, 1, v8)) != FMHA_OK) return st;
  if ((st = check_sf(a->sf_p, "sf_p", false, v8, v8, 128, false)) != FMHA_OK) return st;
  if ((st = check_sf(a->sf_o, "sf_o", false, o8, false, 1, false)) != FMHA_OK) return st;
  if (a->p_terms < 0 || a->p_terms > 2) return fail(FMHA_ERR_INVALID_ARG, "p_terms must be 0, 1 or 2");
  if (a->p_terms == 2 && !v8) return fail(FMHA_ERR_INVALID_ARG, "p_terms = 2 needs an E4M3 V");

  // tensors
  const bool paged = pg != nullptr;
  if ((st = check_tensor(a->q, "q", B, Sq, Hq, D)) != FMHA_OK) return st;
  if ((st = check_tensor(a->o, "o", B, Sq, Hq, Dv)) != FMHA_OK) return st;
  if (paged) {
    if (pg->page_size != 16 && pg->page_size != 32 && pg->page_size != 64 && pg->page_size != 128)
      return fail(FMHA_ERR_UNSUPPORTED, "page_size %d (supported: 16, 32, 64, 128)", pg->page_size);
    if (pg->num_pages <= 0) return fail(FMHA_ERR_INVALID_ARG, "num_pages must be positive");
    if (pg->page_table == nullptr) return fail(FMHA_ERR_INVALID_ARG, "page_table is NULL");
    if ((reinterpret_cast<uintptr_t>(pg->page_table) & 3u) != 0)
      return fail(FMHA_ERR_INVALID_ARG, "page_table misaligned");
    if (pg->max_pages_per_seq < ceil_div(Skv, pg->page_size))
      return fail(FMHA_ERR_INVALID_ARG, "max_pages_per_seq %d < ceil(Skv / page_size)", pg->max_pages_per_seq);
    if ((st = check_tensor(a->k, "k", pg->num_pages, pg->page_size, Hkv, D)) != FMHA_OK) return st;
    if ((st = check_tensor(a->v, "v", pg->num_pages, pg->page_size, Hkv, Dv)) != FMHA_OK) return st;
  } else if (Skv > 0) {
    if ((st = check_tensor(a->k, "k", B, Skv, Hkv, D)) != FMHA_OK) return st;
    if ((st = check_tensor(a->v, "v", B, Skv, Hkv, Dv)) != FMHA_OK) return st;
  }
  if (a->lse != nullptr && (reinterpret_cast<uintptr_t>(a->lse) & 3u) != 0)
    return fail(FMHA_ERR_INVALID_ARG, "lse misaligned");
  if (mask != nullptr && (msb < 0 || msh < 0)) return fail(FMHA_ERR_INVALID_ARG, "mask strides must be >= 0");
  if (mask != nullptr && ceil_div(Skv, 128) > 1024)
    return fail(FMHA_ERR_UNSUPPORTED, "block mask: Skv %d > 131072 (1024 KV blocks)", Skv);

  // TMA descriptors
  const int eqk = qk == QK_BF16 ? 2 : 1, ev = pv == PV_BF16 ? 2 : 1;
  CUtensorMap tq, tk, tv, to;
  if (packed) {  // (d, head in group, kv head, token, batch); box = all heads of a group x 128 / group tokens
    const uint64_t dims[5] = {uint64_t(D), uint64_t(group), uint64_t(Hkv), uint64_t(Sq), uint64_t(B)};
    const int64_t qstr[4] = {a->q.stride_h, a->q.stride_h * group, a->q.stride_s, a->q.stride_b};
    const uint32_t box[5] = {uint32_t(128 / eqk), uint32_t(group), 1, uint32_t(128 / group), 1};
    if ((st = make_map_n<5>(&tq, a->q.ptr, eqk, dims, qstr, box, "q")) != FMHA_OK) return st;
    const int64_t ostr[4] = {a->o.stride_h, a->o.stride_h * group, a->o.stride_s, a->o.stride_b};
    const uint32_t obox[5] = {64, uint32_t(group), 1, uint32_t(128 / group), 1};
    if ((st = make_map_n<5>(&to, a->o.ptr, 2, dims, ostr, obox, "o")) != FMHA_OK) return st;
  } else {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(Hq), uint64_t(Sq), uint64_t(B)};
    const int64_t strides[3] = {a->q.stride_h, a->q.stride_s, a->q.stride_b};
    const uint32_t box[4] = {uint32_t(128 / eqk), 1, 128, 1};
    if ((st = make_map(&tq, a->q.ptr, eqk, dims, strides, box, "q")) != FMHA_OK) return st;
    const uint64_t odims[4] = {uint64_t(Dv), uint64_t(Hq), uint64_t(Sq), uint64_t(B)};
    const int64_t ostr[3] = {a->o.stride_h, a->o.stride_s, a->o.stride_b};
    // BF16 O: 64-column (128-byte) boxes; E4M3 O: the whole 128-byte row.
    const uint32_t obox[4] = {o8 ? 128u : 64u, 1, 128, 1};
    if ((st = make_map(&to, a->o.ptr, o8 ? 1 : 2, odims, ostr, obox, "o")) != FMHA_OK) return st;
  }
  if (Skv == 0) {  // no key is ever loaded; any valid descriptor will do
    tk = tq;
    tv = tq;
  } else {
    const fmha_tensor* kv[2] = {&a->k, &a->v};
    CUtensorMap* out[2] = {&tk, &tv};
    for (int i = 0; i < 2; ++i) {
      const int eb = i == 0 ? eqk : ev;
      const int dd = i == 0 ? D : Dv;
      const int64_t strides[3] = {kv[i]->stride_h, kv[i]->stride_s, kv[i]->stride_b};
      if (paged) {
        const uint64_t dims[4] = {uint64_t(dd), uint64_t(Hkv), uint64_t(pg->page_size), uint64_t(pg->num_pages)};
        const uint32_t box[4] = {uint32_t(128 / eb), 1, uint32_t(pg->page_size), 1};
        st = make_map(out[i], kv[i]->ptr, eb, dims, strides, box, i == 0 ? "k pool" : "v pool");
      } else {
        const uint64_t dims[4] = {uint64_t(dd), uint64_t(Hkv), uint64_t(Skv), uint64_t(B)};
        const uint32_t box[4] = {uint32_t(128 / eb), 1, 128, 1};
        st = make_map(out[i], kv[i]->ptr, eb, dims, strides, box, i == 0 ? "k" : "v");
      }
      if (st != FMHA_OK) return st;
    }
  }

  AttnParams p;
  memset(&p, 0, sizeof(p));
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Sq = Sq; p.Skv = Skv; p.group = Hq / Hkv;
  p.n_q_blocks = ceil_div(Sq, 128);
  p.n_kv_blocks = ceil_div(Skv, 128);
  p.pair_mode = query_tiles_per_cta(qk, D) == 1 ? SINGLE : (p.group % 2 == 0) ? PAIR_HEADS : PAIR_ROWS;
  p.n_units = p.pair_mode == PAIR_ROWS ? ceil_div(p.n_q_blocks, 2) : p.n_q_blocks;
  p.causal = a->causal != 0;
  const float scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / std::sqrt(float(D));
  p.scale_log2 = scale * 1.4426950408889634f;
  p.sf_q = a->sf_q.ptr; p.sf_q_kind = a->sf_q.kind; p.sf_q_rpb = a->sf_q.rows_per_block > 0 ? a->sf_q.rows_per_block : 1;
  p.sf_q_nblk = ceil_div(Sq, p.sf_q_rpb);
  p.sf_k = a->sf_k.ptr; p.sf_k_kind = a->sf_k.kind; p.sf_k_rpb = a->sf_k.rows_per_block > 0 ? a->sf_k.rows_per_block : 1;
  p.sf_k_nblk = ceil_div(Skv, p.sf_k_rpb);
  p.sf_v = a->sf_v.ptr; p.sf_v_kind = a->sf_v.kind;
  p.sf_p = a->sf_p.ptr; p.sf_p_kind = a->sf_p.kind; p.sf_p_rpb = a->sf_p.rows_per_block > 0 ? a->sf_p.rows_per_block : 1;
  p.sf_p_nblk = ceil_div(Sq, p.sf_p_rpb);
  p.lse = a->lse;
  p.p_terms = a->p_terms == 2 ? 2 : 1;
  p.o8 = o8 ? 1 : 0;
  p.sf_o = a->sf_o.kind == FMHA_SF_PER_TENSOR ? a->sf_o.ptr : nullptr;
  p.mask = mask; p.mask_sb = msb; p.mask_sh = msh;
  if (paged) {
    p.page_table = pg->page_table; p.num_pages = pg->num_pages; p.page_size = pg->page_size;
    p.max_pages_per_seq = pg->max_pages_per_seq;
  }
  cudaError_t e;
  p.err = device_error_word(&e);
  if (p.err == nullptr) return fail(FMHA_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
  const uint64_t wc = g_wait_cycles.load();
  p.wait_cycles = wc ? wc : kDefaultWaitCycles;

  if (packed) {
    const SplitPlan sp = plan_splits(B, Hq, Hkv, Sq, Skv, D, dec->num_splits);
    p.packed = 1;
    p.group_shift = group_shift;
    p.n_rows = Sq * group;
    // At most 16 packed rows (all in one tile) with BF16 P: the 16-lane softmax pass.
    p.narrow = (pv == PV_BF16 && sp.interleave && p.n_rows <= 16) ? 1 : 0;
    p.n_units = sp.n_units;
    p.n_splits = sp.n_splits;
    p.split_tiles = sp.split_tiles;
    p.kv_interleave = sp.interleave;
    p.n_parts = sp.n_parts;
    if (sp.n_parts > 1) {
      if (dec->workspace == nullptr || !aligned16(dec->workspace))
        return fail(FMHA_ERR_INVALID_ARG, "decode: workspace is NULL or not 16-byte aligned (%d partials)",
                    sp.n_parts);
      if (dec->workspace_bytes < sp.workspace_bytes)
        return fail(FMHA_ERR_INVALID_ARG, "decode: workspace of %zu bytes < %zu needed", dec->workspace_bytes,
                    sp.workspace_bytes);
      p.o_part = static_cast<float*>(dec->workspace);
      const size_t o_elems = static_cast<size_t>(sp.n_parts) * B * Sq * Hq * D;
      p.lse_part = p.o_part + o_elems;
    }
    if (static_cast<long long>(p.n_units) * p.n_splits * Hkv * B >= (1ll << 31))
      return fail(FMHA_ERR_UNSUPPORTED, "grid too large");
    e = launch_attention_packed(qk, pv, paged, p, tq, tk, tv, to, stream);
    if (e != cudaSuccess) return fail(FMHA_ERR_CUDA, "decode attention launch: %s", cudaGetErrorString(e));
    if (sp.n_parts > 1) {
      MergeParams mp;
      mp.o_part = p.o_part;
      mp.lse_part = p.lse_part;
      mp.o = static_cast<uint16_t*>(a->o.ptr);
      mp.o_sb = a->o.stride_b; mp.o_ss = a->o.stride_s; mp.o_sh = a->o.stride_h;
      mp.lse = a->lse;
      mp.n_splits = sp.n_parts; mp.B = B; mp.Sq = Sq; mp.Hq = Hq; mp.D = D;
      e = launch_split_merge(mp, stream);
      if (e != cudaSuccess) return fail(FMHA_ERR_CUDA, "split merge launch: %s", cudaGetErrorString(e));
    }
    return ok_status();
  }
  const long long head_units = p.pair_mode == PAIR_HEADS ? Hq / 2 : Hq;
  if (static_cast<long long>(p.n_units) * head_units * B >= (1ll << 31))
    return fail(FMHA_ERR_UNSUPPORTED, "grid too large");
  e = D == 192 ? launch_attention_d192(qk, pv, paged, p, tq, tk, tv, to, stream)
               : launch_attention(qk, pv, D, paged, p, tq, tk, tv, to, stream);
  if (e != cudaSuccess) return fail(FMHA_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
  return ok_status();
}

// Token rows one CTA of the channel-mean kernel sums: 256 KB of BF16 input, 64
// rows per thread. At 48 registers a thread, 5 CTAs of 256 fit an SM; 128 KB
// chunks gave the Sage workload's K (B1 H24 S16384) 768 CTAs, a second wave of
// 28 on 148 SMs, while 256 KB chunks give 384 CTAs in one wave (2-3 per SM,
// 64-96 KB of loads in flight each) and half the partials for the final sum.
int mean_rows_per_cta(int D) { return D >= 8 ? 131072 / D : 1; }

fmha_status quantize_impl(const fmha_tensor* src, const float* shift, const fmha_tensor* dst, const fmha_sf* sf,
                          int32_t B, int32_t S, int32_t H, int32_t D, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream);

size_t quant_groups(int kind, int B, int H, int D) {
  switch (kind) {
    case FMHA_SF_PER_TENSOR: return 1;
    case FMHA_SF_PER_HEAD: return size_t(B) * H;
    case FMHA_SF_PER_CHANNEL: return size_t(B) * H * D;
    default: return 0;
  }
}

}  // namespace

extern "C" {

fmha_status fmha_quantize_blockwise(const fmha_tensor* src, const fmha_tensor* dst, const fmha_sf* sf, int32_t B,
                                    int32_t S, int32_t H, int32_t D, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream) {
  return quantize_impl(src, nullptr, dst, sf, B, S, H, D, workspace, workspace_bytes, stream);
}

fmha_status fmha_quantize_blockwise_shifted(const fmha_tensor* src, const float* shift, const fmha_tensor* dst,
                                            const fmha_sf* sf, int32_t B, int32_t S, int32_t H, int32_t D,
                                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (shift == nullptr) return fail(FMHA_ERR_INVALID_ARG, "shift is NULL");
  if (reinterpret_cast<uintptr_t>(shift) & 15u) return fail(FMHA_ERR_INVALID_ARG, "shift must be 16-byte aligned");
  return quantize_impl(src, shift, dst, sf, B, S, H, D, workspace, workspace_bytes, stream);
}

size_t fmha_channel_mean_workspace_bytes(int32_t B, int32_t S, int32_t H, int32_t D) {
  if (B <= 0 || S <= 0 || H <= 0 || D < 8) return 0;
  return size_t(B) * H * ceil_div(S, mean_rows_per_cta(D)) * D * sizeof(double);
}

fmha_status fmha_channel_mean(const fmha_tensor* src, float* mean, int32_t B, int32_t S, int32_t H, int32_t D,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (src == nullptr) return fail(FMHA_ERR_INVALID_ARG, "NULL argument");
  if (B < 0 || S < 0 || H < 0 || D < 0) return fail(FMHA_ERR_INVALID_ARG, "negative size");
  if (src->dtype != FMHA_BF16) return fail(FMHA_ERR_UNSUPPORTED, "channel mean input must be BF16");
  if (D < 8 || D > 2048 || (D & (D - 1)) != 0)
    return fail(FMHA_ERR_UNSUPPORTED, "channel mean needs D a power of two in [8, 2048]");
  if (B == 0 || H == 0) return ok_status();
  if (mean == nullptr || (reinterpret_cast<uintptr_t>(mean) & 3u))
    return fail(FMHA_ERR_INVALID_ARG, "mean is NULL or misaligned");
  if (S > 0) {
    fmha_status st;
    if ((st = check_tensor(*src, "src", B, S, H, D)) != FMHA_OK) return st;
    const size_t need = fmha_channel_mean_workspace_bytes(B, S, H, D);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(FMHA_ERR_INVALID_ARG, "workspace needs %zu bytes", need);
    if (reinterpret_cast<uintptr_t>(workspace) & 7u) return fail(FMHA_ERR_INVALID_ARG, "workspace misaligned");
  }
  QuantParams p;
  memset(&p, 0, sizeof(p));
  p.src = static_cast<const uint16_t*>(src->ptr);
  p.s_sb = src->stride_b; p.s_ss = src->stride_s; p.s_sh = src->stride_h;
  p.B = B; p.S = S; p.H = H; p.D = D;
  p.rows_per_cta = mean_rows_per_cta(D);
  p.n_chunks = S > 0 ? ceil_div(S, p.rows_per_cta) : 0;
  p.partial = static_cast<double*>(workspace);
  p.mean = mean;
  if (static_cast<int64_t>(p.n_chunks) > 65535 || H > 65535 || B > 65535)
    return fail(FMHA_ERR_UNSUPPORTED, "grid too large");
  cudaError_t e = launch_channel_mean(p, stream);
  if (e != cudaSuccess) return fail(FMHA_ERR_CUDA, "channel mean launch: %s", cudaGetErrorString(e));
  return ok_status();
}

}  // extern "C"

namespace {

fmha_status quantize_impl(const fmha_tensor* src, const float* shift, const fmha_tensor* dst, const fmha_sf* sf,
                          int32_t B, int32_t S, int32_t H, int32_t D, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
  if (src == nullptr || dst == nullptr || sf == nullptr) return fail(FMHA_ERR_INVALID_ARG, "NULL argument");
  if (B < 0 || S < 0 || H < 0 || D < 0) return fail(FMHA_ERR_INVALID_ARG, "negative size");
  if (src->dtype != FMHA_BF16) return fail(FMHA_ERR_UNSUPPORTED, "quantizer input must be BF16");
  if (dst->dtype != FMHA_INT8 && dst->dtype != FMHA_E4M3)
    return fail(FMHA_ERR_UNSUPPORTED, "quantizer output must be INT8 or E4M3");
  if (D % 8 != 0 || D > 2048 || D == 0) return fail(FMHA_ERR_UNSUPPORTED, "D must be a multiple of 8 in [8, 2048]");
  const int kind = sf->kind;
  if (kind != FMHA_SF_PER_TENSOR && kind != FMHA_SF_PER_HEAD && kind != FMHA_SF_PER_TOKEN_BLOCK &&
      kind != FMHA_SF_PER_CHANNEL)
    return fail(FMHA_ERR_INVALID_ARG, "sf.kind %d is not a quantizer granularity", kind);
  if (kind == FMHA_SF_PER_TOKEN_BLOCK && sf->rows_per_block <= 0)
    return fail(FMHA_ERR_INVALID_ARG, "rows_per_block must be positive");
  if (kind == FMHA_SF_PER_CHANNEL && (256 % (D / 8)) != 0)
    return fail(FMHA_ERR_UNSUPPORTED, "per-channel scales need D a power of two in [8, 2048]");
  if (B == 0 || H == 0) return ok_status();
  if (H > 65535 || B > 65535) return fail(FMHA_ERR_UNSUPPORTED, "grid too large: H and B must be <= 65535");
  if (kind == FMHA_SF_PER_TOKEN_BLOCK && S == 0) return ok_status();  // no block, no scale
  if (sf->ptr == nullptr || (reinterpret_cast<uintptr_t>(sf->ptr) & 3u))
    return fail(FMHA_ERR_INVALID_ARG, "sf.ptr is NULL or misaligned");
  if (S > 0) {
    fmha_status st;
    if ((st = check_tensor(*src, "src", B, S, H, D)) != FMHA_OK) return st;
    if (dst->ptr == nullptr || (reinterpret_cast<uintptr_t>(dst->ptr) & 7u))
      return fail(FMHA_ERR_INVALID_ARG, "dst.ptr is NULL or not 8-byte aligned");
    const int64_t ds[3] = {dst->stride_b, dst->stride_s, dst->stride_h};
    for (int i = 0; i < 3; ++i)
      if (ds[i] % 8 != 0) return fail(FMHA_ERR_INVALID_ARG, "dst strides must be multiples of 8 bytes");
  }
  const size_t need = fmha_quantize_workspace_bytes(kind, B, S, H, D);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need)
      return fail(FMHA_ERR_INVALID_ARG, "workspace needs %zu bytes", need);
    if (reinterpret_cast<uintptr_t>(workspace) & 3u) return fail(FMHA_ERR_INVALID_ARG, "workspace misaligned");
  }
  QuantParams p;
  memset(&p, 0, sizeof(p));
  p.src = static_cast<const uint16_t*>(src->ptr);
  p.s_sb = src->stride_b; p.s_ss = src->stride_s; p.s_sh = src->stride_h;
  p.dst = static_cast<uint8_t*>(dst->ptr);
  p.d_sb = dst->stride_b; p.d_ss = dst->stride_s; p.d_sh = dst->stride_h;
  p.sf = sf->ptr; p.kind = kind; p.rpb = kind == FMHA_SF_PER_TOKEN_BLOCK ? sf->rows_per_block : 1;
  p.nblk = kind == FMHA_SF_PER_TOKEN_BLOCK ? ceil_div(S, p.rpb) : 1;
  p.B = B; p.S = S; p.H = H; p.D = D;
  p.ws = static_cast<uint32_t*>(workspace);
  p.rows_per_cta = 2048 / (D / 8) > 0 ? 2048 / (D / 8) : 1;
  p.shift = shift;
  cudaError_t e;
  p.err = device_error_word(&e);
  if (p.err == nullptr) return fail(FMHA_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
  const uint64_t wc = g_wait_cycles.load();
  p.wait_cycles = wc ? wc : kDefaultWaitCycles;
  // Token blocks of at most 32 KB whose rows TMA can address (16-byte strides,
  // D <= 256 elements per box row, D / 8 a power of two) are staged whole in
  // shared memory by TMA.
  CUtensorMap tm;
  const CUtensorMap* tm_src = nullptr;
  auto stride_ok = [](int64_t st, int n) { return n <= 1 || (st > 0 && st % 8 == 0); };
  if (kind == FMHA_SF_PER_TOKEN_BLOCK && S > 0 && D <= 256 && ((D / 8) & (D / 8 - 1)) == 0 && p.rpb <= 256 &&
      static_cast<int64_t>(p.rpb) * D * 2 <= 32768 && stride_ok(p.s_sh, H) && stride_ok(p.s_ss, S) &&
      stride_ok(p.s_sb, B)) {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(H), uint64_t(S), uint64_t(B)};
    const int64_t strides[3] = {p.s_sh, p.s_ss, p.s_sb};
    const uint32_t box[4] = {uint32_t(D), 1u, uint32_t(p.rpb), 1u};
    if (make_map_n<4>(&tm, src->ptr, 2, dims, strides, box, "src", CU_TENSOR_MAP_SWIZZLE_NONE) == FMHA_OK)
      tm_src = &tm;
  }
  e = launch_quantize(dst->dtype == FMHA_E4M3, p, tm_src, stream);
  if (e != cudaSuccess) return fail(FMHA_ERR_CUDA, "quantizer launch: %s", cudaGetErrorString(e));
  return ok_status();
}

}  // namespace

extern "C" {

size_t fmha_quantize_workspace_bytes(int32_t sf_kind, int32_t B, int32_t S, int32_t H, int32_t D) {
  (void)S;
  return quant_groups(sf_kind, B < 0 ? 0 : B, H < 0 ? 0 : H, D < 0 ? 0 : D) * sizeof(uint32_t);
}

fmha_status fmha_quantize_blockwise_noalloc(const fmha_tensor* src, const fmha_tensor* dst, const fmha_sf* sf,
                                            int32_t B, int32_t S, int32_t H, int32_t D, cudaStream_t stream) {
  if (sf == nullptr) return fail(FMHA_ERR_INVALID_ARG, "NULL argument");
  const size_t need = fmha_quantize_workspace_bytes(sf->kind, B, S, H, D);
  const size_t have = kQuantNoallocScratchWords * sizeof(uint32_t);
  if (need > have)
    return fail(FMHA_ERR_INVALID_ARG,
                "needs %zu bytes of scratch (%zu scale groups); the built-in scratch holds %zu bytes "
                "(%zu groups); use fmha_quantize_blockwise with a workspace",
                need, need / sizeof(uint32_t), have, (size_t)kQuantNoallocScratchWords);
  void* ws = nullptr;
  if (need > 0) {
    cudaError_t e;
    ws = quant_noalloc_scratch(&e);
    if (ws == nullptr) return fail(FMHA_ERR_CUDA, "built-in scratch address: %s", cudaGetErrorString(e));
  }
  return fmha_quantize_blockwise(src, dst, sf, B, S, H, D, ws, need, stream);
}

fmha_status fmha_fwd(const fmha_args* args, cudaStream_t stream) {
  return run_attention(args, nullptr, 0, 0, nullptr, stream);
}

fmha_status fmha_fwd_block_sparse(const fmha_args* args, const uint8_t* mask, int64_t mask_stride_b,
                                  int64_t mask_stride_h, cudaStream_t stream) {
  if (mask == nullptr) return fail(FMHA_ERR_INVALID_ARG, "mask is NULL");
  return run_attention(args, mask, mask_stride_b, mask_stride_h, nullptr, stream);
}

fmha_status fmha_fwd_paged(const fmha_args* args, const int32_t* page_table, int32_t num_pages, int32_t page_size,
                           int32_t max_pages_per_seq, const uint8_t* mask, int64_t mask_stride_b,
                           int64_t mask_stride_h, cudaStream_t stream) {
  const PagedArgs pg{page_table, num_pages, page_size, max_pages_per_seq};
  return run_attention(args, mask, mask_stride_b, mask_stride_h, &pg, stream);
}

fmha_status fmha_quantize_nvfp4(const void* src, int64_t src_row_stride, int32_t rows, int32_t K, uint8_t* codes,
                                int64_t codes_row_stride, uint8_t* block_scales, int64_t block_scales_row_stride,
                                float* token_scales, int32_t fast_math, cudaStream_t stream) {
  if (rows < 0 || K < 0) return fail(FMHA_ERR_INVALID_ARG, "negative size");
  if (rows == 0 || K == 0) return ok_status();
  if (K % 16 != 0 || K > 16384) return fail(FMHA_ERR_UNSUPPORTED, "K = %d (supported: multiples of 16 up to 16384)", K);
  if (src == nullptr || codes == nullptr || block_scales == nullptr || token_scales == nullptr)
    return fail(FMHA_ERR_INVALID_ARG, "a pointer is NULL");
  if (!aligned16(src) || (rows > 1 && ((src_row_stride * 2) % 16 != 0 || src_row_stride < K)))
    return fail(FMHA_ERR_INVALID_ARG, "src must be 16-byte aligned with a row stride >= K, a multiple of 8 elements");
  if ((reinterpret_cast<uintptr_t>(codes) & 7u) != 0 || (rows > 1 && (codes_row_stride % 8 != 0 || codes_row_stride < K / 2)))
    return fail(FMHA_ERR_INVALID_ARG, "codes must be 8-byte aligned with a row stride >= K/2, a multiple of 8 bytes");
  if (rows > 1 && block_scales_row_stride < K / 16)
    return fail(FMHA_ERR_INVALID_ARG, "block_scales row stride < K/16");
  if ((reinterpret_cast<uintptr_t>(token_scales) & 3u) != 0) return fail(FMHA_ERR_INVALID_ARG, "token_scales misaligned");
  Nvfp4Params p;
  p.src = static_cast<const uint16_t*>(src); p.src_rs = src_row_stride;
  p.rows = rows; p.K = K;
  p.codes = codes; p.codes_rs = codes_row_stride;
  p.sb = block_scales; p.sb_rs = block_scales_row_stride;
  p.st = token_scales;
  p.fast = fast_math ? 1 : 0;
  cudaError_t e = launch_nvfp4(p, stream);
  if (e != cudaSuccess) return fail(FMHA_ERR_CUDA, "nvfp4 launch: %s", cudaGetErrorString(e));
  return ok_status();
}

size_t fmha_decode_workspace_bytes(const fmha_args* args, int32_t num_splits) {
  if (args == nullptr || args->B <= 0 || args->Hq <= 0 || args->Hkv <= 0 || args->Sq <= 0 || args->Skv < 0 ||
      args->Hq % args->Hkv != 0 || !packed_rows_fit(args->Sq, args->Hq, args->Hkv))
    return 0;
  return plan_splits(args->B, args->Hq, args->Hkv, args->Sq, args->Skv, args->D, num_splits).workspace_bytes;
}

int32_t fmha_decode_num_splits(const fmha_args* args, int32_t num_splits) {
  if (args == nullptr || args->B <= 0 || args->Hq <= 0 || args->Hkv <= 0 || args->Sq <= 0 || args->Skv < 0 ||
      args->Hq % args->Hkv != 0 || !packed_rows_fit(args->Sq, args->Hq, args->Hkv))
    return 0;
  return plan_splits(args->B, args->Hq, args->Hkv, args->Sq, args->Skv, args->D, num_splits).n_splits;
}

fmha_status fmha_fwd_decode(const fmha_args* args, const int32_t* page_table, int32_t num_pages, int32_t page_size,
                            int32_t max_pages_per_seq, const uint8_t* mask, int64_t mask_stride_b,
                            int64_t mask_stride_h, int32_t num_splits, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  const DecodeArgs dec{num_splits, workspace, workspace_bytes};
  if (page_table == nullptr) return run_attention(args, mask, mask_stride_b, mask_stride_h, nullptr, stream, &dec);
  const PagedArgs pg{page_table, num_pages, page_size, max_pages_per_seq};
  return run_attention(args, mask, mask_stride_b, mask_stride_h, &pg, stream, &dec);
}

fmha_status fmha_get_device_error(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(FMHA_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  uint32_t* w = device_error_word(&e);
  if (w == nullptr) return fail(FMHA_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
  uint32_t word = 0;
  if ((e = cudaMemcpy(&word, w, sizeof(word), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return fail(FMHA_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
  if (word != 0 && (e = cudaMemset(w, 0, sizeof(word))) != cudaSuccess)
    return fail(FMHA_ERR_CUDA, "clear error word: %s", cudaGetErrorString(e));
  if (word & kErrTimeout) return fail(FMHA_ERR_TIMEOUT, "a kernel wait ran out (error word 0x%x)", word);
  if (word & kErrPageIndex) return fail(FMHA_ERR_DEVICE_INDEX, "a page-table entry was out of range");
  return ok_status();
}

const char* fmha_status_string(fmha_status s) {
  switch (s) {
    case FMHA_OK: return "FMHA_OK";
    case FMHA_ERR_INVALID_ARG: return "FMHA_ERR_INVALID_ARG";
    case FMHA_ERR_UNSUPPORTED: return "FMHA_ERR_UNSUPPORTED";
    case FMHA_ERR_CUDA: return "FMHA_ERR_CUDA";
    case FMHA_ERR_TIMEOUT: return "FMHA_ERR_TIMEOUT";
    case FMHA_ERR_DEVICE_INDEX: return "FMHA_ERR_DEVICE_INDEX";
  }
  return "FMHA_ERR_UNKNOWN";
}

const char* fmha_last_error_message(void) { return g_msg; }

void fmha_set_wait_timeout_cycles(uint64_t cycles) { g_wait_cycles.store(cycles); }

}  // extern "C"
