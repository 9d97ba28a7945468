// quantize.cu -- block quantizer: amax -> scale = amax / R -> INT8 / E4M3 codes.
//
// Follows "FlashInfer DiT optimization: SageAttention and Int8/FP8
// mixed-precision kernels" (section 2: block-wise scale factors for Q, K, V;
// "Why" item 2: block-wise beats per-tensor scaling on outlier-heavy maps) and
// the input-staging idea of "FlashInfer per-token NVFP4 quantization kernel"
// (section 2: keep the input on chip so amax and quantization read HBM once).
//
// Arithmetic (the contract in include/fmha.h, bit-exact with the oracle):
//   amax  = max |x|                      (x = bf16 value, exact in fp32)
//   scale = fp32(amax) / fp32(R)         (IEEE round-to-nearest division; 1 if amax == 0)
//   code  = RN(fp32(x) / scale)          (IEEE division per element)
//           INT8: round half to even, clamp [-127, 127]; E4M3: RN-even, saturate to +-448.
//
// Token-block granularity: one CTA per (b, h, token block); each thread keeps
// its 16-byte vectors in registers between the amax and the quantize pass, so
// HBM is read once (2 B/element) and written once (1 B/element).
// Grid-wide granularities (per tensor / head / channel): pass 1 reduces amax
// into the caller's workspace with atomicMax on the (non-negative) fp32 bit
// patterns, pass 2 re-reads and quantizes: 2 + 2 + 1 B/element.
//
// K smoothing (SageAttention, Zhang et al. 2024): every kernel can quantize
// x - shift[b, h, d] instead of x (one fp32 round-to-nearest subtraction per
// element, before the amax). The shift is normally the token mean per channel,
// which channel_mean_* computes: fp64 partial sums per CTA, then a fixed-order
// sum over the CTAs, one fp64 division by S and one rounding to fp32.
#include <algorithm>
#include <mutex>

#include "fmha_internal.h"
#include "ptx_sm100.cuh"

namespace fmha {
namespace {

constexpr int kThreads = 256;
// 16-byte vectors a thread keeps in registers between the amax and the code
// pass: 8 hold a 128 x 128 BF16 block, 4 a 64 x 128 block. The smaller cache
// lets four CTAs share an SM's registers (more loads in flight).
constexpr int kCacheVecsMax = 8;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}

// The 8 values of one 16-byte vector, minus the shift of its 8 channels when
// shift_c (16-byte aligned) is not null.
__device__ __forceinline__ void vals8(const uint4& v, const float* shift_c, float (&x)[8]) {
  unpack8(v, x);
  if (shift_c != nullptr) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(shift_c));
    const float4 c = __ldg(reinterpret_cast<const float4*>(shift_c + 4));
    x[0] = __fsub_rn(x[0], a.x); x[1] = __fsub_rn(x[1], a.y); x[2] = __fsub_rn(x[2], a.z);
    x[3] = __fsub_rn(x[3], a.w); x[4] = __fsub_rn(x[4], c.x); x[5] = __fsub_rn(x[5], c.y);
    x[6] = __fsub_rn(x[6], c.z); x[7] = __fsub_rn(x[7], c.w);
  }
}

__device__ __forceinline__ float amax8(const float (&x)[8]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
  return m;
}

// Shift of column vector c of head (b, h), or null when nothing is subtracted.
__device__ __forceinline__ const float* shift_at(const QuantParams& p, int64_t bh, int c) {
  return p.shift != nullptr ? p.shift + bh * p.D + c * 8 : nullptr;
}

__device__ __forceinline__ uint4 ld16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

template <bool kE4M3>
__device__ __forceinline__ float range_max() { return kE4M3 ? 448.f : 127.f; }

template <bool kE4M3>
__device__ __forceinline__ float scale_from_amax(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, range_max<kE4M3>()) : 1.f;
}

template <bool kE4M3>
__device__ __forceinline__ uint32_t code4(float a, float b, float c, float d, float sa, float sb, float sc,
                                          float sd) {
  const float qa = __fdiv_rn(a, sa), qb = __fdiv_rn(b, sb), qc = __fdiv_rn(c, sc), qd = __fdiv_rn(d, sd);
  if constexpr (kE4M3) {
    return ptx::pack_e4m3x2(qa, qb) | (ptx::pack_e4m3x2(qc, qd) << 16);
  } else {
    auto cl = [](float q) {
      int i = __float2int_rn(q);  // round half to even
      i = max(-127, min(127, i));
      return static_cast<uint32_t>(i) & 0xFFu;
    };
    return cl(qa) | (cl(qb) << 8) | (cl(qc) << 16) | (cl(qd) << 24);
  }
}

template <bool kE4M3>
__device__ __forceinline__ uint2 code8(const float (&x)[8], const float (&s)[8]) {
  return make_uint2(code4<kE4M3>(x[0], x[1], x[2], x[3], s[0], s[1], s[2], s[3]),
                    code4<kE4M3>(x[4], x[5], x[6], x[7], s[4], s[5], s[6], s[7]));
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kThreads / 32 ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// One CTA per (token block, h, b).
template <bool kE4M3, int kCacheVecs>
__global__ void __launch_bounds__(kThreads, kCacheVecs <= 4 ? 4 : 0) quant_token_block_kernel(const QuantParams p) {
  __shared__ float red[kThreads / 32];
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int s0 = blk * p.rpb;
  const int rows = min(p.S - s0, p.rpb);
  const int vpr = p.D >> 3;
  const int nvec = rows * vpr;
  const uint16_t* src = p.src + b * p.s_sb + static_cast<int64_t>(s0) * p.s_ss + h * p.s_sh;
  uint8_t* dst = p.dst + b * p.d_sb + static_cast<int64_t>(s0) * p.d_ss + h * p.d_sh;

  const int64_t bh = static_cast<int64_t>(b) * p.H + h;

  uint4 cache[kCacheVecs];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kCacheVecs; ++i) {
    const int v = threadIdx.x + i * kThreads;
    if (v < nvec) {
      const int r = v / vpr, c = v - r * vpr;
      cache[i] = ld16(src + r * p.s_ss + c * 8);
      float x[8];
      vals8(cache[i], shift_at(p, bh, c), x);
      amax = fmaxf(amax, amax8(x));
    }
  }
  for (int v = threadIdx.x + kCacheVecs * kThreads; v < nvec; v += kThreads) {
    const int r = v / vpr, c = v - r * vpr;
    float x[8];
    vals8(ld16(src + r * p.s_ss + c * 8), shift_at(p, bh, c), x);
    amax = fmaxf(amax, amax8(x));
  }
  amax = block_reduce_max(amax, red);
  const float scale = scale_from_amax<kE4M3>(amax);
  float s8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s8[i] = scale;
#pragma unroll
  for (int i = 0; i < kCacheVecs; ++i) {
    const int v = threadIdx.x + i * kThreads;
    if (v < nvec) {
      const int r = v / vpr, c = v - r * vpr;
      float x[8];
      vals8(cache[i], shift_at(p, bh, c), x);
      *reinterpret_cast<uint2*>(dst + r * p.d_ss + c * 8) = code8<kE4M3>(x, s8);
    }
  }
  for (int v = threadIdx.x + kCacheVecs * kThreads; v < nvec; v += kThreads) {
    const int r = v / vpr, c = v - r * vpr;
    float x[8];
    vals8(ld16(src + r * p.s_ss + c * 8), shift_at(p, bh, c), x);
    *reinterpret_cast<uint2*>(dst + r * p.d_ss + c * 8) = code8<kE4M3>(x, s8);
  }
  if (threadIdx.x == 0) p.sf[bh * p.nblk + blk] = scale;
}

// Grid-wide kinds, pass 1: per-CTA amax over rows [chunk*rows_per_cta, ...) of
// (b, h), merged into the workspace with atomicMax on fp32 bits (valid: amax >= 0).
// Per-channel needs 256 % (D/8) == 0 so each thread owns one fixed column vector.
__global__ void __launch_bounds__(kThreads) quant_amax_kernel(const QuantParams p) {
  __shared__ float red[kThreads * 8];
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int s0 = chunk * p.rows_per_cta;
  const int rows = min(p.S - s0, p.rows_per_cta);
  const int vpr = p.D >> 3;
  const int nvec = rows * vpr;
  const uint16_t* src = p.src + b * p.s_sb + static_cast<int64_t>(s0) * p.s_ss + h * p.s_sh;
  const int64_t bh = static_cast<int64_t>(b) * p.H + h;
  if (p.kind == FMHA_SF_PER_CHANNEL) {
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
      const int r = v / vpr, c = v - r * vpr;
      float x[8];
      vals8(ld16(src + r * p.s_ss + c * 8), shift_at(p, bh, c), x);
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(x[i]));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[threadIdx.x * 8 + i] = m[i];
    __syncthreads();
    const int step = kThreads / vpr;  // threads sharing one column vector are tid % vpr apart
    for (int ch = threadIdx.x; ch < p.D; ch += kThreads) {
      const int cv = ch >> 3, j = ch & 7;
      float a = 0.f;
      for (int k = 0; k < step; ++k) a = fmaxf(a, red[(cv + k * vpr) * 8 + j]);
      atomicMax(p.ws + bh * p.D + ch, __float_as_uint(a));
    }
  } else {
    float m = 0.f;
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
      const int r = v / vpr, c = v - r * vpr;
      float x[8];
      vals8(ld16(src + r * p.s_ss + c * 8), shift_at(p, bh, c), x);
      m = fmaxf(m, amax8(x));
    }
    m = block_reduce_max(m, red);
    if (threadIdx.x == 0) {
      const int64_t g = p.kind == FMHA_SF_PER_HEAD ? bh : 0;
      atomicMax(p.ws + g, __float_as_uint(m));
    }
  }
}

// Grid-wide kinds, pass 2: quantize with the merged amax; chunk 0 writes the scales.
template <bool kE4M3>
__global__ void __launch_bounds__(kThreads) quant_apply_kernel(const QuantParams p) {
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int s0 = chunk * p.rows_per_cta;
  const int rows = min(p.S - s0, p.rows_per_cta);
  const int vpr = p.D >> 3;
  const int nvec = rows * vpr;
  const uint16_t* src = p.src + b * p.s_sb + static_cast<int64_t>(s0) * p.s_ss + h * p.s_sh;
  uint8_t* dst = p.dst + b * p.d_sb + static_cast<int64_t>(s0) * p.d_ss + h * p.d_sh;
  const int64_t bh = static_cast<int64_t>(b) * p.H + h;
  float s8[8];
  if (p.kind == FMHA_SF_PER_CHANNEL) {
    const int cv = threadIdx.x % vpr;  // fixed column vector of this thread (256 % vpr == 0)
#pragma unroll
    for (int i = 0; i < 8; ++i) s8[i] = scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + i]));
  } else {
    const float s = scale_from_amax<kE4M3>(__uint_as_float(p.ws[p.kind == FMHA_SF_PER_HEAD ? bh : 0]));
#pragma unroll
    for (int i = 0; i < 8; ++i) s8[i] = s;
  }
  for (int v = threadIdx.x; v < nvec; v += kThreads) {
    const int r = v / vpr, c = v - r * vpr;
    float x[8];
    vals8(ld16(src + r * p.s_ss + c * 8), shift_at(p, bh, c), x);
    *reinterpret_cast<uint2*>(dst + r * p.d_ss + c * 8) = code8<kE4M3>(x, s8);
  }
  if (chunk == 0) {
    if (p.kind == FMHA_SF_PER_CHANNEL) {
      for (int ch = threadIdx.x; ch < p.D; ch += kThreads)
        p.sf[bh * p.D + ch] = scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + ch]));
    } else if (threadIdx.x == 0) {
      if (p.kind == FMHA_SF_PER_HEAD)
        p.sf[bh] = s8[0];
      else if (b == 0 && h == 0)
        p.sf[0] = s8[0];
    }
  }
}

// S == 0 for a grid-wide kind: every group's amax is 0, so every scale is 1.
__global__ void __launch_bounds__(kThreads) fill_unit_scales_kernel(float* sf, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * kThreads)
    sf[i] = 1.f;
}

template <bool kE4M3>
cudaError_t launch_quantize_t(const QuantParams& p, cudaStream_t stream) {
  if (p.kind == FMHA_SF_PER_TOKEN_BLOCK) {
    dim3 grid(p.nblk, p.H, p.B);
    if (static_cast<int64_t>(p.rpb) * (p.D >> 3) <= 4 * kThreads)
      quant_token_block_kernel<kE4M3, 4><<<grid, kThreads, 0, stream>>>(p);
    else
      quant_token_block_kernel<kE4M3, kCacheVecsMax><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
  }
  const size_t groups = p.kind == FMHA_SF_PER_CHANNEL ? static_cast<size_t>(p.B) * p.H * p.D
                        : p.kind == FMHA_SF_PER_HEAD  ? static_cast<size_t>(p.B) * p.H
                                                      : 1;
  if (p.S == 0) {  // no token: no amax pass (its grid would be empty), unit scales
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((groups + kThreads - 1) / kThreads, 1024));
    fill_unit_scales_kernel<<<blocks, kThreads, 0, stream>>>(p.sf, static_cast<int64_t>(groups));
    return cudaGetLastError();
  }
  cudaError_t e = cudaMemsetAsync(p.ws, 0, groups * sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  dim3 grid((p.S + p.rows_per_cta - 1) / p.rows_per_cta, p.H, p.B);
  quant_amax_kernel<<<grid, kThreads, 0, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  quant_apply_kernel<kE4M3><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

// Token mean, pass 1: CTA (chunk, h, b) sums rows [chunk * rows_per_cta, ...)
// of (b, h) per channel in fp64. Each thread owns one column vector (256 is a
// multiple of D / 8) and a fixed set of rows; the threads of a column vector
// are then added in thread order, so the partial sums do not depend on timing.
__global__ void __launch_bounds__(kThreads) channel_mean_partial_kernel(const QuantParams p) {
  __shared__ double red[kThreads * 8];
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int s0 = chunk * p.rows_per_cta;
  const int rows = min(p.S - s0, p.rows_per_cta);
  const int vpr = p.D >> 3;
  const int cv = threadIdx.x % vpr, row_step = kThreads / vpr;
  const uint16_t* src = p.src + b * p.s_sb + static_cast<int64_t>(s0) * p.s_ss + h * p.s_sh + cv * 8;
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll 8
  for (int r = threadIdx.x / vpr; r < rows; r += row_step) {
    float x[8];
    unpack8(ld16(src + r * p.s_ss), x);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(x[i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[threadIdx.x * 8 + i] = acc[i];
  __syncthreads();
  const int64_t bh = static_cast<int64_t>(b) * p.H + h;
  for (int ch = threadIdx.x; ch < p.D; ch += kThreads) {
    const int c = ch >> 3, j = ch & 7;
    double a = 0.0;
    for (int k = 0; k < row_step; ++k) a += red[(c + k * vpr) * 8 + j];
    p.partial[(bh * p.n_chunks + chunk) * p.D + ch] = a;
  }
}

// Token mean, pass 2: one thread per (b, h, d) adds the chunks in order,
// divides by S in fp64 and rounds once to fp32.
__global__ void __launch_bounds__(kThreads) channel_mean_final_kernel(const QuantParams p) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (i >= static_cast<int64_t>(p.B) * p.H * p.D) return;
  const int64_t bh = i / p.D, ch = i - bh * p.D;
  const double* part = p.partial + bh * p.n_chunks * p.D + ch;
  double a = 0.0;
#pragma unroll 8
  for (int c = 0; c < p.n_chunks; ++c) a += part[static_cast<int64_t>(c) * p.D];
  p.mean[i] = __double2float_rn(__ddiv_rn(a, static_cast<double>(p.S)));
}

}  // namespace

cudaError_t launch_quantize(bool to_e4m3, const QuantParams& p, cudaStream_t stream) {
  return to_e4m3 ? launch_quantize_t<true>(p, stream) : launch_quantize_t<false>(p, stream);
}

cudaError_t launch_channel_mean(const QuantParams& p, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(p.B) * p.H * p.D;
  if (n == 0) return cudaSuccess;
  if (p.S == 0) return cudaMemsetAsync(p.mean, 0, n * sizeof(float), stream);
  dim3 grid(p.n_chunks, p.H, p.B);
  channel_mean_partial_kernel<<<grid, kThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  channel_mean_final_kernel<<<static_cast<unsigned>((n + kThreads - 1) / kThreads), kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

// Built-in scratch for fmha_quantize_blockwise_noalloc: the amax accumulators
// of the grid-wide granularities live in this file-scope device array instead
// of a caller buffer, so that entry point never allocates. Every device that
// loads the library holds it (256 KB) until the process exits. In host code the
// name is only a stand-in for the symbol: kernels get the real device address
// from cudaGetSymbolAddress, looked up once per device below.
static __device__ __align__(256) uint32_t g_quant_noalloc_scratch[kQuantNoallocScratchWords];

uint32_t* quant_noalloc_scratch(cudaError_t* err) {
  constexpr int kMaxDevices = 64;
  static uint32_t* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  *err = cudaGetDevice(&dev);  // the caller's current device is the one the kernels run on
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_quant_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint32_t*>(p);
  }
  *err = cudaSuccess;
  return addr[dev];
}

}  // namespace fmha
