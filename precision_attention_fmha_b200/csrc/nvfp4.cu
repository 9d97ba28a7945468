// Per-token NVFP4 quantization ("FlashInfer per-token NVFP4 quantization
// kernel"): E2M1 codes, one E4M3 scale per 16 elements, one fp32 scale per
// token (row).
//   s_t  = amax_row / 2688 (1 when the row is zero)
//   sb   = E4M3((amax_blk / s_t) / 6)           (IEEE divisions, RN, satfinite)
//   e    = decode(sb) * s_t
//   code = E2M1(x / e), or E2M1(x * (1 / e)) on the fast path; 0 when e == 0
// The exact path takes x / e as Markstein's FMA-corrected quotient (P.
// Markstein, IBM J. Res. Dev. 34(1), 1990) from one correctly rounded
// reciprocal per block: q0 = RN(x r), q = RN(q0 + (x - q0 e) r), with the
// sign of x (so -0 keeps its code). It is the correctly rounded quotient, so
// the codes equal the IEEE division's, while e >= 2^-60 keeps every quotient
// that can reach a nonzero code (|q| >= 2^-2) and its residual in the normal
// range; blocks with a smaller e divide.
// One CTA per row. Each thread keeps its 16-element blocks in registers from
// the amax pass to the quantize pass (the row is read from HBM once, as the
// page's kernel caches its input on chip), so HBM sees 2 B read and
// 0.5 + 1/16 B written per element plus 4 B per row.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fmha_internal.h"
#include "ptx_sm100.cuh"

namespace fmha {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Eight fp32 values -> eight E2M1 codes, element 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t pack_e2m1x8(const float (&y)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return r;
}

template <int NB, bool FAST>
__global__ void __launch_bounds__(kThreads) nvfp4_quant_kernel(const Nvfp4Params p) {
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nblk = p.K >> 4;
  const uint16_t* src = p.src + static_cast<int64_t>(row) * p.src_rs;
  uint4 v[NB][2];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int blk = tid + i * kThreads;
    if (blk < nblk) {
      const uint4* s = reinterpret_cast<const uint4*>(src + 16 * blk);
      v[i][0] = __ldg(s);
      v[i][1] = __ldg(s + 1);
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i][0]);
#pragma unroll
      for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
    } else {
      v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __shared__ float red[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float s_t = amax > 0.f ? __fdiv_rn(amax, 2688.f) : 1.f;
  uint8_t* codes = p.codes + static_cast<int64_t>(row) * p.codes_rs;
  uint8_t* sbs = p.sb + static_cast<int64_t>(row) * p.sb_rs;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int blk = tid + i * kThreads;
    if (blk >= nblk) continue;
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i][0]);
    float x[16];
    float amax_b = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      x[2 * k] = bf16_lo(w[k]);
      x[2 * k + 1] = bf16_hi(w[k]);
      amax_b = fmaxf(amax_b, fmaxf(fabsf(x[2 * k]), fabsf(x[2 * k + 1])));
    }
    const float q = __fdiv_rn(__fdiv_rn(amax_b, s_t), 6.f);
    const uint32_t sb_code = ptx::pack_e4m3x2(q, 0.f) & 0xffu;
    const uint32_t sb_h = ptx::e4m3x2_to_f16x2(sb_code);  // exact: E4M3 values are F16 values
    const float sb = __half2float(__ushort_as_half(static_cast<unsigned short>(sb_h & 0xffffu)));
    const float e = __fmul_rn(sb, s_t);
    uint2 out = make_uint2(0u, 0u);
    if (e != 0.f) {
      float y[16];
      if (FAST) {
        const float r = __fdiv_rn(1.f, e);
#pragma unroll
        for (int k = 0; k < 16; ++k) y[k] = __fmul_rn(x[k], r);
      } else if (e >= 0x1p-60f) {
        const float r = __frcp_rn(e);
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          float q0a, q0b, ea, eb, qa, qb;
          ptx::ffma2(q0a, q0b, x[k], x[k + 1], r, r, -0.f, -0.f);       // RN(x r)
          ptx::ffma2(ea, eb, -q0a, -q0b, e, e, x[k], x[k + 1]);         // x - q0 e, one rounding
          ptx::ffma2(qa, qb, ea, eb, r, r, q0a, q0b);                   // RN(q0 + res r)
          y[k] = copysignf(qa, x[k]);
          y[k + 1] = copysignf(qb, x[k + 1]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) y[k] = __fdiv_rn(x[k], e);
      }
      float lo[8], hi[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        lo[k] = y[k];
        hi[k] = y[8 + k];
      }
      out.x = pack_e2m1x8(lo);
      out.y = pack_e2m1x8(hi);
    }
    *reinterpret_cast<uint2*>(codes + 8 * blk) = out;
    sbs[blk] = static_cast<uint8_t>(sb_code);
  }
  if (tid == 0) p.st[row] = s_t;
}

template <int NB>
cudaError_t launch_nb(const Nvfp4Params& p, cudaStream_t s) {
  if (p.fast)
    nvfp4_quant_kernel<NB, true><<<p.rows, kThreads, 0, s>>>(p);
  else
    nvfp4_quant_kernel<NB, false><<<p.rows, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_nvfp4(const Nvfp4Params& p, cudaStream_t s) {
  if (p.rows == 0) return cudaSuccess;
  const int nblk = p.K >> 4;
  if (nblk <= kThreads) return launch_nb<1>(p, s);
  if (nblk <= 2 * kThreads) return launch_nb<2>(p, s);
  if (nblk <= 4 * kThreads) return launch_nb<4>(p, s);
  return launch_nb<8>(p, s);
}

}  // namespace fmha
