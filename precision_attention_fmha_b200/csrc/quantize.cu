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
//   code  = RN(fp32(x) / scale)          (the correctly rounded quotient: one
//           reciprocal per scale and two FMAs per element, Divisor below)
//           INT8: round half to even, clamp [-127, 127]; E4M3: RN-even, saturate to +-448.
//
// Token-block granularity: CTAs walk the (b, token block, h) blocks, loading
// the next block while they reduce and encode the current one; each thread
// keeps its 16-byte vectors in registers between the amax and the quantize
// pass, so HBM is read once (2 B/element) and written once (1 B/element).
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

// Streaming multiprocessors of the current device (the token-block grid is a
// multiple of the CTAs they hold at once).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

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

// Quotients x / s rounded to nearest, for one scale s: Markstein's
// FMA-corrected quotient (P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
// r = RN(1/s), q0 = RN(x r), e = x - q0 s (exact in one FMA), q = RN(q0 + e r).
// With r correctly rounded, q is the correctly rounded quotient while e and
// q0 stay in the normal range. The guard s >= 2^-60 (uniform over a block)
// keeps them there for every quotient large enough to reach a nonzero code
// (|q| >= 2^-11); below it the IEEE division is used. The result takes the
// sign of x, as the quotient does (x = -0 gives -0, E4M3 code 0x80). For BF16
// inputs the codes were compared with the IEEE quotient's codes for every x
// and every scale RN(amax / R), R = 127 and 448.
struct Divisor {
  float s, r;
  bool fast;
  __device__ explicit Divisor(float s_) : s(s_), r(0.f), fast(s_ >= 0x1p-60f) { r = __frcp_rn(s_); }
  __device__ __forceinline__ float quot(float x) const {
    if (!fast) return __fdiv_rn(x, s);
    const float q0 = __fmul_rn(x, r);
    // The sign of x (s > 0): the correction step turns a quotient of -0 into +0.
    return copysignf(__fmaf_rn(__fmaf_rn(-q0, s, x), r, q0), x);
  }
};

template <bool kE4M3>
__device__ __forceinline__ uint32_t code4(float qa, float qb, float qc, float qd) {
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

// Codes of 8 values with one divisor, or with one divisor per value.
template <bool kE4M3>
__device__ __forceinline__ uint2 code8(const float (&x)[8], const Divisor& d) {
  return make_uint2(code4<kE4M3>(d.quot(x[0]), d.quot(x[1]), d.quot(x[2]), d.quot(x[3])),
                    code4<kE4M3>(d.quot(x[4]), d.quot(x[5]), d.quot(x[6]), d.quot(x[7])));
}
template <bool kE4M3>
__device__ __forceinline__ uint2 code8(const float (&x)[8], const Divisor (&d)[8]) {
  return make_uint2(code4<kE4M3>(d[0].quot(x[0]), d[1].quot(x[1]), d[2].quot(x[2]), d[3].quot(x[3])),
                    code4<kE4M3>(d[4].quot(x[4]), d[5].quot(x[5]), d[6].quot(x[6]), d[7].quot(x[7])));
}

template <int kThr = kThreads>
__device__ __forceinline__ float block_reduce_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kThr / 32 ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// Token-block granularity. Work items are the (b, token block, h) blocks in
// that order (neighbouring heads share rows of the [B, S, H, D] tensor); a CTA
// walks items blockIdx.x, blockIdx.x + gridDim.x, ... and issues the loads of
// its next item before it reduces and encodes the current one, so HBM reads
// stay in flight through the block reduction and the encoding. Each thread
// keeps up to kCache 16-byte vectors of an item in registers (HBM read once);
// vectors past kThr * kCache (blocks larger than the cache) are re-read.
// Position (b, token block, h) of a work item, in that order (h fastest), and
// its advance by a fixed stride without a division per item: the stride is
// decomposed once (dh heads, then dblk blocks and db batches with carries).
struct ItemCursor {
  int b, blk, h;
  int dh, dblk, db;
  __device__ ItemCursor(int64_t item, int64_t stride, int H, int nblk) {
    h = static_cast<int>(item % H);
    const int64_t bb = item / H;
    blk = static_cast<int>(bb % nblk);
    b = static_cast<int>(bb / nblk);
    dh = static_cast<int>(stride % H);
    const int64_t sb = stride / H;
    dblk = static_cast<int>(sb % nblk);
    db = static_cast<int>(sb / nblk);
  }
  __device__ __forceinline__ void advance(int H, int nblk) {
    h += dh;
    int carry = h >= H;
    h -= carry ? H : 0;
    blk += dblk + carry;
    carry = blk >= nblk;
    blk -= carry ? nblk : 0;
    b += db + carry;
  }
};

// CTAs per SM the register budget is set for: 64 registers a thread without a
// shift; the shifted values need a few more (3 CTAs of 256, 1 of 512).
constexpr int token_block_min_ctas(int threads, bool shift) {
  return shift ? (threads == 256 ? 3 : 1) : 2048 / threads / 2;
}

template <bool kE4M3, int kThr, bool kShift>
__global__ void __launch_bounds__(kThr, token_block_min_ctas(kThr, kShift))
    quant_token_block_kernel(const QuantParams p, int64_t n_items) {
  constexpr int kCache = 4;
  // The shift pointer is known at compile time: without one, no shift registers.
  auto shift_of = [&](int64_t bh, int c) -> const float* { return kShift ? shift_at(p, bh, c) : nullptr; };
  __shared__ float red[2][kThr / 32];  // alternating buffers: no barrier between items
  const int vpr = p.D >> 3;
  auto load = [&](const ItemCursor& ic, uint4 (&c)[kCache]) {
    const int b = ic.b, h = ic.h, blk = ic.blk;
    const int s0 = blk * p.rpb;
    const int nvec = min(p.S - s0, p.rpb) * vpr;
    const uint16_t* src = p.src + b * p.s_sb + static_cast<int64_t>(s0) * p.s_ss + h * p.s_sh;
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
      const int v = threadIdx.x + i * kThr;
      if (v < nvec) {
        const int r = v / vpr, cc = v - r * vpr;
        c[i] = ld16(src + r * p.s_ss + cc * 8);
      }
    }
  };
  uint4 cur[kCache], nxt[kCache];
  int64_t item = blockIdx.x;
  ItemCursor ic(item, gridDim.x, p.H, p.nblk);
  if (item < n_items) load(ic, cur);
  for (int it = 0; item < n_items; ++it) {
    const int64_t next = item + gridDim.x;
    const int b = ic.b, h = ic.h, blk = ic.blk;
    ic.advance(p.H, p.nblk);
    if (next < n_items) load(ic, nxt);  // in flight while this item is reduced and encoded
    const int s0 = blk * p.rpb;
    const int nvec = min(p.S - s0, p.rpb) * vpr;
    const uint16_t* src = p.src + b * p.s_sb + static_cast<int64_t>(s0) * p.s_ss + h * p.s_sh;
    uint8_t* dst = p.dst + b * p.d_sb + static_cast<int64_t>(s0) * p.d_ss + h * p.d_sh;
    const int64_t bh = static_cast<int64_t>(b) * p.H + h;

    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
      const int v = threadIdx.x + i * kThr;
      if (v < nvec) {
        float x[8];
        vals8(cur[i], shift_of(bh, v % vpr), x);
        amax = fmaxf(amax, amax8(x));
      }
    }
    for (int v = threadIdx.x + kCache * kThr; v < nvec; v += kThr) {
      const int r = v / vpr, c = v - r * vpr;
      float x[8];
      vals8(ld16(src + r * p.s_ss + c * 8), shift_of(bh, c), x);
      amax = fmaxf(amax, amax8(x));
    }
    amax = block_reduce_max<kThr>(amax, red[it & 1]);
    const Divisor dv(scale_from_amax<kE4M3>(amax));
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
      const int v = threadIdx.x + i * kThr;
      if (v < nvec) {
        const int r = v / vpr, c = v - r * vpr;
        float x[8];
        vals8(cur[i], shift_of(bh, c), x);
        *reinterpret_cast<uint2*>(dst + r * p.d_ss + c * 8) = code8<kE4M3>(x, dv);
      }
    }
    for (int v = threadIdx.x + kCache * kThr; v < nvec; v += kThr) {
      const int r = v / vpr, c = v - r * vpr;
      float x[8];
      vals8(ld16(src + r * p.s_ss + c * 8), shift_of(bh, c), x);
      *reinterpret_cast<uint2*>(dst + r * p.d_ss + c * 8) = code8<kE4M3>(x, dv);
    }
    if (threadIdx.x == 0) p.sf[bh * p.nblk + blk] = dv.s;
#pragma unroll
    for (int i = 0; i < kCache; ++i) cur[i] = nxt[i];
    item = next;
  }
}

// Token-block granularity with TMA staging: the same walk over the (b, token
// block, h) items, but every block is copied whole into a ring of shared-memory
// slots by the tensor-memory accelerator (one 4-D box [D, 1, rpb, 1] per
// item), `stages` items ahead of the one being encoded. Many more bytes are then
// in flight per SM than registers could hold; rows past S arrive as zeros
// (they do not change the amax and get no codes). Thread 0 refills a slot as
// soon as the block reduction shows that every thread has read it.
//
// The per-element work is cut to a few instructions so that the kernel stays
// bound by HBM: D / 8 is a power of two, so a thread's column vector is fixed
// and its rows are a shift away (no integer division); without a shift the
// amax is taken on the BF16 pairs themselves (max of magnitudes, two per
// instruction); the quotient's three operations run on packed fp32 pairs; an
// INT8 code is rint(q) read from the low byte of
// q + 1.5 * 2^23 (exact for |q| < 2^22; |q| <= 127 here), bytes gathered with
// byte permutes; an E4M3 code takes the sign bit of x (so -0 keeps 0x80).
constexpr int kMaxStages = 4;
constexpr uint32_t kQuantWaitSleepNs = 500;

// max(|a|, |b|) of BF16 pairs; the sign bits hold garbage (masked at the end).
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Codes of the 8 values of one vector (x: the values, w: their BF16 words when
// there is no shift) with one fast divisor (s >= 2^-60).
template <bool kE4M3, bool kShift>
__device__ __forceinline__ uint2 code8_fast(const float (&x)[8], const uint4& w, const Divisor& d) {
  float q[8];
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    float q0a, q0b, ea, eb;
    ptx::ffma2(q0a, q0b, x[j], x[j + 1], d.r, d.r, -0.f, -0.f);       // RN(x r)
    ptx::ffma2(ea, eb, -q0a, -q0b, d.s, d.s, x[j], x[j + 1]);         // x - q0 s, one rounding
    ptx::ffma2(q[j], q[j + 1], ea, eb, d.r, d.r, q0a, q0b);           // RN(q0 + e r)
  }
  if constexpr (kE4M3) {
    uint32_t lo = ptx::pack_e4m3x2(q[0], q[1]) | (ptx::pack_e4m3x2(q[2], q[3]) << 16);
    uint32_t hi = ptx::pack_e4m3x2(q[4], q[5]) | (ptx::pack_e4m3x2(q[6], q[7]) << 16);
    if constexpr (kShift) {  // sign bits of the fp32 values
      uint32_t sl = 0, sh = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sl |= (__float_as_uint(x[j]) >> 31) << (8 * j + 7);
        sh |= (__float_as_uint(x[4 + j]) >> 31) << (8 * j + 7);
      }
      lo |= sl;
      hi |= sh;
    } else {  // sign bits of the BF16 words: bits 15 and 31 of each word -> bit 7 of each byte
      lo |= __byte_perm(w.x, w.y, 0x7531) & 0x80808080u;
      hi |= __byte_perm(w.z, w.w, 0x7531) & 0x80808080u;
    }
    return make_uint2(lo, hi);
  } else {
    uint32_t t[8];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      float a, b;
      ptx::fadd2(a, b, q[j], q[j + 1], 12582912.f, 12582912.f);  // rint(q) in the low mantissa bits
      t[j] = __float_as_uint(a);
      t[j + 1] = __float_as_uint(b);
    }
    const uint32_t lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    return make_uint2(lo, hi);
  }
}

template <bool kE4M3, int kThr, bool kShift>
__global__ void __launch_bounds__(kThr) quant_token_block_tma_kernel(const __grid_constant__ QuantParams p,
                                                                     const __grid_constant__ CUtensorMap tm,
                                                                     int64_t n_items, int stages,
                                                                     uint32_t slot_bytes) {
  using namespace ptx;
  constexpr int kCache = 4;
  extern __shared__ __align__(128) uint8_t qsm[];
  __shared__ alignas(8) uint64_t full[kMaxStages];
  __shared__ float red[2][kThr / 32];
  const int vpr = p.D >> 3;          // a power of two dividing kThr
  const int lg = __ffs(vpr) - 1;
  const int c = threadIdx.x & (vpr - 1);   // this thread's column vector
  const int r0 = threadIdx.x >> lg;        // its row in pass 0
  const int rstep = kThr >> lg;            // rows per pass
  const uint32_t box_bytes = static_cast<uint32_t>(p.rpb) * p.D * 2;  // zero-filled rows count too
  const uint32_t slots = smem_addr(qsm);
  auto issue = [&](int slot, const ItemCursor& ic) {  // thread 0
    const uint32_t bar = smem_addr(&full[slot]);
    mbar_arrive_expect_tx(bar, box_bytes);
    tma_load_4d(slots + slot * slot_bytes, &tm, bar, 0, ic.h, ic.blk * p.rpb, ic.b);
  };
  // Bounded wait for a slot's copy; a timeout is recorded in the error word.
  auto wait_full = [&](int slot, uint32_t parity) {
    const uint32_t bar = smem_addr(&full[slot]);
    if (mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, kQuantWaitSleepNs))
      if (static_cast<uint64_t>(clock64() - t0) > p.wait_cycles) {
        atomicOr(p.err, kErrTimeout);
        return false;
      }
    return true;
  };

  if (threadIdx.x == 0) {
    for (int k = 0; k < stages; ++k) mbar_init(smem_addr(&full[k]), 1);
    fence_barrier_init();
    prefetch_tmap(&tm);
  }
  __syncthreads();
  int issued = 0;  // thread 0: items whose copies were started
  ItemCursor ahead(blockIdx.x, gridDim.x, p.H, p.nblk);  // thread 0: the next item to copy
  if (threadIdx.x == 0)
    for (int k = 0; k < stages && blockIdx.x + static_cast<int64_t>(k) * gridDim.x < n_items; ++k, ++issued) {
      issue(k, ahead);
      ahead.advance(p.H, p.nblk);
    }

  int it = 0;
  ItemCursor ic(blockIdx.x, gridDim.x, p.H, p.nblk);
  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
    const int slot = it % stages;
    if (!__syncthreads_and(wait_full(slot, (it / stages) & 1))) break;
    const int b = ic.b, h = ic.h, blk = ic.blk;
    ic.advance(p.H, p.nblk);
    const int s0 = blk * p.rpb;
    const int rows = min(p.S - s0, p.rpb);
    const uint8_t* tile = qsm + slot * slot_bytes + c * 16;
    const int64_t bh = static_cast<int64_t>(b) * p.H + h;
    [[maybe_unused]] float sh[8];
    if constexpr (kShift) {
      const float* sp = shift_at(p, bh, c);
      const float4 a = __ldg(reinterpret_cast<const float4*>(sp)), e = __ldg(reinterpret_cast<const float4*>(sp + 4));
      sh[0] = a.x; sh[1] = a.y; sh[2] = a.z; sh[3] = a.w; sh[4] = e.x; sh[5] = e.y; sh[6] = e.z; sh[7] = e.w;
    }
    auto values = [&](const uint4& w, float (&x)[8]) {
      unpack8(w, x);
      if constexpr (kShift) {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = __fsub_rn(x[j], sh[j]);
      }
    };
    uint4 cache[kCache];
    float amax = 0.f;
    uint32_t am2 = 0u;  // no shift: max of |x| over BF16 pairs (magnitudes in bits 0-14, 16-30)
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
      const int r = r0 + i * rstep;
      if (r < rows) {
        cache[i] = *reinterpret_cast<const uint4*>(tile + r * (vpr * 16));
        if constexpr (kShift) {
          float x[8];
          values(cache[i], x);
          amax = fmaxf(amax, amax8(x));
        } else {
          am2 = max_abs_bf16x2(am2, max_abs_bf16x2(max_abs_bf16x2(cache[i].x, cache[i].y),
                                                   max_abs_bf16x2(cache[i].z, cache[i].w)));
        }
      }
    }
    if constexpr (!kShift) amax = __uint_as_float(max(am2 & 0x7FFFu, (am2 >> 16) & 0x7FFFu) << 16);
    amax = block_reduce_max<kThr>(amax, red[it & 1]);  // every thread has read the slot
    if (threadIdx.x == 0 && item + static_cast<int64_t>(stages) * gridDim.x < n_items) {
      fence_proxy_async_smem();  // generic reads of the slot before the copy that rewrites it
      issue(slot, ahead);
      ahead.advance(p.H, p.nblk);
      ++issued;
    }
    const Divisor dv(scale_from_amax<kE4M3>(amax));
    uint8_t* dst = p.dst + b * p.d_sb + static_cast<int64_t>(s0) * p.d_ss + h * p.d_sh + c * 8;
    if (dv.fast) {
#pragma unroll
      for (int i = 0; i < kCache; ++i) {
        const int r = r0 + i * rstep;
        if (r < rows) {
          float x[8];
          values(cache[i], x);
          *reinterpret_cast<uint2*>(dst + r * p.d_ss) = code8_fast<kE4M3, kShift>(x, cache[i], dv);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < kCache; ++i) {
        const int r = r0 + i * rstep;
        if (r < rows) {
          float x[8];
          values(cache[i], x);
          *reinterpret_cast<uint2*>(dst + r * p.d_ss) = code8<kE4M3>(x, dv);
        }
      }
    }
    if (threadIdx.x == 0) p.sf[bh * p.nblk + blk] = dv.s;
  }
  // After a timeout, copies may still be landing: shared memory stays until they do.
  if (threadIdx.x == 0) {
    for (int k = it; k < issued; ++k) {
      const uint32_t bar = smem_addr(&full[k % stages]);
      const long long t0 = clock64();
      while (!mbar_try_wait_sleep(bar, (k / stages) & 1, kQuantWaitSleepNs))
        if (static_cast<uint64_t>(clock64() - t0) > (1ull << 32)) break;
    }
  }
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
  if (p.kind == FMHA_SF_PER_CHANNEL) {
    const int cv = threadIdx.x % vpr;  // fixed column vector of this thread (256 % vpr == 0)
    const Divisor d8[8] = {
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 0]))),
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 1]))),
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 2]))),
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 3]))),
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 4]))),
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 5]))),
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 6]))),
        Divisor(scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + cv * 8 + 7])))};
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
      const int r = v / vpr, c = v - r * vpr;
      float x[8];
      vals8(ld16(src + r * p.s_ss + c * 8), shift_at(p, bh, c), x);
      *reinterpret_cast<uint2*>(dst + r * p.d_ss + c * 8) = code8<kE4M3>(x, d8);
    }
    if (chunk == 0)
      for (int ch = threadIdx.x; ch < p.D; ch += kThreads)
        p.sf[bh * p.D + ch] = scale_from_amax<kE4M3>(__uint_as_float(p.ws[bh * p.D + ch]));
  } else {
    const Divisor d(scale_from_amax<kE4M3>(__uint_as_float(p.ws[p.kind == FMHA_SF_PER_HEAD ? bh : 0])));
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
      const int r = v / vpr, c = v - r * vpr;
      float x[8];
      vals8(ld16(src + r * p.s_ss + c * 8), shift_at(p, bh, c), x);
      *reinterpret_cast<uint2*>(dst + r * p.d_ss + c * 8) = code8<kE4M3>(x, d);
    }
    if (chunk == 0 && threadIdx.x == 0) {
      if (p.kind == FMHA_SF_PER_HEAD)
        p.sf[bh] = d.s;
      else if (b == 0 && h == 0)
        p.sf[0] = d.s;
    }
  }
}

// S == 0 for a grid-wide kind: every group's amax is 0, so every scale is 1.
__global__ void __launch_bounds__(kThreads) fill_unit_scales_kernel(float* sf, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * kThreads)
    sf[i] = 1.f;
}

// TMA-staged token-block launch: 256 threads for blocks of up to 1024 16-byte
// vectors (16 KB), 512 up to 2048; as many CTAs as fit an SM's shared memory
// (at most 3), each with a ring of up to 4 slots.
template <bool kE4M3, bool kShift>
cudaError_t launch_token_block_tma(const QuantParams& p, const CUtensorMap& tm, int64_t items, cudaStream_t stream) {
  const uint32_t box = static_cast<uint32_t>(p.rpb) * p.D * 2;
  const uint32_t slot = (box + 127u) & ~127u;
  const bool big = box > 16384u;
  const int stages = big ? 3 : 4;
  const int smem = stages * static_cast<int>(slot);
  const int per_sm = std::max(1, std::min(3, (227 * 1024) / (smem + 2048)));
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(items, static_cast<int64_t>(sm_count()) * per_sm));
  cudaError_t e;
  if (big) {
    auto k = quant_token_block_tma_kernel<kE4M3, 512, kShift>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    k<<<grid, 512, smem, stream>>>(p, tm, items, stages, slot);
  } else {
    auto k = quant_token_block_tma_kernel<kE4M3, 256, kShift>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    k<<<grid, 256, smem, stream>>>(p, tm, items, stages, slot);
  }
  return cudaGetLastError();
}

template <bool kE4M3>
cudaError_t launch_quantize_t(const QuantParams& p, const CUtensorMap* tm, cudaStream_t stream) {
  if (p.kind == FMHA_SF_PER_TOKEN_BLOCK && tm != nullptr) {
    const int64_t items = static_cast<int64_t>(p.B) * p.nblk * p.H;
    return p.shift != nullptr ? launch_token_block_tma<kE4M3, true>(p, *tm, items, stream)
                              : launch_token_block_tma<kE4M3, false>(p, *tm, items, stream);
  }
  if (p.kind == FMHA_SF_PER_TOKEN_BLOCK) {
    // 256 threads for blocks of up to 1024 16-byte vectors (4 per thread), 512 above.
    const int64_t items = static_cast<int64_t>(p.B) * p.nblk * p.H;
    const bool big = static_cast<int64_t>(p.rpb) * (p.D >> 3) > 4 * 256;
    const bool sh = p.shift != nullptr;
    const int64_t resident = static_cast<int64_t>(sm_count()) * token_block_min_ctas(big ? 512 : 256, sh);
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(items, resident));
    if (big && sh) quant_token_block_kernel<kE4M3, 512, true><<<grid, 512, 0, stream>>>(p, items);
    else if (big) quant_token_block_kernel<kE4M3, 512, false><<<grid, 512, 0, stream>>>(p, items);
    else if (sh) quant_token_block_kernel<kE4M3, 256, true><<<grid, 256, 0, stream>>>(p, items);
    else quant_token_block_kernel<kE4M3, 256, false><<<grid, 256, 0, stream>>>(p, items);
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
__global__ void __launch_bounds__(kThreads, 3) channel_mean_partial_kernel(const QuantParams p) {
  __shared__ double red[kThreads * 8];
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int s0 = chunk * p.rows_per_cta;
  const int rows = min(p.S - s0, p.rows_per_cta);
  const int vpr = p.D >> 3;
  const int cv = threadIdx.x % vpr, row_step = kThreads / vpr;
  const uint16_t* src = p.src + b * p.s_sb + static_cast<int64_t>(s0) * p.s_ss + h * p.s_sh + cv * 8;
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  // kU row vectors in flight per thread (3 CTAs of 256 fit an SM at this
  // register count); the thread's rows are still added in ascending order.
  constexpr int kU = 10;
  for (int r0 = threadIdx.x / vpr; r0 < rows; r0 += kU * row_step) {
    uint4 w[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u)  // unpredicated: rows past the end reload the last row
      w[u] = ld16(src + static_cast<int64_t>(min(r0 + u * row_step, rows - 1)) * p.s_ss);
    asm volatile("" ::: "memory");  // every load of the batch is issued before the first use
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (r0 + u * row_step < rows) {
        float x[8];
        unpack8(w[u], x);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(x[i]);
      }
    }
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
// divides by S in fp64 and rounds once to fp32. The partials are loaded 16 at a
// time before any is added (one memory round trip per 16 chunks); the additions
// keep the chunk order.
__global__ void __launch_bounds__(kThreads) channel_mean_final_kernel(const QuantParams p) {
  constexpr int kBatch = 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (i >= static_cast<int64_t>(p.B) * p.H * p.D) return;
  const int64_t bh = i / p.D, ch = i - bh * p.D;
  const double* part = p.partial + bh * p.n_chunks * p.D + ch;
  double a = 0.0;
  for (int c0 = 0; c0 < p.n_chunks; c0 += kBatch) {
    double v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j)  // unpredicated: past the last chunk, reload the last one
      v[j] = part[static_cast<int64_t>(min(c0 + j, p.n_chunks - 1)) * p.D];
    asm volatile("" ::: "memory");  // every load of the batch is issued before the first add
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (c0 + j < p.n_chunks) a += v[j];
  }
  p.mean[i] = __double2float_rn(__ddiv_rn(a, static_cast<double>(p.S)));
}

}  // namespace

cudaError_t launch_quantize(bool to_e4m3, const QuantParams& p, const CUtensorMap* tm_src, cudaStream_t stream) {
  return to_e4m3 ? launch_quantize_t<true>(p, tm_src, stream) : launch_quantize_t<false>(p, tm_src, stream);
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
