"""CPU oracle for the mixed-precision FMHA forward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code, table or constant with the
CUDA library, and it imports nothing from it.

What it computes (plain, slow, obviously correct):

* ``e4m3``      -- the OCP 8-bit float E4M3 ("E4M3FN") codec, written from the
                   format definition (bias 7, no infinities, max 448).
* ``quant``     -- block quantization: amax -> scale = amax/R -> INT8 or E4M3
                   codes, in IEEE float32 exactly as stated (one division for
                   the scale, one per element for the code); the token mean
                   per channel and quantization of x minus a shift, for
                   SageAttention's K smoothing.
* ``nvfp4``     -- per-token NVFP4 quantization: E2M1 codec from the format
                   definition and the two-level (E4M3 per 16 elements, fp32
                   per token) scaling in IEEE float32.
* ``attention`` -- scaled-dot-product attention in float64 on dequantized
                   operands, with causal / 128x128 block masks, GQA and a
                   paged-KV gather.
* ``online_softmax`` -- the same attention through the tiled online softmax
                   (128-key tiles, lazy rescale past 2^tau) with P rounded as
                   the kernels store it (BF16, one or two E4M3 terms with the P
                   scale): a model of the approximation, for checks finer than
                   the stated tolerance.

Sources (page titles; sections):

* "FlashInfer DiT optimization: SageAttention and Int8/FP8 mixed-precision
  kernels" (flashinfer PR #2711), sections 2 (SageAttention scale factors) and
  "Why" item 2 (block-wise scaling beats per-tensor for outlier-heavy maps).
* "FlashInfer FP8/BF16 mixed-precision attention for Blackwell" (flashinfer
  PR #5900), introduction (dense context FMHA, QK-BF16/PV-FP8 and all-FP8),
  sections 1 (P in FP8 staged for the PV product) and 3 (the row max moved
  lazily, past a 2^8 jump).
* "FlashInfer block-sparse attention with PrimTS" (flashinfer PR #4474),
  section 2 (block-sparse API over contiguous and paged K/V).
* "FlashInfer per-token NVFP4 quantization kernel" (flashinfer PR #3237),
  introduction and sections 1-2 (per-token NVFP4 codes, on-chip input
  staging, a switchable fast-math path).

The pages never write the attention formula down; the oracle uses the
textbook definition O = softmax(scale * Q K^T) V. Every reading taken where
the pages are silent is listed in the module that takes it.

Parity pins: every function here is pinned by ``tests/test_oracle_*.py``
against brute force, closed forms, invariants or an independent library
routine. ``attention`` is the definition the tolerances are stated against
(on the dequantized operands). The kernels' internal rounding of the softmax
output P (not an operand) is modelled by ``online_softmax``, which is pinned to
``attention`` when P is kept unrounded and to the formats' rounding bounds
when it is not.
"""

from . import e4m3, quant, attention, online_softmax  # noqa: F401
