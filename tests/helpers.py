"""Shared test helpers: dtype conversions and the parity checks.

Tolerances are the ones the attention path is specified to: BF16 operands
within max-abs 1e-2 of the oracle on unit-variance inputs; 8-bit (E4M3 /
INT8) operands within max-abs 3e-2 and cosine similarity >= 0.999 per head.
The 8-bit max-abs bound is stated for outputs of unit scale; per head it is
multiplied by max(1, max |O_ref|) so that outputs far above unit scale (the
outlier workload reaches |O| ~ 60, where BF16 output rounding alone is
2^-9 |O| ~ 0.12) are held to the same relative accuracy. Cosine similarity
per head stays the binding check.
"""

import numpy as np
import torch

BF16_ATOL = 1e-2
Q8_ATOL = 3e-2
Q8_COS = 0.999


def f64(t):
    """torch tensor (bf16 / fp32 / int8) on any device -> float64 numpy."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def f32(t):
    return t.detach().to("cpu").to(torch.float32).numpy()


def codes_np(t):
    """8-bit codes tensor -> numpy int8 (INT8) or uint8 bit patterns (E4M3)."""
    t = t.detach().to("cpu")
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def to_torch_codes(codes, dtype, device):
    if dtype == torch.float8_e4m3fn:
        return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(device)
    return torch.from_numpy(np.ascontiguousarray(codes)).to(device)


def cos_per_head(o, ref):
    """Cosine similarity per (b, h) over (S, D); o, ref [B, S, H, D] float64."""
    a = np.moveaxis(o, 2, 1).reshape(o.shape[0] * o.shape[2], -1)
    b = np.moveaxis(ref, 2, 1).reshape(ref.shape[0] * ref.shape[2], -1)
    na, nb = np.linalg.norm(a, axis=1), np.linalg.norm(b, axis=1)
    ok = (na > 0) & (nb > 0)
    c = np.ones(a.shape[0])
    c[ok] = np.sum(a[ok] * b[ok], axis=1) / (na[ok] * nb[ok])
    both_zero = (na == 0) & (nb == 0)
    c[~ok & ~both_zero] = 0.0
    return c


def assert_close_bf16(o, ref, atol=BF16_ATOL):
    err = np.abs(o - ref)
    assert np.all(np.isfinite(o)), "non-finite output"
    assert err.max() <= atol, f"max-abs {err.max():.3e} > {atol} (at {np.unravel_index(err.argmax(), err.shape)})"


def assert_close_q8(o, ref, atol=Q8_ATOL, cos_min=Q8_COS):
    assert np.all(np.isfinite(o)), "non-finite output"
    err = np.abs(o - ref)
    err_h = err.max(axis=(1, 3))  # [B, H]
    scale_h = np.maximum(1.0, np.abs(ref).max(axis=(1, 3)))
    worst = np.unravel_index(np.argmax(err_h / scale_h), err_h.shape)
    assert np.all(err_h <= atol * scale_h), (
        f"max-abs {err_h[worst]:.3e} > {atol} x {scale_h[worst]:.2f} (head {worst})")
    c = cos_per_head(o, ref)
    assert c.min() >= cos_min, f"min cos per head {c.min():.6f} < {cos_min}"
