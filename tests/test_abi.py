"""CPU checks of the C ABI: the library loads without a GPU, exports every
function include/fmha.h declares, and rejects bad arguments on the host
before any launch (these calls never reach the GPU)."""

import ctypes
import os
import re

import pytest

from precision_attention_fmha_b200 import build as build_mod
from precision_attention_fmha_b200 import fmha

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fmha.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(fmha.LIB_PATH):
        build_mod.build()
    return fmha.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(fmha_[a-z0-9_]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fmha_quantize_blockwise", "fmha_fwd", "fmha_fwd_block_sparse", "fmha_fwd_paged",
              "fmha_get_device_error", "fmha_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in fmha.STATUS.items():
        assert lib.fmha_status_string(code).decode() == name


def test_workspace_sizes(lib):
    assert fmha.quantize_workspace_bytes("per_token_block", 2, 100, 3, 128) == 0
    assert fmha.quantize_workspace_bytes("per_tensor", 2, 100, 3, 128) == 4
    assert fmha.quantize_workspace_bytes("per_head", 2, 100, 3, 128) == 2 * 3 * 4
    assert fmha.quantize_workspace_bytes("per_channel", 2, 100, 3, 128) == 2 * 3 * 128 * 4


def _args(D=128, dq=fmha.BF16, dv=fmha.BF16, ptr=0x10000, Hq=4, Hkv=2):
    a = fmha._Args()
    for t, dt in ((a.q, dq), (a.k, dq), (a.v, dv), (a.o, fmha.BF16)):
        t.ptr, t.dtype, t.reserved = ptr, dt, 0
        t.stride_b, t.stride_s, t.stride_h = 256 * Hq * D, Hq * D, D
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = 1, Hq, Hkv, 256, 256, D
    return a


@pytest.mark.parametrize("mutate,status", [
    (lambda a: setattr(a, "D", 96), 2),
    (lambda a: setattr(a, "Hkv", 3), 1),
    (lambda a: setattr(a.q, "ptr", 0), 1),
    (lambda a: setattr(a.q, "ptr", 0x10008), 1),
    (lambda a: setattr(a.k, "stride_s", 4 * 128 + 4), 1),
    (lambda a: (setattr(a.o, "dtype", fmha.E4M3), setattr(a, "D", 64)), 2),  # E4M3 O needs D = 128
    (lambda a: setattr(a.o, "dtype", fmha.INT8), 2),
    (lambda a: (setattr(a.sf_o, "kind", 1), setattr(a.sf_o, "ptr", 0x20000)), 2),  # sf_o with a BF16 O
    (lambda a: (setattr(a.o, "dtype", fmha.E4M3), setattr(a.sf_o, "kind", 2),
                setattr(a.sf_o, "ptr", 0x20000)), 2),  # per-head sf_o
    (lambda a: (setattr(a.o, "dtype", fmha.E4M3), setattr(a.sf_o, "kind", 1)), 1),  # sf_o.ptr NULL
    (lambda a: setattr(a.v, "dtype", fmha.INT8), 2),
    (lambda a: setattr(a.q, "reserved", 1), 1),
    (lambda a: setattr(a.sf_q, "kind", 1), 2),  # scale on a BF16 operand
])
def test_bad_arguments_rejected_before_launch(lib, mutate, status):
    a = _args()
    mutate(a)
    assert lib.fmha_fwd(ctypes.byref(a), None) == status
    assert lib.fmha_last_error_message().decode()


def test_empty_problem_is_a_no_op(lib):
    a = _args()
    a.Sq = 0
    assert lib.fmha_fwd(ctypes.byref(a), None) == 0


def test_eight_bit_scale_rules(lib):
    a = _args(dq=fmha.E4M3, dv=fmha.E4M3)
    a.sf_k.kind, a.sf_k.ptr, a.sf_k.rows_per_block = 3, 0x20000, 48  # not a multiple of 32
    assert lib.fmha_fwd(ctypes.byref(a), None) == 2
    a = _args(dq=fmha.E4M3, dv=fmha.E4M3, D=64)
    assert lib.fmha_fwd(ctypes.byref(a), None) == 2


def _wide_args(dq=fmha.BF16, dv=fmha.BF16, Dv=128):
    """D = 192 Q/K with a Dv-wide V / O (strides sized per operand)."""
    a = _args(D=192, dq=dq, dv=dv)
    for t in (a.v, a.o):
        t.stride_b, t.stride_s, t.stride_h = 256 * 4 * Dv, 4 * Dv, Dv
    a.Dv = Dv
    return a


@pytest.mark.parametrize("mutate", [
    lambda a: setattr(a, "Dv", 0),                                    # Dv = D = 192
    lambda a: setattr(a, "Dv", 192),
    lambda a: (setattr(a, "D", 128), setattr(a, "Dv", 64)),           # Dv != D below 192
    lambda a: (setattr(a.q, "dtype", fmha.INT8), setattr(a.k, "dtype", fmha.INT8),
               setattr(a.v, "dtype", fmha.E4M3)),                     # INT8 Q/K
    lambda a: setattr(a.o, "dtype", fmha.E4M3),                       # E4M3 O
    lambda a: (setattr(a.v, "dtype", fmha.E4M3), setattr(a, "p_terms", 2)),  # two-term P
])
def test_wide_qk_head_dim_rules(lib, mutate):
    """D = 192 takes Dv = 128, BF16 or E4M3 Q/K, one-term P and a BF16 O."""
    a = _wide_args()
    mutate(a)
    assert lib.fmha_fwd(ctypes.byref(a), None) == 2
    assert lib.fmha_last_error_message().decode()


def test_wide_qk_bf16_key_limit(lib):
    """D = 192 with BF16 Q/K deals key blocks through a 1024-bit set: Skv <= 131072."""
    a = _wide_args()
    a.Skv = 131072 + 1
    for t in (a.k, a.v):
        t.stride_b = (131072 + 1) * t.stride_s
    assert lib.fmha_fwd(ctypes.byref(a), None) == 2
    assert "131072" in lib.fmha_last_error_message().decode()


def test_paged_argument_checks(lib):
    a = _args()
    assert lib.fmha_fwd_paged(ctypes.byref(a), 0x30000, 8, 48, 4, None, 0, 0, None) == 2  # page size
    assert lib.fmha_fwd_paged(ctypes.byref(a), None, 8, 64, 4, None, 0, 0, None) == 1      # no table
    assert lib.fmha_fwd_paged(ctypes.byref(a), 0x30000, 8, 64, 3, None, 0, 0, None) == 1   # too few pages


def test_header_declares_decode_and_nvfp4(lib):
    names = declared_functions()
    for n in ("fmha_fwd_decode", "fmha_decode_workspace_bytes", "fmha_decode_num_splits", "fmha_quantize_nvfp4"):
        assert n in names and hasattr(lib, n)


def test_nvfp4_argument_checks(lib):
    f = lib.fmha_quantize_nvfp4
    src, codes, sb, st = 0x10000, 0x20000, 0x30000, 0x40000
    assert f(src, 64, 4, 40, codes, 32, sb, 4, st, 0, None) == 2       # K not a multiple of 16
    assert f(src, 32768, 4, 32768, codes, 16384, sb, 2048, st, 0, None) == 2  # K above 16384
    assert f(src + 2, 64, 4, 64, codes, 32, sb, 4, st, 0, None) == 1   # src misaligned
    assert f(src, 60, 4, 64, codes, 32, sb, 4, st, 0, None) == 1       # src row stride < K
    assert f(src, 64, 4, 64, codes + 4, 32, sb, 4, st, 0, None) == 1   # codes misaligned
    assert f(src, 64, 4, 64, codes, 28, sb, 4, st, 0, None) == 1       # codes row stride
    assert f(src, 64, 4, 64, codes, 32, sb, 3, st, 0, None) == 1       # block-scale row stride
    assert f(None, 64, 4, 64, codes, 32, sb, 4, st, 0, None) == 1      # NULL
    assert f(src, 64, 0, 64, codes, 32, sb, 4, st, 0, None) == 0       # nothing to do


def test_decode_rejects_e4m3_output(lib):
    a = _args()
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = 1, 4, 2, 1, 256, 128
    a.o.dtype = fmha.E4M3
    assert lib.fmha_fwd_decode(ctypes.byref(a), None, 0, 0, 0, None, 0, 0, 0, None, 0, None) == 2


def test_decode_plan_on_host(lib):
    a = _args()
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = 4, 64, 8, 1, 16384, 128
    splits = lib.fmha_decode_num_splits(ctypes.byref(a), 4)
    assert splits == 4
    # 8 partials (4 splits x the 2 interleaved query tiles), each O [B, Sq, Hq, D] fp32 + lse
    assert lib.fmha_decode_workspace_bytes(ctypes.byref(a), 4) == 8 * 4 * 1 * 64 * 129 * 4 + 16
    assert lib.fmha_decode_num_splits(ctypes.byref(a), 1000) == 128
    a.Sq = 40  # 320 packed rows: no interleave; one split = one partial, no workspace
    assert lib.fmha_decode_workspace_bytes(ctypes.byref(a), 1) == 0
    a.Sq = 2 ** 28  # x 8 query heads per KV head: 2^31 packed rows, beyond 32-bit row counts
    assert lib.fmha_decode_num_splits(ctypes.byref(a), 4) == 0
    assert lib.fmha_decode_workspace_bytes(ctypes.byref(a), 4) == 0
    a.Sq = 2 ** 28 - 1
    assert lib.fmha_decode_num_splits(ctypes.byref(a), 4) == 4


def test_decode_rejects_packed_rows_beyond_32_bits(lib):
    """Sq * Hq / Hkv >= 2^31 packed rows: FMHA_ERR_UNSUPPORTED before any launch."""
    a = _args()
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = 1, 16, 1, 2 ** 27, 1024, 128
    for t, h in ((a.q, 16), (a.o, 16), (a.k, 1), (a.v, 1)):
        t.stride_h, t.stride_s, t.stride_b = 128, h * 128, h * 128 * (2 ** 27)
    st = lib.fmha_fwd_decode(ctypes.byref(a), None, 0, 0, 0, None, 0, 0, 0, None, 0, None)
    assert st == 2 and "packed rows" in lib.fmha_last_error_message().decode()


def _bf16_tensor(B, S, H, D, ptr=0x10000):
    t = fmha._Tensor()
    t.ptr, t.dtype, t.reserved = ptr, fmha.BF16, 0
    t.stride_b, t.stride_s, t.stride_h = S * H * D, H * D, D
    return t


def test_k_smoothing_entry_points_on_host(lib):
    names = declared_functions()
    for n in ("fmha_channel_mean", "fmha_channel_mean_workspace_bytes", "fmha_quantize_blockwise_shifted"):
        assert n in names and hasattr(lib, n)
    # 1024 rows of D = 128 per CTA: fp64 partial sums [B, H, chunks, D]
    assert fmha.channel_mean_workspace_bytes(2, 100, 3, 128) == 2 * 3 * 1 * 128 * 8
    assert fmha.channel_mean_workspace_bytes(2, 2100, 3, 128) == 2 * 3 * 3 * 128 * 8
    assert fmha.channel_mean_workspace_bytes(2, 0, 3, 128) == 0
    src = _bf16_tensor(2, 2100, 3, 128)
    mean, ws, need = 0x40000, 0x80000, 2 * 3 * 3 * 128 * 8
    f = lib.fmha_channel_mean
    assert f(ctypes.byref(_bf16_tensor(2, 2100, 3, 96)), mean, 2, 2100, 3, 96, ws, need, None) == 2  # D not 2^k
    assert f(ctypes.byref(src), mean + 2, 2, 2100, 3, 128, ws, need, None) == 1   # mean misaligned
    assert f(ctypes.byref(src), None, 2, 2100, 3, 128, ws, need, None) == 1       # mean NULL
    assert f(ctypes.byref(src), mean, 2, 2100, 3, 128, ws, need - 8, None) == 1   # workspace too small
    assert f(ctypes.byref(src), mean, 2, 2100, 3, 128, ws + 4, need, None) == 1   # workspace misaligned
    assert f(ctypes.byref(src), mean, 0, 2100, 3, 128, None, 0, None) == 0        # nothing to do
    g = lib.fmha_quantize_blockwise_shifted
    dst = _bf16_tensor(2, 300, 3, 128, ptr=0x100000)
    dst.dtype = fmha.INT8
    sf = fmha._Sf(0x200000, fmha.SF_KINDS["per_token_block"], 64)
    assert g(ctypes.byref(src), None, ctypes.byref(dst), ctypes.byref(sf), 2, 300, 3, 128, None, 0, None) == 1
    assert g(ctypes.byref(src), 0x40004, ctypes.byref(dst), ctypes.byref(sf), 2, 300, 3, 128, None, 0, None) == 1
    assert g(ctypes.byref(src), 0x40000, ctypes.byref(dst), ctypes.byref(sf), 0, 300, 3, 128, None, 0, None) == 0


def test_masked_launch_limits_key_blocks(lib):
    """A block mask needs Skv <= 131072 (the CTA's 1024-bit keep set); without a mask there is no limit."""
    a = _args()
    a.Skv = 131072 + 1
    for t in (a.k, a.v):
        t.stride_b = a.Skv * a.Hkv * a.D
    assert lib.fmha_fwd_block_sparse(ctypes.byref(a), 0x40000, 0, 0, None) == 2
    assert "131072" in lib.fmha_last_error_message().decode()


def test_quantizer_grid_limit_on_host(lib):
    x = fmha._Tensor(0x10000, fmha.BF16, 0, 70000 * 8 * 128, 70000 * 128, 128)
    y = fmha._Tensor(0x20000, fmha.INT8, 0, 70000 * 8 * 128, 70000 * 128, 128)
    sf = fmha._Sf(0x30000, 3, 64)
    assert lib.fmha_quantize_blockwise(ctypes.byref(x), ctypes.byref(y), ctypes.byref(sf), 1, 8, 70000, 128,
                                       None, 0, None) == 2
