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
    (lambda a: setattr(a.o, "dtype", fmha.E4M3), 2),
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


def test_paged_argument_checks(lib):
    a = _args()
    assert lib.fmha_fwd_paged(ctypes.byref(a), 0x30000, 8, 48, 4, None, 0, 0, None) == 2  # page size
    assert lib.fmha_fwd_paged(ctypes.byref(a), None, 8, 64, 4, None, 0, 0, None) == 1      # no table
    assert lib.fmha_fwd_paged(ctypes.byref(a), 0x30000, 8, 64, 3, None, 0, 0, None) == 1   # too few pages
