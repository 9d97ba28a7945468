"""The no-allocation quantizer entry point, through the C ABI.

fmha_quantize_blockwise_noalloc serves callers that cannot allocate device
memory for a call (an engine that owns all device memory and exposes no
allocator; a latency-critical path where cudaMalloc is not allowed). It keeps
its amax accumulators in a device array built into the library instead of a
caller workspace. Its codes and scales must equal those of the ordinary entry
point, call after call: the shared array keeps the previous call's contents,
so two different calls in a row also check that each call clears what it uses.
This file is collected last so a failure here cannot hide the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

from precision_attention_fmha_b200 import fmha, workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
KINDS = {"per_tensor": 1, "per_head": 2, "per_token_block": 3, "per_channel": 4}


def _lib():
    lib = fmha.load_library()
    f = lib.fmha_quantize_blockwise_noalloc
    f.argtypes = [ctypes.POINTER(fmha._Tensor), ctypes.POINTER(fmha._Tensor), ctypes.POINTER(fmha._Sf),
                  ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return lib


def _noalloc(x, out_dtype, kind, rows_per_block=0):
    lib = _lib()
    B, S, H, D = x.shape
    codes = torch.empty(x.shape, dtype=out_dtype, device=DEV)
    scales = torch.empty(fmha.scale_shape(kind, B, S, H, D, rows_per_block or 1), dtype=torch.float32, device=DEV)
    src, dst = fmha._tensor(x), fmha._tensor(codes)
    sf = fmha._Sf(scales.data_ptr(), KINDS[kind], rows_per_block)
    st = lib.fmha_quantize_blockwise_noalloc(ctypes.byref(src), ctypes.byref(dst), ctypes.byref(sf), B, S, H, D,
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, codes, scales


def _bits(t):
    t = t.cpu()
    return t.view(torch.uint8).numpy() if t.dtype == torch.float8_e4m3fn else t.numpy()


@pytest.mark.parametrize("kind,out,rpb", [("per_tensor", torch.float8_e4m3fn, 0), ("per_head", torch.int8, 0),
                                          ("per_channel", torch.float8_e4m3fn, 0),
                                          ("per_token_block", torch.int8, 64)])
def test_noalloc_matches_workspace_entry_point_twice(kind, out, rpb):
    for call, seed in enumerate((101, 202)):  # two calls in a row, different data
        x, _, _ = workloads.outlier_qkv(seed, 2, 500 + 37 * call, 3, 128)
        x = x.to(DEV)
        st, codes, scales = _noalloc(x, out, kind, rpb)
        assert st == 0, _lib().fmha_last_error_message().decode()
        ref_codes, ref_scales = fmha.fmha_quantize_blockwise(x, out, kind, rpb or None)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(codes), _bits(ref_codes)), f"codes differ on call {call}"
        assert np.array_equal(scales.cpu().numpy(), ref_scales.cpu().numpy()), f"scales differ on call {call}"


def test_noalloc_rejects_more_groups_than_the_builtin_scratch():
    x, _, _ = workloads.normal_qkv(5, 1, 8, 8, 2, 2, 128)
    x = x.to(DEV)
    lib = _lib()
    codes = torch.empty(x.shape, dtype=torch.int8, device=DEV)
    scales = torch.empty(1, dtype=torch.float32, device=DEV)
    src, dst = fmha._tensor(x), fmha._tensor(codes)
    sf = fmha._Sf(scales.data_ptr(), KINDS["per_channel"], 0)
    # 1 x 513 x 128 = 65664 per-channel groups > 65536: rejected before anything runs
    st = lib.fmha_quantize_blockwise_noalloc(ctypes.byref(src), ctypes.byref(dst), ctypes.byref(sf), 1, 8, 513, 128,
                                            None)
    assert st == 1
    assert "65536" in lib.fmha_last_error_message().decode()


@pytest.mark.parametrize("kind", ["per_tensor", "per_head", "per_channel", "per_token_block"])
def test_noalloc_empty_sequence(kind):
    """S == 0 through the no-allocation entry point: no code, unit scales for the grid-wide kinds,
    the same as the workspace entry point."""
    x = torch.zeros((2, 0, 3, 128), dtype=torch.bfloat16, device=DEV)
    st, codes, scales = _noalloc(x, torch.int8, kind, 64 if kind == "per_token_block" else 0)
    assert st == 0, _lib().fmha_last_error_message().decode()
    _, ref_scales = fmha.fmha_quantize_blockwise(x, torch.int8, kind, 64 if kind == "per_token_block" else None)
    torch.cuda.synchronize()
    assert codes.numel() == 0
    assert np.array_equal(scales.cpu().numpy(), ref_scales.cpu().numpy())
    if kind != "per_token_block":
        assert np.all(scales.cpu().numpy() == 1.0)
