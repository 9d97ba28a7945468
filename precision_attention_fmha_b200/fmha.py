"""ctypes binding of libfmha.so (include/fmha.h).

Argument marshalling only: every step of the computation runs in the CUDA
library. PyTorch supplies device memory (outputs are allocated with
``torch.empty``) and the current stream. If the library is missing the first
call raises -- there is no fallback implementation.

Tensors are token-major [B, S, H, D] with the last dim contiguous. 8-bit
operands are ``torch.int8`` (INT8) or ``torch.float8_e4m3fn`` (E4M3). A scale
factor is given as ``Scale(tensor, kind, rows_per_block)`` with ``kind`` one
of "per_tensor", "per_head", "per_token_block", "per_channel".
"""

import ctypes
import math
import os
from collections import namedtuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfmha.so")

BF16, FP16, FP32, E4M3, INT8 = 0, 1, 2, 3, 4
SF_KINDS = {None: 0, "none": 0, "per_tensor": 1, "per_head": 2, "per_token_block": 3, "per_channel": 4}
STATUS = {0: "FMHA_OK", 1: "FMHA_ERR_INVALID_ARG", 2: "FMHA_ERR_UNSUPPORTED", 3: "FMHA_ERR_CUDA",
          4: "FMHA_ERR_TIMEOUT", 5: "FMHA_ERR_DEVICE_INDEX"}
FMHA_OK, FMHA_ERR_INVALID_ARG, FMHA_ERR_UNSUPPORTED, FMHA_ERR_CUDA, FMHA_ERR_TIMEOUT, FMHA_ERR_DEVICE_INDEX = range(6)

Scale = namedtuple("Scale", ["tensor", "kind", "rows_per_block"], defaults=[0])


class FmhaError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class _Tensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("stride_b", ctypes.c_int64), ("stride_s", ctypes.c_int64), ("stride_h", ctypes.c_int64)]


class _Sf(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("kind", ctypes.c_int32), ("rows_per_block", ctypes.c_int32)]


class _Args(ctypes.Structure):
    _fields_ = [("q", _Tensor), ("k", _Tensor), ("v", _Tensor), ("o", _Tensor),
                ("sf_q", _Sf), ("sf_k", _Sf), ("sf_v", _Sf), ("sf_p", _Sf),
                ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("Sq", ctypes.c_int32), ("Skv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("causal", ctypes.c_int32), ("lse", ctypes.c_void_p),
                ("p_terms", ctypes.c_int32), ("Dv", ctypes.c_int32), ("sf_o", _Sf)]


_lib = None


def load_library(path=None):
    """Loads libfmha.so once (raises if it is missing) and declares the C signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libfmha.so not built ({path}); run `python -m precision_attention_fmha_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.fmha_quantize_blockwise.argtypes = [ctypes.POINTER(_Tensor), ctypes.POINTER(_Tensor), ctypes.POINTER(_Sf),
                                            i32, i32, i32, i32, vp, sz, vp]
    lib.fmha_quantize_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.fmha_quantize_workspace_bytes.restype = sz
    lib.fmha_quantize_blockwise_shifted.argtypes = [ctypes.POINTER(_Tensor), vp, ctypes.POINTER(_Tensor),
                                                    ctypes.POINTER(_Sf), i32, i32, i32, i32, vp, sz, vp]
    lib.fmha_channel_mean.argtypes = [ctypes.POINTER(_Tensor), vp, i32, i32, i32, i32, vp, sz, vp]
    lib.fmha_channel_mean_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.fmha_channel_mean_workspace_bytes.restype = sz
    lib.fmha_fwd.argtypes = [ctypes.POINTER(_Args), vp]
    lib.fmha_fwd_block_sparse.argtypes = [ctypes.POINTER(_Args), vp, i64, i64, vp]
    lib.fmha_fwd_paged.argtypes = [ctypes.POINTER(_Args), vp, i32, i32, i32, vp, i64, i64, vp]
    lib.fmha_get_device_error.argtypes = [vp]
    lib.fmha_fwd_decode.argtypes = [ctypes.POINTER(_Args), vp, i32, i32, i32, vp, i64, i64, i32, vp, sz, vp]
    lib.fmha_quantize_nvfp4.argtypes = [vp, i64, i32, i32, vp, i64, vp, i64, vp, i32, vp]
    lib.fmha_decode_workspace_bytes.argtypes = [ctypes.POINTER(_Args), i32]
    lib.fmha_decode_workspace_bytes.restype = sz
    lib.fmha_decode_num_splits.argtypes = [ctypes.POINTER(_Args), i32]
    lib.fmha_decode_num_splits.restype = i32
    lib.fmha_status_string.argtypes = [ctypes.c_int]
    lib.fmha_status_string.restype = ctypes.c_char_p
    lib.fmha_last_error_message.restype = ctypes.c_char_p
    lib.fmha_set_wait_timeout_cycles.argtypes = [ctypes.c_uint64]
    for f in ("fmha_quantize_blockwise", "fmha_fwd", "fmha_fwd_block_sparse", "fmha_fwd_paged",
              "fmha_get_device_error", "fmha_quantize_blockwise_shifted", "fmha_channel_mean"):
        getattr(lib, f).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status):
    if status != 0:
        msg = load_library().fmha_last_error_message().decode()
        raise FmhaError(status, msg)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return FP16
    if t.dtype == torch.float8_e4m3fn:
        return E4M3
    if t.dtype == torch.int8:
        return INT8
    raise TypeError(f"unsupported dtype {t.dtype}")


def _tensor(t):
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, S, H, D] tensor with a contiguous last dim")
    return _Tensor(t.data_ptr(), _dtype_code(t), 0, t.stride(0), t.stride(1), t.stride(2))


def _sf(s):
    if s is None:
        return _Sf(None, 0, 0)
    if not isinstance(s, Scale):
        raise TypeError("scale factors are Scale(tensor, kind, rows_per_block)")
    if s.tensor.dtype != torch.float32 or not s.tensor.is_contiguous():
        raise ValueError("scale tensors must be contiguous float32")
    return _Sf(s.tensor.data_ptr(), SF_KINDS[s.kind], int(s.rows_per_block or 0))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def quantize_workspace_bytes(kind, B, S, H, D):
    return load_library().fmha_quantize_workspace_bytes(SF_KINDS[kind], B, S, H, D)


def scale_shape(kind, B, S, H, D, rows_per_block=None):
    if kind == "per_tensor":
        return (1,)
    if kind == "per_head":
        return (B, H)
    if kind == "per_token_block":
        return (B, H, math.ceil(S / rows_per_block))
    if kind == "per_channel":
        return (B, H, D)
    raise ValueError(kind)


def fmha_quantize_blockwise(x, out_dtype, kind, rows_per_block=None, out=None, scales=None, workspace=None,
                            stream=None, shift=None):
    """BF16 x [B,S,H,D] -> (codes, fp32 scales). out_dtype: torch.int8 or torch.float8_e4m3fn.

    shift (optional, contiguous fp32 [B, H, D] on the device): quantize
    x - shift instead of x (K smoothing; see ``channel_mean``).
    """
    lib = load_library()
    if shift is not None and (shift.dtype != torch.float32 or not shift.is_contiguous()
                              or tuple(shift.shape) != (x.shape[0], x.shape[2], x.shape[3])):
        raise ValueError("shift must be a contiguous float32 [B, H, D] tensor")
    B, S, H, D = x.shape
    if out is None:
        out = torch.empty((B, S, H, D), dtype=out_dtype, device=x.device)
    if scales is None:
        scales = torch.empty(scale_shape(kind, B, S, H, D, rows_per_block), dtype=torch.float32, device=x.device)
    need = lib.fmha_quantize_workspace_bytes(SF_KINDS[kind], B, S, H, D)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    src, dst = _tensor(x), _tensor(out)
    sf = _Sf(scales.data_ptr(), SF_KINDS[kind], int(rows_per_block or 0))
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if shift is None:
        _check(lib.fmha_quantize_blockwise(ctypes.byref(src), ctypes.byref(dst), ctypes.byref(sf), B, S, H, D,
                                           ws_ptr, ws_bytes, _stream(stream)))
    else:
        _check(lib.fmha_quantize_blockwise_shifted(ctypes.byref(src), shift.data_ptr(), ctypes.byref(dst),
                                                   ctypes.byref(sf), B, S, H, D, ws_ptr, ws_bytes, _stream(stream)))
    return out, scales


def channel_mean_workspace_bytes(B, S, H, D):
    return load_library().fmha_channel_mean_workspace_bytes(B, S, H, D)


def channel_mean(x, out=None, workspace=None, stream=None):
    """Token mean per (b, h, d) of BF16 x [B, S, H, D] -> fp32 [B, H, D] (fp64 sums)."""
    lib = load_library()
    B, S, H, D = x.shape
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=x.device)
    need = lib.fmha_channel_mean_workspace_bytes(B, S, H, D)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    src = _tensor(x)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.fmha_channel_mean(ctypes.byref(src), out.data_ptr(), B, S, H, D, ws_ptr, ws_bytes,
                                 _stream(stream)))
    return out


def quantize_smoothed(x, out_dtype, kind, rows_per_block=None, stream=None):
    """SageAttention K smoothing: (codes, scales, mean) with codes * scales ~= x - mean."""
    mean = channel_mean(x, stream=stream)
    codes, scales = fmha_quantize_blockwise(x, out_dtype, kind, rows_per_block, stream=stream, shift=mean)
    return codes, scales, mean


def _args(q, k, v, out, sf_q, sf_k, sf_v, sf_p, softmax_scale, causal, lse, Skv=None, p_terms=1, sf_o=None):
    B, Sq, Hq, D = q.shape
    Hkv = k.shape[2]
    a = _Args()
    a.q, a.k, a.v, a.o = _tensor(q), _tensor(k), _tensor(v), _tensor(out)
    a.sf_q, a.sf_k, a.sf_v, a.sf_p = _sf(sf_q), _sf(sf_k), _sf(sf_v), _sf(sf_p)
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = B, Hq, Hkv, Sq, k.shape[1] if Skv is None else Skv, D
    a.softmax_scale = float(softmax_scale) if softmax_scale else 0.0
    a.causal = 1 if causal else 0
    a.lse = lse.data_ptr() if lse is not None else None
    a.p_terms = int(p_terms)
    a.Dv = v.shape[3]
    a.sf_o = _sf(sf_o)
    return a


def _out_like(q, v, out):
    """O is [B, Sq, Hq, Dv]: Dv, the head dim of V, differs from q's for D = 192 / 128."""
    if out is None:
        out = torch.empty(q.shape[:3] + v.shape[3:], dtype=torch.bfloat16, device=q.device)
    return out


def fmha_fwd(q, k, v, out=None, sf_q=None, sf_k=None, sf_v=None, sf_p=None, softmax_scale=None, causal=False,
             lse=None, stream=None, p_terms=1, sf_o=None):
    """Dense attention. Returns O (BF16 [B, Sq, Hq, Dv]). p_terms=2 splits an E4M3 P into two terms.

    Head dims: q / k D and v / out Dv, equal (64 or 128), or D = 192 with Dv = 128.

    An E4M3 ``out`` (torch.float8_e4m3fn, D = 128) receives E4M3(O / sf_o),
    with sf_o an optional per-tensor Scale (1.0 when None)."""
    lib = load_library()
    out = _out_like(q, v, out)
    a = _args(q, k, v, out, sf_q, sf_k, sf_v, sf_p, softmax_scale, causal, lse, p_terms=p_terms, sf_o=sf_o)
    _check(lib.fmha_fwd(ctypes.byref(a), _stream(stream)))
    return out


def fmha_fwd_block_sparse(q, k, v, mask, out=None, sf_q=None, sf_k=None, sf_v=None, sf_p=None,
                          softmax_scale=None, causal=False, lse=None, stream=None, p_terms=1, sf_o=None):
    """Attention restricted by a uint8 128x128 block mask [B or 1, Hkv or 1, ceil(Sq/128), ceil(Skv/128)]."""
    lib = load_library()
    out = _out_like(q, v, out)
    a = _args(q, k, v, out, sf_q, sf_k, sf_v, sf_p, softmax_scale, causal, lse, p_terms=p_terms, sf_o=sf_o)
    msb, msh = _mask_strides(mask, q.shape[1], k.shape[1])
    _check(lib.fmha_fwd_block_sparse(ctypes.byref(a), mask.data_ptr(), msb, msh, _stream(stream)))
    return out


def _mask_strides(mask, Sq, Skv):
    if mask.dtype != torch.uint8 or mask.dim() != 4:
        raise ValueError("mask must be uint8 [B, Hkv, ceil(Sq/128), ceil(Skv/128)]")
    nq, nk = math.ceil(Sq / 128), math.ceil(Skv / 128)
    if mask.shape[2] != nq or mask.shape[3] != nk or mask.stride(3) != 1 or mask.stride(2) != nk:
        raise ValueError(f"mask inner dims must be contiguous [{nq}, {nk}]")
    return (mask.stride(0) if mask.shape[0] > 1 else 0), (mask.stride(1) if mask.shape[1] > 1 else 0)


def fmha_fwd_paged(q, k_pool, v_pool, page_table, Skv, mask=None, out=None, sf_q=None, sf_k=None, sf_v=None,
                   sf_p=None, softmax_scale=None, causal=False, lse=None, stream=None, p_terms=1, sf_o=None):
    """Attention over a paged K/V pool [num_pages, page_size, Hkv, D] through page_table int32 [B, max_pages]."""
    lib = load_library()
    out = _out_like(q, v_pool, out)
    if page_table.dtype != torch.int32 or page_table.dim() != 2 or not page_table.is_contiguous():
        raise ValueError("page_table must be contiguous int32 [B, max_pages_per_seq]")
    a = _args(q, k_pool, v_pool, out, sf_q, sf_k, sf_v, sf_p, softmax_scale, causal, lse, Skv=Skv, p_terms=p_terms,
              sf_o=sf_o)
    mptr, msb, msh = None, 0, 0
    if mask is not None:
        msb, msh = _mask_strides(mask, q.shape[1], Skv)
        mptr = mask.data_ptr()
    _check(lib.fmha_fwd_paged(ctypes.byref(a), page_table.data_ptr(), k_pool.shape[0], k_pool.shape[1],
                              page_table.shape[1], mptr, msb, msh, _stream(stream)))
    return out


def fmha_fwd_decode(q, k, v, page_table=None, Skv=None, mask=None, num_splits=0, workspace=None, out=None,
                    sf_q=None, sf_k=None, sf_v=None, sf_p=None, softmax_scale=None, causal=False, lse=None,
                    stream=None):
    """Decode-shaped attention (few query tokens, GQA-packed tiles, split-KV).

    k / v: contiguous [B, Skv, Hkv, D], or page pools [num_pages, page_size, Hkv, D]
    with page_table int32 [B, max_pages] and Skv. The workspace (uint8 CUDA tensor)
    is allocated here when not given. Returns O (BF16 [B, Sq, Hq, D])."""
    lib = load_library()
    out = _out_like(q, v, out)
    if page_table is not None:
        if page_table.dtype != torch.int32 or page_table.dim() != 2 or not page_table.is_contiguous():
            raise ValueError("page_table must be contiguous int32 [B, max_pages_per_seq]")
        if Skv is None:
            raise ValueError("Skv is required with a page table")
    a = _args(q, k, v, out, sf_q, sf_k, sf_v, sf_p, softmax_scale, causal, lse, Skv=Skv)
    mptr, msb, msh = None, 0, 0
    if mask is not None:
        msb, msh = _mask_strides(mask, q.shape[1], a.Skv)
        mptr = mask.data_ptr()
    need = lib.fmha_decode_workspace_bytes(ctypes.byref(a), int(num_splits))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wptr, wbytes = (workspace.data_ptr(), workspace.numel() * workspace.element_size()) if workspace is not None \
        else (None, 0)
    if page_table is not None:
        pt, npages, psize, maxp = page_table.data_ptr(), k.shape[0], k.shape[1], page_table.shape[1]
    else:
        pt, npages, psize, maxp = None, 0, 0, 0
    _check(lib.fmha_fwd_decode(ctypes.byref(a), pt, npages, psize, maxp, mptr, msb, msh, int(num_splits), wptr,
                               wbytes, _stream(stream)))
    return out


def decode_num_splits(q, k, Skv=None, num_splits=0):
    """KV splits fmha_fwd_decode uses for these shapes (host only)."""
    B, Sq, Hq, D = q.shape
    a = _Args()
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = B, Hq, k.shape[2], Sq, k.shape[1] if Skv is None else Skv, D
    return load_library().fmha_decode_num_splits(ctypes.byref(a), int(num_splits))


def quantize_nvfp4(x, fast_math=False, codes=None, block_scales=None, token_scales=None, stream=None):
    """Per-token NVFP4 of a BF16 CUDA matrix [rows, K] (row stride x.stride(0)).

    Returns (codes uint8 [rows, K/2], block_scales float8_e4m3fn [rows, K/16],
    token_scales float32 [rows])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a BF16 [rows, K] matrix with unit column stride")
    rows, K = x.shape
    dev = x.device
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    block_scales = torch.empty((rows, K // 16), dtype=torch.uint8, device=dev) if block_scales is None \
        else block_scales.view(torch.uint8)
    token_scales = torch.empty((rows,), dtype=torch.float32, device=dev) if token_scales is None else token_scales
    _check(load_library().fmha_quantize_nvfp4(x.data_ptr(), x.stride(0), rows, K, codes.data_ptr(), codes.stride(0),
                                              block_scales.data_ptr(), block_scales.stride(0),
                                              token_scales.data_ptr(), 1 if fast_math else 0, _stream(stream)))
    return codes, block_scales.view(torch.float8_e4m3fn), token_scales


def decode_workspace_bytes(q, k, Skv=None, num_splits=0):
    """Workspace bytes fmha_fwd_decode needs for these shapes (host only)."""
    B, Sq, Hq, D = q.shape
    a = _Args()
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = B, Hq, k.shape[2], Sq, k.shape[1] if Skv is None else Skv, D
    return load_library().fmha_decode_workspace_bytes(ctypes.byref(a), int(num_splits))


def decode_num_parts(q, k, Skv=None, num_splits=0):
    """Partial outputs fmha_fwd_decode merges (1: no merge launch)."""
    need = decode_workspace_bytes(q, k, Skv, num_splits)
    if need == 0:
        return 1
    B, Sq, Hq, D = q.shape
    return (need - 16) // (B * Sq * Hq * (D + 1) * 4)


def get_device_error(stream=None):
    """Synchronises the stream and raises FmhaError if a kernel recorded a device-side error."""
    _check(load_library().fmha_get_device_error(_stream(stream)))


def set_wait_timeout_cycles(cycles):
    load_library().fmha_set_wait_timeout_cycles(int(cycles))
