"""Thin ctypes binding of libattn_b200.so (C ABI in include/attn.h).

Argument marshalling only: shapes are read from the torch tensors, device pointers and the
current CUDA stream are passed through, and every step of the computation runs in the CUDA
library. Importing this module raises if the library has not been built; there is no fallback.

Functions keep the C names; q, k, v (and o) are all bf16 or all fp16, and the element type is
taken from q (the C ``*_typed`` entry points receive it):
    attn_fwd(q, k, v, causal=..., scale=None, out=None, lse=None)          -> (o, lse)
    attn_fwd_sparse(q, k, v, block_idx, block_cnt, causal=..., ...)        -> (o, lse)
    attn_decode(q, k, v, causal=..., dv=None, num_splits=0, impl=0, ...)   -> (o, lse)
    attn_combine(o_part, lse_part, out=None, lse=None, dtype=bf16)         -> (o, lse)
    attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, num_splits)         -> int
    attn_status_string(code), attn_check_device(), attn_selftest_wait_timeout(limit_us)
plus attn_fwd_host(...): host tensors in, host tensors out (the C attn_fwd_host pipeline).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn_b200.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m exact_attention_139_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_lib.attn_fwd.restype = _i
_lib.attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 7 + [_f, _i, _vp]
_lib.attn_fwd_typed.restype = _i
_lib.attn_fwd_typed.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 7 + [_f, _i, _i, _vp]
_lib.attn_fwd_sparse_typed.restype = _i
_lib.attn_fwd_sparse_typed.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 7 + [_f, _i, _vp, _vp, _i, _i, _vp]
_lib.attn_decode_workspace_size.restype = _sz
_lib.attn_decode_workspace_size.argtypes = [_i] * 7
_lib.attn_decode.restype = _i
_lib.attn_decode.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _i, _vp, _sz, _vp]
_lib.attn_decode_ex.restype = _i
_lib.attn_decode_ex.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _i, _vp, _sz, _i, _vp]
_lib.attn_decode_typed.restype = _i
_lib.attn_decode_typed.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _i, _vp, _sz, _i, _i, _vp]
_lib.attn_combine.restype = _i
_lib.attn_combine.argtypes = [_vp, _vp, _vp, _vp] + [_i] * 5 + [_vp]
_lib.attn_combine_typed.restype = _i
_lib.attn_combine_typed.argtypes = [_vp, _vp, _vp, _vp] + [_i] * 6 + [_vp]
_lib.attn_fwd_host.restype = _i
_lib.attn_fwd_host.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 7 + [_f, _i, _i, _vp, _sz, _i, _vp]
_lib.attn_fwd_host_scratch_size.restype = _sz
_lib.attn_fwd_host_scratch_size.argtypes = [_i] * 7
_lib.attn_decode_default_splits.restype = _i
_lib.attn_decode_default_splits.argtypes = [_i] * 8
_lib.attn_check_device.restype = _i
_lib.attn_check_device.argtypes = [_vp]
_lib.attn_selftest_wait_timeout.restype = _i
_lib.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint, _vp]
_lib.attn_status_string.restype = ctypes.c_char_p
_lib.attn_status_string.argtypes = [_i]
_lib.attn_abi_version.restype = _i
_lib.attn_abi_version.argtypes = []

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_MISALIGNED = 0, 1, 2, 3
ATTN_ERR_WORKSPACE, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT = 4, 5, 6
ATTN_DECODE_AUTO, ATTN_DECODE_CUDA_CORE, ATTN_DECODE_TCGEN05_T, ATTN_DECODE_TCGEN05_N = 0, 1, 2, 3
ATTN_DTYPE_BF16, ATTN_DTYPE_F16 = 0, 1
_DTYPE_CODE = {torch.bfloat16: ATTN_DTYPE_BF16, torch.float16: ATTN_DTYPE_F16}


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {attn_status_string(code)} (status {code})")
        self.code = code


def lib() -> ctypes.CDLL:
    return _lib


def attn_status_string(code: int) -> str:
    return _lib.attn_status_string(int(code)).decode()


def attn_abi_version() -> int:
    return _lib.attn_abi_version()


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(code: int, where: str):
    if code != ATTN_OK:
        raise AttnError(code, where)


def _need(t: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape(t: torch.Tensor, name: str, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _same_device(where: str, *ts):
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError(f"{where}: tensors on different devices {sorted(map(str, devs))}")


def _qkv_dims(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """(B, Hq, Lq, d, Hkv, Lk, ldv) of q [B,Hq,Lq,d], k [B,Hkv,Lk,d], v [B,Hkv,Lk,ldv].

    The C entry points receive only pointers and these sizes, and the kernels' tensor maps span
    exactly those sizes: a k or v smaller than q implies would be read past its end, so every
    shape is checked against q's here."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.dim() != 4:
            raise ValueError(f"{n} must be 4-D [B, heads, length, dim], got shape {tuple(t.shape)}")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    _shape(k, "k", (B, Hkv, Lk, d))
    ldv = v.shape[-1]
    _shape(v, "v", (B, Hkv, Lk, ldv))
    return B, Hq, Lq, d, Hkv, Lk, ldv


def _outputs(out, lse, shape_o, shape_l, dtype, device, want_lse=True):
    """Caller-given or fresh O (``dtype``) and LSE (fp32) buffers, checked against their shapes."""
    if out is None:
        out = torch.empty(shape_o, dtype=dtype, device=device)
    _need(out, "out", dtype)
    _shape(out, "out", shape_o)
    if lse is None and want_lse:
        lse = torch.empty(shape_l, dtype=torch.float32, device=device)
    if lse is not None:
        _need(lse, "lse", torch.float32)
        _shape(lse, "lse", shape_l)
    _same_device("outputs", out, lse)
    if out.device != torch.device(device):
        raise ValueError(f"out is on {out.device}, the inputs on {device}")
    return out, lse


def _elem_code(q: torch.Tensor) -> int:
    if q.dtype not in _DTYPE_CODE:
        raise ValueError(f"q must be bfloat16 or float16, got {q.dtype}")
    return _DTYPE_CODE[q.dtype]


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, scale: float | None = None,
             out: torch.Tensor | None = None, lse: torch.Tensor | None = None, want_lse: bool = True):
    """O [B,Hq,Lq,dv] (q's dtype) and LSE [B,Hq,Lq] fp32 for q [B,Hq,Lq,d], k/v [B,Hkv,Lk,d/dv]."""
    code_t = _elem_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _same_device("attn_fwd", q, k, v)
    B, Hq, Lq, d, Hkv, Lk, dv = _qkv_dims(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out, lse = _outputs(out, lse, (B, Hq, Lq, dv), (B, Hq, Lq), q.dtype, q.device, want_lse)
    with torch.cuda.device(q.device):
        code = _lib.attn_fwd_typed(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Lq, Lk, d, dv,
                                   scale, int(bool(causal)), code_t, _stream_handle(q.device))
    _check(code, "attn_fwd")
    return out, lse


SPARSE_BLOCK = 128  # query rows / keys per block of attn_fwd_sparse's index lists


def attn_fwd_sparse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_idx: torch.Tensor,
                    block_cnt: torch.Tensor, *, causal: bool, scale: float | None = None,
                    out: torch.Tensor | None = None, lse: torch.Tensor | None = None):
    """Block-sparse attention: block_idx int32 [B, Hq, ceil(Lq/128), max_blocks] (sorted, distinct
    128-key block ids per query block), block_cnt int32 [B, Hq, ceil(Lq/128)] (entries used)."""
    code_t = _elem_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(block_idx, "block_idx", torch.int32)
    _need(block_cnt, "block_cnt", torch.int32)
    _same_device("attn_fwd_sparse", q, k, v, block_idx, block_cnt)
    B, Hq, Lq, d, Hkv, Lk, dv = _qkv_dims(q, k, v)
    nqb = (Lq + SPARSE_BLOCK - 1) // SPARSE_BLOCK
    if block_cnt.shape != (B, Hq, nqb) or block_idx.dim() != 4 or block_idx.shape[:3] != (B, Hq, nqb):
        raise ValueError(f"block lists must be [B, Hq, {nqb}, max_blocks] and [B, Hq, {nqb}]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out, lse = _outputs(out, lse, (B, Hq, Lq, dv), (B, Hq, Lq), q.dtype, q.device)
    with torch.cuda.device(q.device):
        code = _lib.attn_fwd_sparse_typed(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                          B, Hq, Hkv, Lq, Lk, d, dv, scale, int(bool(causal)), block_idx.data_ptr(),
                                          block_cnt.data_ptr(), block_idx.shape[3], code_t, _stream_handle(q.device))
    _check(code, "attn_fwd_sparse")
    return out, lse


def attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, num_splits=0) -> int:
    return int(_lib.attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, num_splits))


def attn_decode_default_splits(B, Hq, Hkv, Lq, Lk, d, dv, latent: bool) -> int:
    return int(_lib.attn_decode_default_splits(B, Hq, Hkv, Lq, Lk, d, dv, int(latent)))


def attn_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, scale: float | None = None,
                dv: int | None = None, num_splits: int = 0, impl: int = ATTN_DECODE_AUTO,
                workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None):
    """Split-KV decode. ``v is k`` selects the latent layout (V = first ``dv`` columns of K)."""
    code_t = _elem_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _same_device("attn_decode", q, k, v, workspace)
    B, Hq, Lq, d, Hkv, Lk, ldv = _qkv_dims(q, k, v)
    dv = ldv if dv is None else int(dv)
    if not 1 <= dv <= ldv:
        raise ValueError(f"dv = {dv} must be in [1, {ldv}] (the width of v)")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    need = attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    elif not (workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    out, lse = _outputs(out, lse, (B, Hq, Lq, dv), (B, Hq, Lq), q.dtype, q.device)
    with torch.cuda.device(q.device):
        code = _lib.attn_decode_typed(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                      B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, int(bool(causal)), int(num_splits),
                                      workspace.data_ptr(), workspace.numel() * workspace.element_size(), int(impl),
                                      code_t, _stream_handle(q.device))
    _check(code, "attn_decode")
    return out, lse


def attn_combine(o_part: torch.Tensor, lse_part: torch.Tensor, *, B: int, Hq: int, Lq: int,
                 out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                 dtype: torch.dtype = torch.bfloat16):
    """o_part fp32 [S, B*Hq*Lq, dv], lse_part fp32 [S, B*Hq*Lq] -> O [B,Hq,Lq,dv] (``dtype``), LSE."""
    _need(o_part, "o_part", torch.float32)
    _need(lse_part, "lse_part", torch.float32)
    if dtype not in _DTYPE_CODE:
        raise ValueError(f"dtype must be bfloat16 or float16, got {dtype}")
    if o_part.dim() != 3:
        raise ValueError(f"o_part must be 3-D [splits, rows, dv], got shape {tuple(o_part.shape)}")
    S, rows, dv = o_part.shape
    if rows != B * Hq * Lq:
        raise ValueError(f"o_part has {rows} rows, B*Hq*Lq = {B * Hq * Lq}")
    _shape(lse_part, "lse_part", (S, rows))
    _same_device("attn_combine", o_part, lse_part)
    out, lse = _outputs(out, lse, (B, Hq, Lq, dv), (B, Hq, Lq), dtype, o_part.device)
    with torch.cuda.device(o_part.device):
        code = _lib.attn_combine_typed(o_part.data_ptr(), lse_part.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                       B, Hq, Lq, dv, S, _DTYPE_CODE[dtype], _stream_handle(o_part.device))
    _check(code, "attn_combine")
    return out, lse


def attn_check_device(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device error status."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(_lib.attn_check_device(_stream_handle(dev)))


def attn_selftest_wait_timeout(limit_us: int, device=None):
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check(_lib.attn_selftest_wait_timeout(int(limit_us), _stream_handle(dev)), "attn_selftest_wait_timeout")


def attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, scale: float | None = None,
                  device="cuda:0", bufs: dict | None = None, pieces: int = 0):
    """Host (CPU, pinned) tensors in, host tensors out, through the C entry point attn_fwd_host
    (copy-in, compute and copy-out pipelined over pieces of the (batch, kv head) grid inside the
    library). ``bufs`` may hold the device scratch and the pinned outputs between calls. Waits for
    the call to finish (the returned host tensors are then valid)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda:
            raise ValueError(f"{n} must be a host tensor (pinned for overlapped copies)")
        if t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous {q.dtype}")
    B, Hq, Lq, d, Hkv, Lk, dv = _qkv_dims(q, k, v)
    if Hq % Hkv != 0:
        raise ValueError(f"Hq = {Hq} is not a multiple of Hkv = {Hkv}")
    dev = torch.device(device)
    bufs = {} if bufs is None else bufs
    key = (tuple(q.shape), tuple(k.shape), tuple(v.shape), q.dtype)
    if "key" in bufs and bufs["key"] != key:
        raise ValueError("bufs holds buffers of another shape or dtype; pass a fresh dict")
    if "key" not in bufs:
        nbytes = int(_lib.attn_fwd_host_scratch_size(B, Hq, Hkv, Lq, Lk, d, dv))
        if nbytes == 0:
            raise ValueError("invalid sizes")
        bufs["key"] = key
        bufs["scratch"] = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        bufs["o_host"] = torch.empty((B, Hq, Lq, dv), dtype=q.dtype, pin_memory=True)
        bufs["lse_host"] = torch.empty((B, Hq, Lq), dtype=torch.float32, pin_memory=True)
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        _check(_lib.attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), bufs["o_host"].data_ptr(),
                                  bufs["lse_host"].data_ptr(), B, Hq, Hkv, Lq, Lk, d, dv, sc, int(bool(causal)),
                                  _elem_code(q), bufs["scratch"].data_ptr(), bufs["scratch"].numel(),
                                  int(pieces), stream.cuda_stream), "attn_fwd_host")
    stream.synchronize()
    return bufs["o_host"], bufs["lse_host"]
