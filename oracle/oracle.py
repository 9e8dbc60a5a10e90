"""fp64 CPU oracle for exact scaled-dot-product attention (ctypes wrapper over attn_oracle.c).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` are the only callers. The CUDA library and its binding never import this module and
share no code with it.

Definitions followed (see attn_oracle.c for the full list of readings):
  * "Resumen Tecnico: FlashMLA-ETAP" (gist.science 2506.01969), section "Mecanismo Central":
    S = Q.K^T, P = softmax(S), O = P.V and the transposed flow O = (V^T.P^T)^T.
  * "Activar Flash Attention con llama.cpp" (quellm.com), FAQ on GQA: shared K/V heads.

Inputs are bf16 or fp16 tensors (torch, CPU) or numpy uint16 arrays holding bit patterns (bf16
unless ``elem="f16"`` is passed); q, k and v share one element type and each value is widened
exactly to double. Outputs are float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")

_i64 = ctypes.c_int64
_dp = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.c_void_p


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so"
    return os.path.join(_HERE, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile attn_oracle.c with gcc (mutant != 0 plants one deliberate mistake)."""
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-shared", "-fPIC", "-pthread", f"-DORACLE_MUTANT={int(mutant)}",
           _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


_LIBS: dict[int, ctypes.CDLL] = {}


def _lib(mutant: int = 0) -> ctypes.CDLL:
    if mutant not in _LIBS:
        L = ctypes.CDLL(build(mutant))
        L.oracle_attn_rows.restype = ctypes.c_int
        L.oracle_attn_rows.argtypes = [_u16p, _u16p, _u16p] + [_i64] * 8 + [
            ctypes.c_double, ctypes.c_int, _i64, _i64, ctypes.POINTER(_i64), _i64, _dp, _dp,
            ctypes.c_int, ctypes.c_int]
        L.oracle_softmax_row.restype = ctypes.c_int
        L.oracle_softmax_row.argtypes = [_u16p, _u16p] + [_i64] * 6 + [
            ctypes.c_double, ctypes.c_int, _i64, _dp, ctypes.c_int]
        L.oracle_attn_transposed_head.restype = ctypes.c_int
        L.oracle_attn_transposed_head.argtypes = [_u16p, _u16p, _u16p] + [_i64] * 8 + [
            ctypes.c_double, ctypes.c_int, _i64, _i64, _dp, _dp, ctypes.c_int]
        L.oracle_attn_rows_sparse.restype = ctypes.c_int
        L.oracle_attn_rows_sparse.argtypes = [_u16p, _u16p, _u16p] + [_i64] * 8 + [
            ctypes.c_double, ctypes.c_int, _i64, _i64, ctypes.c_void_p, ctypes.c_void_p, _i64,
            ctypes.POINTER(_i64), _i64, _dp, _dp, ctypes.c_int, ctypes.c_int]
        L.oracle_widen.restype = ctypes.c_int
        L.oracle_widen.argtypes = [_u16p, _i64, ctypes.c_int, _dp]
        L.oracle_combine.restype = ctypes.c_int
        L.oracle_combine.argtypes = [_dp, _dp, _i64, _i64, _i64, _dp, _dp]
        L.oracle_mutant_id.restype = ctypes.c_int
        _LIBS[mutant] = L
    return _LIBS[mutant]


ELEM_CODES = {"bf16": 0, "f16": 1}


def bits16(x, elem: str | None = None) -> tuple[np.ndarray, str]:
    """16-bit torch tensor or uint16 array -> (C-contiguous uint16 bit patterns, element type).

    A torch tensor's element type comes from its dtype; a numpy array is bf16 unless ``elem``
    says otherwise."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy input must hold 16-bit patterns as uint16")
        return np.ascontiguousarray(x), elem or "bf16"
    import torch  # the oracle accepts torch CPU tensors as a convenience
    kinds = {torch.bfloat16: "bf16", torch.float16: "f16"}
    if x.dtype not in kinds:
        raise TypeError(f"expected bfloat16 or float16, got {x.dtype}")
    if elem is not None and elem != kinds[x.dtype]:
        raise TypeError(f"tensor is {kinds[x.dtype]}, elem says {elem}")
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16), kinds[x.dtype]


def bf16_bits(x) -> np.ndarray:
    """bf16 torch tensor or uint16 array -> C-contiguous uint16 numpy array of bit patterns."""
    b, kind = bits16(x)
    if kind != "bf16":
        raise TypeError(f"expected bfloat16, got {kind}")
    return b


def _operands(q, k, v, elem):
    qb, eq = bits16(q, elem)
    kb, ek = bits16(k, elem)
    if v is None:
        vb, ev = None, ek
    elif v is k:
        vb, ev = kb, ek
    else:
        vb, ev = bits16(v, elem)
    if not (eq == ek == ev):
        raise TypeError(f"q, k, v element types differ: {eq}, {ek}, {ev}")
    return qb, kb, vb, ELEM_CODES[eq]


def widen(bits, elem: str = "bf16", mutant: int = 0) -> np.ndarray:
    """The oracle's exact widening of 16-bit patterns (uint16 array) to float64."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16).reshape(-1))
    out = np.empty(b.size, dtype=np.float64)
    rc = _lib(mutant).oracle_widen(_ptr(b), b.size, ELEM_CODES[elem], _dptr(out))
    if rc != 0:
        raise ValueError(f"oracle_widen rejected its arguments (code {rc})")
    return out


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def attn_rows(q, k, v, rows, *, B, Hq, Hkv, Lq, Lk, d, dv, ldv=None, scale, causal,
              kv_range=None, blocks=None, nthreads=None, elem=None, mutant: int = 0):
    """O (n_rows x dv) and LSE (n_rows) for the flat row ids ``rows`` = (b*Hq + h)*Lq + i.

    ``kv_range=(j0, j1)`` restricts the keys to [j0, j1): the split partial (O normalised by its
    own sum, LSE of that range, -inf when no key is visible). ``v`` may be the same array as
    ``k`` (latent KV: V is the first dv columns of each K row, ldv = d).

    ``blocks=(idx, cnt, blk_q, blk_k)`` gives block-sparse attention: idx int32
    [B, Hq, ceil(Lq/blk_q), max_blk] and cnt int32 [B, Hq, ceil(Lq/blk_q)]; query block qb of head
    (b, h) sees only the key blocks idx[b, h, qb, :cnt[b, h, qb]] (and the causal mask).
    """
    qb, kb, vb, ec = _operands(q, k, v, elem)
    ldv = dv if ldv is None else ldv
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    j0, j1 = (0, Lk) if kv_range is None else kv_range
    o = np.empty((rows.size, dv), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    assert qb.size == B * Hq * Lq * d and kb.size == B * Hkv * Lk * d
    assert vb.size == B * Hkv * Lk * ldv
    if blocks is not None:
        if kv_range is not None:
            raise ValueError("kv_range and blocks are exclusive")
        idx, cnt, blk_q, blk_k = blocks
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
        cnt = np.ascontiguousarray(np.asarray(cnt, dtype=np.int32))
        nqb = -(-Lq // blk_q)
        assert cnt.shape == (B, Hq, nqb) and idx.shape[:3] == (B, Hq, nqb) and idx.ndim == 4
        rc = _lib(mutant).oracle_attn_rows_sparse(
            _ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d, dv, ldv, float(scale), int(causal),
            int(blk_q), int(blk_k), _ptr(idx), _ptr(cnt), idx.shape[3],
            rows.ctypes.data_as(ctypes.POINTER(_i64)), rows.size, _dptr(o), _dptr(lse), ec,
            nthreads or default_threads())
    else:
        rc = _lib(mutant).oracle_attn_rows(
            _ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d, dv, ldv, float(scale), int(causal),
            j0, j1, rows.ctypes.data_as(ctypes.POINTER(_i64)), rows.size, _dptr(o), _dptr(lse), ec,
            nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_attn_rows rejected its arguments (code {rc})")
    return o, lse


def attn(q, k, v, *, B, Hq, Hkv, Lq, Lk, d, dv, ldv=None, scale, causal, kv_range=None,
         blocks=None, nthreads=None, elem=None, mutant: int = 0):
    """Full attention: O [B,Hq,Lq,dv] and LSE [B,Hq,Lq] in float64."""
    rows = np.arange(B * Hq * Lq, dtype=np.int64)
    o, lse = attn_rows(q, k, v, rows, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d, dv=dv, ldv=ldv,
                       scale=scale, causal=causal, kv_range=kv_range, blocks=blocks,
                       nthreads=nthreads, elem=elem, mutant=mutant)
    return o.reshape(B, Hq, Lq, dv), lse.reshape(B, Hq, Lq)


def softmax_row(q, k, row, *, B, Hq, Hkv, Lq, Lk, d, scale, causal, elem=None, mutant: int = 0):
    """The materialised probability row P[row, :] (length Lk, zeros at masked keys)."""
    qb, kb, _, ec = _operands(q, k, None, elem)
    p = np.empty(Lk, dtype=np.float64)
    rc = _lib(mutant).oracle_softmax_row(_ptr(qb), _ptr(kb), B, Hq, Hkv, Lq, Lk, d,
                                         float(scale), int(causal), int(row), _dptr(p), ec)
    if rc != 0:
        raise ValueError(f"oracle_softmax_row rejected its arguments (code {rc})")
    return p


def attn_transposed_head(q, k, v, b, h, *, B, Hq, Hkv, Lq, Lk, d, dv, ldv=None, scale, causal,
                         elem=None, mutant: int = 0):
    """The transposed flow (S^T = K.Q^T, column softmax, O = (V^T.P^T)^T) for one (b, h)."""
    qb, kb, vb, ec = _operands(q, k, v, elem)
    ldv = dv if ldv is None else ldv
    o = np.empty((Lq, dv), dtype=np.float64)
    lse = np.empty(Lq, dtype=np.float64)
    rc = _lib(mutant).oracle_attn_transposed_head(
        _ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d, dv, ldv, float(scale), int(causal),
        int(b), int(h), _dptr(o), _dptr(lse), ec)
    if rc != 0:
        raise ValueError(f"oracle_attn_transposed_head rejected its arguments (code {rc})")
    return o, lse


def combine(o_parts, lse_parts, mutant: int = 0):
    """Log-sum-exp merge of split partials: o_parts [S, R, dv], lse_parts [S, R] (float64)."""
    op = np.ascontiguousarray(o_parts, dtype=np.float64)
    lp = np.ascontiguousarray(lse_parts, dtype=np.float64)
    S, R, dv = op.shape
    assert lp.shape == (S, R)
    o = np.empty((R, dv), dtype=np.float64)
    lse = np.empty(R, dtype=np.float64)
    rc = _lib(mutant).oracle_combine(_dptr(op), _dptr(lp), S, R, dv, _dptr(o), _dptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_combine rejected its arguments (code {rc})")
    return o, lse
