"""fp64 CPU oracle for exact scaled-dot-product attention (ctypes wrapper over attn_oracle.c).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` are the only callers. The CUDA library and its binding never import this module and
share no code with it.

Definitions followed (see attn_oracle.c for the full list of readings):
  * "Resumen Tecnico: FlashMLA-ETAP" (gist.science 2506.01969), section "Mecanismo Central":
    S = Q.K^T, P = softmax(S), O = P.V and the transposed flow O = (V^T.P^T)^T.
  * "Activar Flash Attention con llama.cpp" (quellm.com), FAQ on GQA: shared K/V heads.

Inputs are bf16 tensors (torch, CPU) or numpy uint16 arrays holding bf16 bit patterns; each
value is widened exactly to double. Outputs are float64 numpy arrays.
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
            ctypes.c_int]
        L.oracle_softmax_row.restype = ctypes.c_int
        L.oracle_softmax_row.argtypes = [_u16p, _u16p] + [_i64] * 6 + [
            ctypes.c_double, ctypes.c_int, _i64, _dp]
        L.oracle_attn_transposed_head.restype = ctypes.c_int
        L.oracle_attn_transposed_head.argtypes = [_u16p, _u16p, _u16p] + [_i64] * 8 + [
            ctypes.c_double, ctypes.c_int, _i64, _i64, _dp, _dp]
        L.oracle_combine.restype = ctypes.c_int
        L.oracle_combine.argtypes = [_dp, _dp, _i64, _i64, _i64, _dp, _dp]
        L.oracle_mutant_id.restype = ctypes.c_int
        _LIBS[mutant] = L
    return _LIBS[mutant]


def bf16_bits(x) -> np.ndarray:
    """bf16 torch tensor or uint16 array -> C-contiguous uint16 numpy array of bit patterns."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy input must hold bf16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch  # the oracle accepts torch CPU tensors as a convenience
    if x.dtype != torch.bfloat16:
        raise TypeError(f"expected bfloat16, got {x.dtype}")
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def attn_rows(q, k, v, rows, *, B, Hq, Hkv, Lq, Lk, d, dv, ldv=None, scale, causal,
              kv_range=None, nthreads=None, mutant: int = 0):
    """O (n_rows x dv) and LSE (n_rows) for the flat row ids ``rows`` = (b*Hq + h)*Lq + i.

    ``kv_range=(j0, j1)`` restricts the keys to [j0, j1): the split partial (O normalised by its
    own sum, LSE of that range, -inf when no key is visible). ``v`` may be the same array as
    ``k`` (latent KV: V is the first dv columns of each K row, ldv = d).
    """
    qb, kb = bf16_bits(q), bf16_bits(k)
    vb = kb if v is k else bf16_bits(v)
    ldv = dv if ldv is None else ldv
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    j0, j1 = (0, Lk) if kv_range is None else kv_range
    o = np.empty((rows.size, dv), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    assert qb.size == B * Hq * Lq * d and kb.size == B * Hkv * Lk * d
    assert vb.size == B * Hkv * Lk * ldv
    rc = _lib(mutant).oracle_attn_rows(
        _ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d, dv, ldv, float(scale), int(causal),
        j0, j1, rows.ctypes.data_as(ctypes.POINTER(_i64)), rows.size, _dptr(o), _dptr(lse),
        nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_attn_rows rejected its arguments (code {rc})")
    return o, lse


def attn(q, k, v, *, B, Hq, Hkv, Lq, Lk, d, dv, ldv=None, scale, causal, kv_range=None,
         nthreads=None, mutant: int = 0):
    """Full attention: O [B,Hq,Lq,dv] and LSE [B,Hq,Lq] in float64."""
    rows = np.arange(B * Hq * Lq, dtype=np.int64)
    o, lse = attn_rows(q, k, v, rows, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d, dv=dv, ldv=ldv,
                       scale=scale, causal=causal, kv_range=kv_range, nthreads=nthreads,
                       mutant=mutant)
    return o.reshape(B, Hq, Lq, dv), lse.reshape(B, Hq, Lq)


def softmax_row(q, k, row, *, B, Hq, Hkv, Lq, Lk, d, scale, causal, mutant: int = 0):
    """The materialised probability row P[row, :] (length Lk, zeros at masked keys)."""
    qb, kb = bf16_bits(q), bf16_bits(k)
    p = np.empty(Lk, dtype=np.float64)
    rc = _lib(mutant).oracle_softmax_row(_ptr(qb), _ptr(kb), B, Hq, Hkv, Lq, Lk, d,
                                         float(scale), int(causal), int(row), _dptr(p))
    if rc != 0:
        raise ValueError(f"oracle_softmax_row rejected its arguments (code {rc})")
    return p


def attn_transposed_head(q, k, v, b, h, *, B, Hq, Hkv, Lq, Lk, d, dv, ldv=None, scale, causal,
                         mutant: int = 0):
    """The transposed flow (S^T = K.Q^T, column softmax, O = (V^T.P^T)^T) for one (b, h)."""
    qb, kb = bf16_bits(q), bf16_bits(k)
    vb = kb if v is k else bf16_bits(v)
    ldv = dv if ldv is None else ldv
    o = np.empty((Lq, dv), dtype=np.float64)
    lse = np.empty(Lq, dtype=np.float64)
    rc = _lib(mutant).oracle_attn_transposed_head(
        _ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d, dv, ldv, float(scale), int(causal),
        int(b), int(h), _dptr(o), _dptr(lse))
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
