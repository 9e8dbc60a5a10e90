"""Helpers for the GPU parity tests: run the CUDA path, run the oracle, compare.

Tolerances, fp32 accumulation on the tensor cores and an fp32 softmax in both cases:
  * bf16 inputs and output: O max-abs <= 2e-2 and relative L2 <= 5e-3; LSE max-abs <= 1e-3.
    (P is rounded to bf16 before P.V, relative step 2^-8; O is rounded once more at the end.)
  * fp16 inputs and output: eight times tighter on O, max-abs <= 2.5e-3 and relative L2
    <= 6.25e-4 (fp16 has three more mantissa bits, relative step 2^-11); LSE as for bf16,
    since it never passes through the 16-bit type.
"""
from __future__ import annotations

import os

import numpy as np
import torch

from oracle import oracle

O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
TOL = {
    torch.bfloat16: (O_MAX_ABS, O_REL_L2, LSE_MAX_ABS),
    torch.float16: (O_MAX_ABS / 8, O_REL_L2 / 8, LSE_MAX_ABS),
}


def rows_per_head(default: int) -> int:
    return int(os.environ.get("ATTN_PARITY_ROWS_PER_HEAD", default))


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """o_gpu/lse_gpu: torch (any device) for the compared rows; o_ref/lse_ref: float64 numpy.
    The tolerance follows o_gpu's dtype."""
    o_max_abs, o_rel_l2, lse_max_abs = TOL[o_gpu.dtype]
    og = o_gpu.detach().float().cpu().double().numpy().reshape(o_ref.shape)
    assert np.all(np.isfinite(og)), f"{what}: non-finite output"
    err = np.abs(og - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(og - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    assert max_abs <= o_max_abs, f"{what}: O max-abs {max_abs:.3e}"
    assert rel <= o_rel_l2, f"{what}: O rel-L2 {rel:.3e}"
    stats = {"o_max_abs": max_abs, "o_rel_l2": rel, "o_rmse": float(np.sqrt(np.mean(err ** 2)))}
    if lse_gpu is not None:
        lg = lse_gpu.detach().float().cpu().double().numpy().reshape(lse_ref.shape)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin), f"{what}: LSE finiteness differs"
        lerr = float(np.abs(lg[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
        assert lerr <= lse_max_abs, f"{what}: LSE max-abs {lerr:.3e}"
        stats["lse_max_abs"] = lerr
    return stats


def oracle_rows(w, q, k, v, rows, kv_range=None, elem=None):
    return oracle.attn_rows(q, k, (k if w.latent else v), rows, B=w.B, Hq=w.Hq, Hkv=w.Hkv, Lq=w.Lq, Lk=w.Lk,
                            d=w.d, dv=w.dv, ldv=w.ldv, scale=w.scale, causal=w.causal, kv_range=kv_range,
                            elem=elem)


def take_rows(o, lse, rows):
    """Select flat rows (b*Hq + h)*Lq + i of O [B,Hq,Lq,dv] and LSE [B,Hq,Lq] (on device)."""
    idx = torch.as_tensor(np.asarray(rows), device=o.device, dtype=torch.long)
    return o.reshape(-1, o.shape[-1]).index_select(0, idx), lse.reshape(-1).index_select(0, idx)
