"""fp16 inputs and outputs (the *_typed entry points through the binding) against the fp64 oracle.

The same kernels run with the fp16 tensor-core operand format, fp16 TMA element type and fp16
rounding of P and O; the oracle widens the same fp16 bit patterns exactly. Tolerances are the
fp16 ones of gpu_util (eight times tighter on O than for bf16).
"""
import numpy as np
import pytest
import torch

from exact_attention_139_b200.inputs import WORKLOADS, Workload, make_inputs, sample_rows
from oracle import oracle
from tests.gpu_util import compare, oracle_rows, rows_per_head, take_rows

pytestmark = pytest.mark.gpu

CC, TC, TN = 1, 2, 3


def f16(w):
    return w.with_(dtype="f16", name=w.name + "_f16")


@pytest.mark.parametrize("w", [
    f16(WORKLOADS["tiny_d64"]),
    f16(WORKLOADS["tiny_d64_causal"]),
    Workload("f16_sweep_a", 2, 4, 2, 127, 129, 128, 128, True, seed=31, dtype="f16"),
    Workload("f16_sweep_b", 1, 8, 8, 129, 200, 64, 64, False, seed=32, dtype="f16"),
    Workload("f16_sweep_c", 1, 2, 1, 1000, 1000, 128, 128, True, seed=33, dtype="f16"),
], ids=lambda w: w.name)
def test_prefill_f16_all_rows(w, cuda_device):
    from exact_attention_139_b200 import attn
    q, k, v = make_inputs(w)
    o, lse = attn.attn_fwd(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=w.causal,
                           scale=w.scale)
    assert attn.attn_check_device() == 0
    assert o.dtype == torch.float16
    rows = np.arange(w.B * w.Hq * w.Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows, elem="f16")
    compare(o.reshape(-1, w.dv), lse.reshape(-1), o_ref, l_ref, w.name)


def test_prefill_f16_llama8b_sampled(cuda_device):
    from exact_attention_139_b200 import attn
    w = f16(WORKLOADS["llama8b_prefill_8k"])
    q, k, v = make_inputs(w)
    o, lse = attn.attn_fwd(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=True,
                           scale=w.scale)
    assert attn.attn_check_device() == 0
    rows = sample_rows(w, rows_per_head(16)).numpy()
    o_ref, l_ref = oracle_rows(w, q, k, v, rows, elem="f16")
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, w.name)


def _decode(w, dev, impl, num_splits=0):
    from exact_attention_139_b200 import attn
    q, k, v = make_inputs(w)
    qd, kd = q.to(dev), k.to(dev)
    vd = kd if w.latent else v.to(dev)
    o, lse = attn.attn_decode(qd, kd, vd, causal=w.causal, scale=w.scale, dv=w.dv, impl=impl,
                              num_splits=num_splits)
    assert attn.attn_check_device() == 0
    assert o.dtype == torch.float16
    return q, k, v, o, lse


@pytest.mark.parametrize("impl", [TN, TC])
def test_mla_decode_64k_f16(impl, cuda_device):
    w = f16(WORKLOADS["mla_decode_64k"])
    q, k, v, o, lse = _decode(w, cuda_device, impl)
    nb = min(w.B, max(1, rows_per_head(8) // 2))
    rows = np.arange(nb * w.Hq * w.Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows, elem="f16")
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, f"mla f16 impl={impl}")


def test_gqa_decode_32k_f16(cuda_device):
    w = f16(WORKLOADS["gqa_decode_32k"])
    q, k, v, o, lse = _decode(w, cuda_device, TN)
    rows = np.arange(w.B * w.Hq * w.Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows, elem="f16")
    compare(o.reshape(-1, w.dv), lse.reshape(-1), o_ref, l_ref, "gqa f16")


@pytest.mark.parametrize("impl", [CC, TN])
@pytest.mark.parametrize("splits", [1, 7])
def test_decode_f16_small(impl, splits, cuda_device):
    w = Workload("f16_dec", 2, 16, 2, 2, 1500, 128, 128, True, seed=41, dtype="f16")
    q, k, v, o, lse = _decode(w, cuda_device, impl, num_splits=splits)
    rows = np.arange(w.B * w.Hq * w.Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows, elem="f16")
    compare(o.reshape(-1, w.dv), lse.reshape(-1), o_ref, l_ref, f"f16 small impl={impl} s={splits}")


def test_combine_f16(cuda_device):
    """attn_combine writing fp16 against the oracle's log-sum-exp merge of the same partials."""
    from exact_attention_139_b200 import attn
    g = torch.Generator().manual_seed(5)
    S, B, Hq, Lq, dv = 5, 2, 4, 2, 64
    R = B * Hq * Lq
    op = torch.rand((S, R, dv), generator=g, dtype=torch.float32) * 2 - 1
    lp = torch.randn((S, R), generator=g, dtype=torch.float32) * 3
    lp[1, 3] = -float("inf")
    lp[:, 5] = -float("inf")  # a row with no visible key at all
    o, lse = attn.attn_combine(op.to(cuda_device), lp.to(cuda_device), B=B, Hq=Hq, Lq=Lq,
                               dtype=torch.float16)
    torch.cuda.synchronize()
    assert o.dtype == torch.float16
    o_ref, l_ref = oracle.combine(op.double().numpy(), lp.double().numpy())
    compare(o.reshape(R, dv), lse.reshape(R), o_ref, l_ref, "combine f16")
