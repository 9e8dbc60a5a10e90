"""attn_decode (split-KV, both kernels) and attn_combine against the fp64 oracle."""
import numpy as np
import pytest
import torch

from exact_attention_139_b200.inputs import WORKLOADS, Workload, make_inputs, sample_rows
from oracle import oracle
from tests.gpu_util import compare, oracle_rows, rows_per_head, take_rows

pytestmark = pytest.mark.gpu

CC, TC, TN = 1, 2, 3


def run(w, dev, impl=0, num_splits=0):
    from exact_attention_139_b200 import attn
    q, k, v = make_inputs(w)
    qd, kd = q.to(dev), k.to(dev)
    vd = kd if w.latent else v.to(dev)
    o, lse = attn.attn_decode(qd, kd, vd, causal=w.causal, scale=w.scale, dv=w.dv, impl=impl,
                              num_splits=num_splits)
    assert attn.attn_check_device() == 0
    return q, k, v, o, lse


@pytest.mark.parametrize("impl", [TN, TC, CC])
def test_mla_decode_64k(impl, cuda_device):
    w = WORKLOADS["mla_decode_64k"]
    q, k, v, o, lse = run(w, cuda_device, impl=impl)
    # every row of the first nb batches (all 32 batches by default: the full output)
    nb = min(w.B, max(1, rows_per_head(2 * w.B) // 2))
    rows = np.arange(nb * w.Hq * w.Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, f"mla impl={impl}")


@pytest.mark.parametrize("impl", [TN, CC])
def test_gqa_decode_32k(impl, cuda_device):
    """GQA decode with a dense V (16 x 32 query heads on 8 kv heads, 32K keys): every row."""
    w = WORKLOADS["gqa_decode_32k"]
    q, k, v, o, lse = run(w, cuda_device, impl=impl)
    rows = np.arange(w.B * w.Hq * w.Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    compare(o.reshape(-1, w.dv), lse.reshape(-1), o_ref, l_ref, f"gqa impl={impl}")


SMALL = [
    # B, Hq, Hkv, Lq, Lk, d, dv, latent, causal
    (2, 16, 1, 2, 1000, 576, 512, True, True),
    (1, 16, 1, 1, 64, 576, 512, True, True),
    (3, 16, 1, 2, 4097, 576, 512, True, True),
    (2, 8, 1, 2, 333, 256, 128, True, False),
    (2, 8, 2, 1, 777, 128, 128, False, True),
    (1, 4, 4, 2, 65, 64, 64, False, True),
    (2, 32, 8, 2, 1500, 128, 128, False, True),
    (1, 8, 1, 1, 3, 128, 128, True, True),
    (3, 16, 2, 2, 1000, 256, 256, False, True),
    (2, 32, 1, 1, 4000, 128, 128, False, True),
]


@pytest.mark.parametrize("splits", [0, 1, 3, 16])  # 0: the library's schedule (balanced for TN)
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B{}_H{}x{}_Lq{}_Lk{}_d{}_{}".format(*s[:7]))
def test_small_shapes(shape, splits, cuda_device):
    from exact_attention_139_b200 import attn
    B, Hq, Hkv, Lq, Lk, d, dv, latent, causal = shape
    w = Workload("dec", B, Hq, Hkv, Lq, Lk, d, dv, causal, latent=latent, seed=2000 + Lk + d)
    q, k, v = make_inputs(w)
    rows = np.arange(B * Hq * Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    impls = [CC]
    R = (Hq // Hkv) * Lq
    if latent and d % 64 == 0 and dv % 128 == 0 and R <= 32:
        impls += [TC, TN]
    if not latent and dv == d and d in (128, 256) and R <= 32:
        impls += [TN]
    qd, kd = q.to(cuda_device), k.to(cuda_device)
    vd = kd if latent else v.to(cuda_device)
    for impl in impls:
        o, lse = attn.attn_decode(qd, kd, vd, causal=causal, scale=w.scale, dv=dv, impl=impl, num_splits=splits)
        assert attn.attn_check_device() == 0
        compare(o.reshape(-1, dv), lse.reshape(-1), o_ref, l_ref, f"{shape} splits={splits} impl={impl}")


def test_split_count_invariance(cuda_device):
    from exact_attention_139_b200 import attn
    w = Workload("inv", 2, 16, 1, 2, 5000, 576, 512, True, latent=True, seed=31)
    q, k, _ = (t.to(cuda_device) for t in make_inputs(w))
    outs = [attn.attn_decode(q, k, k, causal=True, dv=512, num_splits=s)[0].float() for s in (1, 5, 40, 0)]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 1e-2


def test_decode_matches_prefill_last_row(cuda_device):
    from exact_attention_139_b200 import attn
    w = Workload("dp", 2, 8, 2, 1, 3000, 128, 128, True, seed=41)
    q, k, v = (t.to(cuda_device) for t in make_inputs(w))
    od, ld = attn.attn_decode(q, k, v, causal=True)
    of, lf = attn.attn_fwd(q, k, v, causal=True)
    assert (od.float() - of.float()).abs().max().item() <= 2e-2
    assert (ld - lf).abs().max().item() <= 1e-3


def test_combine_against_oracle_merge(cuda_device):
    from exact_attention_139_b200 import attn
    w = Workload("cmb", 1, 4, 1, 3, 300, 64, 64, True, seed=51)
    q, k, v = make_inputs(w)
    rows = np.arange(w.B * w.Hq * w.Lq)
    cuts = [0, 100, 100, 250, 299, 300]  # includes an empty range and a one-key range
    parts = [oracle_rows(w, q, k, v, rows, kv_range=(cuts[s], cuts[s + 1])) for s in range(len(cuts) - 1)]
    op = np.stack([p[0] for p in parts])
    lp = np.stack([p[1] for p in parts])
    o_ref, l_ref = oracle.combine(op, lp)
    o, lse = attn.attn_combine(torch.tensor(op, dtype=torch.float32, device=cuda_device),
                               torch.tensor(lp, dtype=torch.float32, device=cuda_device), B=w.B, Hq=w.Hq, Lq=w.Lq)
    compare(o.reshape(-1, w.dv), lse.reshape(-1), o_ref, l_ref, "combine")
    # a row whose every split is empty
    lp_empty = np.full((2, 1), -np.inf)
    op_empty = np.zeros((2, 1, 64))
    o2, l2 = attn.attn_combine(torch.tensor(op_empty, dtype=torch.float32, device=cuda_device),
                               torch.tensor(lp_empty, dtype=torch.float32, device=cuda_device), B=1, Hq=1, Lq=1)
    assert torch.all(o2 == 0) and torch.isinf(l2).all() and (l2 < 0).all()


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,latent", [(3, 16, 1, 2, 1000, True), (5, 16, 1, 2, 4097, True),
                                                  (2, 32, 8, 1, 3001, False), (7, 8, 2, 2, 777, False)])
def test_balanced_schedule_vs_oracle(B, Hq, Hkv, Lq, Lk, latent, cuda_device):
    """num_splits = 0 on the queries-on-M kernel: CTAs take equal ranges of the flattened
    (unit, key) space, so ranges straddle units and the last piece of a unit may hold only keys
    that the causal mask hides from its first query row."""
    from exact_attention_139_b200 import attn
    d, dv = (576, 512) if latent else (128, 128)
    w = Workload("bal", B, Hq, Hkv, Lq, Lk, d, dv, True, latent=latent, seed=2500 + Lk)
    q, k, v, o, lse = run(w, cuda_device, impl=TN, num_splits=0)
    rows = np.arange(B * Hq * Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    compare(o.reshape(-1, dv), lse.reshape(-1), o_ref, l_ref, f"balanced B{B} Lk{Lk}")
