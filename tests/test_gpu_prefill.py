"""attn_fwd (tcgen05 prefill kernel) against the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

from exact_attention_139_b200.inputs import WORKLOADS, Workload, make_inputs, sample_rows
from tests.gpu_util import compare, oracle_rows, rows_per_head, take_rows

pytestmark = pytest.mark.gpu


def run(w: Workload, dev):
    from exact_attention_139_b200 import attn
    q, k, v = make_inputs(w)
    o, lse = attn.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=w.causal, scale=w.scale)
    assert attn.attn_check_device() == 0
    return q, k, v, o, lse


@pytest.mark.parametrize("name", ["tiny_d64", "tiny_d64_causal"])
def test_tiny_full(name, cuda_device):
    w = WORKLOADS[name]
    q, k, v, o, lse = run(w, cuda_device)
    rows = np.arange(w.B * w.Hq * w.Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    compare(o.reshape(-1, w.dv), lse.reshape(-1), o_ref, l_ref, name)


SWEEP = [
    # B, Hq, Hkv, Lq, Lk, d, causal
    (1, 1, 1, 1, 1, 64, False),
    (1, 1, 1, 1, 1, 128, True),
    (1, 2, 1, 17, 17, 128, True),
    (2, 4, 2, 127, 129, 128, True),
    (1, 8, 2, 129, 127, 128, False),
    (1, 4, 1, 200, 1000, 128, True),
    (2, 2, 2, 1000, 1000, 64, True),
    (1, 8, 8, 129, 200, 64, False),
    (3, 16, 2, 17, 1000, 128, False),
    (1, 4, 4, 1000, 1000, 128, False),
    (1, 2, 1, 256, 640, 128, True),
]


@pytest.mark.parametrize("shape", SWEEP, ids=lambda s: "B{}_H{}x{}_L{}x{}_d{}_{}".format(*s[:6], "c" if s[6] else "n"))
def test_shape_sweep(shape, cuda_device):
    B, Hq, Hkv, Lq, Lk, d, causal = shape
    w = Workload("sweep", B, Hq, Hkv, Lq, Lk, d, d, causal, seed=1000 + sum(shape[:6]))
    q, k, v, o, lse = run(w, cuda_device)
    rows = np.arange(B * Hq * Lq)
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    compare(o.reshape(-1, d), lse.reshape(-1), o_ref, l_ref, str(shape))


@pytest.mark.parametrize("name,per_head", [("batched_prefill_256", 256), ("batched_prefill_2k", 2048),
                                           ("llama8b_prefill_8k", 8192)])
def test_full_size_every_row(name, per_head, cuda_device):
    """The full-size configs in the launch configuration bench.py times, every row against the
    oracle (about 550 GFLOP of fp64 work each for the 2K and 8K configs; ATTN_PARITY_ROWS_PER_HEAD
    caps the rows per head for a quicker run)."""
    w = WORKLOADS[name]
    q, k, v, o, lse = run(w, cuda_device)
    rows = sample_rows(w, rows_per_head(per_head)).numpy()
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, name)


def _ramp_inputs(w: Workload, beta: float):
    """Inputs that make the lazy O rescale fire in every key tile for half of the warps: query
    rows alternate by 32 (one warp of a softmax warpgroup) between +u and -u plus N(0, 1) noise,
    and key t carries beta * t / 128 along u (u = the all-ones direction) plus N(0, 1) noise, so
    along the keys the + rows' scores climb by beta * sqrt(d) per 128-key tile while the - rows'
    fall. V is N(0, 1). All draws from one seeded CPU generator, rounded once to bf16."""
    g = torch.Generator().manual_seed(w.seed)
    u = torch.ones(w.d)
    sign = torch.where((torch.arange(w.Lq) // 32) % 2 == 0, 1.0, -1.0)
    q = torch.randn((w.B, w.Hq, w.Lq, w.d), generator=g) + sign[None, None, :, None] * u
    ramp = beta * torch.arange(w.Lk, dtype=torch.float32) / 128.0
    k = torch.randn((w.B, w.Hkv, w.Lk, w.d), generator=g) + ramp[None, None, :, None] * u
    v = torch.randn((w.B, w.Hkv, w.Lk, w.dv), generator=g)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def _lazy_rescales(w: Workload, q, k, rows):
    """Per row, how many 128-key tiles after the first raise the row max by more than the lazy
    threshold (2^8) over the last max used, in fp64 from the bf16 inputs."""
    qf, kf = q.double(), k.double()
    G = w.Hq // w.Hkv
    off = w.Lk - w.Lq
    out = []
    for r in rows:
        b, rem = divmod(int(r), w.Hq * w.Lq)
        h, i = divmod(rem, w.Lq)
        s = (kf[b, h // G] @ qf[b, h, i]).numpy() * w.scale * math.log2(math.e)
        last = min(w.Lk - 1, i + off) if w.causal else w.Lk - 1
        used, n = None, 0
        for t0 in range(0, last + 1, 128):
            m = s[t0:min(last, t0 + 127) + 1].max()
            if used is None:
                used = m
            elif m > used + 8.0:
                used, n = m, n + 1
        out.append(n)
    return np.array(out)


@pytest.mark.parametrize("shape", [(1, 4, 2, 1024, 128, True), (1, 4, 2, 1024, 128, False),
                                   (1, 3, 1, 1000, 128, True), (1, 4, 2, 1024, 64, True)],
                         ids=lambda s: "B{}_H{}x{}_L{}_d{}_{}".format(*s[:5], "c" if s[5] else "n"))
def test_rescale_in_every_tile(shape, cuda_device):
    """The lazy O rescale in every key tile for the + warps and never for the - warps of each
    softmax warpgroup, so that within one tile some warps hand the first half of P over early and
    others only after rescaling O: every row against the oracle (sibling-head units at G = 2,
    adjacent row tiles at G = 3; causal and not; d = 128 and 64)."""
    from exact_attention_139_b200 import attn
    B, Hq, Hkv, L, d, causal = shape
    w = Workload("rescale", B, Hq, Hkv, L, L, d, d, causal, seed=4242 + L + d)
    q, k, v = _ramp_inputs(w, beta=1.0 if d == 128 else 1.4)
    rows = np.arange(B * Hq * L)
    probe = rows[(rows % L) >= L - 256]  # rows that see at least 6 key tiles
    n = _lazy_rescales(w, q, k, probe)
    plus = ((probe % L) // 32) % 2 == 0
    assert n[plus].min() >= 3 and n[~plus].max() == 0, (n[plus].min(), n[~plus].max())
    o, lse = attn.attn_fwd(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=causal, scale=w.scale)
    assert attn.attn_check_device() == 0
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    compare(o.reshape(-1, d), lse.reshape(-1), o_ref, l_ref, f"rescale {shape}")


def test_long_context_sampled(cuda_device):
    """131072-token causal prefill with vertical key bias; sampled rows per head."""
    w = WORKLOADS["long_prefill_128k"]
    q, k, v, o, lse = run(w, cuda_device)
    rows = sample_rows(w, rows_per_head(256)).numpy()
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, w.name)


def test_deterministic(cuda_device):
    from exact_attention_139_b200 import attn
    w = Workload("det", 1, 4, 2, 300, 700, 128, 128, True, seed=77)
    q, k, v = (t.to(cuda_device) for t in make_inputs(w))
    o1, l1 = attn.attn_fwd(q, k, v, causal=True)
    o2, l2 = attn.attn_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("B,Hq,Hkv,pieces", [(1, 32, 8, 0), (1, 32, 8, 4), (2, 4, 2, 0), (2, 4, 2, 3),
                                             (3, 2, 1, 1), (3, 2, 1, 64), (5, 6, 3, 0)])
def test_host_path_matches_device_path(B, Hq, Hkv, pieces, cuda_device):
    """attn_fwd_host (the C entry point: pinned host buffers, pieces pipelined over copy and
    compute streams) gives the device call's O and LSE bit for bit."""
    from exact_attention_139_b200 import attn
    w = Workload("host", B, Hq, Hkv, 300, 300, 128, 128, True, seed=6000 + B)
    q, k, v = make_inputs(w)
    o_d, l_d = attn.attn_fwd(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=True)
    bufs = {}
    for _ in range(2):  # the second call reuses the scratch and the pinned outputs
        o_h, l_h = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=True,
                                      device=cuda_device, bufs=bufs, pieces=pieces)
        assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())
    assert attn.attn_check_device() == attn.ATTN_OK


def test_host_path_full_size_against_oracle(cuda_device):
    """The 8K prefill through the host entry point, sampled rows against the oracle."""
    from exact_attention_139_b200 import attn
    w = WORKLOADS["llama8b_prefill_8k"]
    q, k, v = make_inputs(w)
    o_h, l_h = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=True,
                                  device=cuda_device)
    assert attn.attn_check_device() == attn.ATTN_OK
    rows = sample_rows(w, 32).numpy()
    o_ref, l_ref = oracle_rows(w, q, k, v, rows)
    og, lg = take_rows(o_h, l_h, rows)
    compare(og, lg, o_ref, l_ref, "host path 8K")


def test_binding_rejects_mismatched_tensors(cuda_device):
    """Shapes that disagree with q are refused in the binding, before anything is launched."""
    from exact_attention_139_b200 import attn
    bf = dict(dtype=torch.bfloat16, device=cuda_device)
    q = torch.zeros(1, 4, 256, 128, **bf)
    k = torch.zeros(1, 2, 256, 128, **bf)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, k, torch.zeros(1, 2, 128, 128, **bf), causal=True)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, k, k, causal=True, out=torch.empty(1, 4, 128, 128, **bf))
    with pytest.raises(ValueError):
        attn.attn_fwd(q, k, k, causal=True, lse=torch.empty(4, 256, dtype=torch.float32, device=cuda_device))
    with pytest.raises(ValueError):
        attn.attn_decode(q[:, :, :1].contiguous(), k, k, causal=True, dv=256)
    op = torch.zeros(2, 8, 128, dtype=torch.float32, device=cuda_device)
    with pytest.raises(ValueError):
        attn.attn_combine(op, torch.zeros(2, 8, dtype=torch.float32, device=cuda_device), B=1, Hq=4, Lq=1)
    with pytest.raises(ValueError):
        attn.attn_combine(op, torch.zeros(2, 7, dtype=torch.float32, device=cuda_device), B=1, Hq=8, Lq=1)
    o, _ = attn.attn_fwd(q, k, k, causal=True)  # the same call with matching shapes runs
    assert attn.attn_check_device() == attn.ATTN_OK and o.shape == q.shape
