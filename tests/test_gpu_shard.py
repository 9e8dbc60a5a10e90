"""Head-sharded calls (the per-GPU work of tensor parallelism over heads) on one GPU.

Each shard is an ordinary, independent call on its slice of the heads; nothing waits on another
shard. Heads do not interact, so the shards gathered in rank order must equal the unsharded call
bit for bit (the decode split count is fixed so that both sides cut the keys the same way), and
each shard's output must match the fp64 oracle run on that shard's own q, k and v slices.
"""
import numpy as np
import pytest
import torch

from exact_attention_139_b200.inputs import Workload, make_inputs
from exact_attention_139_b200.shard import gather_heads, head_shard, shard_inputs
from tests.gpu_util import compare, oracle_rows, take_rows


def _check_shard_against_oracle(w, sh, qs, ks, vs, o, lse, what, n_rows=96):
    """Sampled rows of one shard's output (always its first and last row) against the oracle on
    the shard's slices, at the parity tolerances."""
    ws = w.with_(Hq=sh.Hq, Hkv=sh.Hkv)
    total = ws.B * ws.Hq * ws.Lq
    rng = np.random.default_rng(4242 + sh.rank)
    rows = np.unique(np.concatenate([[0, total - 1], rng.choice(total, size=min(n_rows, total), replace=False)]))
    o_ref, l_ref = oracle_rows(ws, qs.cpu(), ks.cpu(), vs.cpu(), rows)
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, f"{what} rank {sh.rank}/{sh.world}")

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
def test_prefill_head_shards_bitwise(world, cuda_device):
    from exact_attention_139_b200 import attn
    w = Workload("shard_pf", 2, 16, 4, 700, 700, 128, 128, True, seed=5000)
    q, k, v = (t.to(cuda_device) for t in make_inputs(w))
    o, lse = attn.attn_fwd(q, k, v, causal=True)
    parts = []
    for r in range(world):
        sh = head_shard(w.Hq, w.Hkv, world, r)
        qs, ks, vs = shard_inputs(q, k, v, sh)
        parts.append(attn.attn_fwd(qs, ks, vs, causal=True))
        _check_shard_against_oracle(w, sh, qs, ks, vs, *parts[-1], "prefill")
    torch.cuda.synchronize()
    assert attn.attn_check_device() == attn.ATTN_OK
    assert torch.equal(gather_heads(p[0] for p in parts), o)
    assert torch.equal(gather_heads(p[1] for p in parts), lse)


@pytest.mark.parametrize("latent", [False, True])
def test_decode_head_shards_bitwise(latent, cuda_device):
    from exact_attention_139_b200 import attn
    if latent:  # 16 heads on one latent head: a 2-way split replicates the latent head
        w = Workload("shard_mla", 4, 16, 1, 2, 5000, 576, 512, True, latent=True, seed=5001)
    else:
        w = Workload("shard_gqa", 4, 32, 8, 1, 5000, 128, 128, True, seed=5002)
    q, k, v = (t.to(cuda_device) for t in make_inputs(w))
    v = k if latent else v
    o, lse = attn.attn_decode(q, k, v, causal=True, dv=w.dv, num_splits=5)
    parts = []
    for r in range(2):
        sh = head_shard(w.Hq, w.Hkv, 2, r)
        qs, ks, vs = shard_inputs(q, k, v, sh)
        parts.append(attn.attn_decode(qs, ks, vs, causal=True, dv=w.dv, num_splits=5))
        _check_shard_against_oracle(w, sh, qs, ks, vs, *parts[-1], "decode")
    torch.cuda.synchronize()
    assert attn.attn_check_device() == attn.ATTN_OK
    assert torch.equal(gather_heads(p[0] for p in parts), o)
    assert torch.equal(gather_heads(p[1] for p in parts), lse)
