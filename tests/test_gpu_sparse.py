"""attn_fwd_sparse (block-sparse prefill over given key-block lists) against the fp64 oracle.

Reading of the MInference article's sparse patterns: with a given index, the result is the exact
softmax restricted to the listed 128-key blocks of each 128-row query block (causal mask still
applied; a row that sees no key gets O = 0 and LSE = -inf).
"""
import numpy as np
import pytest
import torch

from exact_attention_139_b200.inputs import Workload, make_inputs, sample_rows
from oracle import oracle
from tests.gpu_util import compare, take_rows

pytestmark = pytest.mark.gpu

BLK = 128


def random_lists(B, Hq, nqb, nkb, seed, p_keep=0.5, extra=2):
    g = np.random.default_rng(seed)
    max_blk = nkb + extra
    idx = np.full((B, Hq, nqb, max_blk), 12345, dtype=np.int32)  # junk past the counts
    cnt = np.zeros((B, Hq, nqb), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            for qb in range(nqb):
                keep = np.flatnonzero(g.random(nkb) < p_keep)
                if (b * 7 + h * 3 + qb) % 6 == 5:
                    keep = keep[:0]  # an empty list
                idx[b, h, qb, :keep.size] = keep
                cnt[b, h, qb] = keep.size
    return idx, cnt


def run_sparse(w, q, k, v, idx, cnt, dev):
    from exact_attention_139_b200 import attn
    o, lse = attn.attn_fwd_sparse(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(idx).to(dev),
                                  torch.from_numpy(cnt).to(dev), causal=w.causal, scale=w.scale)
    assert attn.attn_check_device() == attn.ATTN_OK
    return o, lse


def oracle_sparse(w, q, k, v, idx, cnt, rows):
    return oracle.attn_rows(q, k, v, rows, B=w.B, Hq=w.Hq, Hkv=w.Hkv, Lq=w.Lq, Lk=w.Lk, d=w.d, dv=w.dv,
                            scale=w.scale, causal=w.causal, blocks=(idx, cnt, BLK, BLK))


SHAPES = [
    # B, Hq, Hkv, Lq, Lk, d, causal
    (1, 4, 2, 700, 900, 128, True),
    (2, 2, 1, 300, 1000, 64, False),
    (1, 2, 2, 1000, 1000, 128, True),
    (1, 8, 2, 129, 1500, 128, True),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_H{}x{}_L{}x{}_d{}_{}".format(*s[:6], "c" if s[6] else "n"))
def test_full_lists_equal_dense_bitwise(shape, cuda_device):
    """Listing every block runs the same products in the same order as attn_fwd."""
    from exact_attention_139_b200 import attn
    B, Hq, Hkv, Lq, Lk, d, causal = shape
    w = Workload("sp_full", B, Hq, Hkv, Lq, Lk, d, d, causal, seed=4000 + Lq)
    q, k, v = make_inputs(w)
    nqb, nkb = -(-Lq // BLK), -(-Lk // BLK)
    idx = np.tile(np.arange(nkb, dtype=np.int32), (B, Hq, nqb, 1))
    cnt = np.full((B, Hq, nqb), nkb, dtype=np.int32)
    o_s, l_s = run_sparse(w, q, k, v, idx, cnt, cuda_device)
    o_d, l_d = attn.attn_fwd(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o_s, o_d) and torch.equal(l_s, l_d)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_H{}x{}_L{}x{}_d{}_{}".format(*s[:6], "c" if s[6] else "n"))
def test_random_lists_vs_oracle(shape, dtype, cuda_device):
    B, Hq, Hkv, Lq, Lk, d, causal = shape
    w = Workload("sp_rand", B, Hq, Hkv, Lq, Lk, d, d, causal, seed=4100 + Lq + Lk, dtype=dtype)
    q, k, v = make_inputs(w)
    nqb, nkb = -(-Lq // BLK), -(-Lk // BLK)
    idx, cnt = random_lists(B, Hq, nqb, nkb, seed=Lq + 7 * Lk)
    o, lse = run_sparse(w, q, k, v, idx, cnt, cuda_device)
    rows = np.arange(B * Hq * Lq)
    o_ref, l_ref = oracle_sparse(w, q, k, v, idx, cnt, rows)
    assert np.isfinite(l_ref).any()
    compare(o.reshape(-1, d), lse.reshape(-1), o_ref, l_ref, f"sparse {shape} {dtype}")


def test_rows_that_see_no_key(cuda_device):
    """Lk = Lq + 64: with only block 1 listed, rows 0..63 of query block 0 see no key."""
    w = Workload("sp_edge", 1, 2, 1, 200, 264, 128, 128, True, seed=4200)
    q, k, v = make_inputs(w)
    idx = np.zeros((1, 2, 2, 3), dtype=np.int32)
    cnt = np.zeros((1, 2, 2), dtype=np.int32)
    idx[0, :, 0, :1] = [1]
    cnt[0, :, 0] = 1
    idx[0, :, 1, :2] = [0, 2]
    cnt[0, :, 1] = 2
    o, lse = run_sparse(w, q, k, v, idx, cnt, cuda_device)
    rows = np.arange(w.B * w.Hq * w.Lq)
    o_ref, l_ref = oracle_sparse(w, q, k, v, idx, cnt, rows)
    assert np.isinf(l_ref.reshape(2, 200)[:, :64]).all()
    compare(o.reshape(-1, 128), lse.reshape(-1), o_ref, l_ref, "no-key rows")
    assert (o[0, :, :64] == 0).all()


def test_a_shape_long_sampled(cuda_device):
    """A-shape pattern (first block + a local window of 8 blocks) on a 32K causal prefill."""
    w = Workload("sp_ashape", 1, 8, 2, 32768, 32768, 128, 128, True, seed=4300)
    q, k, v = make_inputs(w)
    nqb = w.Lq // BLK
    idx = np.zeros((1, 8, nqb, 9), dtype=np.int32)
    cnt = np.zeros((1, 8, nqb), dtype=np.int32)
    for qb in range(nqb):
        lst = sorted({0} | set(range(max(0, qb - 7), qb + 1)))
        idx[0, :, qb, :len(lst)] = lst
        cnt[0, :, qb] = len(lst)
    o, lse = run_sparse(w, q, k, v, idx, cnt, cuda_device)
    rows = sample_rows(w, 12).numpy()
    o_ref, l_ref = oracle_sparse(w, q, k, v, idx, cnt, rows)
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, "a-shape 32k")


def test_bad_list_is_reported(cuda_device):
    """An unsorted list is read up to the offending entry and reported; the next call is clean."""
    from exact_attention_139_b200 import attn
    w = Workload("sp_bad", 1, 2, 1, 256, 256, 128, 128, True, seed=4400)
    q, k, v = (t.to(cuda_device) for t in make_inputs(w))
    # query block 1 of head 0 lists block 1 then block 0 (block 0 alone would be fine for
    # query block 0: a list is only read up to its first block above the causal diagonal)
    idx = torch.tensor([[[[0, 1], [1, 0]], [[0, 1], [0, 1]]]], dtype=torch.int32, device=cuda_device)
    cnt = torch.full((1, 2, 2), 2, dtype=torch.int32, device=cuda_device)
    attn.attn_fwd_sparse(q, k, v, idx, cnt, causal=True)
    assert attn.attn_check_device() == attn.ATTN_ERR_INVALID_ARG
    idx[0, 0, 1] = torch.tensor([0, 1], dtype=torch.int32)
    attn.attn_fwd_sparse(q, k, v, idx, cnt, causal=True)
    assert attn.attn_check_device() == attn.ATTN_OK


def test_sparse_prefill_128k_sampled(cuda_device):
    """The benchmarked sparse workload (128K causal, A-shape + vertical blocks), in the launch
    configuration bench.py times, on sampled rows of every head."""
    from exact_attention_139_b200.inputs import WORKLOADS, block_lists
    w = WORKLOADS["sparse_prefill_128k"]
    q, k, v = make_inputs(w)
    idx, cnt = block_lists(w)
    o, lse = run_sparse(w, q, k, v, idx, cnt, cuda_device)
    rows = sample_rows(w, 4).numpy()
    o_ref, l_ref = oracle_sparse(w, q, k, v, idx, cnt, rows)
    og, lg = take_rows(o, lse, rows)
    compare(og, lg, o_ref, l_ref, w.name)
