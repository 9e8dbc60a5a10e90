"""Multi-rank host logic of bench.py on CPU: two gloo ranks (spawned processes).

Each rank runs its own independent batch (weak scaling): the job time is the max over ranks and
the reported value counts the work of every rank. No data-path collective exists.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from exact_attention_139_b200.inputs import WORKLOADS, make_inputs
    ms_local = 1.0 + rank  # the slower rank sets the job time
    ms = bench.max_over_ranks(ms_local, world, device="cpu")
    w = bench.rank_workload(WORKLOADS["tiny_d64"], rank)
    q, _, _ = make_inputs(w)
    digest = float(q.float().sum())
    out[rank] = (ms, w.seed, digest, bench.dist_env())
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_batches():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.0
    assert res[0][1] != res[1][1]          # each rank draws its own batch
    assert res[0][2] != res[1][2]
    assert res[0][3] == (2, 0, 0) and res[1][3] == (2, 1, 1)


def test_reference_arm_only_rank0_prints(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        workload = "tiny_d64"
        steps = 1
        warmup = 0
        cpu_seconds = 0.1
    bench.run_reference(A())
    assert capsys.readouterr().out == ""


# ------------------------------------------------------------------------------------------------
# head sharding (tensor parallel over heads, no collective on the data path)
# ------------------------------------------------------------------------------------------------
def test_head_shard_rules():
    from exact_attention_139_b200.shard import head_shard
    # Llama-3-8B shape over 4 ranks: whole groups of 4 query heads and their kv heads
    s = [head_shard(32, 8, 4, r) for r in range(4)]
    assert [x.q_heads for x in s] == [(0, 8), (8, 16), (16, 24), (24, 32)]
    assert [x.kv_heads for x in s] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    # MLA: 128 query heads on one latent head over 8 GPUs, 16 heads each, latent head replicated
    s = [head_shard(128, 1, 8, r) for r in range(8)]
    assert all(x.Hq == 16 and x.kv_heads == (0, 1) for x in s)
    # a group of 8 spread over 2 ranks of 4 heads: each holds a copy of its kv head
    assert head_shard(16, 2, 4, 3).kv_heads == (1, 2)
    # uneven heads, groups of 6 cut into 4s, rank out of range, Hq not a multiple of Hkv
    for bad in [(32, 8, 3, 0), (24, 4, 6, 0), (32, 8, 4, 4), (30, 4, 2, 0)]:
        with pytest.raises(ValueError):
            head_shard(*bad)


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np
    from exact_attention_139_b200.inputs import Workload, make_inputs
    from exact_attention_139_b200.shard import head_shard, shard_inputs
    from oracle import oracle
    results = {}
    for name, w in [("gqa", Workload("sh", 2, 8, 2, 9, 13, 16, 16, True, seed=77)),
                    ("mla", Workload("sh_mla", 2, 8, 1, 2, 21, 24, 16, True, latent=True, seed=78))]:
        q, k, v = make_inputs(w)  # every rank draws the same global inputs
        sh = head_shard(w.Hq, w.Hkv, world, rank)
        qs, ks, vs = shard_inputs(q, k, v, sh)
        o, lse = oracle.attn(qs, ks, vs, B=w.B, Hq=sh.Hq, Hkv=sh.Hkv, Lq=w.Lq, Lk=w.Lk, d=w.d, dv=w.dv,
                             ldv=w.ldv, scale=w.scale, causal=w.causal)
        results[name] = (o, lse)
    out[rank] = results
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_head_shards_reassemble_the_layer():
    """Each of two gloo ranks computes its head shard; the shards, gathered in rank order, equal
    the unsharded layer (heads are independent: no exchange is needed)."""
    import numpy as np
    from exact_attention_139_b200.inputs import Workload, make_inputs
    from oracle import oracle
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for name, w in [("gqa", Workload("sh", 2, 8, 2, 9, 13, 16, 16, True, seed=77)),
                    ("mla", Workload("sh_mla", 2, 8, 1, 2, 21, 24, 16, True, latent=True, seed=78))]:
        q, k, v = make_inputs(w)
        o, lse = oracle.attn(q, k, v, B=w.B, Hq=w.Hq, Hkv=w.Hkv, Lq=w.Lq, Lk=w.Lk, d=w.d, dv=w.dv, ldv=w.ldv,
                             scale=w.scale, causal=w.causal)
        og = np.concatenate([res[r][name][0] for r in range(world)], axis=1)
        lg = np.concatenate([res[r][name][1] for r in range(world)], axis=1)
        assert np.array_equal(og, o) and np.array_equal(lg, lse)


def test_bench_job_workload_modes():
    import bench
    from exact_attention_139_b200.inputs import WORKLOADS
    w = WORKLOADS["llama8b_prefill_8k"]
    b = bench.job_workload(w, 4, 1, "batch")
    assert (b.Hq, b.Hkv, b.B) == (32, 8, 1) and b.seed != w.seed
    h = bench.job_workload(w, 4, 1, "heads")
    assert (h.Hq, h.Hkv, h.Lq) == (8, 2, 8192)
    assert h.flops() * 4 == w.flops()  # the shards add up to the layer
    m = bench.job_workload(WORKLOADS["mla_decode_64k"], 8, 7, "heads")
    assert (m.Hq, m.Hkv, m.latent) == (2, 1, True) and m.kv_bytes() == WORKLOADS["mla_decode_64k"].kv_bytes()
    assert bench.job_workload(w, 1, 0, "heads") == w


def test_sparse_workload_index_structure():
    """The sparse workload's given index: per query block a sorted, distinct list inside the causal
    range that holds the first block, the diagonal block and the blocks of the biased keys."""
    import numpy as np
    from exact_attention_139_b200.inputs import Workload, block_lists, sparse_visible_pairs, vertical_positions
    w = Workload("sp", 1, 4, 2, 2048, 2048, 16, 16, True, vertical_keys=8, vertical_bias=2.0, seed=5,
                 sparse_window=3)
    idx, cnt = block_lists(w)
    pos = vertical_positions(w)
    for h in range(w.Hq):
        vb = set((pos[h // 2].numpy() // 128).tolist())
        for qb in range(16):
            lst = idx[0, h, qb, :cnt[0, h, qb]].tolist()
            assert lst == sorted(set(lst)) and lst[0] == 0 and lst[-1] == qb
            assert set(range(max(0, qb - 2), qb + 1)) <= set(lst)
            assert {b for b in vb if b <= qb} <= set(lst)
            assert all(b <= qb for b in lst)
    full = sparse_visible_pairs(w, np.tile(np.arange(16, dtype=np.int32), (1, 4, 16, 1)),
                                np.full((1, 4, 16), 16, dtype=np.int32))
    assert full == w.visible_pairs()  # every block listed: the dense causal count
