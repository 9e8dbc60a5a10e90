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
    with mp.Manager() as mgr:
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
