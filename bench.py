"""Benchmark: exact attention on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one pass of the hot path over one batch of synthetic input. The default workload is the
Llama-3-8B-shaped causal GQA prefill (B=1, Hq=32, Hkv=8, L=8192, d=128): metric attention TFLOPS
(algorithmic flops = 2*(d+dv) per visible query/key pair). The same JSON line also carries the
MLA-shaped split-KV decode (B=32, 16 heads on one 576/512 latent head, Lq=2, Lk=65536) and the GQA
decode (B=16, 32 query heads on 8 kv heads, Lk=32768) measured in HBM GB/s, and the fp16-input
variants of the prefill and of the MLA decode, the 16 x 2K batched causal prefill, the 256-token
batched prefill (against the larger of its compute and HBM times), and the 128K long-context
prefill, dense and block-sparse over its given index, each with its roofline fraction against
MEASURED_PEAKS.json.

Timing: W untimed warm-up steps, then K steps each bracketed by CUDA events on the launching stream;
L2 is flushed (a 256 MiB write) before every timed step, outside the events. Multi-GPU (torchrun):
every rank runs its own copy of the workload (independent batches: weak scaling, no collective on
the data path); the per-rank time is max-reduced and value = total flops of all ranks / max time.

--impl reference times the fp64 CPU oracle on a bounded seeded sample of the same workload (the
reference arm: the pages ship no runnable code, so the oracle is the reference program).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from exact_attention_139_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
# DRAM bytes (read + write) per launch of the timed kernel, from one ncu capture of the current
# kernels (dram__bytes.sum.per_second x gpu__time_duration.sum; see profiles/): reported as the
# roofline "traffic". Re-measure whenever one of these kernels changes.
NCU_TRAFFIC_BYTES = {
    "llama8b_prefill_8k": 137.9e6,   # prefill2_kernel<128, bf16, dense> (registers 184 / 64 / 80)
    "batched_prefill_2k": 839.9e6,   # same kernel
    "batched_prefill_256": 53.8e6,   # same kernel (O still in L2 when it ends)
    "mla_decode_64k": 2421.4e6,      # decode_tn_kernel<9,2,48,3,latent,bf16>, balanced grid
    "gqa_decode_32k": 2150.9e6,      # decode_tn_kernel<2,1,48,3,dense V,bf16>, balanced grid
}
# the profiles/ summary each figure above comes from
NCU_TRAFFIC_SOURCE = {
    "llama8b_prefill_8k": "profiles/prefill2_kernel_llama8b_prefill_8k.md",
    "batched_prefill_2k": "profiles/prefill2_kernel_batched_prefill_2k.md",
    "batched_prefill_256": "profiles/prefill2_kernel_batched_prefill_256.md",
    "mla_decode_64k": "profiles/decode_tn_kernel_mla_decode_64k.md",
    "gqa_decode_32k": "profiles/decode_tn_kernel_gqa_decode_32k.md",
}


def traffic(name: str, exact_shape: bool):
    """(traffic bytes per launch, source) of the profiled kernel for this workload, or (None, None)
    when this rank's shape is not the profiled one."""
    if not exact_shape or name not in NCU_TRAFFIC_BYTES:
        return None, None
    return NCU_TRAFFIC_BYTES[name], NCU_TRAFFIC_SOURCE[name]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of one GPU every ~10 ms from a
    background thread through NVML (read-only queries), during the timed region."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.thread = None

    def _run(self):
        import pynvml
        try:
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            while not self.stop_flag:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                try:
                    reasons = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except AttributeError:
                    reasons = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((sm, reasons))
                time.sleep(0.01)
        except Exception as e:  # clocks are reported as unavailable, the run itself continues
            self.error = str(e)

    def start(self):
        import threading
        self.stop_flag = False
        self.error = None
        self.max_mhz = None
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        time.sleep(0.05)

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=5)
        if not self.samples:
            return {"error": self.error} if self.error else None
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# timing helpers
# ------------------------------------------------------------------------------------------------
class Flusher:
    def __init__(self, dev):
        self.buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.fill_(1)


def time_steps(step, steps, warmup, flush, stream):
    """Per-step CUDA-event durations (ms) of `step` on `stream`, L2 flushed before each step."""
    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """Max of a per-rank scalar over the process group (the slowest rank sets the job time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank: int):
    """Each rank processes its own independent batch (same shape, its own seed)."""
    return w if rank == 0 else w.with_(seed=w.seed + 1000 * rank)


def job_workload(w, world: int, rank: int, shard: str):
    """This rank's part of the job: its own batch of the full shape (shard == "batch", weak
    scaling), or its head shard of one layer (shard == "heads", strong scaling: Hq / world query
    heads and the kv heads they read, replicated where a group spans ranks)."""
    if shard == "batch" or world == 1:
        return rank_workload(w, rank)
    from exact_attention_139_b200.shard import head_shard
    sh = head_shard(w.Hq, w.Hkv, world, rank)
    return w.with_(Hq=sh.Hq, Hkv=sh.Hkv, seed=w.seed + 1000 * rank)


def bench_config(w, world: int, shard: str) -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Lq": w.Lq, "Lk": w.Lk, "d": w.d,
            "dv": w.dv, "causal": w.causal, "flops_per_step_per_gpu": w.flops(),
            "l2": "flushed (256 MiB write) before every timed step",
            "parallelism": ("single GPU" if world == 1 else
                            f"head-sharded x{world} ({w.Hq} query heads per GPU)" if shard == "heads"
                            else f"independent replicas x{world}")}


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


# ------------------------------------------------------------------------------------------------
# CPU baseline / reference arm: the fp64 oracle on a bounded sample
# ------------------------------------------------------------------------------------------------
def oracle_sample_rate(w, target_s: float, q=None, k=None, v=None):
    """Time the oracle on seeded rows of workload w; returns (flops/s, rows, seconds, threads)."""
    from oracle import oracle
    if q is None:
        q, k, v = make_inputs(w)
    g = np.random.default_rng(12345)
    threads = oracle.default_threads()
    # calibrate on a small batch, then size the sample to ~target_s seconds
    n = 64
    total_rows = w.B * w.Hq * w.Lq
    while True:
        rows = np.sort(g.choice(total_rows, size=min(n, total_rows), replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attn_rows(q, k, (k if w.latent else v), rows, B=w.B, Hq=w.Hq, Hkv=w.Hkv, Lq=w.Lq, Lk=w.Lk, d=w.d,
                         dv=w.dv, ldv=w.ldv, scale=w.scale, causal=w.causal, nthreads=threads)
        dt = time.perf_counter() - t0
        if dt >= target_s or n >= total_rows:
            break
        n = int(min(total_rows, max(2 * n, n * target_s / max(dt, 1e-3) * 1.05)))
    flops = 0.0
    off = w.Lk - w.Lq
    for r in rows:
        i = int(r) % w.Lq
        vis = min(w.Lk, i + off + 1) if w.causal else w.Lk
        flops += vis * 2.0 * (w.d + w.dv)
    return flops / dt, len(rows), dt, threads


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
def bench_prefill(w, dev, steps, warmup, flush, stream):
    from exact_attention_139_b200 import attn
    q, k, v = make_inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty((w.B, w.Hq, w.Lq, w.dv), dtype=w.torch_dtype, device=dev)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)
    step = lambda: attn.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale, out=o, lse=lse)
    times = time_steps(step, steps, warmup, flush, stream)
    if attn.attn_check_device() != attn.ATTN_OK:
        raise RuntimeError("device error during the prefill benchmark")
    return times, (q, k, v)


def bench_prefill_sparse(w, dev, steps, warmup, flush, stream, dense_steps=0):
    """Block-sparse prefill over the workload's given index (inputs.block_lists); with dense_steps
    > 0 also the dense causal prefill of the same inputs (the 128K long-context config: the sparse
    workload shares its seeded Q, K, V)."""
    from exact_attention_139_b200 import attn
    from exact_attention_139_b200.inputs import block_lists, sparse_visible_pairs
    q, k, v = make_inputs(w)
    idx, cnt = block_lists(w)
    pairs = sparse_visible_pairs(w, idx, cnt)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    del q, k, v
    idx_d, cnt_d = torch.from_numpy(idx).to(dev), torch.from_numpy(cnt).to(dev)
    o = torch.empty((w.B, w.Hq, w.Lq, w.dv), dtype=w.torch_dtype, device=dev)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)
    step = lambda: attn.attn_fwd_sparse(qd, kd, vd, idx_d, cnt_d, causal=w.causal, scale=w.scale, out=o, lse=lse)
    times = time_steps(step, steps, warmup, flush, stream)
    dense_times = []
    if dense_steps > 0:
        dstep = lambda: attn.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale, out=o, lse=lse)
        dense_times = time_steps(dstep, dense_steps, 1, flush, stream)
    if attn.attn_check_device() != attn.ATTN_OK:
        raise RuntimeError("device error during the 128K prefill benchmarks")
    return times, pairs, dense_times


def host_link_ms(dev, h2d_bytes: int, d2h_bytes: int, reps: int = 5):
    """Time (ms) to move h2d_bytes host -> device and d2h_bytes device -> host concurrently, as
    two plain copies on two streams between pinned host memory and the device: the bound of any
    end-to-end call that moves those bytes over the host link."""
    hi = torch.empty(h2d_bytes, dtype=torch.uint8, pin_memory=True)
    ho = torch.empty(d2h_bytes, dtype=torch.uint8, pin_memory=True)
    di = torch.empty(h2d_bytes, dtype=torch.uint8, device=dev)
    do = torch.empty(d2h_bytes, dtype=torch.uint8, device=dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    main = torch.cuda.current_stream(dev)
    best = float("inf")
    for _ in range(reps):
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(main)
        s_in.wait_stream(main)
        s_out.wait_stream(main)
        with torch.cuda.stream(s_in):
            di.copy_(hi, non_blocking=True)
        with torch.cuda.stream(s_out):
            ho.copy_(do, non_blocking=True)
        main.wait_stream(s_in)
        main.wait_stream(s_out)
        b.record(main)
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b))
    return best


def bench_prefill_e2e(w, dev, steps, warmup, host):
    """End to end through the library's host entry point (attn_fwd_host): pinned host inputs ->
    device, the prefill, O and LSE back to pinned host memory, all inside the timed region."""
    from exact_attention_139_b200 import attn
    q, k, v = (t.pin_memory() for t in host)
    bufs = {}
    for _ in range(max(1, warmup)):
        attn.attn_fwd_host(q, k, v, causal=w.causal, scale=w.scale, device=dev, bufs=bufs)
    stream = torch.cuda.current_stream(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        attn.attn_fwd_host(q, k, v, causal=w.causal, scale=w.scale, device=dev, bufs=bufs)
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = bufs["o_host"].numel() * bufs["o_host"].element_size() + bufs["lse_host"].numel() * 4
    return ms, h2d, d2h


DECODE_IMPLS = {"auto": 0, "cuda_core": 1, "keys_on_m": 2, "queries_on_m": 3}  # attn_decode_impl


def bench_decode(w, dev, steps, warmup, flush, stream, impl="auto", num_splits=0):
    """Decode steps (split kernel + combine). impl / num_splits select the kernel and the split
    count (0: the library's own schedule, balanced over the SMs for the tensor-core kernel)."""
    from exact_attention_139_b200 import attn
    q, k, v = make_inputs(w)
    qd, kd = q.to(dev), k.to(dev)
    vd = kd if w.latent else v.to(dev)
    del q, k, v
    # `splits` reports the partial-slot count
    splits = num_splits or attn.attn_decode_default_splits(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, w.dv, w.latent)
    ws = torch.empty(attn.attn_decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.dv, num_splits),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((w.B, w.Hq, w.Lq, w.dv), dtype=w.torch_dtype, device=dev)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)
    step = lambda: attn.attn_decode(qd, kd, vd, causal=w.causal, scale=w.scale, dv=w.dv, num_splits=num_splits,
                                    impl=DECODE_IMPLS[impl], workspace=ws, out=o, lse=lse)
    times = time_steps(step, steps, warmup, flush, stream)
    if attn.attn_check_device() != attn.ATTN_OK:
        raise RuntimeError("device error during the decode benchmark")
    # time the split kernel alone (the combine is the second launch of each step)
    return times, splits


def run_ours(args):
    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    w = job_workload(WORKLOADS[args.workload], world, rank, args.shard)
    stream = torch.cuda.current_stream(dev)
    flush = Flusher(dev)
    clocks = ClockSampler(torch.cuda.current_device())

    barrier(world)
    clocks.start()
    times, host = bench_prefill(w, dev, args.steps, args.warmup, flush, stream)
    clk = clocks.stop()
    barrier(world)
    ms_local = sum(times) / len(times)
    ms = max_over_ranks(ms_local, world)
    flops = w.flops()
    value = flops * world / (ms * 1e-3) / 1e12
    per_gpu_tflops = flops / (ms * 1e-3) / 1e12
    peak_tf = float(peaks["bf16_tflops"])
    # kernels that run for milliseconds (the 128K legs: one launch of ~12 ms sparse, ~120 ms dense)
    # hold the tensor cores busy long enough for the power cap to lower the SM clock, so their
    # denominator is the sustained figure (a seconds-long GEMM loop) rather than the burst one
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak_tf))
    sus_src = f"{peak_src} bf16_tflops_sustained (kernel of milliseconds under the power cap)"

    extras = {}
    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h = bench_prefill_e2e(w, dev, max(2, args.steps // 2), 1, host)
        e_ms = max_over_ranks(e_ms, world)
        link_ms = host_link_ms(dev, h2d, d2h)
        e2e = {"value": round(flops * world / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4), "call": "attn_fwd_host (C ABI, host buffers)",
               "host_link_ms": round(link_ms, 4), "frac_of_host_link": round(link_ms / e_ms, 4)}
    del host
    launches = args.steps  # one prefill kernel per step
    if not args.no_extras:
        wd = job_workload(WORKLOADS["mla_decode_64k"], world, rank, args.shard)
        clocks_d = ClockSampler(torch.cuda.current_device())
        clocks_d.start()
        dtimes, splits = bench_decode(wd, dev, args.steps, args.warmup, flush, stream, args.decode_impl,
                                      args.decode_splits)
        dflt = args.decode_impl == "auto" and args.decode_splits == 0  # the profiled configuration
        dclk = clocks_d.stop()
        dms = max_over_ranks(sum(dtimes) / len(dtimes), world)
        gbs = wd.kv_bytes() / (dms * 1e-3) / 1e9
        wg = job_workload(WORKLOADS["gqa_decode_32k"], world, rank, args.shard)
        gtimes, gsplits = bench_decode(wg, dev, args.steps, args.warmup, flush, stream)
        gms = max_over_ranks(sum(gtimes) / len(gtimes), world)
        ggbs = wg.kv_bytes() / (gms * 1e-3) / 1e9
        extras["decode_gqa"] = {
            "workload": wg.name, "metric": "KV-read HBM GB/s", "value": round(ggbs * world, 1),
            "per_gpu_gbs": round(ggbs, 1), "ms_per_step": round(gms, 4), "num_splits": gsplits, "schedule": "balanced grid (num_splits = most partials per kv head)",
            "roofline": {"bound": "hbm", "achieved": round(ggbs, 1), "peak": float(peaks["hbm_gbs"]),
                         "unit": "GB/s", "frac": round(ggbs / float(peaks["hbm_gbs"]), 4),
                         "algorithmic_bytes_per_launch": wg.kv_bytes(),
                         "traffic": traffic(wg.name, wg.Hq == 32)[0],
                         "traffic_source": traffic(wg.name, wg.Hq == 32)[1]}}
        launches += 2 * args.steps
        extras["decode"] = {
            "workload": wd.name, "metric": "KV-read HBM GB/s", "value": round(gbs * world, 1),
            "per_gpu_gbs": round(gbs, 1), "ms_per_step": round(dms, 4), "num_splits": splits,
            "schedule": ("balanced grid (num_splits = most partials per kv head)" if args.decode_splits == 0
                         else f"{args.decode_splits} equal splits per kv head"),
            "kernel": args.decode_impl, "kernels_per_step": 2,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                         "frac": round(gbs / float(peaks["hbm_gbs"]), 4), "peak_source": peak_src,
                         "algorithmic_bytes_per_launch": wd.kv_bytes(),
                         "traffic": traffic(wd.name, wd.Hq == 16 and dflt)[0],
                         "traffic_source": traffic(wd.name, wd.Hq == 16 and dflt)[1],
                         "note": "step = split kernel + combine kernel"},
            "tflops": round(wd.flops() / (dms * 1e-3) / 1e12, 1), "clocks": dclk}
        launches += 2 * args.steps
        # 256-token batched sweep: reported against the larger of its compute and HBM times (Q, K, V
        # and O are 84 MB; the L2 is flushed before every step, so they come from HBM)
        wsh = job_workload(WORKLOADS["batched_prefill_256"], world, rank, args.shard)
        shtimes, _ = bench_prefill(wsh, dev, args.steps, args.warmup, flush, stream)
        shms = max_over_ranks(sum(shtimes) / len(shtimes), world)
        sh_bytes = 2 * (2 * wsh.B * wsh.Hq * wsh.Lq * wsh.d + wsh.B * wsh.Hkv * wsh.Lk * (wsh.d + wsh.dv))
        t_bound = max(wsh.flops() / (peak_tf * 1e12), sh_bytes / (float(peaks["hbm_gbs"]) * 1e9))
        extras["prefill_short"] = {
            "workload": wsh.name, "metric": "attention TFLOPS", "value": round(wsh.flops() * world / (shms * 1e-3) / 1e12, 2),
            "ms_per_step": round(shms, 4),
            "roofline": {"bound": "max(tensor, hbm)", "achieved_ms": round(shms, 4), "bound_ms": round(t_bound * 1e3, 4),
                         "frac": round(t_bound * 1e3 / shms, 4), "algorithmic_flops_per_launch": wsh.flops(),
                         "algorithmic_bytes_per_launch": sh_bytes,
                         "traffic": traffic(wsh.name, world == 1 or args.shard == "batch")[0],
                         "traffic_source": traffic(wsh.name, world == 1 or args.shard == "batch")[1]}}
        launches += args.steps
        # batched causal prefill, B = 16 at 2K tokens (the batched configuration of the Llama-3-8B
        # shape): compute-bound like the 8K prefill, against the same tensor peak
        wb = job_workload(WORKLOADS["batched_prefill_2k"], world, rank, args.shard)
        btimes, _ = bench_prefill(wb, dev, args.steps, args.warmup, flush, stream)
        bms = max_over_ranks(sum(btimes) / len(btimes), world)
        btf = wb.flops() / (bms * 1e-3) / 1e12
        b_exact = world == 1 or args.shard == "batch"
        extras["prefill_batched_2k"] = {
            "workload": wb.name, "metric": "attention TFLOPS", "value": round(btf * world, 2),
            "ms_per_step": round(bms, 4),
            "roofline": {"bound": "tensor", "achieved": round(btf, 2), "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": round(btf / peak_tf, 4), "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "algorithmic_flops_per_launch": wb.flops(),
                         "traffic": traffic(wb.name, b_exact)[0], "traffic_source": traffic(wb.name, b_exact)[1]}}
        launches += args.steps
        if not args.no_f16:
            # fp16 inputs: same kernels with the fp16 operand format; fp16 and bf16 share one
            # nominal tensor rate on B200, so the measured bf16 peak is the fp16 denominator
            wf = job_workload(WORKLOADS[args.workload].with_(dtype="f16"), world, rank, args.shard)
            ftimes, _ = bench_prefill(wf, dev, args.steps, args.warmup, flush, stream)
            fms = max_over_ranks(sum(ftimes) / len(ftimes), world)
            ftf = wf.flops() / (fms * 1e-3) / 1e12
            extras["prefill_f16"] = {
                "workload": wf.name + " (fp16 inputs)", "metric": "attention TFLOPS", "value": round(ftf * world, 2),
                "ms_per_step": round(fms, 4),
                "roofline": {"bound": "tensor", "achieved": round(ftf, 2), "peak": peak_tf, "unit": "TFLOP/s",
                             "frac": round(ftf / peak_tf, 4),
                             "peak_source": f"{peak_src} bf16_tflops (burst) x 1 (fp16:bf16 nominal ratio)"}}
            wdf = job_workload(WORKLOADS["mla_decode_64k"].with_(dtype="f16"), world, rank, args.shard)
            dftimes, dfsplits = bench_decode(wdf, dev, args.steps, args.warmup, flush, stream)
            dfms = max_over_ranks(sum(dftimes) / len(dftimes), world)
            dfgbs = wdf.kv_bytes() / (dfms * 1e-3) / 1e9
            extras["decode_f16"] = {
                "workload": wdf.name + " (fp16 inputs)", "metric": "KV-read HBM GB/s", "value": round(dfgbs * world, 1),
                "ms_per_step": round(dfms, 4), "num_splits": dfsplits, "schedule": "balanced grid (num_splits = most partials per kv head)",
                "roofline": {"bound": "hbm", "achieved": round(dfgbs, 1), "peak": float(peaks["hbm_gbs"]),
                             "unit": "GB/s", "frac": round(dfgbs / float(peaks["hbm_gbs"]), 4)}}
            launches += args.steps + 2 * args.steps
        if not args.no_sparse:
            ws_ = job_workload(WORKLOADS["sparse_prefill_128k"], world, rank, args.shard)
            sp_steps = max(3, args.steps // 10)  # ~13 ms per step
            long_steps = max(2, args.steps // 50)  # ~130 ms per step
            stimes, pairs, ltimes = bench_prefill_sparse(ws_, dev, sp_steps, min(args.warmup, 5), flush, stream,
                                                         dense_steps=long_steps)
            sms = max_over_ranks(sum(stimes) / len(stimes), world)
            sflops = pairs * 2.0 * (ws_.d + ws_.dv)
            stf = sflops / (sms * 1e-3) / 1e12
            extras["prefill_sparse"] = {
                "workload": ws_.name, "metric": "attention TFLOPS over the visible (listed, causal) pairs",
                "value": round(stf * world, 2), "ms_per_step": round(sms, 4), "steps": sp_steps,
                "density": round(pairs / ws_.visible_pairs(), 4),
                "dense_equivalent_tflops": round(ws_.flops() / (sms * 1e-3) / 1e12, 1),
                "roofline": {"bound": "tensor", "achieved": round(stf, 2), "peak": peak_sus, "unit": "TFLOP/s",
                             "frac": round(stf / peak_sus, 4), "peak_source": sus_src,
                             "frac_of_burst": round(stf / peak_tf, 4), "algorithmic_flops_per_launch": sflops}}
            launches += sp_steps
            wl = job_workload(WORKLOADS["long_prefill_128k"], world, rank, args.shard)
            lms = max_over_ranks(sum(ltimes) / len(ltimes), world)
            ltf = wl.flops() / (lms * 1e-3) / 1e12
            extras["prefill_long"] = {
                "workload": wl.name, "metric": "attention TFLOPS", "value": round(ltf * world, 2),
                "ms_per_step": round(lms, 3), "steps": long_steps,
                "roofline": {"bound": "tensor", "achieved": round(ltf, 2), "peak": peak_sus, "unit": "TFLOP/s",
                             "frac": round(ltf / peak_sus, 4), "peak_source": sus_src,
                             "frac_of_burst": round(ltf / peak_tf, 4), "algorithmic_flops_per_launch": wl.flops()}}
            launches += long_steps

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, nrows, secs, threads = oracle_sample_rate(w, args.cpu_seconds)
        cpu = {"value": round(rate / 1e12, 6), "unit": "TFLOPS", "cores": threads, "kind": "oracle",
               "sample": f"{nrows} seeded query rows of {w.name} (fp64 oracle, {secs:.1f} s)",
               "extrapolated_full_step_s": round(flops / rate, 1)}

    if rank == 0:
        line = {
            "metric": "attention TFLOPS (causal GQA prefill, Llama-3-8B shape)" if w.causal else "attention TFLOPS",
            "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "strong" if (args.shard == "heads" and world > 1) else "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
            "config": bench_config(w, world, args.shard),
            "roofline": {"bound": "tensor", "achieved": round(per_gpu_tflops, 2), "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": round(per_gpu_tflops / peak_tf, 4), "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "algorithmic_flops_per_launch": flops,
                         "traffic": traffic(w.name, world == 1 or args.shard == "batch")[0],
                         "traffic_source": traffic(w.name, world == 1 or args.shard == "batch")[1]},
            "e2e": e2e,
            "gpu_launches": args.steps,  # one prefill kernel per timed step of the headline leg
            "gpu_launches_all_legs": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
            "extras": extras,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    q, k, v = make_inputs(w)
    per_step = []
    for _ in range(args.warmup):
        oracle_sample_rate(w, min(2.0, args.cpu_seconds / 4), q, k, v)
    rows_used, threads = 0, 1
    step_secs = []
    for _ in range(args.steps):
        rate, rows_used, secs, threads = oracle_sample_rate(w, args.cpu_seconds / max(1, args.steps), q, k, v)
        per_step.append(rate)
        step_secs.append(secs)
    value = statistics.mean(per_step) / 1e12
    line = {
        "impl": "reference", "metric": "attention TFLOPS (causal GQA prefill, Llama-3-8B shape)",
        "value": round(value, 6), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.mean(step_secs), 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16)",
        "config": bench_config(w, 1, "batch"),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": f"{rows_used} seeded query rows per step of {w.name} (fp64 oracle)",
                         "extrapolated_full_step_s": round(w.flops() / (value * 1e12), 1)},
        "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b_prefill_8k", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU (oracle) baseline")
    ap.add_argument("--no-extras", action="store_true", help="skip the decode measurement")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--no-f16", action="store_true", help="skip the fp16-input measurements")
    ap.add_argument("--no-sparse", action="store_true", help="skip the block-sparse prefill measurement")
    ap.add_argument("--decode-impl", choices=sorted(DECODE_IMPLS), default="auto",
                    help="kernel of the MLA decode leg (auto: the library's choice, queries on M)")
    ap.add_argument("--decode-splits", type=int, default=0,
                    help="split count of the MLA decode leg (0: the library's balanced schedule)")
    ap.add_argument("--shard", choices=["batch", "heads"], default="batch",
                    help="N > 1: each rank runs its own batch (weak scaling) or a head shard of one layer "
                         "(strong scaling, no collective)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
