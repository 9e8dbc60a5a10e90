"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle's tests.

This module holds no attention arithmetic: it only draws N(0, 1) values, adds the optional
'vertical' key bias and rounds once to the workload's 16-bit type (bf16, or fp16 for the
``*_f16`` variants made with ``with_(dtype="f16")``). Everything is generated on the CPU with a seeded
``torch.Generator`` so both sides see the same bits.

Workloads (the shapes of the pages' settings; no dataset or model weights are used):
  * ``tiny_d64``: B=1, H=2, L=128, d=dv=64, causal and non-causal.
  * ``llama8b_prefill_8k``: Llama-3-8B-shaped causal GQA prefill, B=1, Hq=32, Hkv=8, L=8192,
    d=dv=128 (model shape named by the MInference article on 7minutos.es).
  * ``batched_prefill_2k`` / ``batched_prefill_256``: B=16, Hq=32, Hkv=8, L=2048 / 256, causal
    (batch 8-16 and the <256-token regime of the "Flash Attention en Modelos Pequenos" notes).
  * ``mla_decode_64k``: MLA-shaped decode, B=32, 16 query heads on one latent KV head, Lq=2,
    Lk=65536, d=576, dv=512 with V = first 512 columns of the latent row (FlashMLA-ETAP
    summary, "Planteamiento del Problema" and "Limitaciones").
  * ``long_prefill_128k``: B=1, Hq=32, Hkv=8, L=131072, causal, K biased by +2.0 on 64 random
    key positions per KV head (the vertical-column pattern of the MInference article).
  * ``gqa_decode_32k``: GQA decode with a dense V, B=16, Hq=32, Hkv=8, Lq=1, Lk=32768,
    d=dv=128 (the batch 8-16 regime of the "Flash Attention en Modelos Pequenos" notes on the
    Llama-3-8B head shape).
  * ``sparse_prefill_128k``: the 128K vertical-bias prefill with a given block-sparse index
    (``block_lists``): every 128-row query block sees the first key block, a local window of
    16 blocks ending at its diagonal block, and the blocks that hold its kv head's biased
    "vertical" keys (the A-shape and vertical-bar patterns of the MInference article, at block
    granularity). The index is an input here; building one from attention scores is not.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

BASE_SEED = 20261202


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    d: int
    dv: int
    causal: bool
    latent: bool = False          # V is the first dv columns of K (ldv = d)
    vertical_keys: int = 0        # number of biased key positions per KV head
    vertical_bias: float = 0.0
    seed: int = BASE_SEED
    dtype: str = "bf16"           # element type of q, k, v and o: "bf16" or "f16"
    sparse_window: int = 0        # > 0: block-sparse index with a local window of this many blocks

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"bf16": torch.bfloat16, "f16": torch.float16}[self.dtype]

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def ldv(self) -> int:
        return self.d if self.latent else self.dv

    def visible_pairs(self) -> int:
        """Number of (query row, key) pairs that take part, summed over batch and heads."""
        if not self.causal:
            per_head = self.Lq * self.Lk
        else:
            off = self.Lk - self.Lq
            per_head = sum(min(self.Lk, i + off + 1) for i in range(self.Lq))
        return per_head * self.B * self.Hq

    def flops(self) -> float:
        """Algorithmic flops: 2*(d + dv) per visible pair (masked work not counted)."""
        return float(self.visible_pairs()) * 2.0 * (self.d + self.dv)

    def kv_bytes(self) -> int:
        """K/V bytes read once (the latent row is read once and serves as both K and V)."""
        per_row = self.d if self.latent else self.d + self.dv
        return self.B * self.Hkv * self.Lk * per_row * 2

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_d64": Workload("tiny_d64", 1, 2, 2, 128, 128, 64, 64, False, seed=BASE_SEED + 1),
    "tiny_d64_causal": Workload("tiny_d64_causal", 1, 2, 2, 128, 128, 64, 64, True,
                                seed=BASE_SEED + 1),
    "llama8b_prefill_8k": Workload("llama8b_prefill_8k", 1, 32, 8, 8192, 8192, 128, 128, True,
                                   seed=BASE_SEED + 2),
    "batched_prefill_2k": Workload("batched_prefill_2k", 16, 32, 8, 2048, 2048, 128, 128, True,
                                   seed=BASE_SEED + 3),
    "batched_prefill_256": Workload("batched_prefill_256", 16, 32, 8, 256, 256, 128, 128, True,
                                    seed=BASE_SEED + 3),
    "mla_decode_64k": Workload("mla_decode_64k", 32, 16, 1, 2, 65536, 576, 512, True,
                               latent=True, seed=BASE_SEED + 4),
    "long_prefill_128k": Workload("long_prefill_128k", 1, 32, 8, 131072, 131072, 128, 128, True,
                                  vertical_keys=64, vertical_bias=2.0, seed=BASE_SEED + 5),
    "gqa_decode_32k": Workload("gqa_decode_32k", 16, 32, 8, 1, 32768, 128, 128, True,
                               seed=BASE_SEED + 6),
    "sparse_prefill_128k": Workload("sparse_prefill_128k", 1, 32, 8, 131072, 131072, 128, 128, True,
                                    vertical_keys=64, vertical_bias=2.0, seed=BASE_SEED + 5,
                                    sparse_window=16),
}

SPARSE_BLOCK = 128


def block_lists(w: Workload):
    """(idx, cnt) int32 numpy arrays [B, Hq, nqb, max] / [B, Hq, nqb] of the block-sparse index of
    ``w``: for query block qb of head (b, h), the sorted distinct key blocks {0}, the window
    qb - sparse_window + 1 .. qb (shifted by the causal offset), and the blocks holding the
    vertical keys of kv head h // (Hq / Hkv), each kept only when at or below the diagonal."""
    import numpy as np
    nqb = -(-w.Lq // SPARSE_BLOCK)
    nkb = -(-w.Lk // SPARSE_BLOCK)
    off_blocks = (w.Lk - w.Lq) // SPARSE_BLOCK
    pos = vertical_positions(w)
    G = w.Hq // w.Hkv
    lists = {}
    for b in range(w.B):
        for hk in range(w.Hkv):
            vb = np.unique(pos[b * w.Hkv + hk].numpy() // SPARSE_BLOCK) if pos else np.zeros(0, np.int64)
            for qb in range(nqb):
                diag = min(nkb - 1, qb + off_blocks) if w.causal else nkb - 1
                s = {0} | set(range(max(0, diag - w.sparse_window + 1), diag + 1))
                s |= {int(x) for x in vb if x <= diag}
                lists[(b, hk, qb)] = sorted(s)
    max_len = max(len(v) for v in lists.values())
    idx = np.zeros((w.B, w.Hq, nqb, max_len), dtype=np.int32)
    cnt = np.zeros((w.B, w.Hq, nqb), dtype=np.int32)
    for (b, hk, qb), lst in lists.items():
        for h in range(hk * G, (hk + 1) * G):
            idx[b, h, qb, :len(lst)] = lst
            cnt[b, h, qb] = len(lst)
    return idx, cnt


def sparse_visible_pairs(w: Workload, idx, cnt) -> int:
    """(query row, key) pairs inside the listed blocks that the causal mask keeps."""
    import numpy as np
    nqb = idx.shape[2]
    nkb = -(-w.Lk // SPARSE_BLOCK)
    off = w.Lk - w.Lq
    kstart = np.arange(nkb) * SPARSE_BLOCK
    kend = np.minimum(kstart + SPARSE_BLOCK, w.Lk)
    total = 0
    for qb in range(nqb):
        rows = np.arange(qb * SPARSE_BLOCK, min(w.Lq, (qb + 1) * SPARSE_BLOCK))
        if w.causal:
            last = np.minimum(rows[:, None] + off, kend[None, :] - 1)
            per_kb = np.clip(last - kstart[None, :] + 1, 0, None).sum(axis=0)
        else:
            per_kb = (kend - kstart) * rows.size
        for b in range(w.B):
            for h in range(w.Hq):
                total += int(per_kb[idx[b, h, qb, :cnt[b, h, qb]]].sum())
    return total


def _planes(g: torch.Generator, lead: int, rows: int, cols: int, dtype=torch.bfloat16) -> torch.Tensor:
    """lead x rows x cols 16-bit values, drawn plane by plane as fp32 N(0,1), rounded once."""
    out = torch.empty((lead, rows, cols), dtype=dtype)
    for p in range(lead):
        out[p] = torch.randn((rows, cols), generator=g, dtype=torch.float32).to(dtype)
    return out


def make_inputs(w: Workload):
    """(q, k, v) CPU tensors of ``w.torch_dtype`` for workload ``w``; v is k itself for latent
    workloads. The fp16 variant draws the same fp32 values as the bf16 one.

    Draw order: Q planes, K planes, V planes (each (b, h) plane in order), then the biased key
    positions (one ``randperm`` per (b, kv head)). The bias is added to the fp32 draw before the
    single rounding to bf16, so K is regenerated plane by plane when a bias is requested.
    """
    g = torch.Generator().manual_seed(w.seed)
    dt = w.torch_dtype
    q = _planes(g, w.B * w.Hq, w.Lq, w.d, dt).view(w.B, w.Hq, w.Lq, w.d)
    if w.vertical_keys == 0:
        k = _planes(g, w.B * w.Hkv, w.Lk, w.d, dt).view(w.B, w.Hkv, w.Lk, w.d)
        v = k if w.latent else _planes(g, w.B * w.Hkv, w.Lk, w.dv, dt).view(w.B, w.Hkv, w.Lk, w.dv)
        return q, k, v
    # keep the fp32 K draw (one plane at a time) until the positions are known
    kstate = g.get_state()
    for _ in range(w.B * w.Hkv):
        torch.randn((w.Lk, w.d), generator=g, dtype=torch.float32)
    v = None if w.latent else _planes(g, w.B * w.Hkv, w.Lk, w.dv, dt).view(w.B, w.Hkv, w.Lk, w.dv)
    positions = [torch.randperm(w.Lk, generator=g)[: w.vertical_keys]
                 for _ in range(w.B * w.Hkv)]
    g2 = torch.Generator()
    g2.set_state(kstate)
    k = torch.empty((w.B * w.Hkv, w.Lk, w.d), dtype=dt)
    for p in range(w.B * w.Hkv):
        plane = torch.randn((w.Lk, w.d), generator=g2, dtype=torch.float32)
        plane[positions[p]] += w.vertical_bias
        k[p] = plane.to(dt)
    k = k.view(w.B, w.Hkv, w.Lk, w.d)
    return q, k, (k if w.latent else v)


def vertical_positions(w: Workload):
    """The biased key positions of ``w`` (list over (b, kv head)), re-drawn like make_inputs."""
    if w.vertical_keys == 0:
        return []
    g = torch.Generator().manual_seed(w.seed)
    for _ in range(w.B * w.Hq):
        torch.randn((w.Lq, w.d), generator=g, dtype=torch.float32)
    for _ in range(w.B * w.Hkv):
        torch.randn((w.Lk, w.d), generator=g, dtype=torch.float32)
    if not w.latent:
        for _ in range(w.B * w.Hkv):
            torch.randn((w.Lk, w.dv), generator=g, dtype=torch.float32)
    return [torch.randperm(w.Lk, generator=g)[: w.vertical_keys] for _ in range(w.B * w.Hkv)]


def sample_rows(w: Workload, per_head: int, seed: int = 7, always=(0, 1, 127, 128, 255, 256)):
    """Flat row ids (b*Hq + h)*Lq + i: ``per_head`` rows for every (b, h), seeded, always
    including the listed positions and the last row (those below Lq)."""
    g = torch.Generator().manual_seed(w.seed + seed)
    fixed = sorted({i for i in always if i < w.Lq} | {w.Lq - 1})
    rows = []
    for bh in range(w.B * w.Hq):
        n_rand = max(0, min(per_head, w.Lq) - len(fixed))
        pick = torch.randperm(w.Lq, generator=g)[: n_rand + len(fixed)].tolist()
        chosen = list(fixed) + [i for i in pick if i not in fixed][:n_rand]
        rows.extend(bh * w.Lq + i for i in sorted(chosen))
    return torch.tensor(rows, dtype=torch.int64)
