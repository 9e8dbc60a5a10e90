"""Pins for the fp64 oracle: checks against facts fixed by the pages and by mathematics.

Each ``pin_*`` function raises AssertionError when the oracle built with ``mutant`` violates it.
``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutants.py`` runs them on
builds with one planted mistake each and requires every mutant to fail at least one pin.

Sources of the facts:
  * definition S = Q.K^T, P = softmax(S), O = P.V and its transposed form
    ("Resumen Tecnico: FlashMLA-ETAP", section "Mecanismo Central", items 1-2);
  * shared K/V heads (GQA FAQ of "Activar Flash Attention con llama.cpp");
  * closed forms and invariants of softmax (rows sum to one, shift invariance, constant and
    one-hot value rows, log-sum-exp merge of disjoint key sets);
  * a library routine: torch's fp64 CPU scaled_dot_product_attention with an explicit mask,
    for bf16 and for fp16 inputs;
  * library conversions of every 16-bit pattern (numpy float16, torch bfloat16) for the
    oracle's exact widening;
  * a hand-derived worked example in tests/golden/.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rnd_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


def f64(x):
    return x.to(torch.float64)


def bottom_right_mask(Lq, Lk, causal):
    i = torch.arange(Lq).view(-1, 1)
    j = torch.arange(Lk).view(1, -1)
    return (j <= i + (Lk - Lq)) if causal else torch.ones(Lq, Lk, dtype=torch.bool)


SHAPES = [
    # B, Hq, Hkv, Lq, Lk, d, dv, causal
    (1, 2, 2, 5, 5, 8, 8, False),
    (2, 4, 2, 6, 9, 8, 4, True),
    (1, 4, 1, 3, 7, 16, 16, True),
    (2, 2, 1, 7, 7, 4, 6, True),
]


def _args(B, Hq, Hkv, Lq, Lk, d, dv, causal, scale=None):
    return dict(B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d, dv=dv,
                scale=(1.0 / math.sqrt(d)) if scale is None else scale, causal=causal)


def pin_rows_sum_to_one(mutant=0):
    for n, (B, Hq, Hkv, Lq, Lk, d, dv, causal) in enumerate(SHAPES):
        q = rnd_bf16((B, Hq, Lq, d), 10 + n, 2.0)
        k = rnd_bf16((B, Hkv, Lk, d), 20 + n, 2.0)
        mask = bottom_right_mask(Lq, Lk, causal)
        for row in range(B * Hq * Lq):
            p = oracle.softmax_row(q, k, row, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d,
                                   scale=1.0 / math.sqrt(d), causal=causal, mutant=mutant)
            assert abs(p.sum() - 1.0) <= 1e-12, (row, p.sum())
            assert np.all(p >= 0)
            i = row % Lq
            assert np.all(p[~mask[i].numpy()] == 0.0)


def pin_transposed_flow(mutant=0):
    for n, (B, Hq, Hkv, Lq, Lk, d, dv, causal) in enumerate(SHAPES):
        q = rnd_bf16((B, Hq, Lq, d), 30 + n)
        k = rnd_bf16((B, Hkv, Lk, d), 40 + n)
        v = rnd_bf16((B, Hkv, Lk, dv), 50 + n)
        a = _args(B, Hq, Hkv, Lq, Lk, d, dv, causal)
        o, lse = oracle.attn(q, k, v, mutant=mutant, **a)
        for b in range(B):
            for h in range(Hq):
                ot, lt = oracle.attn_transposed_head(q, k, v, b, h, mutant=mutant, **a)
                assert np.max(np.abs(ot - o[b, h])) <= 1e-12
                assert np.max(np.abs(lt - lse[b, h])) <= 1e-12


def pin_constant_v(mutant=0):
    B, Hq, Hkv, Lq, Lk, d, dv = 1, 2, 1, 6, 11, 8, 5
    q = rnd_bf16((B, Hq, Lq, d), 60, 3.0)
    k = rnd_bf16((B, Hkv, Lk, d), 61, 3.0)
    r = rnd_bf16((dv,), 62)
    v = r.view(1, 1, 1, dv).expand(B, Hkv, Lk, dv).contiguous()
    for causal in (False, True):
        o, _ = oracle.attn(q, k, v, mutant=mutant, **_args(B, Hq, Hkv, Lq, Lk, d, dv, causal))
        assert np.max(np.abs(o - f64(r).numpy())) <= 1e-12


def pin_one_hot(mutant=0):
    # scale 1, d 4: the chosen key scores 64, every other key scores 0 (margin 64 >= 50).
    B, Hq, Hkv, Lq, Lk, d, dv = 1, 1, 1, 3, 9, 4, 3
    q = torch.zeros(B, Hq, Lq, d)
    q[..., 0] = 8.0
    k = torch.zeros(B, Hkv, Lk, d)
    jstar = 2
    k[0, 0, jstar, 0] = 8.0
    v = rnd_bf16((B, Hkv, Lk, dv), 63)
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    o, lse = oracle.attn(q, k, v, mutant=mutant, **_args(B, Hq, Hkv, Lq, Lk, d, dv, False, 1.0))
    for i in range(Lq):
        assert np.max(np.abs(o[0, 0, i] - f64(v[0, 0, jstar]).numpy())) <= 1e-12
        # LSE = 64 + ln(1 + 8 e^-64): the second term is below double rounding
        assert abs(lse[0, 0, i] - 64.0) <= 1e-12


def pin_closed_forms(mutant=0):
    # (a) causal with Lq = Lk: row 0 sees key 0 only -> O_0 = v_0, LSE_0 = s_00.
    B, Hq, Hkv, L, d, dv = 1, 2, 1, 6, 8, 4
    q = rnd_bf16((B, Hq, L, d), 70)
    k = rnd_bf16((B, Hkv, L, d), 71)
    v = rnd_bf16((B, Hkv, L, dv), 72)
    sc = 1.0 / math.sqrt(d)
    o, lse = oracle.attn(q, k, v, mutant=mutant, **_args(B, Hq, Hkv, L, L, d, dv, True))
    for h in range(Hq):
        assert np.max(np.abs(o[0, h, 0] - f64(v[0, 0, 0]).numpy())) <= 1e-12
        s00 = sc * float((f64(q[0, h, 0]) * f64(k[0, 0, 0])).sum())
        assert abs(lse[0, h, 0] - s00) <= 1e-12
    # (b) a single key: every row returns v_0.
    k1, v1 = k[:, :, :1].contiguous(), v[:, :, :1].contiguous()
    q1 = q[:, :, :1].contiguous()
    o, _ = oracle.attn(q, k1, v1, mutant=mutant, **_args(B, Hq, Hkv, L, 1, d, dv, False))
    assert np.max(np.abs(o - f64(v1[0, 0, 0]).numpy())) <= 1e-12
    o, _ = oracle.attn(q1, k1, v1, mutant=mutant, **_args(B, Hq, Hkv, 1, 1, d, dv, True))
    assert np.max(np.abs(o - f64(v1[0, 0, 0]).numpy())) <= 1e-12
    # (c) q = 0: uniform scores; O = mean of the visible V rows, LSE = ln(#visible).
    Lq, Lk = 4, 7
    qz = torch.zeros(B, Hq, Lq, d, dtype=torch.bfloat16)
    kz = rnd_bf16((B, Hkv, Lk, d), 73)
    vz = rnd_bf16((B, Hkv, Lk, dv), 74)
    o, lse = oracle.attn(qz, kz, vz, mutant=mutant, **_args(B, Hq, Hkv, Lq, Lk, d, dv, True))
    V = f64(vz[0, 0]).numpy()
    for i in range(Lq):
        nvis = i + (Lk - Lq) + 1
        assert np.max(np.abs(o[0, 0, i] - V[:nvis].mean(axis=0))) <= 1e-12
        assert abs(lse[0, 0, i] - math.log(nvis)) <= 1e-12


def pin_shift_invariance(mutant=0):
    # one extra dimension with q = c/scale and k = 1 adds c to every score of the row.
    B, Hq, Hkv, Lq, Lk, d, dv = 1, 2, 1, 5, 8, 7, 4
    scale = 0.5
    q = rnd_bf16((B, Hq, Lq, d), 80)
    k = rnd_bf16((B, Hkv, Lk, d), 81)
    v = rnd_bf16((B, Hkv, Lk, dv), 82)
    base_o, base_l = oracle.attn(q, k, v, mutant=mutant,
                                 **_args(B, Hq, Hkv, Lq, Lk, d, dv, True, scale))
    for c in (1.0, 1000.0):
        qe = torch.cat([q, torch.full((B, Hq, Lq, 1), c / scale).to(torch.bfloat16)], -1)
        ke = torch.cat([k, torch.ones(B, Hkv, Lk, 1, dtype=torch.bfloat16)], -1)
        assert float(qe[0, 0, 0, -1]) == c / scale  # exactly representable in bf16
        o, l = oracle.attn(qe, ke, v, mutant=mutant,
                           **_args(B, Hq, Hkv, Lq, Lk, d + 1, dv, True, scale))
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(l))
        assert np.max(np.abs(o - base_o)) <= 1e-12
        assert np.max(np.abs((l - base_l) - c)) <= 1e-12 * max(1.0, c)


def pin_gqa_equals_repeated_mha(mutant=0):
    B, Hq, Hkv, Lq, Lk, d, dv = 2, 6, 2, 5, 6, 8, 8
    G = Hq // Hkv
    q = rnd_bf16((B, Hq, Lq, d), 90)
    k = rnd_bf16((B, Hkv, Lk, d), 91)
    v = rnd_bf16((B, Hkv, Lk, dv), 92)
    o, l = oracle.attn(q, k, v, mutant=mutant, **_args(B, Hq, Hkv, Lq, Lk, d, dv, True))
    kr = k.repeat_interleave(G, dim=1).contiguous()
    vr = v.repeat_interleave(G, dim=1).contiguous()
    o2, l2 = oracle.attn(q, kr, vr, mutant=mutant, **_args(B, Hq, Hq, Lq, Lk, d, dv, True))
    assert np.max(np.abs(o - o2)) <= 1e-12 and np.max(np.abs(l - l2)) <= 1e-12


def pin_split_merge(mutant=0):
    B, Hq, Hkv, Lq, Lk, d, dv = 1, 2, 1, 3, 13, 8, 4
    q = rnd_bf16((B, Hq, Lq, d), 100)
    k = rnd_bf16((B, Hkv, Lk, d), 101)
    v = rnd_bf16((B, Hkv, Lk, dv), 102)
    a = _args(B, Hq, Hkv, Lq, Lk, d, dv, True)
    o, l = oracle.attn(q, k, v, mutant=mutant, **a)
    rows = np.arange(B * Hq * Lq)
    for cuts in ([0, 5, 13], [0, 1, 2, 12, 13], [0, 11, 12, 13]):
        parts = [oracle.attn_rows(q, k, v, rows, kv_range=(cuts[s], cuts[s + 1]),
                                  mutant=mutant, **a) for s in range(len(cuts) - 1)]
        op = np.stack([p[0] for p in parts])
        lp = np.stack([p[1] for p in parts])
        om, lm = oracle.combine(op, lp, mutant=mutant)
        assert np.max(np.abs(om - o.reshape(-1, dv))) <= 1e-12
        assert np.max(np.abs(lm - l.reshape(-1))) <= 1e-12
    # the last key is invisible to row 0 (causal, Lq = 3): its one-key range is empty there
    _, lp = oracle.attn_rows(q, k, v, rows, kv_range=(12, 13), mutant=mutant, **a)
    assert lp[0] == -math.inf and np.all(np.isfinite(lp[2::Lq]))


def pin_library_sdpa(mutant=0):
    """torch's fp64 CPU scaled_dot_product_attention with an explicit bottom-right mask."""
    for n, (B, Hq, Hkv, Lq, Lk, d, dv, causal) in enumerate(SHAPES):
        q = rnd_bf16((B, Hq, Lq, d), 110 + n)
        k = rnd_bf16((B, Hkv, Lk, d), 120 + n)
        v = rnd_bf16((B, Hkv, Lk, dv), 130 + n)
        o, lse = oracle.attn(q, k, v, mutant=mutant, **_args(B, Hq, Hkv, Lq, Lk, d, dv, causal))
        G = Hq // Hkv
        kr, vr = f64(k).repeat_interleave(G, 1), f64(v).repeat_interleave(G, 1)
        mask = bottom_right_mask(Lq, Lk, causal)
        ref = torch.nn.functional.scaled_dot_product_attention(
            f64(q), kr, vr, attn_mask=mask, scale=1.0 / math.sqrt(d))
        assert np.max(np.abs(o - ref.numpy())) <= 1e-12
        s = torch.einsum("bhid,bhjd->bhij", f64(q), kr) / math.sqrt(d)
        ref_l = torch.logsumexp(s.masked_fill(~mask, -math.inf), dim=-1)
        assert np.max(np.abs(lse - ref_l.numpy())) <= 1e-12


def pin_latent_kv(mutant=0):
    """V = first dv columns of the latent K row (ldv = d) equals a separate dense V copy."""
    B, Hq, Hkv, Lq, Lk, d, dv = 2, 4, 1, 2, 9, 12, 8
    q = rnd_bf16((B, Hq, Lq, d), 140)
    k = rnd_bf16((B, Hkv, Lk, d), 141)
    a = _args(B, Hq, Hkv, Lq, Lk, d, dv, True)
    o, l = oracle.attn(q, k, k, ldv=d, mutant=mutant, **a)
    vd = k[..., :dv].contiguous()
    o2, l2 = oracle.attn(q, k, vd, mutant=mutant, **a)
    assert np.max(np.abs(o - o2)) <= 1e-12 and np.max(np.abs(l - l2)) <= 1e-12


def pin_golden_worked_example(mutant=0):
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        ex = json.load(f)
    q = torch.tensor(ex["q"], dtype=torch.bfloat16).view(1, 1, ex["Lq"], ex["d"])
    k = torch.tensor(ex["k"], dtype=torch.bfloat16).view(1, 1, ex["Lk"], ex["d"])
    v = torch.tensor(ex["v"], dtype=torch.bfloat16).view(1, 1, ex["Lk"], ex["dv"])
    env = {"e": math.e, "ln": math.log, "__builtins__": {}}
    for case in ex["cases"]:
        o_ref = np.array([[eval(x, env) for x in row] for row in case["o_expr"]])
        lse_ref = np.array([eval(x, env) for x in case["lse_expr"]])
        o, lse = oracle.attn(q, k, v, B=1, Hq=1, Hkv=1, Lq=ex["Lq"], Lk=ex["Lk"], d=ex["d"],
                             dv=ex["dv"], scale=ex["scale"], causal=case["causal"],
                             mutant=mutant)
        assert np.max(np.abs(o[0, 0] - o_ref)) <= 1e-12, case["name"]
        assert np.max(np.abs(lse[0, 0] - lse_ref)) <= 1e-12, case["name"]


def pin_widen_tables(mutant=0):
    """Every one of the 65536 bit patterns widens to the value numpy (fp16) and torch (bf16)
    give it: IEEE binary16 incl. subnormals, infinities and NaN; bf16 likewise."""
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.widen(bits, "f16", mutant=mutant)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    got = oracle.widen(bits, "bf16", mutant=mutant)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_library_sdpa_f16(mutant=0):
    """fp16 inputs (some subnormal values in V) against torch's fp64 scaled_dot_product_attention."""
    for n, (B, Hq, Hkv, Lq, Lk, d, dv, causal) in enumerate(SHAPES):
        g = torch.Generator().manual_seed(150 + n)
        q = torch.randn((B, Hq, Lq, d), generator=g).to(torch.float16)
        k = torch.randn((B, Hkv, Lk, d), generator=g).to(torch.float16)
        v = (torch.randn((B, Hkv, Lk, dv), generator=g) * 1e-5).to(torch.float16)
        assert (v.abs() < 2.0 ** -14).any()  # subnormal fp16 values take part
        o, lse = oracle.attn(q, k, v, mutant=mutant, **_args(B, Hq, Hkv, Lq, Lk, d, dv, causal))
        G = Hq // Hkv
        kr, vr = f64(k).repeat_interleave(G, 1), f64(v).repeat_interleave(G, 1)
        mask = bottom_right_mask(Lq, Lk, causal)
        ref = torch.nn.functional.scaled_dot_product_attention(
            f64(q), kr, vr, attn_mask=mask, scale=1.0 / math.sqrt(d))
        assert np.max(np.abs(o - ref.numpy())) <= 1e-12 * 1e-5
        s = torch.einsum("bhid,bhjd->bhij", f64(q), kr) / math.sqrt(d)
        ref_l = torch.logsumexp(s.masked_fill(~mask, -math.inf), dim=-1)
        assert np.max(np.abs(lse - ref_l.numpy())) <= 1e-12


def random_block_lists(B, Hq, nqb, nkb, seed, p_keep=0.5, max_blk=None):
    """Sorted unique key-block lists per (b, h, query block), some of them empty."""
    g = np.random.default_rng(seed)
    max_blk = nkb if max_blk is None else max_blk
    idx = np.full((B, Hq, nqb, max_blk), -7, dtype=np.int32)  # unused entries hold junk
    cnt = np.zeros((B, Hq, nqb), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            for qb in range(nqb):
                keep = np.flatnonzero(g.random(nkb) < p_keep)[:max_blk]
                if (b + h + qb) % 5 == 3:
                    keep = keep[:0]
                idx[b, h, qb, :keep.size] = keep
                cnt[b, h, qb] = keep.size
    return idx, cnt


def block_mask(idx, cnt, Lq, Lk, blk_q, blk_k, causal):
    """Boolean [B, Hq, Lq, Lk] visibility mask built from block lists (and the causal rule)."""
    B, Hq, nqb, _ = idx.shape
    m = np.zeros((B, Hq, Lq, Lk), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            for qb in range(nqb):
                for kb in idx[b, h, qb, :cnt[b, h, qb]]:
                    m[b, h, qb * blk_q:(qb + 1) * blk_q, kb * blk_k:(kb + 1) * blk_k] = True
    if causal:
        m &= bottom_right_mask(Lq, Lk, True).numpy()[None, None]
    return torch.from_numpy(m)


SPARSE_SHAPES = [
    # B, Hq, Hkv, Lq, Lk, d, blk_q, blk_k, causal
    (1, 2, 1, 11, 13, 8, 4, 3, True),
    (2, 4, 2, 9, 9, 4, 3, 2, False),
    (1, 2, 2, 5, 12, 8, 2, 5, True),
]


def pin_sparse_full_lists_equal_dense(mutant=0):
    """Listing every key block reduces block-sparse attention to the dense definition."""
    for n, (B, Hq, Hkv, Lq, Lk, d, bq, bk, causal) in enumerate(SPARSE_SHAPES):
        q = rnd_bf16((B, Hq, Lq, d), 300 + n)
        k = rnd_bf16((B, Hkv, Lk, d), 310 + n)
        v = rnd_bf16((B, Hkv, Lk, d), 320 + n)
        nqb, nkb = -(-Lq // bq), -(-Lk // bk)
        idx = np.tile(np.arange(nkb, dtype=np.int32), (B, Hq, nqb, 1))
        cnt = np.full((B, Hq, nqb), nkb, dtype=np.int32)
        a = _args(B, Hq, Hkv, Lq, Lk, d, d, causal)
        o, l = oracle.attn(q, k, v, blocks=(idx, cnt, bq, bk), mutant=mutant, **a)
        o2, l2 = oracle.attn(q, k, v, mutant=mutant, **a)
        assert np.array_equal(o, o2) and np.array_equal(l, l2)


def pin_sparse_library_sdpa(mutant=0):
    """Random block lists against torch's fp64 SDPA with the explicit block mask; rows that see
    no key are O = 0, LSE = -inf."""
    for n, (B, Hq, Hkv, Lq, Lk, d, bq, bk, causal) in enumerate(SPARSE_SHAPES):
        q = rnd_bf16((B, Hq, Lq, d), 330 + n)
        k = rnd_bf16((B, Hkv, Lk, d), 340 + n)
        v = rnd_bf16((B, Hkv, Lk, d), 350 + n)
        nqb, nkb = -(-Lq // bq), -(-Lk // bk)
        idx, cnt = random_block_lists(B, Hq, nqb, nkb, 360 + n)
        o, lse = oracle.attn(q, k, v, blocks=(idx, cnt, bq, bk), mutant=mutant,
                             **_args(B, Hq, Hkv, Lq, Lk, d, d, causal))
        mask = block_mask(idx, cnt, Lq, Lk, bq, bk, causal)
        G = Hq // Hkv
        kr, vr = f64(k).repeat_interleave(G, 1), f64(v).repeat_interleave(G, 1)
        s = torch.einsum("bhid,bhjd->bhij", f64(q), kr) / math.sqrt(d)
        s = s.masked_fill(~mask, -math.inf)
        seen = mask.any(-1).numpy()
        assert (~seen).any() and seen.any()
        ref_l = torch.logsumexp(s, dim=-1).numpy()
        ref_o = torch.einsum("bhij,bhjd->bhid", torch.softmax(s, -1).nan_to_num(0.0), vr).numpy()
        assert np.max(np.abs(o[seen] - ref_o[seen])) <= 1e-12
        assert np.max(np.abs(lse[seen] - ref_l[seen])) <= 1e-12
        assert np.all(o[~seen] == 0.0) and np.all(lse[~seen] == -math.inf)


def pin_sparse_equals_merged_block_partials(mutant=0):
    """Block-sparse O/LSE equal the log-sum-exp merge of the per-block split partials of the
    listed blocks (each partial from the contiguous key range of one block)."""
    B, Hq, Hkv, Lq, Lk, d, bq, bk, causal = 1, 2, 1, 8, 14, 8, 4, 4, True
    q = rnd_bf16((B, Hq, Lq, d), 370)
    k = rnd_bf16((B, Hkv, Lk, d), 371)
    v = rnd_bf16((B, Hkv, Lk, d), 372)
    nqb, nkb = -(-Lq // bq), -(-Lk // bk)
    idx = np.full((B, Hq, nqb, 3), 0, dtype=np.int32)
    idx[..., :] = [0, 2, 3]
    cnt = np.full((B, Hq, nqb), 3, dtype=np.int32)
    a = _args(B, Hq, Hkv, Lq, Lk, d, d, causal)
    rows = np.arange(B * Hq * Lq)
    o, l = oracle.attn_rows(q, k, v, rows, blocks=(idx, cnt, bq, bk), mutant=mutant, **a)
    parts = [oracle.attn_rows(q, k, v, rows, kv_range=(kb * bk, min(Lk, kb * bk + bk)), mutant=mutant, **a)
             for kb in (0, 2, 3)]
    om, lm = oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]), mutant=mutant)
    fin = np.isfinite(l)
    assert np.array_equal(fin, np.isfinite(lm))
    assert np.max(np.abs(o - om)) <= 1e-12 and np.max(np.abs(l[fin] - lm[fin])) <= 1e-12


ALL_PINS = [pin_rows_sum_to_one, pin_transposed_flow, pin_constant_v, pin_one_hot,
            pin_closed_forms, pin_shift_invariance, pin_gqa_equals_repeated_mha,
            pin_split_merge, pin_library_sdpa, pin_latent_kv, pin_golden_worked_example,
            pin_widen_tables, pin_library_sdpa_f16, pin_sparse_full_lists_equal_dense,
            pin_sparse_library_sdpa, pin_sparse_equals_merged_block_partials]
