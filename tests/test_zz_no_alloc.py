"""attn_decode_noalloc: the decode entry point for callers that cannot allocate device memory.

Some callers (code running while another part of the process captures a CUDA graph, serving
processes with a fixed memory pool, plugins that only receive input and output pointers) cannot
allocate or pass a workspace. attn_decode_noalloc keeps the split partials in a scratch array that
is part of the library instead. These tests call it through the C ABI and compare its output with
attn_decode (caller workspace) on two calls in a row, with partials of another layout left in the
scratch before each, check calls of different shapes one after another, and check the size limit
and that invalid arguments are reported as they are by attn_decode. This file is
collected last on purpose.
"""
import ctypes

import pytest
import torch

from exact_attention_139_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20
O_MAX_ABS, O_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3


def _noalloc(lib, q, k, v, o, lse, w, splits=0, **override):
    """attn_decode_noalloc through the C ABI; keyword arguments override the workload's sizes."""
    f = lib.attn_decode_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 8 + [ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                                                ctypes.c_void_p]
    a = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, Lq=w.Lq, Lk=w.Lk, d=w.d, dv=w.dv, ldv=w.ldv)
    a.update(override)
    return f(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), a["B"], a["Hq"], a["Hkv"],
             a["Lq"], a["Lk"], a["d"], a["dv"], a["ldv"], w.scale, int(w.causal), splits,
             torch.cuda.current_stream().cuda_stream)


def _close(a, b, la, lb):
    a, b = a.float(), b.float()
    assert (a - b).abs().max().item() <= O_MAX_ABS
    assert ((a - b).norm() / b.norm()).item() <= O_REL_L2
    assert (la - lb).abs().max().item() <= LSE_MAX_ABS


MLA = Workload("noalloc_mla", 2, 16, 1, 2, 3000, 576, 512, True, latent=True, seed=301)
GQA = Workload("noalloc_gqa", 3, 8, 2, 1, 1500, 128, 128, True, seed=302)


def _device_inputs(w, dev):
    q, k, v = make_inputs(w)
    qd, kd = q.to(dev), k.to(dev)
    return qd, kd, (kd if w.latent else v.to(dev))


@pytest.mark.parametrize("w", [MLA, GQA], ids=lambda w: w.name)
def test_matches_workspace_entry_point_twice(w, cuda_device):
    from exact_attention_139_b200 import attn
    qd, kd, vd = _device_inputs(w, cuda_device)
    o_ref, l_ref = attn.attn_decode(qd, kd, vd, causal=w.causal, scale=w.scale, dv=w.dv)
    assert attn.attn_check_device() == attn.ATTN_OK
    lib = attn.lib()
    for _ in range(2):
        # leave partials of another layout in the scratch first (16 equal splits), so that a read
        # of bytes the next call did not write would show up in its result
        o = torch.empty_like(o_ref)
        lse = torch.empty_like(l_ref)
        assert _noalloc(lib, qd, kd, vd, o, lse, w, splits=16) == attn.ATTN_OK
        assert attn.attn_check_device() == attn.ATTN_OK
        _close(o, o_ref, lse, l_ref)
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(l_ref, float("nan"))
        assert _noalloc(lib, qd, kd, vd, o, lse, w) == attn.ATTN_OK
        assert attn.attn_check_device() == attn.ATTN_OK
        _close(o, o_ref, lse, l_ref)


def test_alternating_shapes_share_the_scratch(cuda_device):
    """Calls of different shapes and split plans one after the other on the shared scratch."""
    from exact_attention_139_b200 import attn
    lib = attn.lib()
    refs = {}
    for w in (MLA, GQA):
        qd, kd, vd = _device_inputs(w, cuda_device)
        refs[w.name] = (qd, kd, vd) + attn.attn_decode(qd, kd, vd, causal=w.causal, scale=w.scale, dv=w.dv)
    for w, splits in ((MLA, 0), (GQA, 16), (MLA, 5), (GQA, 0), (MLA, 0)):
        qd, kd, vd, o_ref, l_ref = refs[w.name]
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(l_ref, float("nan"))
        assert _noalloc(lib, qd, kd, vd, o, lse, w, splits=splits) == attn.ATTN_OK
        assert attn.attn_check_device() == attn.ATTN_OK
        _close(o, o_ref, lse, l_ref)


def test_rejects_shapes_beyond_the_scratch(cuda_device):
    from exact_attention_139_b200 import attn
    w = Workload("noalloc_big", 32, 16, 1, 2, 65536, 576, 512, True, latent=True)
    splits = 256  # 256 splits x 1024 rows x 512 x 4 B of partials is far beyond the scratch
    assert attn.attn_decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.dv, splits) > SCRATCH_BYTES
    q = torch.zeros((w.B, w.Hq, w.Lq, w.d), dtype=torch.bfloat16, device=cuda_device)
    k = torch.zeros((1, 1, 64, w.d), dtype=torch.bfloat16, device=cuda_device)  # never read
    o = torch.empty((w.B, w.Hq, w.Lq, w.dv), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=cuda_device)
    assert _noalloc(attn.lib(), q, k, k, o, lse, w, splits=splits) == attn.ATTN_ERR_WORKSPACE


def test_invalid_arguments_reported_before_the_size_check(cuda_device):
    """An invalid call gets attn_decode's error code even when its partials would not fit."""
    from exact_attention_139_b200 import attn
    w = Workload("noalloc_bad", 32, 16, 1, 2, 65536, 576, 512, True, latent=True)
    q = torch.zeros((w.B, w.Hq, w.Lq, w.d), dtype=torch.bfloat16, device=cuda_device)
    k = torch.zeros((1, 1, 64, w.d), dtype=torch.bfloat16, device=cuda_device)  # never read
    o = torch.empty((w.B, w.Hq, w.Lq, w.dv), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=cuda_device)
    lib = attn.lib()
    # each of these would also need more partials than the scratch holds (256 splits)
    assert _noalloc(lib, q, k, k, o, lse, w, splits=256, dv=516) == attn.ATTN_ERR_MISALIGNED
    assert _noalloc(lib, q, k, k, o, lse, w, splits=256, ldv=256) == attn.ATTN_ERR_INVALID_ARG
    assert _noalloc(lib, q, k, k, o, lse, w, splits=256, Hq=15, Hkv=2) == attn.ATTN_ERR_INVALID_ARG
    assert _noalloc(lib, q, k, k, o, lse, w, splits=257) == attn.ATTN_ERR_INVALID_ARG
