"""attn_decode_noalloc: the decode entry point for callers that cannot allocate device memory.

Some callers (code running while another part of the process captures a CUDA graph, serving
processes with a fixed memory pool, plugins that only receive input and output pointers) cannot
allocate or pass a workspace. attn_decode_noalloc keeps the split partials in a scratch array that
is part of the library instead. These tests call it through the C ABI and compare its output with
attn_decode (caller workspace) on two calls in a row, and check the size limit. This file is
collected last on purpose.
"""
import ctypes

import pytest
import torch

from exact_attention_139_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20
O_MAX_ABS, O_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3


def _noalloc(lib, q, k, v, o, lse, w, splits=0):
    f = lib.attn_decode_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 8 + [ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                                                ctypes.c_void_p]
    return f(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.Hq, w.Hkv, w.Lq, w.Lk,
             w.d, w.dv, w.ldv, w.scale, int(w.causal), splits, torch.cuda.current_stream().cuda_stream)


def _close(a, b, la, lb):
    a, b = a.float(), b.float()
    assert (a - b).abs().max().item() <= O_MAX_ABS
    assert ((a - b).norm() / b.norm()).item() <= O_REL_L2
    assert (la - lb).abs().max().item() <= LSE_MAX_ABS


@pytest.mark.parametrize("w", [
    Workload("noalloc_mla", 2, 16, 1, 2, 3000, 576, 512, True, latent=True, seed=301),
    Workload("noalloc_gqa", 3, 8, 2, 1, 1500, 128, 128, True, seed=302),
], ids=lambda w: w.name)
def test_matches_workspace_entry_point_twice(w, cuda_device):
    from exact_attention_139_b200 import attn
    q, k, v = make_inputs(w)
    qd, kd = q.to(cuda_device), k.to(cuda_device)
    vd = kd if w.latent else v.to(cuda_device)
    o_ref, l_ref = attn.attn_decode(qd, kd, vd, causal=w.causal, scale=w.scale, dv=w.dv)
    assert attn.attn_check_device() == attn.ATTN_OK
    lib = attn.lib()
    for _ in range(2):  # the scratch keeps the previous call's contents: results must not depend on it
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(l_ref, float("nan"))
        assert _noalloc(lib, qd, kd, vd, o, lse, w) == attn.ATTN_OK
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
