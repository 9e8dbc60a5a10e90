"""The FMA-pipe exp2 of the prefill softmax: its coefficients come from the committed Remez fit
and meet the stated error bound (CPU); the device function matches CUDA's exp2f (GPU)."""
import os
import re

import numpy as np
import pytest

from tests import exp2_poly_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def kernel_coefficients():
    text = open(os.path.join(ROOT, "exact_attention_139_b200", "csrc", "sm100.cuh")).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1)) for i in range(4)]


def test_coefficients_match_the_fit():
    fit = exp2_poly_fit.fp32_coefficients()
    assert np.allclose(kernel_coefficients(), fit, rtol=0, atol=1e-9)


def test_fp32_error_bound():
    assert exp2_poly_fit.max_rel_error(kernel_coefficients()) < 1e-4


def test_range_reduction_on_cpu():
    """The full recipe (shifter rounding, polynomial, exponent add) in fp32 numpy."""
    c = np.float32(kernel_coefficients())
    x = np.concatenate([np.linspace(-125, 64, 200001), [-0.5, 0.5, 0.0, -1e-7, 63.49]]).astype(np.float32)
    sh = np.float32(12582912.0)
    t = (x + sh).astype(np.float32)
    n = (t - sh).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = exp2_poly_fit.horner_fp32(c, f)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    y = bits.view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.abs(f) <= 0.5)
    assert np.max(np.abs(y / ref - 1)) < 1e-4
    # below the range the results are subnormal or clamped: only their smallness matters
    xs = np.float32([-125.5, -126.0, -200.0, -np.inf])
    xc = np.maximum(xs, np.float32(-126.0))
    ts = (xc + sh).astype(np.float32)
    ps = exp2_poly_fit.horner_fp32(c, (xc - (ts - sh)).astype(np.float32))
    ys = (ps.view(np.uint32) + (ts.view(np.uint32) << np.uint32(23))).astype(np.uint32).view(np.float32)
    assert np.all((ys >= 0) & (ys < 2.0 ** -124))


@pytest.mark.gpu
def test_device_matches_cuda_exp2(cuda_device):
    import torch
    from exact_attention_139_b200 import attn
    x = torch.cat([torch.linspace(-125, 64, 1 << 20), torch.tensor([-300.0, -127.5, 0.0, 1.0, 7.99])]).to(cuda_device)
    y = torch.empty_like(x)
    lib = attn.lib()
    import ctypes
    lib.attn_selftest_exp2.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.attn_selftest_exp2.restype = ctypes.c_int
    assert lib.attn_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(),
                                  torch.cuda.current_stream().cuda_stream) == 0
    ref = torch.exp2(x)  # CUDA's exp2f
    inside = torch.cat([torch.arange(1 << 20), torch.tensor([(1 << 20) + 2, (1 << 20) + 3, (1 << 20) + 4])]).to(cuda_device)
    rel = ((y[inside].double() / ref[inside].double()) - 1).abs().max().item()
    assert rel < 1e-4
    below = y[(1 << 20):(1 << 20) + 2]  # x = -300 and -127.5: below the range the result is 0
    assert (below == 0).all()
    lo = torch.tensor([-float("inf"), -126.5, -1000.0], device=cuda_device)
    ylo = torch.empty_like(lo)
    assert lib.attn_selftest_exp2(lo.data_ptr(), ylo.data_ptr(), 3, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert (ylo == 0).all()  # masked scores (-inf) give exactly zero weight
