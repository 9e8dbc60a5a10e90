"""The bounded-wait error path on the GPU: a wait on a barrier nothing arrives on runs out,
the status reaches the host, and the context stays usable."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_wait_timeout_reported_and_context_usable(cuda_device):
    from exact_attention_139_b200 import attn
    from exact_attention_139_b200.inputs import Workload, make_inputs
    assert attn.attn_check_device() == attn.ATTN_OK
    attn.attn_selftest_wait_timeout(20000)  # 20 ms
    assert attn.attn_check_device() == attn.ATTN_ERR_TIMEOUT
    assert attn.attn_check_device() == attn.ATTN_OK  # cleared
    w = Workload("after", 1, 2, 1, 130, 130, 64, 64, True, seed=5)
    q, k, v = (t.to(cuda_device) for t in make_inputs(w))
    o, _ = attn.attn_fwd(q, k, v, causal=True)
    assert attn.attn_check_device() == attn.ATTN_OK
    assert torch.isfinite(o.float()).all()
