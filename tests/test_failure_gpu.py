"""Failure detection on the GPU without a fault: every wait inside the kernel
is bounded.  Shortening the limit makes the waits give up; the kernel must
report SSA_ERR_TIMEOUT through the status word, unwind cleanly, and leave the
context usable -- the next call with the default limit gives the same result
as before."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs():
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 1024, 4, 128, generator=g)
    k = torch.randn(1, 1024, 2, 128, generator=g)
    v = torch.randn(1, 1024, 2, 128, generator=g)
    return [t.bfloat16().cuda() for t in (q, k, v)]


def test_short_wait_limit_reports_timeout_and_context_survives():
    from softmax_ssa_fwd_b200 import ssa
    q, k, v = _inputs()
    ref = ssa.attention(q, k, v, causal=True, mode=ssa.MODE_SKIP, lam=1e-3)
    assert ssa.ssa_device_status() == ssa.SSA_OK
    try:
        ssa.ssa_set_wait_timeout_ns(1)  # every pipeline wait gives up almost at once
        ssa.attention(q, k, v, causal=True, mode=ssa.MODE_SKIP, lam=1e-3)
        assert ssa.ssa_device_status() == ssa.SSA_ERR_TIMEOUT
    finally:
        ssa.ssa_set_wait_timeout_ns(0)
    assert ssa.ssa_device_status() == ssa.SSA_OK  # the word was cleared
    again = ssa.attention(q, k, v, causal=True, mode=ssa.MODE_SKIP, lam=1e-3)
    assert ssa.ssa_device_status() == ssa.SSA_OK
    torch.cuda.synchronize()
    assert torch.equal(again[0], ref[0]) and torch.equal(again[1], ref[1])
    assert torch.equal(again[2], ref[2])
