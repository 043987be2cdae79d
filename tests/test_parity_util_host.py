"""Host test of the GPU/oracle comparison (tests/parity_util.py), no GPU:
the "kernel result" handed to compare() is built from the oracle itself, with
planted differences, to check that compare() accepts exactly what the method
statement's tolerances allow -- a decision taken the other way inside the band
-- and rejects a decision outside it and a wrong output."""
import math

import numpy as np
import pytest
import torch

from oracle import run_items
from parity_util import compare
from softmax_ssa_fwd_b200.inputs import MODE_SKIP

D = 16


def _inputs():
    # two query rows, three one-key tiles (see the margin pins): key 0 sets the
    # running max, key 1 sits at ratio exp(-4) for row 0, key 2 is negligible
    q = torch.zeros(1, 2, 1, D)
    q[0, 0, 0, 0] = 1.0
    q[0, 1, 0, 1] = 1.0
    k = torch.zeros(1, 3, 1, D)
    k[0, 1, 0, 0], k[0, 1, 0, 1] = -4.0, -6.0
    k[0, 2, 0, 0], k[0, 2, 0, 1] = -40.0, -40.0
    v = torch.zeros(1, 3, 1, D)
    v[0, 0, 0, :] = 1.0
    v[0, 1, 0, :] = -3.0
    v[0, 2, 0, :] = 2.0
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def _as_gpu(res, flip_to=None):
    """Shape an oracle result like the kernel's outputs (CPU tensors)."""
    out = torch.from_numpy(res.out[0, :2][None, :, None, :]).to(torch.bfloat16)
    lse = torch.from_numpy(res.lse[0, :2][None, None, :]).float()
    cnt = torch.tensor([[[int(res.skip_count[0])]]], dtype=torch.int32)
    sb = torch.from_numpy(res.skip_bits[0].view(np.int32).copy()).view(1, 1, 1, -1)
    return out, lse, cnt, sb, None


KW = dict(causal=False, scale=1.0, mode=MODE_SKIP, Br=2, Bc=1)


def test_identical_results_pass():
    q, k, v = _inputs()
    lam = math.exp(-4.0) / (1 + 0.5e-3)
    res = run_items(q, k, v, lam=lam, **KW)
    rep = compare(q, k, v, [(0, 0, 0)], lam=lam, gpu=_as_gpu(res), **KW)
    assert rep.marginal_mismatch == 0 and rep.marginal_tiles == 1


def test_other_decision_inside_the_band_is_settled_and_compared():
    q, k, v = _inputs()
    lam = math.exp(-4.0) / (1 + 0.5e-3)          # oracle keeps tile 1 (ratio just above lambda)
    other = run_items(q, k, v, lam=lam, flip_bits=np.array([[0b010]], np.uint32), **KW)
    rep = compare(q, k, v, [(0, 0, 0)], lam=lam, gpu=_as_gpu(other), **KW)
    assert rep.marginal_mismatch == 1 and rep.skipped_gpu == 2


def test_other_decision_with_a_wrong_output_fails():
    q, k, v = _inputs()
    lam = math.exp(-4.0) / (1 + 0.5e-3)
    other = run_items(q, k, v, lam=lam, flip_bits=np.array([[0b010]], np.uint32), **KW)
    out, lse, cnt, sb, kb = _as_gpu(other)
    out = out + 0.05
    with pytest.raises(AssertionError):
        compare(q, k, v, [(0, 0, 0)], lam=lam, gpu=(out, lse, cnt, sb, kb), **KW)


def test_other_decision_outside_the_band_fails():
    q, k, v = _inputs()
    lam = math.exp(-4.0) / (1 + 2e-3)             # kept, 2e-3 above: outside the band
    res = run_items(q, k, v, lam=lam, **KW)
    out, lse, cnt, sb, kb = _as_gpu(res)
    sb = sb ^ 0b010                               # the kernel "skipped" tile 1
    cnt = cnt + 1
    with pytest.raises(AssertionError, match="outside the tolerance band"):
        compare(q, k, v, [(0, 0, 0)], lam=lam, gpu=(out, lse, cnt, sb, kb), **KW)


def test_wrong_count_fails():
    q, k, v = _inputs()
    lam = 1e-3
    res = run_items(q, k, v, lam=lam, **KW)
    out, lse, cnt, sb, kb = _as_gpu(res)
    with pytest.raises(AssertionError):
        compare(q, k, v, [(0, 0, 0)], lam=lam, gpu=(out, lse, cnt + 1, sb, kb), **KW)
