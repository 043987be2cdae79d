"""Pins for the split-KV decode oracle (oracle/decode.py), each against
something other than itself:
  * one split is the prefill rule for a single query tile: it must agree with
    the independent C oracle (oracle/ssa_oracle.c), lambda > 1 included;
  * with lambda = 0 nothing is skipped and splitting is exact: any number of
    splits gives dense softmax attention (numpy brute force);
  * for lambda <= 1 each split's decisions have the closed form "skip key tile
    kt iff every row's tile max lies ln(1/lambda) below the max of the split's
    earlier tiles", computed here on the dense score matrix;
  * skip counts are monotone in lambda (lambda <= 1).
"""
import math

import numpy as np
import pytest
import torch

from oracle import run_items
from oracle.decode import decode
from softmax_ssa_fwd_b200.inputs import MODE_SKIP


def _gen(B, Hq, Hkv, Lq, Lk, d, seed, sink_coef=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, Hq, d, generator=g)
    k = torch.randn(B, Lk, Hkv, d, generator=g)
    v = torch.randn(B, Lk, Hkv, d, generator=g)
    if sink_coef:
        u = torch.randn(d, generator=g)
        u /= u.norm()
        q += sink_coef * u
        k[:, :4] += sink_coef * u
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def _scores(q, k, causal, scale):
    qn, kn = q.double().numpy(), k.double().numpy()
    B, Lq, Hq, d = qn.shape
    Lk, Hkv = kn.shape[1], kn.shape[2]
    scale = float(np.float32(scale))
    s = np.zeros((B, Hq, Lq, Lk))
    for b in range(B):
        for h in range(Hq):
            s[b, h] = scale * qn[b, :, h] @ kn[b, :, h // (Hq // Hkv)].T
    if causal:
        vis = np.arange(Lk)[None, :] <= (np.arange(Lq) + Lk - Lq)[:, None]
        s = np.where(vis[None, None], s, -np.inf)
    return s


@pytest.mark.parametrize("Lq,causal,lam", [(1, True, 0.0), (1, True, 1e-3), (3, True, 1e-2),
                                           (3, False, 1e-2), (4, True, 2.0), (1, False, 5e-2)])
def test_one_split_equals_the_prefill_oracle(Lq, causal, lam):
    q, k, v = _gen(2, 4, 2, Lq, 700, 32, seed=11 + Lq, sink_coef=9.0)
    scale = 32 ** -0.5
    dec = decode(q, k, v, causal=causal, scale=scale, lam=lam, Bc=64, num_splits=1)
    ref = run_items(q, k, v, causal=causal, scale=scale, mode=MODE_SKIP, lam=lam, Br=64, Bc=64)
    for it, (b, h, t) in enumerate(ref.items):
        assert t == 0
        np.testing.assert_allclose(dec.out[b, :, h], ref.out[it, :Lq], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dec.lse[b, h], ref.lse[it, :Lq], rtol=1e-12, atol=1e-12)
        assert dec.skip_count[b, h] == ref.skip_count[it]
    if lam >= 1e-2:
        assert dec.skip_count.sum() > 0  # the case exercises the skip


@pytest.mark.parametrize("splits", [1, 2, 5, 40])
@pytest.mark.parametrize("causal", [True, False])
def test_lambda0_any_split_count_is_dense_attention(splits, causal):
    q, k, v = _gen(1, 4, 1, 2, 333, 16, seed=5, sink_coef=6.0)
    scale = 0.3
    dec = decode(q, k, v, causal=causal, scale=scale, lam=0.0, Bc=32, num_splits=splits)
    s = _scores(q, k, causal, scale)
    vn = v.double().numpy()
    mx = s.max(axis=-1, keepdims=True)
    p = np.exp(s - mx)
    l = p.sum(axis=-1, keepdims=True)
    for h in range(4):
        o = (p[0, h] @ vn[0, :, 0]) / l[0, h]
        np.testing.assert_allclose(dec.out[0, :, h], o, rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(dec.lse[0, h], (mx + np.log(l))[0, h, :, 0], rtol=1e-12)
    assert dec.skip_count.sum() == 0


@pytest.mark.parametrize("lam", [1e-4, 1e-2, 0.3])
@pytest.mark.parametrize("splits", [1, 3, 7])
def test_skips_follow_the_per_split_closed_form(lam, splits):
    Bc = 32
    q, k, v = _gen(1, 4, 2, 2, 600, 16, seed=21, sink_coef=8.0)
    dec = decode(q, k, v, causal=True, scale=0.25, lam=lam, Bc=Bc, num_splits=splits)
    s = _scores(q, k, True, 0.25)
    nK = -(-600 // Bc)
    T = -(-nK // splits)
    for h in range(4):
        for sp in range(splits):
            prev = np.full(2, -np.inf)
            for kt in range(sp * T, min(nK, (sp + 1) * T)):
                mt = s[0, h, :, kt * Bc:(kt + 1) * Bc].max(axis=1)
                rows = []
                for i in range(2):
                    if mt[i] == -np.inf:
                        rows.append(True)
                    elif prev[i] == -np.inf:
                        rows.append(False)
                    else:
                        rows.append(mt[i] < prev[i] + math.log(lam))
                assert dec.skip_bits[0, h, kt] == all(rows), (h, sp, kt)
                prev = np.maximum(prev, mt)
    assert dec.skip_count.sum() == dec.skip_bits.sum()


def test_skip_count_is_monotone_in_lambda():
    q, k, v = _gen(1, 4, 4, 1, 900, 16, seed=3, sink_coef=10.0)
    counts = [decode(q, k, v, causal=True, scale=0.25, lam=lam, Bc=64, num_splits=3).skip_count.sum()
              for lam in (0.0, 1e-6, 1e-4, 1e-2, 0.5, 1.0)]
    assert counts == sorted(counts) and counts[-1] > 0
