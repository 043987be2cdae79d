"""Pins for the block-selection oracle (oracle/blockmask.py), each against
something other than itself:
  * a mask selecting every block is plain skip-softmax: it must agree with the
    independent C oracle (lambda > 1 included);
  * with lambda = 0 the result is dense softmax attention over the keys of the
    selected, visible blocks (numpy brute force), and the visited count is the
    number of such blocks;
  * padding bits past the last key block are ignored; an empty selection gives
    zero output and lse = -inf.
"""
import numpy as np
import pytest
import torch

from oracle import run_items
from oracle.blockmask import run as mask_run
from softmax_ssa_fwd_b200.inputs import MODE_SKIP


def _gen(B, Hq, Hkv, L, d, seed, sink_coef=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, d, generator=g)
    k = torch.randn(B, L, Hkv, d, generator=g)
    v = torch.randn(B, L, Hkv, d, generator=g)
    if sink_coef:
        u = torch.randn(d, generator=g)
        u /= u.norm()
        q += sink_coef * u
        k[:, :4] += sink_coef * u
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def _mask(B, Hkv, nQ, nK, density, seed, pad_ones=False):
    rng = np.random.default_rng(seed)
    nKw = -(-nK // 32)
    bits = rng.random((B, Hkv, nQ, nKw * 32)) < density
    if not pad_ones:
        bits[..., nK:] = False
    words = np.zeros((B, Hkv, nQ, nKw), dtype=np.uint32)
    for w in range(nKw):
        for i in range(32):
            words[..., w] |= bits[..., 32 * w + i].astype(np.uint32) << np.uint32(i)
    return words, bits[..., :nK]


@pytest.mark.parametrize("causal,lam,Br,Bc", [(True, 1e-3, 64, 64), (True, 1e-2, 128, 64),
                                              (False, 1e-2, 64, 128), (True, 3.0, 64, 64),
                                              (True, 0.0, 128, 128)])
def test_full_mask_equals_the_c_oracle(causal, lam, Br, Bc):
    q, k, v = _gen(1, 4, 2, 300, 32, seed=3, sink_coef=9.0)
    nQ, nK = -(-300 // Br), -(-300 // Bc)
    words, _ = _mask(1, 2, nQ, nK, 1.0, 0)
    out, lse, sk, vis = mask_run(q, k, v, words, causal=causal, scale=0.2, lam=lam, Br=Br, Bc=Bc)
    ref = run_items(q, k, v, causal=causal, scale=0.2, mode=MODE_SKIP, lam=lam, Br=Br, Bc=Bc)
    for it, (b, h, t) in enumerate(ref.items):
        r0, r1 = t * Br, min(300, t * Br + Br)
        np.testing.assert_allclose(out[b, r0:r1, h], ref.out[it, : r1 - r0], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[b, h, r0:r1], ref.lse[it, : r1 - r0], rtol=1e-12, atol=1e-12)
        assert sk[b, h, t] == ref.skip_count[it]
        assert vis[b, h, t] == ref.visited[it]


@pytest.mark.parametrize("causal", [True, False])
def test_lambda0_is_dense_attention_over_selected_blocks(causal):
    B, Hq, Hkv, L, d, Br, Bc = 2, 4, 2, 200, 16, 64, 32
    q, k, v = _gen(B, Hq, Hkv, L, d, seed=8, sink_coef=4.0)
    nQ, nK = -(-L // Br), -(-L // Bc)
    words, bits = _mask(B, Hkv, nQ, nK, 0.5, 1)
    bits[:, :, :, 0] = True  # every query block sees at least its first key block
    for w in range(words.shape[-1]):
        words[..., w] = 0
        for i in range(32):
            if 32 * w + i < nK:
                words[..., w] |= bits[..., 32 * w + i].astype(np.uint32) << np.uint32(i)
    out, lse, sk, vis = mask_run(q, k, v, words, causal=causal, scale=0.3, lam=0.0, Br=Br, Bc=Bc)
    qn, kn, vn = (t.double().numpy() for t in (q, k, v))
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            s = float(np.float32(0.3)) * qn[b, :, h] @ kn[b, :, kv].T  # the scale the kernel receives
            keep = np.repeat(np.repeat(bits[b, kv], Br, axis=0)[:L], Bc, axis=1)[:, :L]
            if causal:
                keep &= np.arange(L)[None, :] <= np.arange(L)[:, None]
            s = np.where(keep, s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            p = np.where(keep, np.exp(s - mx), 0.0)
            np.testing.assert_allclose(out[b, :, h], (p @ vn[b, :, kv]) / p.sum(1, keepdims=True),
                                       rtol=1e-10, atol=1e-12)
            for t in range(nQ):
                last = min(nK - 1, (min(L, t * Br + Br) - 1) // Bc) if causal else nK - 1
                assert vis[b, h, t] == bits[b, kv, t, : last + 1].sum()
    assert sk.sum() == 0


def test_padding_bits_ignored_and_empty_selection():
    q, k, v = _gen(1, 2, 1, 150, 16, seed=4)
    nQ, nK = 3, 3  # Br = Bc = 64
    words, _ = _mask(1, 1, nQ, nK, 0.7, 2)
    padded = words | np.uint32(0xFFFFFFF8)  # bits 3..31 lie past the last key block
    a = mask_run(q, k, v, words, causal=True, scale=0.25, lam=1e-3, Br=64, Bc=64)
    b = mask_run(q, k, v, padded, causal=True, scale=0.25, lam=1e-3, Br=64, Bc=64)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    empty = np.zeros_like(words)
    out, lse, sk, vis = mask_run(q, k, v, empty, causal=True, scale=0.25, lam=1e-3, Br=64, Bc=64)
    assert not out.any() and np.isneginf(lse).all() and vis.sum() == 0
