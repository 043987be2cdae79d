"""Pins for the proxy-compensation oracle (oracle/proxy.py), each against
something other than itself:
  * every block selected: no proxy is used and the result is dense softmax
    attention (numpy brute force);
  * keys equal inside every block: a block's mean key is each of its keys, so
    the proxy of an omitted block is exact and ANY selection gives dense
    attention -- with a ragged last block, so the true block length (not Bc)
    must be the token mass, and the value summary must be the sum;
  * blocks of one key: every summary is exact, any selection gives dense
    attention;
  * the summaries themselves: mean of the keys and sum of the values over the
    true length of each block;
  * padding bits past the last block change nothing.
"""
import numpy as np
import pytest
import torch

from oracle.proxy import block_summaries, run


def _gen(B, Hq, Hkv, Lq, Lk, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, Hq, d, generator=g).double()
    k = torch.randn(B, Lk, Hkv, d, generator=g).double()
    v = torch.randn(B, Lk, Hkv, d, generator=g).double()
    return q.numpy(), k.numpy(), v.numpy()


def _dense(q, k, v, scale):
    B, Lq, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = float(np.float32(scale))
    out = np.zeros_like(q)
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, :, h] @ k[b, :, h // (Hq // Hkv)].T
            mx = s.max(axis=1, keepdims=True)
            p = np.exp(s - mx)
            out[b, :, h] = p @ v[b, :, h // (Hq // Hkv)] / p.sum(axis=1, keepdims=True)
            lse[b, h] = (mx + np.log(p.sum(axis=1, keepdims=True)))[:, 0]
    return out, lse


def _masks(rng, B, Hkv, nQ, nK, kind):
    words = -(-nK // 32)
    m = np.zeros((B, Hkv, nQ, words), dtype=np.uint32)
    for idx in np.ndindex(B, Hkv, nQ):
        for kt in range(nK):
            on = {"all": True, "none": False, "random": rng.random() < 0.4}[kind]
            if on:
                m[idx + (kt >> 5,)] |= np.uint32(1 << (kt & 31))
    return m


SHAPE = dict(B=2, Hq=4, Hkv=2, Lq=70, Lk=150, d=16)  # Bc = 32: five blocks, the last of 22 keys


def test_all_blocks_selected_is_dense_attention():
    q, k, v = _gen(**SHAPE, seed=1)
    Br, Bc, scale = 32, 32, 0.3
    km, vs = block_summaries(k, v, Bc)
    mask = _masks(np.random.default_rng(0), 2, 2, 3, 5, "all")
    out, lse = run(q, k, v, mask, km, vs, scale=scale, Br=Br, Bc=Bc)
    ref, rlse = _dense(q, k, v, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, rlse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["none", "random"])
@pytest.mark.parametrize("Bc", [32, 16])
def test_constant_keys_per_block_make_every_proxy_exact(kind, Bc):
    q, k, v = _gen(**SHAPE, seed=2)
    Lk = SHAPE["Lk"]
    for c0 in range(0, Lk, Bc):
        k[:, c0:min(Lk, c0 + Bc)] = k[:, c0:c0 + 1]  # every key of the block equals its first
    km, vs = block_summaries(k, v, Bc)
    nK = -(-Lk // Bc)
    mask = _masks(np.random.default_rng(3), 2, 2, 3, nK, kind)
    out, lse = run(q, k, v, mask, km, vs, scale=0.3, Br=32, Bc=Bc)
    ref, rlse = _dense(q, k, v, 0.3)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(lse, rlse, rtol=1e-12, atol=1e-11)


def test_one_key_blocks_are_exact_for_any_selection():
    q, k, v = _gen(B=1, Hq=2, Hkv=1, Lq=9, Lk=37, d=8, seed=4)
    km, vs = block_summaries(k, v, 1)
    mask = _masks(np.random.default_rng(5), 1, 1, 3, 37, "random")
    out, lse = run(q, k, v, mask, km, vs, scale=0.5, Br=4, Bc=1)
    ref, rlse = _dense(q, k, v, 0.5)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(lse, rlse, rtol=1e-12, atol=1e-11)


def test_summaries_use_the_true_block_length():
    k = np.arange(1 * 7 * 1 * 2, dtype=np.float64).reshape(1, 7, 1, 2)
    v = k * 10.0
    km, vs = block_summaries(k, v, 3)  # blocks of 3, 3 and 1 keys
    assert km.shape == (1, 3, 1, 2)
    np.testing.assert_array_equal(km[0, :, 0], [[2.0, 3.0], [8.0, 9.0], [12.0, 13.0]])
    np.testing.assert_array_equal(vs[0, :, 0], [[60.0, 90.0], [240.0, 270.0], [120.0, 130.0]])


def test_padding_bits_are_ignored():
    q, k, v = _gen(**SHAPE, seed=6)
    km, vs = block_summaries(k, v, 32)
    mask = _masks(np.random.default_rng(7), 2, 2, 3, 5, "random")
    padded = mask | np.uint32(0xFFFFFFE0)  # bits 5..31: past the five blocks
    a = run(q, k, v, mask, km, vs, scale=0.3, Br=32, Bc=32)
    b = run(q, k, v, padded, km, vs, scale=0.3, Br=32, Bc=32)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_omitted_blocks_change_the_result_with_varied_keys():
    """With ordinary keys the proxies approximate: the selection matters (a
    guard against an oracle that ignores the mask)."""
    q, k, v = _gen(**SHAPE, seed=8)
    km, vs = block_summaries(k, v, 32)
    full = run(q, k, v, _masks(np.random.default_rng(9), 2, 2, 3, 5, "all"), km, vs, scale=0.3, Br=32, Bc=32)
    none = run(q, k, v, _masks(np.random.default_rng(9), 2, 2, 3, 5, "none"), km, vs, scale=0.3, Br=32, Bc=32)
    assert np.abs(full[0] - none[0]).max() > 1e-3
