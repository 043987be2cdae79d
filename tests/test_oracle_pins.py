"""Pins for the CPU oracle: each test checks it against something other than
itself -- a library routine (torch SDPA in fp64), closed forms, brute-force
enumeration on tiny inputs, invariants, and a hand-worked example.

Definitions pinned (pages: "Skip-Softmax Sparse Attention for Diffusion
Models", intro + "Threshold Modes"; "Attention Sparsity for HuggingFace
Models", "N:M Sparse Softmax" + custom configuration):
  * skip-softmax with lambda = 0 is dense softmax attention;
  * N:M with N = M is dense softmax attention;
  * for lambda <= 1 a skipped tile never raises the running max, so the skip
    decision has a closed form on the dense score matrix;
  * N:M keeps exactly N keys per M-group outside the dense windows, the top-N
    by score with ties to the lowest index.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import run_items, visited_tiles
from softmax_ssa_fwd_b200.inputs import MODE_DENSE, MODE_NM, MODE_SKIP, Workload, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(t):
    return t.to(torch.float64).numpy()


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


def _visible(Lq, Lk, causal):
    i = np.arange(Lq)[:, None] + (Lk - Lq)
    j = np.arange(Lk)[None, :]
    return (j <= i) if causal else np.ones((Lq, Lk), bool)


def _assemble(res, B, Hq, Lq, Br, d):
    """Scatter per-item oracle results into [B, Lq, Hq, d] / [B, Hq, Lq]."""
    out = np.zeros((B, Lq, Hq, d))
    lse = np.zeros((B, Hq, Lq))
    for it, (b, h, t) in enumerate(res.items):
        r0, r1 = t * Br, min(Lq, t * Br + Br)
        out[b, r0:r1, h] = res.out[it, : r1 - r0]
        lse[b, h, r0:r1] = res.lse[it, : r1 - r0]
    return out, lse


def _sdpa_ref(q, k, v, causal, scale):
    """Dense attention through torch's own SDPA in float64 (library special case)."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    qq = q.to(torch.float64).permute(0, 2, 1, 3)
    kk = k.to(torch.float64).repeat_interleave(g, dim=2).permute(0, 2, 1, 3)
    vv = v.to(torch.float64).repeat_interleave(g, dim=2).permute(0, 2, 1, 3)
    mask = torch.from_numpy(_visible(Lq, Lk, causal))
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
    s = (qq @ kk.transpose(-1, -2)) * scale
    s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


def _numpy_ref(q, k, v, causal, scale, keep=None):
    """Brute-force softmax(S) V in numpy fp64 over an explicit keep mask
    [B, Hq, Lq, Lk] (default: the visible keys)."""
    qn, kn, vn = _f64(q), _f64(k), _f64(v)
    B, Lq, Hq, d = qn.shape
    Lk, Hkv = kn.shape[1], kn.shape[2]
    out = np.zeros((B, Lq, Hq, d))
    lse = np.zeros((B, Hq, Lq))
    vis = _visible(Lq, Lk, causal)
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            s = scale * (qn[b, :, h] @ kn[b, :, kv].T)
            msk = vis if keep is None else keep[b, h]
            s = np.where(msk, s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            p = np.exp(s - mx)
            p = np.where(msk, p, 0.0)
            l = p.sum(axis=1, keepdims=True)
            out[b, :, h] = (p @ vn[b, :, kv]) / l
            lse[b, h] = (mx + np.log(l))[:, 0]
    return out, lse


CASES = [
    # B, Hq, Hkv, Lq, Lk, d, causal, Br, Bc
    (1, 2, 2, 128, 128, 64, True, 64, 64),
    (1, 4, 2, 100, 100, 32, True, 64, 64),      # ragged tail, GQA 2:1
    (2, 2, 1, 77, 130, 16, True, 32, 64),       # Lq < Lk: bottom-right causal
    (1, 2, 2, 96, 96, 64, False, 64, 32),
    (1, 2, 2, 200, 200, 64, True, 128, 64),     # Br != Bc
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("mode", [MODE_DENSE, MODE_SKIP])
def test_lambda0_is_dense_attention(case, mode):
    B, Hq, Hkv, Lq, Lk, d, causal, Br, Bc = case
    q, k, v = _gen(B, Hq, Hkv, Lq, Lk, d, seed=11)
    scale = float(np.float32(1.0 / math.sqrt(d)))
    res = run_items(q, k, v, causal=causal, scale=scale, mode=mode, lam=0.0, Br=Br, Bc=Bc)
    out, lse = _assemble(res, B, Hq, Lq, Br, d)
    ref_o, ref_l = _sdpa_ref(q, k, v, causal, scale)
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
    np_o, _ = _numpy_ref(q, k, v, causal, scale)
    np.testing.assert_allclose(out, np_o, rtol=0, atol=1e-12)
    assert res.skip_count.sum() == 0


@pytest.mark.parametrize("m", [4, 8])
def test_nm_with_n_equal_m_is_dense(m):
    B, Hq, Hkv, L, d = 1, 2, 1, 150, 32
    q, k, v = _gen(B, Hq, Hkv, L, L, d, seed=5)
    scale = float(np.float32(1.0 / math.sqrt(d)))
    res = run_items(q, k, v, causal=True, scale=scale, mode=MODE_NM, n=m, m=m, sink=0, recent=0,
                    Br=64, Bc=64)
    out, lse = _assemble(res, B, Hq, L, 64, d)
    ref_o, ref_l = _sdpa_ref(q, k, v, True, scale)
    np.testing.assert_allclose(out, ref_o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, ref_l, atol=1e-12, rtol=0)


def _brute_nm_keep(q, k, causal, n, m, sink, recent):
    """Keep mask by enumerating all C(M, N) subsets of each group: the subset
    with the largest fp32 score sum wins, ties to the lexicographically lowest
    index set; masked keys carry a huge negative finite score so they lose to
    any visible key.  Then keep = visible and (window or chosen)."""
    qn, kn = _f64(q), _f64(k)
    B, Lq, Hq, d = qn.shape
    Lk, Hkv = kn.shape[1], kn.shape[2]
    vis = _visible(Lq, Lk, causal)
    keep = np.zeros((B, Hq, Lq, Lk), bool)
    subsets = list(itertools.combinations(range(m), n))
    for b in range(B):
        for h in range(Hq):
            x = (qn[b, :, h] @ kn[b, :, h // (Hq // Hkv)].T).astype(np.float32).astype(np.float64)
            for i in range(Lq):
                pos = i + Lk - Lq
                for g0 in range(0, Lk, m):
                    vals = [x[i, j] if (j < Lk and vis[i, j]) else -1e30 for j in range(g0, g0 + m)]
                    best = max(subsets, key=lambda S: (sum(vals[t] for t in S), [-t for t in S]))
                    for t in range(m):
                        j = g0 + t
                        if j >= Lk or not vis[i, j]:
                            continue
                        win = j < sink or 0 <= pos - j < recent
                        keep[b, h, i, j] = win or (t in best)
    return keep


def _bits_to_mask(res, B, Hq, Lq, Lk, Br):
    keep = np.zeros((B, Hq, Lq, Lk), bool)
    for it, (b, h, t) in enumerate(res.items):
        r0, r1 = t * Br, min(Lq, t * Br + Br)
        bits = np.unpackbits(res.keep_bits[it].view(np.uint8), axis=-1, bitorder="little")[:, :Lk]
        keep[b, h, r0:r1] = bits[: r1 - r0].astype(bool)
    return keep


@pytest.mark.parametrize("m,n", [(4, 1), (4, 2), (4, 3), (8, 1), (8, 3), (8, 5), (8, 7)])
@pytest.mark.parametrize("sink,recent", [(0, 0), (4, 8), (3, 5)])
def test_nm_matches_subset_enumeration(m, n, sink, recent):
    B, Hq, Hkv, L, d = 1, 2, 1, 40, 16
    q, k, v = _gen(B, Hq, Hkv, L, L, d, seed=100 * m + n)
    k[:, 9] = k[:, 8]    # exact ties: duplicated keys give identical scores
    k[:, 21] = k[:, 20]
    k[:, 22] = k[:, 20]
    scale = float(np.float32(0.25))
    res = run_items(q, k, v, causal=True, scale=scale, mode=MODE_NM, n=n, m=m, sink=sink,
                    recent=recent, Br=16, Bc=8, keep_bits=True)
    got = _bits_to_mask(res, B, Hq, L, L, 16)
    want = _brute_nm_keep(q, k, True, n, m, sink, recent)
    assert (got == want).all()
    # and the output is softmax restricted to exactly that keep mask
    out, lse = _assemble(res, B, Hq, L, 16, d)
    ref_o, ref_l = _numpy_ref(q, k, v, True, scale, keep=want)
    np.testing.assert_allclose(out, ref_o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, ref_l, atol=1e-12, rtol=0)


def test_nm_tie_goes_to_lowest_index():
    B, Hq, Hkv, L, d = 1, 1, 1, 16, 8
    q, k, v = _gen(B, Hq, Hkv, L, L, d, seed=3)
    k[:, 4:8] = k[:, 4:5]   # a whole group of equal keys: 2:4 must keep 4 and 5
    res = run_items(q, k, v, causal=False, scale=1.0, mode=MODE_NM, n=2, m=4, Br=16, Bc=16,
                    keep_bits=True)
    keep = _bits_to_mask(res, B, Hq, L, L, 16)[0, 0]
    assert keep[:, 4].all() and keep[:, 5].all()
    assert not keep[:, 6].any() and not keep[:, 7].any()


def test_nm_keep_count_invariant():
    w = Workload("t", 1, 4, 2, 300, 64, True, 64, 64, MODE_NM, (0.0,), n=2, m=4, sink=4,
                 recent=20, seed=9, rope="1d", rope_base=5e5)
    q, k, v = make_inputs(w)
    res = run_items(q, k, v, causal=True, scale=w.scale, mode=MODE_NM, n=2, m=4, sink=4, recent=20,
                    Br=64, Bc=64, keep_bits=True)
    keep = _bits_to_mask(res, 1, 4, 300, 300, 64)
    vis = _visible(300, 300, True)
    for i in range(300):
        for g0 in range(0, 300, 4):
            grp = range(g0, g0 + 4)
            in_win = [j < 4 or 0 <= i - j < 20 for j in grp]
            if all(vis[i, j] for j in grp) and not any(in_win):
                assert (keep[:, :, i, g0:g0 + 4].sum(-1) == 2).all()
            for t, j in enumerate(grp):
                if in_win[t] and vis[i, j]:
                    assert keep[:, :, i, j].all()
                if not vis[i, j]:
                    assert not keep[:, :, i, j].any()


def _closed_form_skip(q, k, causal, scale, lam, Br, Bc):
    """Skip bits for lambda <= 1 from the dense score matrix: tile kt of query
    tile qt is skipped iff every row i has tile max < (max over earlier
    visited tiles) + ln(lambda) (rows with an all-masked tile count as
    satisfied; a row with no earlier visible key cannot be satisfied)."""
    qn, kn = _f64(q), _f64(k)
    B, Lq, Hq, d = qn.shape
    Lk, Hkv = kn.shape[1], kn.shape[2]
    vis = _visible(Lq, Lk, causal)
    nQ, nK = -(-Lq // Br), -(-Lk // Bc)
    bits = np.zeros((B, Hq, nQ, nK), bool)
    for b in range(B):
        for h in range(Hq):
            s = scale * (qn[b, :, h] @ kn[b, :, h // (Hq // Hkv)].T)
            s = np.where(vis, s, -np.inf)
            for qt in range(nQ):
                rows = s[qt * Br: min(Lq, qt * Br + Br)]
                nv = visited_tiles(causal, Lq, Lk, Br, Bc, qt)
                tmax = np.stack([rows[:, kt * Bc: (kt + 1) * Bc].max(axis=1) for kt in range(nv)], 1)
                for kt in range(1, nv):
                    prefix = tmax[:, :kt].max(axis=1)
                    cur = tmax[:, kt]
                    with np.errstate(invalid="ignore"):
                        ok = (cur == -np.inf) | ((prefix > -np.inf) & (cur < prefix + math.log(lam)))
                    bits[b, h, qt, kt] = ok.all()
    return bits


def _skip_bits_dense(res, B, Hq, nQ, nK):
    bits = np.zeros((B, Hq, nQ, nK), bool)
    for it, (b, h, t) in enumerate(res.items):
        bits[b, h, t] = np.unpackbits(res.skip_bits[it].view(np.uint8), bitorder="little")[:nK]
    return bits


@pytest.mark.parametrize("lam", [1e-4, 1e-3, 1e-2, 0.3, 1.0])
@pytest.mark.parametrize("shape", [(1, 2, 2, 256, 256, 64, True, 64, 64),
                                   (1, 2, 1, 190, 190, 32, True, 64, 32),
                                   (1, 2, 2, 160, 160, 32, False, 32, 32)])
def test_skip_matches_closed_form(lam, shape):
    B, Hq, Hkv, Lq, Lk, d, causal, Br, Bc = shape
    q, k, v = _gen(B, Hq, Hkv, Lq, Lk, d, seed=21, sink_coef=12.0)
    scale = float(np.float32(1.0 / math.sqrt(d)))
    res = run_items(q, k, v, causal=causal, scale=scale, mode=MODE_SKIP, lam=lam, Br=Br, Bc=Bc)
    nQ, nK = -(-Lq // Br), -(-Lk // Bc)
    got = _skip_bits_dense(res, B, Hq, nQ, nK)
    want = _closed_form_skip(q, k, causal, scale, lam, Br, Bc)
    assert (got == want).all()
    assert res.skip_count.sum() == want.sum()
    # outputs are softmax restricted to the keys of the kept tiles
    vis = _visible(Lq, Lk, causal)
    keep = np.broadcast_to(vis, (B, Hq, Lq, Lk)).copy()
    for b in range(B):
        for h in range(Hq):
            for qt in range(nQ):
                for kt in range(nK):
                    if want[b, h, qt, kt]:
                        keep[b, h, qt * Br:(qt + 1) * Br, kt * Bc:(kt + 1) * Bc] = False
    out, lse = _assemble(res, B, Hq, Lq, Br, d)
    ref_o, ref_l = _numpy_ref(q, k, v, causal, scale, keep=keep)
    np.testing.assert_allclose(out, ref_o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, ref_l, atol=1e-12, rtol=0)


def test_skip_actually_happens_and_is_monotone():
    q, k, v = _gen(1, 2, 2, 256, 256, 64, seed=21, sink_coef=12.0)
    counts = []
    for lam in [0.0, 1e-6, 1e-4, 1e-3, 1e-2, 0.1, 0.5, 1.0]:
        r = run_items(q, k, v, causal=True, scale=0.125, mode=MODE_SKIP, lam=lam, Br=64, Bc=64)
        counts.append(int(r.skip_count.sum()))
    assert counts[0] == 0 and counts[-1] > 0
    assert all(a <= b for a, b in zip(counts, counts[1:]))


def test_skip_with_nm_uses_masked_scores():
    """Combined mode: the skip test runs on the N:M-masked scores; pinned by
    the closed form applied to the brute-force N:M keep mask."""
    B, Hq, Hkv, L, d, Br, Bc = 1, 2, 1, 64, 16, 16, 16
    q, k, v = _gen(B, Hq, Hkv, L, L, d, seed=77, sink_coef=8.0)
    scale, lam = 0.25, 1e-2
    res = run_items(q, k, v, causal=True, scale=scale, mode=MODE_SKIP | MODE_NM, lam=lam, n=2, m=4,
                    sink=4, recent=4, Br=Br, Bc=Bc, keep_bits=True)
    keep = _brute_nm_keep(q, k, True, 2, 4, 4, 4)
    qn, kn = _f64(q), _f64(k)
    nQ = nK = L // Bc
    want = np.zeros((B, Hq, nQ, nK), bool)
    final_keep = keep.copy()
    for h in range(Hq):
        s = scale * (qn[0, :, h] @ kn[0, :, 0].T)
        s = np.where(keep[0, h], s, -np.inf)
        for qt in range(nQ):
            rows = s[qt * Br:(qt + 1) * Br]
            tmax = [rows[:, kt * Bc:(kt + 1) * Bc].max(1) for kt in range(qt + 1)]
            for kt in range(1, qt + 1):
                prefix = np.max(np.stack(tmax[:kt], 1), 1)
                with np.errstate(invalid="ignore"):
                    ok = (tmax[kt] == -np.inf) | ((prefix > -np.inf) & (tmax[kt] < prefix + math.log(lam)))
                if ok.all():
                    want[0, h, qt, kt] = True
                    final_keep[0, h, qt * Br:(qt + 1) * Br, kt * Bc:(kt + 1) * Bc] = False
    got = _skip_bits_dense(res, B, Hq, nQ, nK)
    assert (got == want).all() and want.sum() > 0
    out, _ = _assemble(res, B, Hq, L, Br, d)
    ref_o, _ = _numpy_ref(q, k, v, True, scale, keep=final_keep)
    np.testing.assert_allclose(out, ref_o, atol=1e-12, rtol=0)


def test_lambda_above_one_worked_example():
    """Hand-worked sequential example (lambda > 1, where decisions depend on
    the path): values and derivation in tests/golden/lambda_gt1_example.json."""
    with open(os.path.join(GOLDEN, "lambda_gt1_example.json")) as f:
        g = json.load(f)
    s = np.array(g["scores"], np.float32)
    L = len(s)
    q = torch.zeros(1, 1, 1, 2)
    q[0, 0, 0, 0] = 1.0
    k = torch.zeros(1, L, 1, 2)
    k[0, :, 0, 0] = torch.from_numpy(s)
    v = torch.zeros(1, L, 1, 2)
    v[0, :, 0, 0] = torch.tensor(g["values"], dtype=torch.float32)
    q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    assert (k.float()[0, :, 0, 0].numpy() == s).all()   # the scores are exact in bf16
    res = run_items(q, k, v, causal=False, scale=1.0, mode=MODE_SKIP, lam=g["lambda"], Br=1, Bc=1)
    bits = np.unpackbits(res.skip_bits[0].view(np.uint8), bitorder="little")[:L]
    assert bits.tolist() == g["skipped"]
    assert res.out[0, 0, 0] == pytest.approx(g["out"], abs=1e-15)
    assert res.lse[0, 0] == pytest.approx(g["lse"], abs=1e-15)


def test_rows_without_visible_keys():
    """Lq > Lk with bottom-right causal alignment leaves the first rows with no
    visible key: out = 0 and lse = -inf (reading R7)."""
    q, k, v = _gen(1, 1, 1, 70, 40, 16, seed=4)
    res = run_items(q, k, v, causal=True, scale=0.25, mode=MODE_SKIP, lam=1e-3, Br=32, Bc=32)
    out, lse = _assemble(res, 1, 1, 70, 32, 16)
    assert np.all(out[0, :30] == 0) and np.all(np.isneginf(lse[0, 0, :30]))
    ref_o, ref_l = _numpy_ref(q[:, 30:], k, v, True, 0.25)
    np.testing.assert_allclose(out[:, 30:], ref_o, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal,Lq,Lk,Br,Bc,qt,want", [
    (False, 300, 300, 128, 128, 0, 3),
    (True, 256, 256, 64, 64, 0, 1),
    (True, 256, 256, 64, 64, 3, 4),
    (True, 300, 300, 128, 128, 2, 3),     # ragged last tile
    (True, 100, 300, 64, 128, 0, 3),      # bottom-right: row 63 sits at key 263
    (True, 300, 100, 128, 64, 0, 0),      # rows 0..127 see no key at all
    (True, 8192, 8192, 128, 128, 63, 64),
])
def test_visited_tiles_closed_form(causal, Lq, Lk, Br, Bc, qt, want):
    assert visited_tiles(causal, Lq, Lk, Br, Bc, qt) == want
