"""Pins for the two oracle flags that excuse a GPU/oracle difference.

Every difference the GPU parity tests forgive passes through one of them, so
each is pinned here against constructed inputs whose scores are exact, and a
mutation test shows that an oracle which over-marks turns a pin red.

* N:M near ties ("Attention Sparsity for HuggingFace Models", "N:M Sparse
  Softmax": keep the top-N of every M consecutive keys).  The method statement
  wants keep masks bit-exact; the kernel ranks fp32 tensor-core scores, so the
  oracle marks the keys whose fate hangs on two raw q.k scores (the N-th and
  the (N+1)-th largest of the group, rounded to fp32) lying within
  1e-4 * (1 + |s_N|) of each other.  Keys inside the sink / recent windows
  are kept whatever their rank and are never marked.
* Skip-decision margin (the method statement's tolerance: decisions match
  except tiles whose margin |exp(m_tile - m) - lambda| < 1e-3 * lambda).  The
  tile is skipped iff its largest row ratio exp(m_tile_r - m_r) is below
  lambda, so that largest ratio is the tile's margin quantity; a row that does
  not decide the tile never marks it.

Scores are built as q.k with q = (1, 2^-16, 0, ...) and k = (a, n, 0, ...),
a and n small bf16-exact numbers: s = a + n * 2^-16 exactly, in fp64 and in
fp32 (and so on the GPU too).
"""
import math
import re
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle.oracle as orc
from oracle import run_items
from oracle import blockmask as bm_oracle
from oracle.decode import decode
from softmax_ssa_fwd_b200.inputs import MODE_NM, MODE_SKIP

U = 2.0 ** -16
D = 16


def _keys(pairs):
    """k rows (a, n, 0, ...) for a list of (a, n)."""
    k = torch.zeros(1, len(pairs), 1, D)
    for j, (a, n) in enumerate(pairs):
        k[0, j, 0, 0] = a
        k[0, j, 0, 1] = n
    kb = k.bfloat16()
    assert torch.equal(kb.float(), k)           # exact in bf16
    return kb


def _query():
    q = torch.zeros(1, 1, 1, D)
    q[0, 0, 0, 0] = 1.0
    q[0, 0, 0, 1] = U
    return q.bfloat16()


# ---------------------------------------------------------------- N:M near ties

# Groups of M = 4, N = 2, one query row.  Per group: the raw scores (a + n U)
# and the keys whose fate is a near tie.  tol = 1e-4 * (1 + |s_N|).
TIE_GROUPS = [
    # s_N = 1.0, tol = 2e-4: gap 13 U = 1.98e-4 (just under) -> keys 1, 2
    ([(3.0, 0), (1.0, 0), (1.0, -13), (-2.0, 0)], {1, 2}),
    # gap 14 U = 2.14e-4 (just over) -> none
    ([(1.0, 0), (1.0, -14), (3.0, 0), (-2.0, 0)], set()),
    # s_N = 4.0, tol = 5e-4: gap 32 U = 4.88e-4 -> keys 0, 3
    ([(4.0, 0), (-1.0, 0), (8.0, 0), (4.0, -32)], {0, 3}),
    # gap 33 U = 5.04e-4 -> none
    ([(4.0, 0), (-1.0, 0), (8.0, 0), (4.0, -33)], set()),
    # s_N = -3.0, tol = 4e-4: gap 26 U = 3.97e-4 -> keys 2, 3 (s_N is key 2)
    ([(5.0, 0), (-6.0, 0), (-3.0, 0), (-3.0, -26)], {2, 3}),
    # gap 27 U = 4.12e-4 -> none
    ([(5.0, 0), (-6.0, 0), (-3.0, 0), (-3.0, -27)], set()),
    # an exact tie at the boundary (equal scores) is a near tie too -> keys 1, 2
    ([(2.0, 0), (0.5, 0), (0.5, 0), (-1.0, 0)], {1, 2}),
    # well separated: integers -> none
    ([(2.0, 0), (-1.0, 0), (7.0, 0), (0.0, 0)], set()),
]


def _tie_run(lib=None, tie_tol=1e-4, sink=0, recent=0, scale=0.125):
    pairs = [p for grp, _ in TIE_GROUPS for p in grp]
    k = _keys(pairs)
    L = len(pairs)
    q = _query()
    v = torch.zeros_like(k)
    res = run_items(q, k, v, causal=False, scale=scale, mode=MODE_NM, n=2, m=4, sink=sink,
                    recent=recent, Br=1, Bc=L, keep_bits=True, tie_tol=tie_tol, lib=lib)
    ties = np.unpackbits(res.tie_bits[0, 0].view(np.uint8), bitorder="little")[:L].astype(bool)
    keep = np.unpackbits(res.keep_bits[0, 0].view(np.uint8), bitorder="little")[:L].astype(bool)
    return ties, keep


def _want_ties(excluded=()):
    want = np.zeros(len(TIE_GROUPS) * 4, bool)
    for g, (_, keys) in enumerate(TIE_GROUPS):
        for t in keys:
            if 4 * g + t not in excluded:
                want[4 * g + t] = True
    return want


def tie_pin_holds(lib=None, tie_tol=1e-4) -> bool:
    ties, keep = _tie_run(lib, tie_tol)
    if not np.array_equal(ties, _want_ties()):
        return False
    # the keep mask is the exact top-2 (ties to the lower index) everywhere
    for g, (grp, _) in enumerate(TIE_GROUPS):
        s = [a + n * U for a, n in grp]
        order = sorted(range(4), key=lambda t: (-s[t], t))
        if sorted(np.nonzero(keep[4 * g:4 * g + 4])[0].tolist()) != sorted(order[:2]):
            return False
    return True


def test_tie_bits_exactly_on_the_boundary_keys():
    assert tie_pin_holds()


def test_tie_bits_never_on_window_keys():
    # the sink covers groups 0-1 (keys 0..7): their keys are kept whatever their rank
    ties, keep = _tie_run(sink=8)
    assert np.array_equal(ties, _want_ties(excluded=set(range(8))))
    assert keep[:8].all()


def test_tie_bits_ten_times_wider_tolerance_breaks_the_pin():
    # the same pin, run with a 10x tolerance, must fail: it would mark the
    # "just over" groups as well
    assert not tie_pin_holds(tie_tol=1e-3)


def test_tie_bits_all_clear_on_separated_scores():
    g = torch.Generator().manual_seed(3)
    L = 256
    perm = torch.randperm(L, generator=g)
    k = _keys([(float(int(p) - 128) / 4.0, 0) for p in perm])   # distinct, 0.25 apart
    q = _query()
    res = run_items(q, k, torch.zeros_like(k), causal=False, scale=0.1, mode=MODE_NM, n=2, m=4,
                    Br=1, Bc=128, keep_bits=True)
    assert not res.tie_bits.any()


# ---------------------------------------------------------------- skip margin

def _margin_inputs(a1, b1):
    """Two query rows, three one-key tiles.  Key 0 scores 0 for both rows (it
    sets the running max); key 1 scores a1 (row 0) and b1 (row 1); key 2
    scores -40 for both (far below any threshold used here)."""
    q = torch.zeros(1, 2, 1, D)
    q[0, 0, 0, 0] = 1.0
    q[0, 1, 0, 1] = 1.0
    k = torch.zeros(1, 3, 1, D)
    k[0, 1, 0, 0], k[0, 1, 0, 1] = a1, b1
    k[0, 2, 0, 0], k[0, 2, 0, 1] = -40.0, -40.0
    qb, kb = q.bfloat16(), k.bfloat16()
    assert torch.equal(kb.float(), k)
    return qb, kb, torch.ones_like(kb)


# (scores of key 1 for rows 0 and 1, log of the decisive ratio, relative offset
# eps with lambda = exp(decisive) / (1 + eps), expect marginal, expect skipped)
MARGIN_CASES = [
    (-4.0, -6.0, -4.0, +0.9e-3, True, False),   # just inside the band, kept
    (-4.0, -6.0, -4.0, -0.9e-3, True, True),    # just inside, skipped
    (-4.0, -6.0, -4.0, +1.1e-3, False, False),  # just outside, kept
    (-4.0, -6.0, -4.0, -1.1e-3, False, True),   # just outside, skipped
    (-6.0, -4.0, -4.0, +0.5e-3, True, False),   # the decisive row is row 1
    (-1.0, -4.0, -1.0, None, False, False),     # row 1 sits on lambda but row 0 decides (kept)
]


def _lambda(case):
    a1, b1, dec, eps, _, _ = case
    if eps is None:  # lambda exactly at row 1's ratio, which does not decide
        return math.exp(-4.0) / (1 + 0.5e-3)
    return math.exp(dec) / (1 + eps)


def _c_margin(case, lib=None):
    q, k, v = _margin_inputs(case[0], case[1])
    res = run_items(q, k, v, causal=False, scale=1.0, mode=MODE_SKIP, lam=_lambda(case), Br=2,
                    Bc=1, lib=lib)
    marg = np.unpackbits(res.marginal_bits[0].view(np.uint8), bitorder="little")[:3].astype(bool)
    skip = np.unpackbits(res.skip_bits[0].view(np.uint8), bitorder="little")[:3].astype(bool)
    return marg, skip


def margin_pin_holds(lib=None) -> bool:
    for case in MARGIN_CASES:
        marg, skip = _c_margin(case, lib)
        if marg.tolist() != [False, case[4], False] or skip.tolist() != [False, case[5], True]:
            return False
    return True


def test_c_oracle_margin_bits():
    for case in MARGIN_CASES:
        marg, skip = _c_margin(case)
        assert marg.tolist() == [False, case[4], False], case
        assert skip.tolist() == [False, case[5], True], case


@pytest.mark.parametrize("case", MARGIN_CASES)
def test_decode_oracle_margin_bits(case):
    q, k, v = _margin_inputs(case[0], case[1])
    # decode: the two query rows are the Lq rows of one head, one split
    r = decode(q.view(1, 2, 1, D), k, v, causal=False, scale=1.0, lam=_lambda(case), Bc=1,
               num_splits=1)
    assert r.marginal[0, 0].tolist() == [False, case[4], False]
    assert r.skip_bits[0, 0].tolist() == [False, case[5], True]


@pytest.mark.parametrize("case", MARGIN_CASES)
def test_blockmask_oracle_margin_bits(case):
    q, k, v = _margin_inputs(case[0], case[1])
    words = np.full((1, 1, 1, 1), 0b111, np.uint32)
    sb = np.zeros((1, 1, 1, 3), bool)
    mb = np.zeros((1, 1, 1, 3), bool)
    cnt = np.zeros((1, 1, 1), np.int64)
    bm_oracle.run(q, k, v, words, causal=False, scale=1.0, lam=_lambda(case), Br=2, Bc=1,
                  marginal=cnt, skip_bits=sb, marginal_bits=mb)
    assert mb[0, 0, 0].tolist() == [False, case[4], False]
    assert sb[0, 0, 0].tolist() == [False, case[5], True]
    assert cnt[0, 0, 0] == int(case[4])


def test_margin_bits_all_clear_far_from_lambda():
    g = torch.Generator().manual_seed(5)
    B, Hq, L, d = 1, 2, 384, 32
    q = torch.randn(B, L, Hq, d, generator=g)
    k = torch.randn(B, L, Hq, d, generator=g)
    u = torch.randn(d, generator=g)
    u /= u.norm()
    q += 12 * u
    k[:, :4] += 12 * u
    q, k = q.bfloat16(), k.bfloat16()
    v = torch.randn(B, L, Hq, d, generator=g).bfloat16()
    # the decisive ratio of every visited tile, from the dense scores, to pick
    # a lambda that no tile sits near
    res0 = run_items(q, k, v, causal=True, scale=0.125, mode=MODE_SKIP, lam=1e-2, Br=64, Bc=64)
    assert res0.skip_count.sum() > 0
    s = 0.125 * np.einsum("bqhd,bkhd->bhqk", q.double().numpy(), k.double().numpy())
    vis = np.arange(L)[None, :] <= np.arange(L)[:, None]
    s = np.where(vis, s, -np.inf)
    ratios = []
    for b in range(B):
        for h in range(Hq):
            for qt in range(L // 64):
                rows = s[b, h, qt * 64:(qt + 1) * 64]
                run = np.full(64, -np.inf)
                for kt in range(qt + 1):
                    tm = rows[:, kt * 64:(kt + 1) * 64].max(1)
                    with np.errstate(invalid="ignore"):
                        r = np.where(tm == -np.inf, 0.0,
                                     np.where(run == -np.inf, np.inf, np.exp(tm - run)))
                    ratios.append(r.max())
                    run = np.maximum(run, tm)   # a lambda <= 1 never moves the max on a skip
    ratios = np.array([x for x in ratios if np.isfinite(x) and x > 0])
    lam = 1e-2
    assert np.all(np.abs(ratios - lam) > 5e-3 * lam)
    res = run_items(q, k, v, causal=True, scale=0.125, mode=MODE_SKIP, lam=lam, Br=64, Bc=64)
    assert not res.marginal_bits.any()
    assert res.skip_count.sum() > 0


# ---------------------------------------------------------------- planted mistakes

MUTANTS = {
    # a tie tolerance ten times too wide
    "tie_tol_x10": (r"J->tie_tol \* \(1\.0 \+ fabs\(\(double\)srt\[N - 1\]\)\)",
                    "10.0 * J->tie_tol * (1.0 + fabs((double)srt[N - 1]))", "tie"),
    # the tie tolerance applied to scaled scores instead of raw q.k
    "tie_on_scaled": (r"gx\[t\] = \(j < Lk && kept\[\(size_t\)r \* Bc \+ \(j - c0\)\]\) \? \(float\)x\[",
                      "gx[t] = (j < Lk && kept[(size_t)r * Bc + (j - c0)]) ? (float)J->scale * (float)x[",
                      "tie"),
    # a margin band ten times too wide
    "margin_x10": (r"< 1e-3 \* J->lambda", "< 1e-2 * J->lambda", "margin"),
    # a margin taken on any row instead of the deciding one
    "margin_any_row": (r"if \(ratio > max_ratio\) max_ratio = ratio;",
                       "if (ratio > max_ratio) max_ratio = ratio;\n"
                       "        if (isfinite(ratio) && fabs(ratio - J->lambda) < 1e-3 * J->lambda) max_ratio = J->lambda;",
                       "margin"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_over_marking_turns_a_pin_red(name, tmp_path):
    pat, rep, which = MUTANTS[name]
    src = open(orc._SRC).read()
    mutated, n = re.subn(pat, rep, src)
    assert n >= 1, f"mutation {name} did not apply"
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", str(so), str(c),
                    "-lm"], check=True)
    lib = orc.bind(str(so))
    assert tie_pin_holds() and margin_pin_holds()          # the real oracle passes both
    if which == "tie":
        assert not tie_pin_holds(lib)
    else:
        assert not margin_pin_holds(lib)


# ---------------------------------------------------------------- taking the other decision

def test_flip_is_accepted_only_inside_the_band():
    # just inside the band, kept by the oracle: flipped, the tile is skipped and
    # the output is the softmax over key 0 alone (v = 1 everywhere, so check lse)
    case = MARGIN_CASES[0]
    q, k, v = _margin_inputs(case[0], case[1])
    flip = np.array([[0b010]], np.uint32)
    res = run_items(q, k, v, causal=False, scale=1.0, mode=MODE_SKIP, lam=_lambda(case), Br=2, Bc=1,
                    flip_bits=flip)
    skip = np.unpackbits(res.skip_bits[0].view(np.uint8), bitorder="little")[:3].tolist()
    assert skip == [0, 1, 1]
    np.testing.assert_allclose(res.lse[0, :2], [0.0, 0.0], atol=1e-15)
    plain = run_items(q, k, v, causal=False, scale=1.0, mode=MODE_SKIP, lam=_lambda(case), Br=2, Bc=1)
    np.testing.assert_allclose(plain.lse[0, :2], [math.log1p(math.exp(-4.0)), math.log1p(math.exp(-6.0))],
                               atol=1e-15)
    # just outside the band: the request is refused
    case = MARGIN_CASES[2]
    q, k, v = _margin_inputs(case[0], case[1])
    with pytest.raises(ValueError):
        run_items(q, k, v, causal=False, scale=1.0, mode=MODE_SKIP, lam=_lambda(case), Br=2, Bc=1,
                  flip_bits=flip)


def test_decode_and_blockmask_flip_only_inside_the_band():
    case = MARGIN_CASES[0]
    q, k, v = _margin_inputs(case[0], case[1])
    lam = _lambda(case)
    flip = np.zeros((1, 1, 3), bool)
    flip[0, 0, 1] = True
    r = decode(q.view(1, 2, 1, D), k, v, causal=False, scale=1.0, lam=lam, Bc=1, num_splits=1, flip=flip)
    assert r.skip_bits[0, 0].tolist() == [False, True, True]
    words = np.full((1, 1, 1, 1), 0b111, np.uint32)
    sb = np.zeros((1, 1, 1, 3), bool)
    bm_oracle.run(q, k, v, words, causal=False, scale=1.0, lam=lam, Br=2, Bc=1, skip_bits=sb,
                  flip=flip[:, :, None])
    assert sb[0, 0, 0].tolist() == [False, True, True]
    far = _lambda(MARGIN_CASES[2])
    with pytest.raises(ValueError):
        decode(q.view(1, 2, 1, D), k, v, causal=False, scale=1.0, lam=far, Bc=1, num_splits=1, flip=flip)
    with pytest.raises(ValueError):
        bm_oracle.run(q, k, v, words, causal=False, scale=1.0, lam=far, Br=2, Bc=1, flip=flip[:, :, None])
