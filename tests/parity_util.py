"""Helpers for GPU-vs-oracle parity: run both sides on the same seeded bf16
inputs and compare work item by work item.

Bar (the method statement's tolerances): outputs max-abs <= 2e-2 and
relative L2 <= 5e-3 against the fp64 oracle; lse max-abs <= 1e-3; skip
decisions identical except tiles whose margin |exp(m_tile - m) - lambda| is
below 1e-3 * lambda; N:M keep masks identical except keys whose fate is a
near tie in fp32 (oracle tie bits: the two scores around the N-th place lie
within 1e-4 * (1 + |s|) of each other, raw q.k units).
"""
from __future__ import annotations

import os
from dataclasses import dataclass, field

import numpy as np
import torch

from oracle import run_items

OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
TIE_TOL = 1e-4


MARGINAL_FRAC_MAX = 5e-3   # differing decisions inside the band, per visited tile
TIE_FRAC_MAX = 1e-4        # differing keep bits at near ties, per compared keep bit
REPORTS = []               # (test id, Report) of every compare(); the terminal summary prints them
V_LOADS = []               # (test id, V tiles loaded, key tiles walked) of every gpu_run()


@dataclass
class Report:
    items: int = 0
    out_max_abs: float = 0.0
    out_rel_l2: float = 0.0
    lse_max_abs: float = 0.0
    skipped_gpu: int = 0
    skipped_oracle: int = 0
    visited: int = 0
    marginal_tiles: int = 0        # tiles the oracle flags inside the tolerance band
    marginal_mismatch: int = 0     # of which the kernel took the other decision
    keep_bits_compared: int = 0
    tie_bits: int = 0              # keys the oracle flags as near ties
    keep_mismatch_ties: int = 0    # of which the kernel kept the other key
    notes: list = field(default_factory=list)

    def line(self) -> str:
        return (f"items {self.items}, visited tiles {self.visited}, skipped {self.skipped_gpu} "
                f"(oracle {self.skipped_oracle}), marginal {self.marginal_mismatch}/{self.marginal_tiles} "
                f"taken the other way, near-tie keep bits {self.keep_mismatch_ties}/{self.tie_bits} of "
                f"{self.keep_bits_compared}, out max-abs {self.out_max_abs:.2e} rel-L2 {self.out_rel_l2:.2e}, "
                f"lse max-abs {self.lse_max_abs:.2e}")


def expected_v_loads(sb_words, causal, Lq, Lk, Br, Bc, selected=None):
    """V tiles each CTA of the prefill kernel must load, from the kernel's own
    skip bits (which compare() checks against the oracle): the key tiles that
    at least one of the CTA's query tiles visits and keeps.  A CTA owns query
    rows [256 p, 256 p + 256) of one (batch, head): two 128-row query tiles, or
    four 64-row ones.  ``selected``: bool [B, Hq, nQ, nK] key blocks chosen by a
    bitmap.  Returns int [B, Hq, ceil(nQp / 2)], and the same count without the
    skips (key tiles some query tile of the CTA visits)."""
    from oracle import visited_tiles
    B, Hq, nQ, _ = sb_words.shape
    nK = -(-Lk // Bc)
    skip = _unpack(sb_words, nK)
    vis = np.zeros((nQ, nK), bool)
    for qt in range(nQ):
        vis[qt, :visited_tiles(causal, Lq, Lk, Br, Bc, qt)] = True
    visit = np.broadcast_to(vis[None, None], skip.shape)
    if selected is not None:
        visit = visit & selected
    per = 256 // Br
    npairs = -(-(-(-Lq // 128)) // 2)

    def per_cta(x):
        pad = np.zeros((B, Hq, npairs * per, nK), bool)
        pad[:, :, :nQ] = x
        return pad.reshape(B, Hq, npairs, per, nK).any(axis=3).sum(axis=-1)

    return per_cta(visit & ~skip), per_cta(visit)


def gpu_run(q, k, v, *, causal, scale, mode, lam=0.0, n=0, m=0, sink=0, recent=0, Br=128, Bc=128,
            keep_bits=False):
    """The kernel's outputs with its evidence: per-tile skip bits, keep bits
    (optional), and V tile loads per CTA, which must equal the key tiles the
    CTA's query tiles kept (a tile skipped by all of them loads no V)."""
    from softmax_ssa_fwd_b200 import ssa
    B, Lq, Hq, d = q.shape
    Lk = k.shape[1]
    nQ, nK = -(-Lq // Br), -(-Lk // Bc)
    sb = torch.zeros(B, Hq, nQ, -(-nK // 32), dtype=torch.int32, device=q.device)
    kb = torch.zeros(B, Hq, Lq, -(-Lk // 32), dtype=torch.int32, device=q.device) if keep_bits else None
    npairs = -(-(-(-Lq // 128)) // 2)
    vl = torch.full((B, Hq, npairs), -1, dtype=torch.int32, device=q.device)
    out, lse, cnt = ssa.attention(q, k, v, causal=causal, scale=scale, mode=mode, lam=lam, n=n, m=m,
                                  sink=sink, recent=recent, Br=Br, Bc=Bc, skip_bits=sb, keep_bits=kb,
                                  v_tile_loads=vl)
    st = ssa.ssa_device_status()
    assert st == ssa.SSA_OK, ssa.status_string(st)
    want, walked = expected_v_loads(sb.cpu().numpy().view(np.uint32), causal, Lq, Lk, Br, Bc)
    got = vl.cpu().numpy()
    assert np.array_equal(got, want), (
        f"V tile loads differ from the kept tiles at {np.argwhere(got != want)[:8].tolist()}")
    V_LOADS.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], int(got.sum()),
                    int(walked.sum())))
    return out, lse, cnt, sb, kb


def _unpack(words, nbits):
    w = np.ascontiguousarray(words).view(np.uint32)
    return np.unpackbits(w.view(np.uint8), axis=-1, bitorder="little")[..., :nbits].astype(bool)


def _pack_one(bits, nwords):
    out = np.zeros(nwords, np.uint32)
    for i in np.nonzero(bits)[0]:
        out[i >> 5] |= np.uint32(1) << np.uint32(i & 31)
    return out


def compare(q, k, v, items, *, causal, scale, mode, lam=0.0, n=0, m=0, sink=0, recent=0, Br=128,
            Bc=128, keep_bits=False, gpu=None, qkv_cpu=None) -> Report:
    """Run (or reuse) the GPU result, run the oracle on ``items``, compare.

    Skip decisions must be identical; where the kernel took the other side of a
    tile inside the tolerance band, the oracle is re-run on that work item with
    that decision taken its way (the oracle refuses a tile outside the band),
    and everything else -- later decisions, counts, keep bits, out, lse -- is
    compared against that run.  Such tiles, and keep bits that differ at near
    ties, must stay a small fraction of what is compared."""
    if gpu is None:
        gpu = gpu_run(q, k, v, causal=causal, scale=scale, mode=mode, lam=lam, n=n, m=m, sink=sink,
                      recent=recent, Br=Br, Bc=Bc, keep_bits=keep_bits)
    out, lse, cnt, sb, kb = gpu
    qc, kc, vc = qkv_cpu if qkv_cpu is not None else (q.cpu(), k.cpu(), v.cpu())
    B, Lq, Hq, d = qc.shape
    Lk = kc.shape[1]
    nK = -(-Lk // Bc)
    nKw = -(-nK // 32)
    kw = dict(causal=causal, scale=scale, mode=mode, lam=lam, n=n, m=m, sink=sink, recent=recent,
              Br=Br, Bc=Bc, keep_bits=keep_bits, tie_tol=TIE_TOL)
    res = run_items(qc, kc, vc, items=items, **kw)
    g_sb_all = sb.cpu().numpy().view(np.uint32)
    cnt_all = cnt.cpu().numpy()
    rep = Report(items=len(items))
    # settle the decisions taken the other way inside the band, item by item
    for it, (b, h, t) in enumerate(res.items):
        g_sb = _unpack(g_sb_all[b, h, t], nK)
        flips = np.zeros(nK, bool)
        for _ in range(nK + 1):
            diff = g_sb != _unpack(res.skip_bits[it], nK)
            if not diff.any():
                break
            first = int(np.argmax(diff))
            marg = _unpack(res.marginal_bits[it], nK)
            assert marg[first], (
                f"skip decision mismatch at item {(b, h, t)} tile {first} (outside the tolerance band); "
                f"all differing tiles: {np.nonzero(diff)[0][:8].tolist()}")
            flips[first] = True
            one = run_items(qc, kc, vc, items=[(b, h, t)], flip_bits=_pack_one(flips, nKw)[None], **kw)
            for name in ("out", "lse", "skip_count", "visited", "skip_bits", "marginal_bits",
                         "keep_bits", "tie_bits"):
                arr = getattr(res, name)
                if arr is not None:
                    arr[it] = getattr(one, name)[0]
        if flips.any():
            rep.marginal_mismatch += int(flips.sum())
            rep.notes.append(f"item {(b, h, t)}: tiles {np.nonzero(flips)[0].tolist()} decided the other "
                             f"way inside the band")
    num = den = 0.0
    for it, (b, h, t) in enumerate(res.items):
        r0, r1 = t * Br, min(Lq, t * Br + Br)
        rows = r1 - r0
        g_sb = _unpack(g_sb_all[b, h, t], nK)
        assert (g_sb == _unpack(res.skip_bits[it], nK)).all()
        rep.skipped_gpu += int(g_sb.sum())
        rep.skipped_oracle += int(res.skip_count[it])
        rep.visited += int(res.visited[it])
        rep.marginal_tiles += int(_unpack(res.marginal_bits[it], nK).sum())
        assert int(cnt_all[b, h, t]) == int(g_sb.sum()) == int(res.skip_count[it]), (b, h, t)
        if keep_bits:
            g_kb = _unpack(kb[b, h, r0:r1].cpu().numpy(), Lk)
            o_kb = _unpack(res.keep_bits[it, :rows], Lk)
            ties = _unpack(res.tie_bits[it, :rows], Lk)
            kd = g_kb != o_kb
            assert not (kd & ~ties).any(), (
                f"N:M keep mismatch at item {(b, h, t)}: {np.argwhere(kd & ~ties)[:8].tolist()}")
            rep.keep_mismatch_ties += int(kd.sum())
            rep.tie_bits += int(ties.sum())
            rep.keep_bits_compared += rows * Lk
        go = out[b, r0:r1, h].float().cpu().numpy().astype(np.float64)
        oo = res.out[it, :rows]
        e = np.abs(go - oo)
        rep.out_max_abs = max(rep.out_max_abs, float(e.max()))
        num += float((e ** 2).sum())
        den += float((oo ** 2).sum())
        gl = lse[b, h, r0:r1].cpu().numpy().astype(np.float64)
        ol = res.lse[it, :rows]
        both_inf = np.isneginf(gl) & np.isneginf(ol)
        assert (np.isneginf(gl) == np.isneginf(ol)).all()
        if (~both_inf).any():
            fin = ~both_inf
            rep.lse_max_abs = max(rep.lse_max_abs, float(np.abs(gl[fin] - ol[fin]).max()))
    rep.out_rel_l2 = (num / den) ** 0.5 if den > 0 else 0.0
    REPORTS.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], rep))
    assert rep.out_max_abs <= OUT_MAX_ABS, rep
    assert rep.out_rel_l2 <= OUT_REL_L2, rep
    assert rep.lse_max_abs <= LSE_MAX_ABS, rep
    assert rep.marginal_mismatch <= max(2, MARGINAL_FRAC_MAX * rep.visited), rep
    assert rep.keep_mismatch_ties <= max(4, TIE_FRAC_MAX * rep.keep_bits_compared), rep
    return rep


def all_items(B, Hq, Lq, Br):
    nQ = -(-Lq // Br)
    return [(b, h, t) for b in range(B) for h in range(Hq) for t in range(nQ)]
