"""fp64 oracle of split-KV decode skip-softmax attention (numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring): only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may use it.

What it computes follows "Skip-Softmax Sparse Attention for Diffusion Models"
(intro, "Threshold Modes": a key tile is skipped when its scores are
negligible against the running max, exp(tile_row_max - running_max) <
lambda for every row of the query tile) and "Attention Sparsity for
HuggingFace Models" (custom configuration: skip-softmax has a decode
threshold; N:M is prefill only).  The pages do not say how decoding splits
the keys; the reading taken: the key tiles of a sequence are cut into
``num_splits`` contiguous ranges of ceil(nK / num_splits) tiles, each range
runs the recurrence with its own running max, and the ranges are merged with
the log-sum-exp rule.  The query tile is the Lq rows of one query head.

Steps, per (batch, query head), in the pages' order: scores s = scale * q.k
(scale rounded to fp32, inputs bf16 read exactly), causal mask (bottom-right),
then per split and key tile in order: tile row max; skip if every row is
negligible; otherwise the online-softmax update of the running max, the sum
and the accumulator.  Finally the splits are merged.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass
class DecodeResult:
    out: np.ndarray          # [B, Lq, Hq, d] float64
    lse: np.ndarray          # [B, Hq, Lq] float64 (natural log)
    skip_count: np.ndarray   # [B, Hq] int64
    skip_bits: np.ndarray    # [B, Hq, nK] bool: tile skipped (by its split)
    marginal: np.ndarray     # [B, Hq, nK] bool: the tile's largest row ratio within 1e-3 * lambda of lambda


def _as64(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().cpu().float().numpy()
    return np.asarray(t, dtype=np.float64)


def decode(q, k, v, *, causal: bool, scale: float, lam: float, Bc: int, num_splits: int,
           heads=None, margin_rel: float = 1e-3, flip=None) -> DecodeResult:
    """q [B, Lq, Hq, d], k/v [B, Lk, Hkv, d] (torch or numpy, bf16 values).

    ``heads``: optional list of (b, hq) to evaluate (others are left 0 / -inf).
    ``flip``: optional bool [B, Hq, nK]: key tiles whose skip decision is to be
    the other one; accepted only on marginal tiles (inside the tolerance band),
    else ValueError."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    scale = float(np.float32(scale))
    nK = -(-Lk // Bc)
    T = -(-nK // num_splits)
    out = np.zeros((B, Lq, Hq, d))
    lse = np.full((B, Hq, Lq), -np.inf)
    skip_count = np.zeros((B, Hq), dtype=np.int64)
    skip_bits = np.zeros((B, Hq, nK), dtype=bool)
    marginal = np.zeros((B, Hq, nK), dtype=bool)
    pos = np.arange(Lq) + (Lk - Lq)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, hq in todo:
        hkv = hq // G
        kb, vb = _as64(k[b, :, hkv, :]), _as64(v[b, :, hkv, :])     # [Lk, d]
        s = scale * (_as64(q[b, :, hq, :]) @ kb.T)                  # [Lq, Lk]
        if causal:
            s = np.where(np.arange(Lk)[None, :] > pos[:, None], -np.inf, s)
        parts = []
        for sp in range(num_splits):
            m = np.full(Lq, -np.inf)
            l = np.zeros(Lq)
            acc = np.zeros((Lq, d))
            for kt in range(sp * T, min(nK, (sp + 1) * T)):
                c0, c1 = kt * Bc, min(Lk, (kt + 1) * Bc)
                st = s[:, c0:c1]
                mt = st.max(axis=1)
                # the tile's margin quantity: its largest row ratio exp(mt - m)
                # (0 for a row with no key here, +inf for a row with no kept
                # key yet); skipped iff it is below lambda
                big = 0.0
                for i in range(Lq):
                    if mt[i] == -np.inf:
                        e = 0.0
                    elif m[i] == -np.inf:
                        e = math.inf
                    else:
                        e = math.exp(mt[i] - m[i])
                    big = max(big, e)
                marginal[b, hq, kt] = math.isfinite(big) and abs(big - lam) < margin_rel * lam
                skip = big < lam
                if flip is not None and flip[b, hq, kt]:
                    if not marginal[b, hq, kt]:
                        raise ValueError(f"flip of tile {kt} of {(b, hq)}: not marginal")
                    skip = not skip
                if skip:
                    skip_count[b, hq] += 1
                    skip_bits[b, hq, kt] = True
                    continue
                mn = np.maximum(m, mt)
                alpha = np.where(m == -np.inf, 0.0, np.exp(m - np.where(mn == -np.inf, 0.0, mn)))
                ref = np.where(mn == -np.inf, 0.0, mn)
                p = np.where(st == -np.inf, 0.0, np.exp(st - ref[:, None]))
                l = alpha * l + p.sum(axis=1)
                acc = alpha[:, None] * acc + p @ vb[c0:c1]
                m = mn
            parts.append((m, l, acc))
        # merge the splits: M = max of the splits' maxima (splits that kept a key)
        for i in range(Lq):
            ms = [pt[0][i] for pt in parts if pt[1][i] > 0]
            if not ms:
                continue
            M = max(ms)
            L = 0.0
            o = np.zeros(d)
            for mi, li, ai in parts:
                if li[i] > 0:
                    w = math.exp(mi[i] - M)
                    L += w * li[i]
                    o += w * ai[i]
            out[b, i, hq, :] = o / L
            lse[b, hq, i] = M + math.log(L)
    return DecodeResult(out, lse, skip_count, skip_bits, marginal)
