"""fp64 oracle of skip-softmax attention restricted to caller-selected key
blocks (numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"Skip-Softmax Sparse Attention for Diffusion Models" (intro, "Threshold
Modes") gives the tile skip; the block-sparse page of the same stack ("Bitmask
format" of the PrimTS proxy-compensation pull request) gives the selection
format: a packed uint32 bitmap per (batch, KV head, query block), one bit per
KV block, padding bits past the last block ignored.  Reading taken: a key
tile whose bit is clear is not visited at all (no scores, no exponentials, no
P.V, not counted); the skip-softmax recurrence runs over the selected visible
tiles in order.  Proxy compensation of the omitted blocks is not part of this.
"""
from __future__ import annotations

import math

import numpy as np


def _as64(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().cpu().float().numpy()
    return np.asarray(t, dtype=np.float64)


def block_selected(mask_words, b, hkv, qt, kt) -> bool:
    return bool((int(mask_words[b, hkv, qt, kt >> 5]) >> (kt & 31)) & 1)


def run(q, k, v, mask_words, *, causal: bool, scale: float, lam: float, Br: int, Bc: int,
        items=None, marginal=None, margin_rel: float = 1e-3, skip_bits=None, marginal_bits=None,
        flip=None):
    """q [B, Lq, Hq, d], k/v [B, Lk, Hkv, d]; mask_words [B, Hkv, nQ, ceil(nK/32)] uint32.

    Returns (out [B, Lq, Hq, d], lse [B, Hq, Lq], skip_count [B, Hq, nQ], visited [B, Hq, nQ])
    over ``items`` (b, hq, qt) (all by default); other entries stay 0 / -inf.  If
    ``marginal`` (an int array [B, Hq, nQ]) is given it receives, per query tile, the
    number of visited tiles whose largest row ratio exp(tile_max - running_max) lies within
    margin_rel * lambda of lambda.  ``skip_bits`` / ``marginal_bits`` (bool arrays
    [B, Hq, nQ, nK]), if given, receive per key tile the skip decision and that flag.
    ``flip`` (bool [B, Hq, nQ, nK]): key tiles whose decision is to be the other one;
    accepted only on marginal tiles, else ValueError."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    scale = float(np.float32(scale))
    nQ, nK = -(-Lq // Br), -(-Lk // Bc)
    out = np.zeros((B, Lq, Hq, d))
    lse = np.full((B, Hq, Lq), -np.inf)
    skips = np.zeros((B, Hq, nQ), dtype=np.int64)
    visited = np.zeros((B, Hq, nQ), dtype=np.int64)
    if items is None:
        items = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(nQ)]
    for b, hq, qt in items:
        hkv = hq // G
        r0, r1 = qt * Br, min(Lq, qt * Br + Br)
        rows = r1 - r0
        pos = np.arange(r0, r1) + (Lk - Lq)
        kb, vb = _as64(k[b, :, hkv, :]), _as64(v[b, :, hkv, :])
        s = scale * (_as64(q[b, r0:r1, hq, :]) @ kb.T)
        if causal:
            s = np.where(np.arange(Lk)[None, :] > pos[:, None], -np.inf, s)
        last = nK - 1
        if causal:
            last = min(nK - 1, int(pos[-1]) // Bc) if pos[-1] >= 0 else -1
        m = np.full(rows, -np.inf)
        l = np.zeros(rows)
        acc = np.zeros((rows, d))
        for kt in range(last + 1):
            if not block_selected(mask_words, b, hkv, qt, kt):
                continue
            visited[b, hq, qt] += 1
            c0, c1 = kt * Bc, min(Lk, (kt + 1) * Bc)
            st = s[:, c0:c1]
            mt = st.max(axis=1)
            # the tile's margin quantity: its largest row ratio exp(mt - m)
            # (0 for a row with no key here, +inf for a row with no kept key
            # yet); skipped iff it is below lambda
            big = 0.0
            for i in range(rows):
                if mt[i] == -np.inf:
                    e = 0.0
                elif m[i] == -np.inf:
                    e = math.inf
                else:
                    e = math.exp(mt[i] - m[i])
                big = max(big, e)
            near = math.isfinite(big) and abs(big - lam) < margin_rel * lam
            if near:
                if marginal is not None:
                    marginal[b, hq, qt] += 1
                if marginal_bits is not None:
                    marginal_bits[b, hq, qt, kt] = True
            skip = big < lam
            if flip is not None and flip[b, hq, qt, kt]:
                if not near:
                    raise ValueError(f"flip of tile {kt} of {(b, hq, qt)}: not marginal")
                skip = not skip
            if skip:
                skips[b, hq, qt] += 1
                if skip_bits is not None:
                    skip_bits[b, hq, qt, kt] = True
                continue
            mn = np.maximum(m, mt)
            ref = np.where(mn == -np.inf, 0.0, mn)
            alpha = np.where(m == -np.inf, 0.0, np.exp(m - ref))
            p = np.where(st == -np.inf, 0.0, np.exp(st - ref[:, None]))
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ vb[c0:c1]
            m = mn
        for i in range(rows):
            if l[i] > 0:
                out[b, r0 + i, hq, :] = acc[i] / l[i]
                lse[b, hq, r0 + i] = m[i] + math.log(l[i])
    return out, lse, skips, visited
