"""fp64 oracle of block-sparse attention with proxy compensation of the
omitted key blocks (numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Follows the PrimTS proxy-compensation pull request page (Description,
"Sol-Attn motivation and scope", "Bitmask format"): the key blocks a packed
bitmap selects (per batch, KV head and query block; one bit per KV block;
padding bits of the last word ignored) are computed exactly; every omitted
block is approximated by two caller-provided summaries, the arithmetic mean of
its keys and the sum of its values; the softmax denominator is corrected by
the number of tokens a summary stands for, the true length of a final partial
block included; a block that is computed exactly is not counted again through
its summary.

The page gives no formula.  Reading taken: for query row i and an omitted
block b of n_b keys the proxy score is s_ib = scale * q_i . kmean_b, and the
block contributes n_b * exp(s_ib) to the denominator and exp(s_ib) * vsum_b to
the numerator -- as if each of its n_b keys had the mean key (their values then
sum to vsum_b).  So the output is

    out_i = (sum_{j exact} e^{s_ij} v_j + sum_{b omitted} e^{s_ib} vsum_b)
            / (sum_{j exact} e^{s_ij}  + sum_{b omitted} n_b e^{s_ib})

and lse_i is the log of that denominator.  Non-causal only: the page's
summaries have no meaning for a block that is only partly visible.  No
skip-softmax in this mode (the exact blocks are exact).
"""
from __future__ import annotations

import math

import numpy as np


def _as64(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().cpu().float().numpy()
    return np.asarray(t, dtype=np.float64)


def block_summaries(k, v, Bc: int):
    """Per KV block of Bc keys (the last one possibly shorter): the mean of its
    keys and the sum of its values.  k, v [B, Lk, Hkv, d] -> two [B, nK, Hkv, d]."""
    kk, vv = _as64(k), _as64(v)
    B, Lk, Hkv, d = kk.shape
    nK = -(-Lk // Bc)
    kmean = np.zeros((B, nK, Hkv, d))
    vsum = np.zeros((B, nK, Hkv, d))
    for blk in range(nK):
        c0, c1 = blk * Bc, min(Lk, (blk + 1) * Bc)
        kmean[:, blk] = kk[:, c0:c1].sum(axis=1) / (c1 - c0)
        vsum[:, blk] = vv[:, c0:c1].sum(axis=1)
    return kmean, vsum


def block_selected(mask_words, b, hkv, qt, kt) -> bool:
    return bool((int(mask_words[b, hkv, qt, kt >> 5]) >> (kt & 31)) & 1)


def run(q, k, v, mask_words, kmean, vsum, *, scale: float, Br: int, Bc: int, items=None):
    """q [B, Lq, Hq, d], k/v [B, Lk, Hkv, d]; mask_words [B, Hkv, nQ, ceil(nK/32)]
    uint32; kmean / vsum [B, nK, Hkv, d] (any values: the caller's summaries).

    Returns (out [B, Lq, Hq, d], lse [B, Hq, Lq]) over ``items`` (b, hq, qt), all
    by default; other entries stay 0 / -inf."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    scale = float(np.float32(scale))
    nQ, nK = -(-Lq // Br), -(-Lk // Bc)
    km, vs = _as64(kmean), _as64(vsum)
    out = np.zeros((B, Lq, Hq, d))
    lse = np.full((B, Hq, Lq), -np.inf)
    if items is None:
        items = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(nQ)]
    qq = _as64(q)
    for b, hq, qt in items:
        hkv = hq // G
        kb, vb = _as64(k[b, :, hkv, :]), _as64(v[b, :, hkv, :])
        # the terms of the query block: every key of a selected block, one
        # (mean key, summed value, token count) term per omitted block
        exact_keys, proxy_blocks, n_b = [], [], []
        for blk in range(nK):
            c0, c1 = blk * Bc, min(Lk, (blk + 1) * Bc)
            if block_selected(mask_words, b, hkv, qt, blk):
                exact_keys.extend(range(c0, c1))
            else:
                proxy_blocks.append(blk)
                n_b.append(c1 - c0)
        ke, ve = kb[exact_keys], vb[exact_keys]
        kp, vp = km[b, proxy_blocks, hkv], vs[b, proxy_blocks, hkv]
        n_b = np.array(n_b, dtype=np.float64)
        for i in range(qt * Br, min(Lq, qt * Br + Br)):
            qi = qq[b, i, hq, :]
            # every term as a log weight and a value per unit of that weight:
            # an exact key: s_ij and v_j; a proxy: log n_b + s_ib and vsum_b / n_b
            logw = np.concatenate([scale * (ke @ qi), np.log(n_b) + scale * (kp @ qi)])
            vals = np.concatenate([ve, vp / n_b[:, None]])
            mx = logw.max()
            w = np.exp(logw - mx)
            den = float(w.sum())
            out[b, i, hq, :] = (w[:, None] * vals).sum(axis=0) / den
            lse[b, hq, i] = mx + math.log(den)
    return out, lse
