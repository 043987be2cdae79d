"""GPU parity of ssa_fwd_blockmask_proxy (selected key blocks exact, the
omitted ones through the caller's mean-K / summed-V summaries) against the
fp64 proxy oracle (oracle/proxy.py) on the same seeded bf16 inputs and the
same bf16 summaries: outputs max-abs <= 2e-2 and relative L2 <= 5e-3, lse
max-abs <= 1e-3, on every row.  Cases cover ragged last key blocks (the final
summary stands for fewer keys), a ragged query tail, 64-row query tiles, GQA,
masks selecting every block (= ssa_fwd_blockmask, exact attention) or none
(proxies only), and the shape of the page's benchmark at reduced length."""
import numpy as np
import pytest
import torch

from oracle.proxy import run as proxy_run

pytestmark = pytest.mark.gpu

OUT_MAX_ABS, OUT_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3


def _gen(B, Hq, Hkv, Lq, Lk, d, seed, local=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, Hq, d, generator=g)
    k = torch.randn(B, Lk, Hkv, d, generator=g)
    v = torch.randn(B, Lk, Hkv, d, generator=g)
    if local:
        # a shared direction per head makes some key blocks matter more
        a = torch.randn(Hkv, d, generator=g)
        q += local * a.repeat_interleave(Hq // Hkv, dim=0)[None, None]
        k += local * a[None, None]
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def summaries(k, v, Bc):
    """Caller-side summaries (bf16): mean of each key block's keys, sum of its values."""
    B, Lk, Hkv, d = k.shape
    nK = -(-Lk // Bc)
    km = torch.zeros(B, nK, Hkv, d)
    vs = torch.zeros(B, nK, Hkv, d)
    for blk in range(nK):
        c0, c1 = blk * Bc, min(Lk, blk * Bc + Bc)
        km[:, blk] = k[:, c0:c1].double().mean(dim=1).float()
        vs[:, blk] = v[:, c0:c1].double().sum(dim=1).float()
    return km.bfloat16(), vs.bfloat16()


def _mask(B, Hkv, nQ, nK, density, seed, full=False, empty=False):
    rng = np.random.default_rng(seed)
    nKw = -(-nK // 32)
    bits = rng.random((B, Hkv, nQ, nKw * 32)) < density
    if full:
        bits[:] = True
    if empty:
        bits[:] = False
    words = np.zeros((B, Hkv, nQ, nKw), dtype=np.uint32)
    for i in range(32):
        words |= bits[..., i::32].astype(np.uint32) << np.uint32(i)
    return words  # padding bits past nK are random on purpose: they must be ignored


CASES = [
    # B, Hq, Hkv, Lq, Lk, d, Br, Bc, density, extra
    (1, 4, 2, 640, 1000, 128, 128, 128, 0.3, {}),         # ragged last key block (1000 = 7 x 128 + 104)
    (2, 4, 4, 300, 513, 128, 128, 64, 0.5, {}),           # last block of one key, ragged query tail
    (1, 8, 2, 512, 777, 64, 64, 64, 0.2, {}),             # 64-row query tiles, d = 64
    (1, 4, 2, 384, 384, 128, 128, 128, 0.4, {"local": 2.0}),
    (1, 4, 2, 500, 900, 128, 128, 128, 0.0, {"empty": True}),   # no exact block: proxies only
    (1, 4, 2, 300, 700, 128, 128, 128, 1.0, {"full": True}),    # every block exact: no proxy
    (1, 12, 12, 1024, 4095, 128, 64, 64, 84 / 512, {}),   # the page's benchmark shape, shorter
]


@pytest.mark.parametrize("case", CASES)
def test_proxy_matches_oracle(case):
    from softmax_ssa_fwd_b200 import ssa
    B, Hq, Hkv, Lq, Lk, d, Br, Bc, dens, extra = case
    q, k, v = _gen(B, Hq, Hkv, Lq, Lk, d, seed=Lq + Lk, local=extra.get("local", 0.0))
    nQ, nK = -(-Lq // Br), -(-Lk // Bc)
    words = _mask(B, Hkv, nQ, nK, dens, seed=Lk, full=extra.get("full", False),
                  empty=extra.get("empty", False))
    km, vs = summaries(k, v, Bc)
    scale = d ** -0.5
    mt = torch.from_numpy(words.view(np.int32)).cuda()
    out, lse = ssa.attention_blockmask_proxy(q.cuda(), k.cuda(), v.cuda(), mt, km.cuda(), vs.cuda(),
                                             scale=scale, Br=Br, Bc=Bc)
    torch.cuda.synchronize()
    assert ssa.ssa_device_status() == ssa.SSA_OK
    ro, rl = proxy_run(q, k, v, words, km, vs, scale=scale, Br=Br, Bc=Bc)
    o = out.float().cpu().numpy()
    diff = o - ro
    assert np.abs(diff).max() <= OUT_MAX_ABS, np.abs(diff).max()
    assert np.sqrt((diff ** 2).sum() / max((ro ** 2).sum(), 1e-30)) <= OUT_REL_L2
    ls = lse.cpu().numpy()
    assert np.isfinite(ls).all() and np.isfinite(rl).all()
    assert np.abs(ls - rl).max() <= LSE_MAX_ABS, np.abs(ls - rl).max()
    if extra.get("full"):
        # every block exact: the same bytes as the exact-block path with nothing skipped
        o2, l2, _ = ssa.attention_blockmask(q.cuda(), k.cuda(), v.cuda(), mt, causal=False, scale=scale,
                                            mode=ssa.MODE_DENSE, Br=Br, Bc=Bc)
        torch.cuda.synchronize()
        assert torch.equal(o2, out) and torch.equal(l2, lse)
