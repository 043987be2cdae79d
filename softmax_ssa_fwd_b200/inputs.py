"""Seeded synthetic Q/K/V generators and the workload table.

This module is shared by the tests (oracle side) and the bench (CUDA side).
It holds no arithmetic of the attention method: only random draws, rotary
position embeddings that shape the synthetic activations, and the shapes and
knobs of each workload.

Workloads (shapes from the pages' targets: Llama-3.1-8B / Qwen3-8B prefill in
"Attention Sparsity for HuggingFace Models", Wan 2.2 A14B video DiT in
"Skip-Softmax Sparse Attention for Diffusion Models"):

* ``tiny``        B=1 Hq=Hkv=2 L=256 d=64 causal Br=Bc=64, seed 0, lambda in {0, 1e-3, 1e-2}
* ``llama8k``     B=1 Hq=32 Hkv=8 L=8192 d=128 causal, RoPE base 5e5, seed 1,
                  lambda in {1e-4, 1e-3, 1e-2}
* ``llama4k_nm24`` / ``llama4k_nm48``  L=4096, seed 2, N:M 2:4 (sink 4, recent 128)
                  and 4:8 (sink 0, recent 64)
* ``wan``         B=1 H=40 L=75600 = 21x45x80 tokens, d=128, non-causal,
                  3D RoPE over (t, h, w), seed 3, lambda = 1e-3
* ``qwen32k``     B=2 Hq=32 Hkv=8 L=32768 d=128 causal, RoPE base 1e6, seed 4,
                  skip + N:M 2:4 (sink 4, recent 128), lambda = 1e-3
* ``sol_proxy``   B=1 H=12 L=32760 d=128 non-causal, Br=Bc=64, seed 6: key
                  blocks selected by bitmap (84 of 512 per query block, seeded
                  at random), the others through proxy summaries
* ``qwen32k_decode``  decode: B=8 sequences, one new query row each (the last
                  position) against L=32768 cached keys, Hq=32 Hkv=8 d=128,
                  RoPE base 1e6, seed 5, lambda = 1e-4 (the pages' decode
                  threshold), 16 key splits

Recipe: one torch.Generator per workload seeded as listed.  Draw u ~ N(0, I_d)
and normalise it (a unit "sink direction" shared by every head), then Q, K, V
~ N(0, 1) in fp32.  Apply rotary embeddings to Q and K (rotate-half pairs
(c, c + d/2), positions 0..L-1), then add ``sink_coef * u`` to every query and
to keys 0..3, then round to bf16.  ``wan`` uses a 3D rotary split of the d/2
pairs into 22/21/21 for (t, h, w), base 1e4 per axis, and no sink direction.

Stress variants (labelled, not the literal workloads): ``sink_coef=12``
makes most non-sink tiles negligible; ``local_alpha=2.5`` adds a per-head
shared vector alpha * a_h to Q and K before the 3D rotary embedding, which makes
the video attention spatio-temporally local.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

MODE_DENSE = 0
MODE_SKIP = 1
MODE_NM = 2


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    causal: bool
    Br: int
    Bc: int
    mode: int
    lambdas: tuple
    n: int = 0
    m: int = 0
    sink: int = 0
    recent: int = 0
    seed: int = 0
    rope: str = "none"          # "none" | "1d" | "3d"
    rope_base: float = 10000.0
    sink_coef: float = 3.0      # coefficient of the shared unit direction u
    local_alpha: float = 0.0    # per-head shared pre-rotary vector (3d only)
    grid: tuple = ()            # (T, H, W) for the 3d rotary embedding
    Lq: int = 0                 # decode: query rows (the last Lq positions); 0 = L (prefill)
    splits: int = 0             # decode: key splits

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 256, 64, True, 64, 64, MODE_SKIP, (0.0, 1e-3, 1e-2),
                     seed=0),
    "llama8k": Workload("llama8k", 1, 32, 8, 8192, 128, True, 128, 128, MODE_SKIP,
                        (1e-4, 1e-3, 1e-2), seed=1, rope="1d", rope_base=5e5),
    "llama4k_nm24": Workload("llama4k_nm24", 1, 32, 8, 4096, 128, True, 128, 128, MODE_NM, (0.0,),
                             n=2, m=4, sink=4, recent=128, seed=2, rope="1d", rope_base=5e5),
    "llama4k_nm48": Workload("llama4k_nm48", 1, 32, 8, 4096, 128, True, 128, 128, MODE_NM, (0.0,),
                             n=4, m=8, sink=0, recent=64, seed=2, rope="1d", rope_base=5e5),
    "wan": Workload("wan", 1, 40, 40, 75600, 128, False, 128, 128, MODE_SKIP, (1e-3,), seed=3,
                    rope="3d", rope_base=1e4, sink_coef=0.0, grid=(21, 45, 80)),
    "qwen32k": Workload("qwen32k", 2, 32, 8, 32768, 128, True, 128, 128, MODE_SKIP | MODE_NM,
                        (1e-3,), n=2, m=4, sink=4, recent=128, seed=4, rope="1d", rope_base=1e6),
    # block-sparse attention with proxy compensation, the shape of the PrimTS
    # page's B200 measurement: [1, 32760, 12, 128], Q / KV blocks of 64, 84 of
    # 512 key blocks exact per query block (no skip-softmax, non-causal)
    "sol_proxy": Workload("sol_proxy", 1, 12, 12, 32760, 128, False, 64, 64, MODE_DENSE, (0.0,), seed=6,
                          sink_coef=0.0),
    # decode phase: one new token per sequence against a 32k cache, 8 sequences,
    # the pages' decode threshold 1e-4; no N:M (prefill only)
    "qwen32k_decode": Workload("qwen32k_decode", 8, 32, 8, 32768, 128, True, 128, 128, MODE_SKIP,
                               (1e-4,), seed=5, rope="1d", rope_base=1e6, Lq=1, splits=16),
}


def _rotate(x: torch.Tensor, ang: torch.Tensor) -> torch.Tensor:
    """Rotate-half rotary embedding. x: [B, L, H, d]; ang: [L, d/2] radians."""
    h = x.shape[-1] // 2
    c = torch.cos(ang)[None, :, None, :]
    s = torch.sin(ang)[None, :, None, :]
    x1, x2 = x[..., :h], x[..., h:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def _angles_1d(L: int, d: int, base: float, device) -> torch.Tensor:
    pairs = torch.arange(d // 2, dtype=torch.float64, device=device)
    inv = base ** (-2.0 * pairs / d)
    pos = torch.arange(L, dtype=torch.float64, device=device)
    return (pos[:, None] * inv[None, :]).to(torch.float32)


def _angles_3d(grid, d: int, base: float, device) -> torch.Tensor:
    T, H, W = grid
    npair = d // 2
    nt = npair - 2 * (npair // 3)     # 22 / 21 / 21 for d = 128
    nh = nw = npair // 3
    idx = torch.arange(T * H * W, device=device, dtype=torch.int64)
    pt, ph, pw = idx // (H * W), (idx // W) % H, idx % W
    cols = []
    for p, cnt in ((pt, nt), (ph, nh), (pw, nw)):
        j = torch.arange(cnt, dtype=torch.float64, device=device)
        inv = base ** (-j / cnt)
        cols.append(p.to(torch.float64)[:, None] * inv[None, :])
    return torch.cat(cols, dim=1).to(torch.float32)


def make_inputs(w: Workload, device="cpu"):
    """Return (q, k, v) bf16 tensors: q [B, Lq, Hq, d] (Lq = L unless the
    workload is a decode one), k and v [B, L, Hkv, d]."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    B, L, d = w.B, w.L, w.d
    u = torch.randn(d, generator=g, device=dev, dtype=torch.float32)
    u = u / u.norm()
    Lq = w.Lq if 0 < w.Lq < L else L  # decode: queries at the last Lq positions
    q = torch.randn(B, Lq, w.Hq, d, generator=g, device=dev, dtype=torch.float32)
    k = torch.randn(B, L, w.Hkv, d, generator=g, device=dev, dtype=torch.float32)
    v = torch.randn(B, L, w.Hkv, d, generator=g, device=dev, dtype=torch.float32)
    if w.local_alpha:
        a = torch.randn(w.Hkv, d, generator=g, device=dev, dtype=torch.float32)
        q += w.local_alpha * a.repeat_interleave(w.Hq // w.Hkv, dim=0)[None, None]
        k += w.local_alpha * a[None, None]
    if w.rope == "1d":
        ang = _angles_1d(L, d, w.rope_base, dev)
        q, k = _rotate(q, ang[L - Lq:]), _rotate(k, ang)
    elif w.rope == "3d":
        ang = _angles_3d(w.grid, d, w.rope_base, dev)
        q, k = _rotate(q, ang[L - Lq:]), _rotate(k, ang)
    if w.sink_coef:
        q += w.sink_coef * u
        k[:, :4] += w.sink_coef * u
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def sample_items(w: Workload, count: int, seed: int = 1234, Lq: int | None = None):
    """Seeded sample of (b, hq, qt) work items, always including the first and
    last query tile and, for causal workloads, a few long (late) tiles."""
    Lq = Lq or w.L
    nQ = -(-Lq // w.Br)
    g = torch.Generator().manual_seed(seed)
    fixed = [(0, 0, 0), (w.B - 1, w.Hq - 1, nQ - 1), (0, w.Hq // 2, nQ // 2)]
    rnd = [(int(torch.randint(w.B, (1,), generator=g)), int(torch.randint(w.Hq, (1,), generator=g)),
            int(torch.randint(nQ, (1,), generator=g))) for _ in range(max(0, count - len(fixed)))]
    seen, out = set(), []
    for it in fixed + rnd:
        if it not in seen:
            seen.add(it)
            out.append(it)
    return out[:count]
