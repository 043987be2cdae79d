"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs.  Small shapes are compared on every work item (several
tiles, ragged tails, edge cases); the full workload sizes are compared on a
seeded sample of work items, in the same launch configuration the bench
times."""
import math

import numpy as np
import pytest
import torch

from parity_util import all_items, compare, gpu_run
from softmax_ssa_fwd_b200.inputs import MODE_DENSE, MODE_NM, MODE_SKIP, WORKLOADS, make_inputs, sample_items

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rand(B, Hq, Hkv, Lq, Lk, d, seed, sink_coef=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, Hq, d, generator=g)
    k = torch.randn(B, Lk, Hkv, d, generator=g)
    v = torch.randn(B, Lk, Hkv, d, generator=g)
    if sink_coef:
        u = torch.randn(d, generator=g)
        u /= u.norm()
        q += sink_coef * u
        k[:, :4] += sink_coef * u
    return [t.bfloat16().to(DEV) for t in (q, k, v)]


def _full(q, k, v, Br, **kw):
    B, Lq, Hq, _ = q.shape
    return compare(q, k, v, all_items(B, Hq, Lq, Br), Br=Br, **kw)


# ---------------------------------------------------------------- small, every item

@pytest.mark.parametrize("lam", [0.0, 1e-3, 1e-2])
@pytest.mark.parametrize("sink_coef", [3.0, 9.0, 12.0])
def test_tiny_workload(lam, sink_coef):
    w = WORKLOADS["tiny"].with_(sink_coef=sink_coef)
    q, k, v = make_inputs(w, DEV)
    rep = _full(q, k, v, w.Br, causal=True, scale=w.scale, mode=MODE_SKIP, lam=lam, Bc=w.Bc)
    if lam == 0.0:
        assert rep.skipped_gpu == 0
    if sink_coef == 12.0 and lam == 1e-2:
        assert rep.skipped_gpu > 0


SHAPES = [
    # B, Hq, Hkv, Lq, Lk, d, causal, Br, Bc
    (1, 4, 2, 300, 300, 128, True, 128, 128),    # ragged tail, GQA
    (2, 2, 2, 333, 333, 128, False, 128, 64),
    (1, 2, 1, 200, 450, 128, True, 128, 128),    # Lq < Lk, bottom-right causal
    (1, 2, 2, 300, 130, 64, True, 64, 64),       # Lq > Lk: first rows see nothing
    (1, 4, 1, 257, 257, 128, True, 64, 128),     # Br 64 with Bc 128
    (1, 2, 2, 257, 257, 64, True, 128, 64),
    (1, 2, 2, 1, 1, 64, True, 64, 64),           # single key
    (1, 1, 1, 64, 64, 128, False, 128, 128),     # one partial tile
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mode,lam", [(MODE_DENSE, 0.0), (MODE_SKIP, 1e-3), (MODE_SKIP, 5e-2),
                                      (MODE_SKIP, 2.0)])
def test_shapes(shape, mode, lam):
    B, Hq, Hkv, Lq, Lk, d, causal, Br, Bc = shape
    q, k, v = _rand(B, Hq, Hkv, Lq, Lk, d, seed=7, sink_coef=12.0)
    _full(q, k, v, Br, causal=causal, scale=1 / math.sqrt(d), mode=mode, lam=lam, Bc=Bc)


def test_lambda0_equals_dense_bitwise():
    q, k, v = _rand(1, 4, 2, 700, 700, 128, seed=3, sink_coef=12.0)
    a = gpu_run(q, k, v, causal=True, scale=0.08, mode=MODE_DENSE)
    b = gpu_run(q, k, v, causal=True, scale=0.08, mode=MODE_SKIP, lam=0.0)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert int(b[2].sum()) == 0


@pytest.mark.parametrize("n,m,sink,recent", [(2, 4, 4, 128), (4, 8, 0, 64), (1, 4, 0, 0),
                                             (3, 4, 7, 33), (7, 8, 4, 5), (1, 8, 16, 200)])
@pytest.mark.parametrize("d,Bc", [(128, 128), (64, 64)])
def test_nm_keep_masks_and_outputs(n, m, sink, recent, d, Bc):
    q, k, v = _rand(1, 4, 2, 520, 520, d, seed=11)
    k[:, 40:44] = k[:, 40:41]          # exact ties inside a group
    k[:, 301] = k[:, 300]
    _full(q, k, v, 128, causal=True, scale=1 / math.sqrt(d), mode=MODE_NM, n=n, m=m, sink=sink,
          recent=recent, Bc=Bc, keep_bits=True)


@pytest.mark.parametrize("m", [4, 8])
def test_nm_with_n_equal_m_is_dense_bitwise(m):
    q, k, v = _rand(1, 2, 2, 400, 400, 128, seed=5)
    a = gpu_run(q, k, v, causal=True, scale=0.088, mode=MODE_DENSE)
    b = gpu_run(q, k, v, causal=True, scale=0.088, mode=MODE_NM, n=m, m=m, sink=0, recent=0)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("lam", [1e-3, 3e-2, 1.5])
@pytest.mark.parametrize("n,m", [(2, 4), (4, 8)])
def test_skip_combined_with_nm(lam, n, m):
    q, k, v = _rand(2, 4, 2, 600, 600, 128, seed=9, sink_coef=12.0)
    rep = _full(q, k, v, 128, causal=True, scale=1 / math.sqrt(128), mode=MODE_SKIP | MODE_NM,
                lam=lam, n=n, m=m, sink=4, recent=128, keep_bits=True)
    assert rep.skipped_gpu > 0


# ---------------------------------------------------------------- full sizes, sampled items

def _sampled(w, lam, count, keep_bits=False):
    q, k, v = make_inputs(w, DEV)
    gpu = gpu_run(q, k, v, causal=w.causal, scale=w.scale, mode=w.mode, lam=lam, n=w.n, m=w.m,
                  sink=w.sink, recent=w.recent, Br=w.Br, Bc=w.Bc, keep_bits=keep_bits)
    # the bench's own (non-debug) entry point gives the same bytes
    from softmax_ssa_fwd_b200 import ssa
    o2, l2, c2 = ssa.attention(q, k, v, causal=w.causal, scale=w.scale, mode=w.mode, lam=lam,
                               n=w.n, m=w.m, sink=w.sink, recent=w.recent, Br=w.Br, Bc=w.Bc)
    torch.cuda.synchronize()
    assert torch.equal(o2, gpu[0]) and torch.equal(c2, gpu[2])
    items = sample_items(w, count)
    cpu = (q.cpu(), k.cpu(), v.cpu())
    rep = compare(q, k, v, items, causal=w.causal, scale=w.scale, mode=w.mode, lam=lam, n=w.n,
                  m=w.m, sink=w.sink, recent=w.recent, Br=w.Br, Bc=w.Bc, keep_bits=keep_bits,
                  gpu=gpu, qkv_cpu=cpu)
    return rep, gpu


@pytest.mark.parametrize("lam", [1e-4, 1e-3, 1e-2])
def test_llama8k_sampled(lam):
    rep, _ = _sampled(WORKLOADS["llama8k"], lam, 64)
    print(rep)


def test_llama8k_sink_strong_sampled():
    rep, _ = _sampled(WORKLOADS["llama8k"].with_(sink_coef=12.0), 1e-3, 64)
    assert rep.skipped_gpu > 0
    print(rep)


@pytest.mark.parametrize("name", ["llama4k_nm24", "llama4k_nm48"])
def test_llama4k_nm_sampled(name):
    rep, _ = _sampled(WORKLOADS[name], 0.0, 16, keep_bits=True)
    print(rep)


def test_wan_sampled():
    rep, _ = _sampled(WORKLOADS["wan"], 1e-3, 128)
    print(rep)


def test_wan_local_sampled():
    rep, _ = _sampled(WORKLOADS["wan"].with_(local_alpha=2.5), 1e-3, 128)
    assert rep.skipped_gpu > 0
    print(rep)


def test_qwen32k_sampled():
    # keep bits of the full problem: B * Hq * Lq * Lk / 32 words (8.6 GB), compared on the sampled items
    rep, _ = _sampled(WORKLOADS["qwen32k"], 1e-3, 96, keep_bits=True)
    assert rep.keep_bits_compared > 0
    print(rep)
