"""Host-side checks of the bench's bookkeeping (no GPU): FLOP counts, the
max-over-ranks timing and the whole-job rate, the latter on two gloo ranks."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from softmax_ssa_fwd_b200.inputs import WORKLOADS  # noqa: E402


def test_dense_equiv_flops_matches_pair_count():
    for name in ["tiny", "llama8k", "wan"]:
        w = WORKLOADS[name]
        L = w.L
        pairs = L * (L + 1) // 2 if w.causal else L * L
        assert bench.dense_equiv_flops(w) == 4.0 * w.d * w.B * w.Hq * pairs


def test_dense_equiv_flops_bottom_right_causal_small():
    w = WORKLOADS["tiny"].with_(L=37)
    i = np.arange(37)[:, None]
    j = np.arange(37)[None, :]
    assert bench.dense_equiv_flops(w) == 4.0 * w.d * w.B * w.Hq * int((j <= i).sum())


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = 10.0 + 5.0 * rank                       # the slower rank decides
    got = bench.reduce_max(ms, dist, torch.device("cpu"))
    rate = bench.job_rate(1000.0, world, got)
    q.put((rank, got, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, got, rate in res:
        assert got == 15.0
        assert rate == pytest.approx(world * 1000.0 / 15e-3)


def test_single_process_identity():
    assert bench.reduce_max(3.5, None, torch.device("cpu")) == 3.5
    assert bench.job_rate(10.0, 1, 2.0) == pytest.approx(5000.0)


def test_block_mask_helpers():
    import numpy as np
    import bench
    from oracle.blockmask import block_selected
    from softmax_ssa_fwd_b200.inputs import WORKLOADS
    w = WORKLOADS["llama8k"].with_(L=1000, Hq=4, Hkv=2)
    bits = bench.block_mask_bits(w, 0.3, seed=3)
    words = bench.pack_bits(bits)
    nQ, nK = bits.shape[2], bits.shape[3]
    for qt in range(nQ):
        last = min(nK - 1, (min(w.L, qt * w.Br + w.Br) - 1) // w.Bc)
        assert bits[:, :, qt, 0].all() and bits[:, :, qt, last].all()
        assert not bits[:, :, qt, last + 1:].any()
        for kt in range(nK):
            assert block_selected(words, 0, 1, qt, kt) == bits[0, 1, qt, kt]
