"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/ssa.h declares, and rejects bad arguments
synchronously with the documented status codes before touching CUDA."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssa.h")


@pytest.fixture(scope="module")
def ssa():
    from softmax_ssa_fwd_b200 import build
    build.build()
    from softmax_ssa_fwd_b200 import ssa as mod
    return mod


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    assert _declared_functions() == sorted(
        ["ssa_fwd", "ssa_fwd_debug", "ssa_fwd_noalloc", "ssa_visited_tiles",
         "ssa_set_wait_timeout_ns", "ssa_device_status", "ssa_status_string", "ssa_version",
         "ssa_decode", "ssa_decode_debug", "ssa_decode_workspace_bytes", "ssa_decode_default_splits",
         "ssa_fwd_blockmask", "ssa_fwd_blockmask_debug", "ssa_fwd_blockmask_proxy"])


def test_library_exports_every_declared_symbol(ssa):
    lib = ctypes.CDLL(ssa.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(_declared_functions()) <= set(ssa.EXPORTED)


def test_status_strings_and_version(ssa):
    assert ssa.status_string(0) == "SSA_OK"
    assert ssa.status_string(-1) == "SSA_ERR_INVALID_ARG"
    assert ssa.status_string(-2) == "SSA_ERR_UNSUPPORTED"
    assert ssa.status_string(-3) == "SSA_ERR_CUDA"
    assert ssa.status_string(-4) == "SSA_ERR_TIMEOUT"
    assert ssa.status_string(7) == "SSA_ERR_UNKNOWN"
    assert ssa.ssa_version() >= 100


def _call(ssa, **over):
    a = dict(q=0x1000, k=0x2000, v=0x3000, out=0x4000, lse=0x5000, cnt=0x6000, B=1, Hq=4, Hkv=2,
             Lq=256, Lk=256, d=128, causal=1, scale=0.088, mode=1, lam=1e-3, n=2, m=4, sink=4,
             recent=128, Br=128, Bc=128)
    a.update(over)
    return ssa.ssa_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["cnt"], a["B"], a["Hq"], a["Hkv"],
                       a["Lq"], a["Lk"], a["d"], a["causal"], a["scale"], a["mode"], a["lam"], a["n"],
                       a["m"], a["sink"], a["recent"], a["Br"], a["Bc"], None)


@pytest.mark.parametrize("over", [
    dict(q=0), dict(k=0), dict(v=0), dict(out=0), dict(lse=0), dict(cnt=0),
    dict(B=0), dict(Hq=0), dict(Hkv=0), dict(Lq=0), dict(Lk=-3), dict(d=0),
    dict(Hq=6, Hkv=4), dict(scale=0.0), dict(scale=float("nan")), dict(scale=float("inf")),
    dict(lam=-1.0), dict(lam=float("nan")), dict(lam=float("inf")), dict(mode=4), dict(mode=-1),
    dict(mode=2, sink=-1), dict(mode=3, recent=-5), dict(q=0x1008), dict(cnt=0x6002),
    dict(lse=0x5004),
])
def test_invalid_arguments(ssa, over):
    assert _call(ssa, **over) == ssa.SSA_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [
    dict(d=96), dict(d=256), dict(Br=32), dict(Bc=256), dict(mode=2, m=2, n=1),
    dict(mode=2, m=4, n=0), dict(mode=2, m=4, n=5), dict(mode=3, m=8, n=9), dict(mode=2, m=16, n=4),
])
def test_unsupported_arguments(ssa, over):
    assert _call(ssa, **over) == ssa.SSA_ERR_UNSUPPORTED


def test_disabled_mode_parameters_are_ignored(ssa):
    # lambda is not checked when SKIP is off, nor n/m when N:M is off; with a
    # valid shape the call proceeds to CUDA, which fails only for lack of a GPU.
    import torch
    st = _call(ssa, mode=0, lam=-1.0, n=0, m=3)
    if torch.cuda.is_available():
        pytest.skip("needs the no-GPU path")
    assert st == ssa.SSA_ERR_CUDA


@pytest.mark.parametrize("causal,Lq,Lk,Br,Bc", [
    (1, 8192, 8192, 128, 128), (0, 75600, 75600, 128, 128), (1, 256, 256, 64, 64),
    (1, 300, 1000, 64, 128), (1, 1000, 300, 128, 64), (1, 32768, 32768, 128, 128), (1, 1, 1, 64, 64),
])
def test_visited_tiles_matches_oracle(ssa, causal, Lq, Lk, Br, Bc):
    from oracle import visited_tiles
    nQ = math.ceil(Lq / Br)
    want = sum(visited_tiles(causal, Lq, Lk, Br, Bc, t) for t in range(nQ))
    assert ssa.ssa_visited_tiles(causal, Lq, Lk, Br, Bc) == want


def test_visited_tiles_closed_forms(ssa):
    assert ssa.ssa_visited_tiles(1, 8192, 8192, 128, 128) == 64 * 65 // 2
    assert ssa.ssa_visited_tiles(0, 75600, 75600, 128, 128) == 591 * 591
    assert ssa.ssa_visited_tiles(1, 256, 256, 64, 64) == 10
    assert ssa.ssa_visited_tiles(1, 0, 5, 64, 64) == -1


def _dcall(ssa, **over):
    a = dict(q=0x1000, k=0x2000, v=0x3000, out=0x4000, lse=0x5000, cnt=0x6000, B=2, Hq=8, Hkv=2,
             Lq=1, Lk=4096, d=128, causal=1, scale=0.088, lam=1e-4, Bc=128, splits=4, ws=0x7000,
             wsb=None)
    a.update(over)
    wsb = a["wsb"] if a["wsb"] is not None else ssa.ssa_decode_workspace_bytes(a["B"], a["Hq"], a["Lq"], a["d"],
                                                                               max(a["splits"], 1))
    return ssa.lib.ssa_decode(a["q"], a["k"], a["v"], a["out"], a["lse"], a["cnt"], a["B"], a["Hq"],
                              a["Hkv"], a["Lq"], a["Lk"], a["d"], a["causal"], a["scale"], a["lam"],
                              a["Bc"], a["splits"], a["ws"], wsb, None)


@pytest.mark.parametrize("over", [
    dict(q=0), dict(v=0), dict(ws=0), dict(cnt=0), dict(B=0), dict(Lk=0), dict(splits=0),
    dict(Hq=6, Hkv=4), dict(scale=0.0), dict(lam=-1.0), dict(lam=float("nan")), dict(k=0x2004),
    dict(wsb=16),
])
def test_decode_invalid_arguments(ssa, over):
    assert _dcall(ssa, **over) == ssa.SSA_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [dict(d=96), dict(Bc=32), dict(Lq=9), dict(Hq=64, Hkv=1)])
def test_decode_unsupported_arguments(ssa, over):
    assert _dcall(ssa, **over) == ssa.SSA_ERR_UNSUPPORTED


def test_decode_workspace_bytes(ssa):
    # four partial results per row and split (fp32 accumulator of d, then
    # (max, sum)), then the skip counts per (batch, head, split)
    assert ssa.ssa_decode_workspace_bytes(8, 32, 1, 128, 16) == 8 * 32 * 16 * 4 * (128 * 4 + 8) + 8 * 32 * 16 * 4
    assert ssa.ssa_decode_workspace_bytes(0, 32, 1, 128, 16) == 0


def _busiest_cta_tiles(pairs, nK, s, sms):
    """Key tiles (plus one per split) walked by the busiest CTA when the
    pairs * s work items are handed to sms CTAs round-robin."""
    T = -(-nK // s)
    load = [0] * sms
    for it in range(pairs * s):
        sp = it % s
        nt = max(0, min(nK, (sp + 1) * T) - sp * T)
        load[it % sms] += nt + (1 if nt else 0)
    return max(load)


@pytest.mark.parametrize("B,Hkv,Lk,Bc,sms", [(8, 8, 32768, 128, 148), (1, 8, 4096, 128, 148),
                                             (1, 1, 1000, 64, 148), (64, 8, 8192, 128, 148),
                                             (2, 4, 300000, 128, 132)])
def test_decode_default_splits_balances_the_persistent_grid(ssa, B, Hkv, Lk, Bc, sms):
    nK = -(-Lk // Bc)
    s = ssa.ssa_decode_default_splits(B, Hkv, Lk, Bc, sms)
    assert 1 <= s <= min(nK, 256)
    T = -(-nK // s)
    assert -(-nK // T) == s  # no split is left empty
    # the busiest CTA, simulated item by item, is within 10 % of the best count's
    best = min(_busiest_cta_tiles(B * Hkv, nK, c, sms) for c in range(1, min(nK, 256) + 1))
    assert _busiest_cta_tiles(B * Hkv, nK, s, sms) <= 1.10 * best


def test_decode_default_splits_rejects_bad_arguments(ssa):
    assert ssa.ssa_decode_default_splits(0, 8, 4096, 128, 148) == 0
    assert ssa.ssa_decode_default_splits(1, 8, 4096, 32, 148) == 0
    assert ssa.ssa_decode_default_splits(1, 8, 4096, 128, 0) == 0
    # (sequence, KV head) pairs that fill the GPU evenly: no split
    assert ssa.ssa_decode_default_splits(37, 8, 4096, 128, 148) == 1


def test_blockmask_argument_checks(ssa):
    base = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 1, 4, 2, 256, 256, 128, 1, 0.088, 1,
            1e-3, 2, 4, 4, 128, 128, 128)
    assert ssa.lib.ssa_fwd_blockmask(*base, None, None) == ssa.SSA_ERR_INVALID_ARG      # no mask
    assert ssa.lib.ssa_fwd_blockmask(*base, 0x7002, None) == ssa.SSA_ERR_INVALID_ARG    # misaligned
    long = base[:10] + (2049 * 128,) + base[11:]
    assert ssa.lib.ssa_fwd_blockmask(*long, 0x7000, None) == ssa.SSA_ERR_UNSUPPORTED   # > 2048 key tiles


def test_debug_outputs_argument_checks(ssa):
    base = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 1, 4, 2, 256, 256, 128, 1, 0.088, 1,
            1e-3, 2, 4, 4, 128, 128, 128)
    # misaligned 32-bit evidence outputs are refused before anything runs
    assert ssa.lib.ssa_fwd_debug(*base, None, 0x7002, None, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_fwd_debug(*base, None, None, 0x7001, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_fwd_debug(*base, None, None, None, 0x7003) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_fwd_blockmask_debug(*base, 0x7000, None, 0x8002, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_fwd_blockmask_debug(*base, 0x7000, None, None, 0x8002) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_fwd_blockmask_debug(*base, None, None, 0x8000, None) == ssa.SSA_ERR_INVALID_ARG
    dec = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 2, 8, 2, 1, 4096, 128, 1, 0.088, 1e-4, 128,
           4, 0x7000, ssa.ssa_decode_workspace_bytes(2, 8, 1, 128, 4), None)
    assert ssa.lib.ssa_decode_debug(*dec, None) == ssa.SSA_ERR_INVALID_ARG          # no skip bits
    assert ssa.lib.ssa_decode_debug(*dec, 0x9002) == ssa.SSA_ERR_INVALID_ARG        # misaligned
    bad_cnt = dec[:5] + (0x6002,) + dec[6:]
    assert ssa.lib.ssa_decode(*bad_cnt) == ssa.SSA_ERR_INVALID_ARG


def test_proxy_argument_checks(ssa):
    base = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 1, 4, 2, 256, 256, 128, 0.088, 128, 128)
    f = ssa.lib.ssa_fwd_blockmask_proxy
    assert f(*base, None, 0x7000, 0x8000, None) == ssa.SSA_ERR_INVALID_ARG      # no mask
    assert f(*base, 0x6000, None, 0x8000, None) == ssa.SSA_ERR_INVALID_ARG      # no kmean
    assert f(*base, 0x6000, 0x7000, None, None) == ssa.SSA_ERR_INVALID_ARG      # no vsum
    assert f(*base, 0x6000, 0x7008, 0x8000, None) == ssa.SSA_ERR_INVALID_ARG    # misaligned kmean
    assert f(*base, 0x6000, 0x7000, 0x8004, None) == ssa.SSA_ERR_INVALID_ARG    # misaligned vsum
    bad_d = base[:10] + (96,) + base[11:]
    assert f(*bad_d, 0x6000, 0x7000, 0x8000, None) == ssa.SSA_ERR_UNSUPPORTED
