"""Build and call the plain-C fp64 oracle (``ssa_oracle.c``).

Test infrastructure only; see the package docstring.  Argument marshalling
only: every arithmetic step is in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssa_oracle.c")
_LIB = os.path.join(_HERE, "libssa_oracle.so")
_lib = None

MODE_SKIP = 1
MODE_NM = 2


def lib_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile ssa_oracle.c into libssa_oracle.so (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
               "-ffp-contract=off", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def bind(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    lib.ssa_oracle_items.restype = I
    lib.ssa_oracle_items.argtypes = [P, P, P, I, I, I, I, I, I, I, D, I, D, I, I, I, I, I, I, D,
                                     P, I, P, P, P, P, P, P, P, P, P, I]
    lib.ssa_oracle_visited_tiles.restype = I
    lib.ssa_oracle_visited_tiles.argtypes = [I, I, I, I, I, I]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = bind(_LIB)
    return _lib


def visited_tiles(causal: bool, Lq: int, Lk: int, Br: int, Bc: int, qt: int) -> int:
    return _load().ssa_oracle_visited_tiles(int(causal), Lq, Lk, Br, Bc, qt)


@dataclass
class OracleResult:
    items: np.ndarray        # [n, 3] int32 (b, hq, qt)
    out: np.ndarray          # [n, Br, d] float64
    lse: np.ndarray          # [n, Br] float64
    skip_count: np.ndarray   # [n] int32
    visited: np.ndarray      # [n] int32
    skip_bits: np.ndarray    # [n, nKw] uint32
    marginal_bits: np.ndarray  # [n, nKw] uint32
    keep_bits: np.ndarray | None  # [n, Br, Lkw] uint32
    tie_bits: np.ndarray | None   # [n, Br, Lkw] uint32


def _as_u16(t) -> np.ndarray:
    """Accept a torch bf16 CPU tensor or a uint16 numpy array of bf16 bits."""
    if isinstance(t, np.ndarray):
        a = t
    else:  # torch tensor
        import torch
        a = t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
    assert a.dtype == np.uint16
    return np.ascontiguousarray(a)


def run_items(q, k, v, *, causal: bool, scale: float, mode: int, lam: float = 0.0, n: int = 0,
              m: int = 0, sink: int = 0, recent: int = 0, Br: int = 128, Bc: int = 128,
              items=None, keep_bits: bool = False, tie_tol: float = 1e-4,
              nthreads: int | None = None, lib=None, flip_bits=None) -> OracleResult:
    """Run the oracle on work items (b, hq, qt); all items when ``items`` is None.

    q: [B, Lq, Hq, d], k, v: [B, Lk, Hkv, d], bf16 (torch) or their uint16 bits.
    ``scale`` is rounded to fp32 first, the precision the kernel receives it in.
    ``lib``: a library from ``bind`` to run instead of the built oracle (tests only).
    ``flip_bits`` [n_items, ceil(nK/32)] uint32: key tiles whose skip decision is
    to be the other one -- accepted only on tiles inside the tolerance band
    (marginal), else ValueError.
    """
    lib = lib if lib is not None else _load()
    qa, ka, va = _as_u16(q), _as_u16(k), _as_u16(v)
    B, Lq, Hq, d = qa.shape
    _, Lk, Hkv, _ = ka.shape
    nQ = -(-Lq // Br)
    nK = -(-Lk // Bc)
    if items is None:
        items = np.array([(b, h, t) for b in range(B) for h in range(Hq) for t in range(nQ)],
                         dtype=np.int32).reshape(-1, 3)
    items = np.ascontiguousarray(np.asarray(items, dtype=np.int32).reshape(-1, 3))
    nit = items.shape[0]
    nKw = -(-nK // 32)
    Lkw = -(-Lk // 32)
    out = np.zeros((nit, Br, d), np.float64)
    lse = np.zeros((nit, Br), np.float64)
    cnt = np.zeros(nit, np.int32)
    vis = np.zeros(nit, np.int32)
    sb = np.zeros((nit, nKw), np.uint32)
    mb = np.zeros((nit, nKw), np.uint32)
    kb = np.zeros((nit, Br, Lkw), np.uint32) if keep_bits else None
    tb = np.zeros((nit, Br, Lkw), np.uint32) if keep_bits else None
    if nthreads is None:
        nthreads = len(os.sched_getaffinity(0))
    fb = None
    if flip_bits is not None:
        fb = np.ascontiguousarray(np.asarray(flip_bits, dtype=np.uint32).reshape(nit, nKw))
    scale32 = float(np.float32(scale))
    ptr = lambda a: a.ctypes.data if a is not None else None  # noqa: E731
    rc = lib.ssa_oracle_items(ptr(qa), ptr(ka), ptr(va), B, Hq, Hkv, Lq, Lk, d, int(causal),
                              scale32, int(mode), float(lam), int(n), int(m), int(sink),
                              int(recent), Br, Bc, float(tie_tol), ptr(items), nit, ptr(out),
                              ptr(lse), ptr(cnt), ptr(vis), ptr(sb), ptr(mb), ptr(kb), ptr(tb),
                              ptr(fb), int(nthreads))
    if rc == -2:
        raise ValueError("flip_bits names a tile whose decision is not marginal")
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    return OracleResult(items, out, lse, cnt, vis, sb, mb, kb, tb)
