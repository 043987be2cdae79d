"""Thin ctypes binding of libssa (include/ssa.h): argument marshalling only.

Every step of the attention runs in the CUDA kernels behind the C ABI.  The
binding raises if the library cannot be loaded; there is no CPU fallback.
Functions keep the C names; tensors are passed as torch CUDA tensors (their
device pointers are handed to the library) and the stream defaults to torch's
current stream.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssa.so")

SSA_OK = 0
SSA_ERR_INVALID_ARG = -1
SSA_ERR_UNSUPPORTED = -2
SSA_ERR_CUDA = -3
SSA_ERR_TIMEOUT = -4
MODE_DENSE, MODE_SKIP, MODE_NM = 0, 1, 2

EXPORTED = ["ssa_fwd", "ssa_fwd_debug", "ssa_fwd_noalloc", "ssa_visited_tiles",
            "ssa_set_wait_timeout_ns", "ssa_device_status", "ssa_status_string", "ssa_version",
            "ssa_decode", "ssa_decode_debug", "ssa_decode_workspace_bytes", "ssa_decode_default_splits",
            "ssa_fwd_blockmask", "ssa_fwd_blockmask_debug", "ssa_fwd_blockmask_proxy"]


class SSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libssa.so not built at {LIB_PATH}; run softmax_ssa_fwd_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fwd_args = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, F, I, I, I, I, I, I, P]
    lib.ssa_fwd.restype = I
    lib.ssa_fwd.argtypes = fwd_args
    lib.ssa_fwd_debug.restype = I
    lib.ssa_fwd_debug.argtypes = fwd_args + [P, P, P]
    lib.ssa_fwd_noalloc.restype = I
    lib.ssa_fwd_noalloc.argtypes = fwd_args
    lib.ssa_visited_tiles.restype = ctypes.c_int64
    lib.ssa_visited_tiles.argtypes = [I, I, I, I, I]
    lib.ssa_set_wait_timeout_ns.restype = None
    lib.ssa_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.ssa_device_status.restype = I
    lib.ssa_device_status.argtypes = [P]
    lib.ssa_status_string.restype = ctypes.c_char_p
    lib.ssa_status_string.argtypes = [I]
    lib.ssa_version.restype = I
    lib.ssa_version.argtypes = []
    lib.ssa_fwd_blockmask.restype = I
    lib.ssa_fwd_blockmask.argtypes = fwd_args[:-1] + [P, P]
    lib.ssa_fwd_blockmask_debug.restype = I
    lib.ssa_fwd_blockmask_debug.argtypes = fwd_args[:-1] + [P, P, P, P]
    lib.ssa_fwd_blockmask_proxy.restype = I
    lib.ssa_fwd_blockmask_proxy.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, P, P, P]
    lib.ssa_decode.restype = I
    lib.ssa_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, F, I, I, P, ctypes.c_size_t, P]
    lib.ssa_decode_debug.restype = I
    lib.ssa_decode_debug.argtypes = lib.ssa_decode.argtypes + [P]
    lib.ssa_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.ssa_decode_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.ssa_decode_default_splits.restype = I
    lib.ssa_decode_default_splits.argtypes = [I, I, I, I, I]
    return lib


lib = _load()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return stream


def status_string(status: int) -> str:
    return lib.ssa_status_string(int(status)).decode()


def ssa_version() -> int:
    return lib.ssa_version()


def ssa_visited_tiles(causal, Lq, Lk, Br, Bc) -> int:
    return int(lib.ssa_visited_tiles(int(causal), Lq, Lk, Br, Bc))


def ssa_set_wait_timeout_ns(ns: int) -> None:
    """Limit of each in-kernel pipeline wait (0 = default 2 s); a test knob."""
    lib.ssa_set_wait_timeout_ns(int(ns))


def ssa_device_status(stream=None) -> int:
    return lib.ssa_device_status(_stream(stream))


def ssa_fwd(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode, lam,
            n, m, sink, recent, Br, Bc, stream=None) -> int:
    """Direct call of the C entry point; returns its status code."""
    return lib.ssa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(tile_skip_count),
                       B, Hq, Hkv, Lq, Lk, d, int(causal), float(scale), int(mode), float(lam),
                       int(n), int(m), int(sink), int(recent), Br, Bc, _stream(stream))


def ssa_fwd_noalloc(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                    lam, n, m, sink, recent, Br, Bc, stream=None) -> int:
    """The allocation-free entry point (see include/ssa.h); returns its status code."""
    return lib.ssa_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                               _ptr(tile_skip_count), B, Hq, Hkv, Lq, Lk, d, int(causal),
                               float(scale), int(mode), float(lam), int(n), int(m), int(sink),
                               int(recent), Br, Bc, _stream(stream))


def ssa_fwd_debug(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                  lam, n, m, sink, recent, Br, Bc, stream=None, skip_bits=None, keep_bits=None,
                  v_tile_loads=None) -> int:
    return lib.ssa_fwd_debug(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(tile_skip_count),
                             B, Hq, Hkv, Lq, Lk, d, int(causal), float(scale), int(mode), float(lam),
                             int(n), int(m), int(sink), int(recent), Br, Bc, _stream(stream),
                             _ptr(skip_bits), _ptr(keep_bits), _ptr(v_tile_loads))


def attention(q, k, v, *, causal=True, scale=None, mode=MODE_SKIP, lam=0.0, n=0, m=0, sink=0,
              recent=0, Br=128, Bc=128, stream=None, out=None, lse=None, counts=None,
              skip_bits=None, keep_bits=None, v_tile_loads=None):
    """Allocate outputs (torch) and run the forward through the C ABI.

    q [B, Lq, Hq, d], k/v [B, Lk, Hkv, d] bf16 CUDA tensors.  Returns
    (out [B, Lq, Hq, d] bf16, lse [B, Hq, Lq] fp32, tile_skip_count [B, Hq, nQ] int32).
    """
    B, Lq, Hq, d = q.shape
    _, Lk, Hkv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    nQ = -(-Lq // Br)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device=q.device)
    if counts is None:
        counts = torch.empty(B, Hq, nQ, dtype=torch.int32, device=q.device)
    if skip_bits is None and keep_bits is None and v_tile_loads is None:
        st = ssa_fwd(q, k, v, out, lse, counts, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode, lam,
                     n, m, sink, recent, Br, Bc, stream)
    else:
        st = ssa_fwd_debug(q, k, v, out, lse, counts, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                           lam, n, m, sink, recent, Br, Bc, stream, skip_bits, keep_bits, v_tile_loads)
    if st != SSA_OK:
        raise SSAError(st, "ssa_fwd")
    return out, lse, counts


def ssa_decode_workspace_bytes(B, Hq, Lq, d, num_splits) -> int:
    return int(lib.ssa_decode_workspace_bytes(B, Hq, Lq, d, num_splits))


def ssa_decode_default_splits(B, Hkv, Lk, Bc, num_sms) -> int:
    return int(lib.ssa_decode_default_splits(B, Hkv, Lk, Bc, num_sms))


def ssa_decode(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, lam, Bc,
               num_splits, workspace, workspace_bytes, stream=None) -> int:
    """Direct call of the decode entry point; returns its status code."""
    return lib.ssa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(tile_skip_count),
                          B, Hq, Hkv, Lq, Lk, d, int(causal), float(scale), float(lam), Bc,
                          num_splits, _ptr(workspace), int(workspace_bytes), _stream(stream))


def ssa_decode_debug(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, lam, Bc,
                     num_splits, workspace, workspace_bytes, stream=None, skip_bits=None) -> int:
    return lib.ssa_decode_debug(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(tile_skip_count),
                                B, Hq, Hkv, Lq, Lk, d, int(causal), float(scale), float(lam), Bc,
                                num_splits, _ptr(workspace), int(workspace_bytes), _stream(stream),
                                _ptr(skip_bits))


def decode(q, k, v, *, causal=True, scale=None, lam=0.0, Bc=128, num_splits=None, stream=None,
           out=None, lse=None, counts=None, workspace=None, skip_bits=None):
    """Decode-phase skip-softmax attention through the C ABI (torch allocates).

    q [B, Lq, Hq, d] (a few rows), k/v [B, Lk, Hkv, d] bf16 CUDA tensors.  Returns
    (out [B, Lq, Hq, d] bf16, lse [B, Hq, Lq] fp32, tile_skip_count [B, Hq] int32).
    num_splits defaults to ssa_decode_default_splits for this GPU's SM count (the
    kernel is persistent: one CTA per SM takes the (split, KV head, sequence) items in turn).
    """
    B, Lq, Hq, d = q.shape
    _, Lk, Hkv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    if num_splits is None:
        sms = torch.cuda.get_device_properties(q.device).multi_processor_count
        # 0 for arguments ssa_decode rejects: it then reports why
        num_splits = ssa_decode_default_splits(B, Hkv, Lk, Bc, sms) or 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device=q.device)
    if counts is None:
        counts = torch.empty(B, Hq, dtype=torch.int32, device=q.device)
    nbytes = ssa_decode_workspace_bytes(B, Hq, Lq, d, num_splits)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    nws = workspace.numel() * workspace.element_size()
    if skip_bits is None:
        st = ssa_decode(q, k, v, out, lse, counts, B, Hq, Hkv, Lq, Lk, d, causal, scale, lam, Bc,
                        num_splits, workspace, nws, stream)
    else:  # [B, Hq, ceil(nK / 32)], zeroed by the caller
        st = ssa_decode_debug(q, k, v, out, lse, counts, B, Hq, Hkv, Lq, Lk, d, causal, scale, lam, Bc,
                              num_splits, workspace, nws, stream, skip_bits)
    if st != SSA_OK:
        raise SSAError(st, "ssa_decode")
    return out, lse, counts


def ssa_fwd_blockmask(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                      lam, n, m, sink, recent, Br, Bc, block_mask, stream=None) -> int:
    """The key-block-selecting entry point (see include/ssa.h); returns its status code."""
    return lib.ssa_fwd_blockmask(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                 _ptr(tile_skip_count), B, Hq, Hkv, Lq, Lk, d, int(causal),
                                 float(scale), int(mode), float(lam), int(n), int(m), int(sink),
                                 int(recent), Br, Bc, _ptr(block_mask), _stream(stream))


def ssa_fwd_blockmask_debug(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale,
                            mode, lam, n, m, sink, recent, Br, Bc, block_mask, stream=None, skip_bits=None,
                            v_tile_loads=None) -> int:
    return lib.ssa_fwd_blockmask_debug(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                       _ptr(tile_skip_count), B, Hq, Hkv, Lq, Lk, d, int(causal),
                                       float(scale), int(mode), float(lam), int(n), int(m), int(sink),
                                       int(recent), Br, Bc, _ptr(block_mask), _stream(stream),
                                       _ptr(skip_bits), _ptr(v_tile_loads))


def attention_blockmask(q, k, v, block_mask, *, causal=True, scale=None, mode=MODE_SKIP, lam=0.0,
                        n=0, m=0, sink=0, recent=0, Br=128, Bc=128, stream=None, skip_bits=None,
                        v_tile_loads=None):
    """Forward over the key blocks selected by ``block_mask`` ([B, Hkv, nQ, ceil(nK/32)]
    int32/uint32 CUDA tensor).  Returns (out, lse, tile_skip_count) like ``attention``."""
    B, Lq, Hq, d = q.shape
    _, Lk, Hkv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    nQ = -(-Lq // Br)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device=q.device)
    counts = torch.empty(B, Hq, nQ, dtype=torch.int32, device=q.device)
    if skip_bits is None and v_tile_loads is None:
        st = ssa_fwd_blockmask(q, k, v, out, lse, counts, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                               lam, n, m, sink, recent, Br, Bc, block_mask, stream)
    else:  # skip_bits [B, Hq, nQ, ceil(nK / 32)] zeroed by the caller
        st = ssa_fwd_blockmask_debug(q, k, v, out, lse, counts, B, Hq, Hkv, Lq, Lk, d, causal, scale,
                                     mode, lam, n, m, sink, recent, Br, Bc, block_mask, stream,
                                     skip_bits, v_tile_loads)
    if st != SSA_OK:
        raise SSAError(st, "ssa_fwd_blockmask")
    return out, lse, counts


def ssa_fwd_blockmask_proxy(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, d, scale, Br, Bc, block_mask, kmean, vsum,
                            stream=None) -> int:
    """The proxy-compensated entry point (see include/ssa.h); returns its status code."""
    return lib.ssa_fwd_blockmask_proxy(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lk, d,
                                       float(scale), Br, Bc, _ptr(block_mask), _ptr(kmean), _ptr(vsum),
                                       _stream(stream))


def attention_blockmask_proxy(q, k, v, block_mask, kmean, vsum, *, scale=None, Br=128, Bc=128, stream=None):
    """Selected key blocks exact, omitted ones through the caller's summaries
    (kmean, vsum [B, nK, Hkv, d] bf16).  Returns (out, lse)."""
    B, Lq, Hq, d = q.shape
    _, Lk, Hkv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device=q.device)
    st = ssa_fwd_blockmask_proxy(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, d, scale, Br, Bc, block_mask, kmean,
                                 vsum, stream)
    if st != SSA_OK:
        raise SSAError(st, "ssa_fwd_blockmask_proxy")
    return out, lse
