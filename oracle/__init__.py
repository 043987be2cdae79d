"""CPU oracle for the skip-softmax / N:M sparse attention forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``softmax_ssa_fwd_b200``) never imports it and shares no code with it.

The arithmetic lives in ``ssa_oracle.c`` (plain C, fp64); this module only
compiles it (``build()``) and marshals numpy arrays into it (``run_items``).
"""
from .oracle import build, lib_path, run_items, visited_tiles, OracleResult  # noqa: F401
# fp64 numpy oracles of the two further paths (same test-infrastructure rule):
# oracle.decode (split-KV decode), oracle.blockmask (caller-selected key blocks) and
# oracle.proxy (selected blocks exact, omitted ones through caller-supplied summaries)
