import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """One line per GPU/oracle comparison: what was compared and what the
    tolerance bands excused (visible in -q logs)."""
    mod = sys.modules.get("parity_util")
    if mod is None or not (mod.REPORTS or mod.V_LOADS):
        return
    terminalreporter.write_sep("-", "parity reports")
    for name, rep in mod.REPORTS:
        terminalreporter.write_line(f"{name}: {rep.line()}")
    for name, loaded, walked in mod.V_LOADS:
        terminalreporter.write_line(f"{name}: V tiles loaded {loaded} of {walked} walked "
                                    f"({walked - loaded} skipped by every query tile of their CTA)")
