import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a); runs the C-ABI library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Max |err| against the oracle of every GPU parity comparison this run
    made (out and lse), then the worst case per KV dtype and its margin to
    the tolerance."""
    try:
        from tests import gpu_util
    except Exception:  # pragma: no cover
        return
    recs = gpu_util.RECORDS
    if not recs:
        return
    names = {0: "bf16", 1: "fp8_e4m3", 2: "nvfp4"}
    tr = terminalreporter
    tr.section("parity max|err| against the oracle")
    for what, kv, eo, el in recs:
        tr.write_line(f"{names.get(kv, kv):9s} out {eo:.3e}  lse {el:.3e}  {what}")
    for kv in sorted({r[1] for r in recs}):
        rows = [r for r in recs if r[1] == kv]
        tol = gpu_util.TOL[kv]
        wo = max(rows, key=lambda r: r[2])
        wl = max(rows, key=lambda r: r[3])
        tr.write_line(
            f"worst {names.get(kv, kv)} ({len(rows)} comparisons): out {wo[2]:.3e} "
            f"({tol['out'] / max(wo[2], 1e-300):.0f}x inside {tol['out']}) in {wo[0]}; "
            f"lse {wl[3]:.3e} ({tol['lse'] / max(wl[3], 1e-300):.0f}x inside {tol['lse']}) "
            f"in {wl[0]}")
