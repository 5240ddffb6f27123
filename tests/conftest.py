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
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """How much the gradient comparisons leaned on the relative term of the
    tolerance: per comparison, max |ref|, and the elements whose error is above
    the flat 2e-2 (allowed only where |ref| >= 4, by 2^-8 |ref|)."""
    try:
        from helpers import GRAD_STATS, GRAD_FLAT_BELOW, MAX_ABS
    except Exception:  # pragma: no cover
        return
    if not GRAD_STATS:
        return
    tr = terminalreporter
    tr.section("gradient tolerance use")
    tot = sum(s[2] for s in GRAD_STATS)
    over = sum(s[3] for s in GRAD_STATS)
    tr.write_line(f"{len(GRAD_STATS)} comparisons, {tot} elements, {over} with |err| > {MAX_ABS} "
                  f"(flat bound asserted wherever |ref| < {GRAD_FLAT_BELOW})")
    for name, mref, n, nover, ws in GRAD_STATS:
        tr.write_line(f"  {name}: max|ref| {mref:.3g}, {nover}/{n} above flat, worst |err| at |ref|<4 {ws:.3e}")
