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
        from helpers import GRAD_BINS, GRAD_STATS, GRAD_FLAT_BELOW, MAX_ABS
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
    edges = ", ".join(f"[{a:g},{b:g})" for a, b in zip(GRAD_BINS[:-1], GRAD_BINS[1:]))
    worst = [max((s[5][i] for s in GRAD_STATS if s[5][i] is not None), default=None)
             for i in range(len(GRAD_BINS) - 1)]
    tr.write_line("worst |err| per |ref| bin " + edges + ": "
                  + ", ".join("-" if w is None else f"{w:.3e}" for w in worst))
    for name, mref, n, nover, ws, bins in GRAD_STATS:
        tr.write_line(f"  {name}: max|ref| {mref:.3g}, {nover}/{n} above flat; worst |err| per bin "
                      + ", ".join("-" if b is None else f"{b:.2e}" for b in bins))
