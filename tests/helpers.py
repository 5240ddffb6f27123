"""Shared helpers for the parity tests (sampling rows, error metrics)."""
from __future__ import annotations

import numpy as np
import torch

# Acceptance thresholds for floating-point results against the fp64 oracle:
# max-abs 2e-2 and mean-abs 2e-3 (bf16 inputs, fp32 accumulation, bf16 O).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Gradients are stored in bf16 and can be larger than the forward's outputs:
# rounding a value to bf16 alone moves it by up to 2^-9 of its magnitude (so a
# flat 2e-2 cannot hold once |value| >= 8), and the bf16 P / dS operands of the
# tensor-core products add up to 2^-9 of each term. For dQ, dK and dV the
# per-element bound is therefore 2e-2 + 2^-8 * |ref| (two such roundings), with
# the same mean-abs 2e-3.
GRAD_REL = 2.0 ** -8
# Below this magnitude the flat bound alone must hold for gradients too. The
# backward's own bf16 roundings (D from the bf16 O, P and dS as bf16 operands
# of the tensor-core products) give errors that follow the size of the summed
# terms rather than |ref|: an fp64 model with just those roundings already
# reaches 1.9e-2 in dK at |ref| 1.6 and 1.1e-2 in dQ at |ref| 0.06
# (tests/test_tolerance_model.py), so the flat 2e-2 is asserted only where
# |ref| < 0.5, and the relative term carries the rest.
GRAD_FLAT_BELOW = 0.5
# |ref| bins of the per-magnitude error maxima
GRAD_BINS = (0.0, 0.5, 1.0, 2.0, 4.0, float("inf"))
# (name, max |ref|, elements, elements with |err| > MAX_ABS, worst |err| where
# |ref| < GRAD_FLAT_BELOW, worst |err| per GRAD_BINS bin) of every gradient
# comparison, printed by conftest.py
GRAD_STATS = []


def sample_rows(lengths, N: int, n_random: int, seed: int, cap_doc_edges: int = 64) -> np.ndarray:
    """Stratified query rows: first/last row of documents (up to a cap), the
    first/last row of 128-row tiles near them, the last row, plus uniform
    random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, N - 1}
    starts = np.cumsum([0] + list(lengths))[:-1]
    ends = starts + np.asarray(lengths) - 1
    idx = np.arange(len(lengths))
    if len(idx) > cap_doc_edges:
        idx = np.sort(rng.choice(idx, cap_doc_edges, replace=False))
    for t in idx:
        rows.update([int(starts[t]), int(ends[t])])
        rows.update([int(min(N - 1, (starts[t] // 128) * 128 + 127)), int(min(N - 1, starts[t] + 1))])
    rows.update(rng.integers(0, N, size=n_random).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N), dtype=np.int64)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def err_stats(got: np.ndarray, ref: np.ndarray):
    d = np.abs(got.astype(np.float64) - ref)
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0


def assert_close(name: str, got: np.ndarray, ref: np.ndarray, max_abs=MAX_ABS, mean_abs=MEAN_ABS, rel=0.0):
    """Every element within max_abs + rel*|ref| of the reference, and the mean
    absolute error within mean_abs."""
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    diff = np.abs(got.astype(np.float64) - ref)
    mx, mn = err_stats(got, ref)
    excess = diff - rel * np.abs(ref)
    k = int(np.argmax(excess)) if excess.size else 0
    worst = float(excess.reshape(-1)[k]) if excess.size else 0.0
    where = np.unravel_index(k, got.shape) if excess.size else ()
    assert worst <= max_abs and mn <= mean_abs, (
        f"{name}: worst |err| - {rel:g}|ref| = {worst:.3e} at {tuple(int(x) for x in where)} "
        f"(ref {float(ref[where]) if excess.size else 0:.4f}, got {float(got[where]) if excess.size else 0:.4f}; "
        f"limit {max_abs}), max-abs {mx:.3e}, mean-abs {mn:.3e} (<= {mean_abs})")
    return mx, mn


def assert_grad_close(name: str, got: np.ndarray, ref: np.ndarray):
    """dQ/dK/dV: every element within MAX_ABS + GRAD_REL*|ref|, the flat MAX_ABS
    alone wherever |ref| < GRAD_FLAT_BELOW, and mean-abs within MEAN_ABS. The
    number of elements that needed the relative term is recorded."""
    diff = np.abs(got.astype(np.float64) - ref)
    aref = np.abs(ref)
    bins = []
    for lo, hi in zip(GRAD_BINS[:-1], GRAD_BINS[1:]):
        sel = (aref >= lo) & (aref < hi)
        bins.append(float(diff[sel].max()) if sel.any() else None)
    small = aref < GRAD_FLAT_BELOW
    worst_small = float(diff[small].max()) if small.any() else 0.0
    GRAD_STATS.append((name, float(aref.max()) if ref.size else 0.0, int(ref.size),
                       int((diff > MAX_ABS).sum()), worst_small, bins))
    res = assert_close(name, got, ref, rel=GRAD_REL)
    k = int(np.argmax(np.where(small, diff, -1.0))) if small.any() else 0
    assert worst_small <= MAX_ABS, (f"{name}: |err| {worst_small:.3e} > {MAX_ABS} at |ref| "
                                    f"{float(aref.reshape(-1)[k]):.3f} < {GRAD_FLAT_BELOW}")
    return res


def stratified_long_rows(N: int, tile_stride: int, n_random: int, seed: int) -> np.ndarray:
    """Query rows of one long document: the first and last row of every
    tile_stride-th 128-row tile, the rows on either side of every 8192-key
    boundary, the first, middle and last rows of the last two 128-row tiles
    plus 16 random rows from them, and n_random uniform rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for t in range(0, (N + 127) // 128, tile_stride):
        rows.update([t * 128, min(N - 1, t * 128 + 127)])
    for b in range(8192, N + 1, 8192):
        rows.update([b - 1, b])
    tail = max(0, N - 256)
    rows.update([tail, tail + 1, tail + 63, tail + 127, tail + 128, tail + 191, N - 2, N - 1])
    rows.update(rng.integers(tail, N, size=16).tolist())
    rows.update(rng.integers(0, N, size=n_random).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N), dtype=np.int64)
