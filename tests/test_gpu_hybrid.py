"""Parity of the Ulysses x ring hybrid's kernels with the fp64 oracle.

A ring step is the forward restricted to a query window and a key window
(ulysses_attn_fwd_window); a rank's steps combine through ulysses_attn_merge.
Each is compared with the oracle's own window attention and merge, and the
whole emulated hybrid (P = 8 ranks with 1 or 2 KV heads, so 1- or 2-way
Ulysses times an 8- or 4-way ring) with the oracle's unsharded attention."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, bf16_to_f64, sample_rows
from workloads import WORKLOADS, make_inputs, normal_bf16, random_case

pytestmark = pytest.mark.gpu


def _check_partial(name, o, lse, ro, rl):
    """Rows that see no key must be exactly o = 0, lse = -inf; the others are
    compared at the usual tolerance."""
    lse_n = lse.double().cpu().numpy()
    assert np.array_equal(np.isneginf(lse_n), np.isneginf(rl)), f"{name}: rows without keys differ"
    assert not np.isnan(lse_n).any()
    empty = np.isneginf(rl).T                     # [rows][Hl]
    og = bf16_to_f64(o)
    assert np.all(og[empty] == 0.0), f"{name}: rows without keys must be 0"
    keep = ~empty
    assert_close(f"{name} O", og[keep], ro[keep])
    assert_close(f"{name} LSE", lse_n[~np.isneginf(rl)], rl[~np.isneginf(rl)])


WINDOWS = [  # (q_lo, q_hi, kv_lo, kv_hi)
    (0, 1000, 0, 1000),
    (256, 768, 128, 512),
    (300, 1000, 700, 1000),      # rows before the key window see nothing
    (100, 900, 37, 555),         # neither window on a tile boundary
    (0, 1000, 500, 500),         # empty key window
    (640, 1000, 0, 128),         # one key tile, far below
]


@pytest.mark.parametrize("win", WINDOWS)
@pytest.mark.parametrize("Hl,Hkvl,d", [(4, 2, 128), (3, 1, 64)])
def test_window_matches_oracle(win, Hl, Hkvl, d):
    import long_context_sequence_ulysses_b200 as U
    lengths = [420, 1, 300, 279]
    c = random_case(1000, Hl, Hkvl, d, lengths, seed=91 + Hl, device="cuda")
    q_lo, q_hi, kv_lo, kv_hi = win
    o, lse = U.attn_fwd_window(c["q"], c["k"], c["v"], c["position_ids"], q_lo, q_hi, kv_lo, kv_hi)
    torch.cuda.synchronize()
    rows = np.arange(q_lo, q_hi)
    ro, rl = oracle.attn_fwd_window(c["q"], c["k"], c["v"], c["position_ids"], kv_lo, kv_hi, rows=rows)
    _check_partial(f"window {win}", o, lse, ro, rl)


def test_window_over_everything_equals_attn_fwd():
    import long_context_sequence_ulysses_b200 as U
    c = random_case(1500, 4, 1, 128, [700, 3, 797], seed=5, device="cuda")
    o, lse = U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    ow, lw = U.attn_fwd_window(c["q"], c["k"], c["v"], c["position_ids"], 0, 1500, 0, 1500)
    torch.cuda.synchronize()
    assert torch.equal(o, ow) and torch.equal(lse, lw)


def test_merge_matches_oracle():
    """Seeded partials (some rows without keys in some or all parts) merged by
    the kernel and by the oracle's merge."""
    import long_context_sequence_ulysses_b200 as U
    R, M, Hl, d = 3, 300, 4, 64
    o_parts = normal_bf16((R, M, Hl, d), seed=7, device="cuda", stream_id=9)
    g = torch.Generator(device="cpu")
    g.manual_seed(77)
    lse_parts = (torch.randn((R, Hl, M), generator=g, dtype=torch.float32) * 3.0)
    lse_parts[0, :, :50] = float("-inf")
    lse_parts[:, 1, 100:120] = float("-inf")
    lse_parts = lse_parts.cuda()
    o, lse = U.attn_merge(o_parts, lse_parts)
    torch.cuda.synchronize()
    ro, rl = oracle.merge(bf16_to_f64(o_parts), lse_parts.double().cpu().numpy())
    assert_close("merged O", bf16_to_f64(o), ro)
    l = lse.double().cpu().numpy()
    assert np.array_equal(np.isneginf(l), np.isneginf(rl))
    assert_close("merged LSE", l[np.isfinite(rl)], rl[np.isfinite(rl)])


@pytest.mark.parametrize("Hkv", [1, 2])
def test_hybrid_matches_unsharded(Hkv):
    """P = 8 ranks with fewer KV heads than ranks: Hkv-way Ulysses times an
    (8/Hkv)-way ring, against the oracle's attention of the whole sequence."""
    from long_context_sequence_ulysses_b200 import hybrid
    N, H, d, P = 4096, 8, 128, 8
    c = random_case(N, H, Hkv, d, [1500, 1, 1000, 1595], seed=60 + Hkv, device="cuda")
    o, lse = hybrid.forward(c["q"], c["k"], c["v"], c["position_ids"], P)
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert_close("O", bf16_to_f64(o), ro)
    assert_close("LSE", lse.double().cpu().numpy(), rl)


def test_hybrid_workload():
    """The benchmark's hybrid workload (llama8b's shape with 2 KV heads, P = 8:
    2-way Ulysses times a 4-way ring), sampled rows against the oracle."""
    from long_context_sequence_ulysses_b200 import hybrid
    w = WORKLOADS["hybrid_kv2"]
    inp = make_inputs(w, device="cuda")
    o, lse = hybrid.forward(inp["q"], inp["k"], inp["v"], inp["position_ids"], w.P, w.ulysses)
    torch.cuda.synchronize()
    rows = sample_rows(inp["lengths"], w.N, 64, seed=w.seed)
    # every 8192-token ring chunk boundary, both sides
    rows = np.unique(np.concatenate([rows, [8191, 8192, 16383, 16384, 24575, 24576]]))
    ro, rl = oracle.attn_fwd(inp["q"].cpu(), inp["k"].cpu(), inp["v"].cpu(), inp["position_ids"].cpu(), rows=rows)
    rt = torch.from_numpy(rows).cuda()
    assert_close("O", bf16_to_f64(o[rt]), ro)
    assert_close("LSE", lse[:, rt].double().cpu().numpy(), rl)
