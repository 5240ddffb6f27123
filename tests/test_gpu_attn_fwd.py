"""Parity of the tensor-core attention forward with the fp64 oracle.

Small cases are compared on every row (several 128-row tiles, ragged tails,
packed documents, GQA, every supported head dimension); the five workloads
are compared on stratified samples of rows (each sampled row exact over all
its keys), through the same launch the benchmark times."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, bf16_to_f64, sample_rows, stratified_long_rows
from workloads import WORKLOADS, make_inputs, random_case

pytestmark = pytest.mark.gpu


def _run(c, scale=None):
    import long_context_sequence_ulysses_b200 as U
    o, lse = U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"], scale=scale)
    torch.cuda.synchronize()
    return o, lse


CASES = [
    # (lengths, Hl, Hkvl, d)
    ([256], 2, 2, 32),
    ([128], 1, 1, 128),
    ([1], 1, 1, 128),
    ([300], 2, 1, 128),               # ragged tail
    ([1000], 4, 1, 128),
    ([700, 1, 300, 23, 200], 4, 2, 128),
    ([5] * 60, 2, 2, 64),             # many short documents inside one tile
    ([129, 127, 384, 2], 8, 2, 64),
    ([513, 511], 4, 4, 32),
    ([2048], 1, 1, 64),
    ([3000, 1500, 2], 2, 1, 128),
    ([600, 700, 29], 6, 2, 64),       # odd group size: items pair consecutive tiles
    ([1100, 3], 3, 1, 128),
    ([900, 100, 44], 8, 1, 64),       # group of 8: four head pairs share each K/V tile
    ([600, 33], 2, 1, 32),            # head pairs with the smallest head dimension
]


@pytest.mark.parametrize("lengths,Hl,Hkvl,d", CASES)
def test_fwd_matches_oracle_all_rows(lengths, Hl, Hkvl, d):
    N = sum(lengths)
    c = random_case(N, Hl, Hkvl, d, lengths, seed=N + 7 * Hl + d, device="cuda")
    o, lse = _run(c)
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert_close("O", bf16_to_f64(o), ro)
    assert_close("LSE", lse.double().cpu().numpy(), rl)


def test_fwd_scale_argument():
    lengths = [400, 100]
    c = random_case(500, 2, 1, 128, lengths, seed=3, device="cuda")
    o, lse = _run(c, scale=0.05)
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"], scale=0.05)
    assert_close("O", bf16_to_f64(o), ro)
    assert_close("LSE", lse.double().cpu().numpy(), rl)


def test_fwd_rising_and_jumping_scores():
    """Scores that rise along the sequence (the running maximum of a row grows
    by far more than 2^8 across its key tiles) and one key tile whose scores
    jump by more than 128 in log2 units (its exponentials overflow against the old
    offset): both force the kernel's slow path, which reloads S, takes the row
    maximum and rescales O and the row sum."""
    N, Hl, Hkvl, d = 1000, 2, 1, 128
    lengths = [700, 300]
    c = random_case(N, Hl, Hkvl, d, lengths, seed=11, device="cuda")
    j = torch.arange(N, device="cuda", dtype=torch.float32)[:, None, None]
    q = c["q"].float().abs()
    k = 0.25 * c["k"].float() + 3.0 * j / N
    k[640:672] += 12.0
    c["q"] = q.to(torch.bfloat16)
    c["k"] = k.to(torch.bfloat16)
    o, lse = _run(c)
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert np.isfinite(lse.double().cpu().numpy()).all()
    assert_close("O", bf16_to_f64(o), ro)
    assert_close("LSE", lse.double().cpu().numpy(), rl, rel=1e-5)


def test_fwd_one_token_documents_return_v():
    N, Hl, Hkvl, d = 384, 4, 2, 128
    c = random_case(N, Hl, Hkvl, d, [1] * N, seed=1, device="cuda")
    o, lse = _run(c)
    v = c["v"].repeat_interleave(Hl // Hkvl, dim=1)
    assert torch.equal(o, v)          # one key: weight exactly 1, O is V rounded back to bf16


def test_fwd_uniform_v():
    lengths = [200, 50, 262]
    N = sum(lengths)
    c = random_case(N, 2, 1, 64, lengths, seed=2, device="cuda")
    c["v"][:] = torch.linspace(-2, 2, 64, device="cuda").to(torch.bfloat16)
    o, _ = _run(c)
    ref = c["v"][0, 0].float().expand(N, 2, 64)
    assert (o.float() - ref).abs().max().item() <= 2e-2


def test_fwd_deterministic_and_fused_equals_unfused():
    import long_context_sequence_ulysses_b200 as U
    lengths = [600, 424]
    N, P, H, Hkv, d = 1024, 4, 8, 4, 128
    c = random_case(N, H, Hkv, d, lengths, seed=5, device="cuda")
    o_seq = torch.zeros_like(c["q"])
    for r in range(P):
        qs = U.seq_to_head(c["q"], P, rank=r)
        ks = U.seq_to_head(c["k"], P, rank=r)
        vs = U.seq_to_head(c["v"], P, rank=r)
        o1, l1 = U.attn_fwd(qs, ks, vs, c["position_ids"])
        o2, l2 = U.attn_fwd(qs, ks, vs, c["position_ids"])
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        o3 = torch.zeros_like(c["q"])
        _, l3 = U.attn_fwd_fused(c["q"], c["k"], c["v"], c["position_ids"], P, r, out=o3)
        assert torch.equal(o3[:, r * H // P:(r + 1) * H // P], o1) and torch.equal(l3, l1)
        U.attn_fwd_fused(c["q"], c["k"], c["v"], c["position_ids"], P, r, out=o_seq)
    # sharded (all ranks, fused) equals unsharded attention on all heads at once
    o_all, _ = U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert torch.equal(o_seq, o_all)


def test_fwd_empty():
    import long_context_sequence_ulysses_b200 as U
    z = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    o, lse = U.attn_fwd(z, z[:, :1], z[:, :1], torch.empty(0, dtype=torch.int32, device="cuda"))
    assert o.shape == (0, 2, 128) and lse.shape == (2, 0)


WORKLOAD_SAMPLES = {"tiny": None, "llama8b": 160, "train": 160}
# Single long documents: (tile stride of the first/last-row strata, extra uniform rows).
# long131k: both edge rows of all 1024 tiles; million: of every 32nd of its 8192 tiles.
LONG_STRATA = {"long131k": (1, 64), "million": (32, 32)}


@pytest.mark.parametrize("name", ["tiny", "llama8b", "long131k", "million", "train"])
def test_workload_forward(name):
    """Rank 0's head slice of each workload, produced by the seq->head exchange
    and run through the same forward launch the benchmark times. Every sampled
    row is compared on all of rank 0's heads, exact over all its keys."""
    import long_context_sequence_ulysses_b200 as U
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda", with_grad_out=False)
    rank = 0
    q = U.seq_to_head(inp["q"], w.P, rank=rank)
    k = U.seq_to_head(inp["k"], w.P, rank=rank)
    v = U.seq_to_head(inp["v"], w.P, rank=rank)
    del inp["q"], inp["k"], inp["v"]
    o, lse = U.attn_fwd(q, k, v, inp["position_ids"])
    torch.cuda.synchronize()
    if name in LONG_STRATA:
        stride, n_rand = LONG_STRATA[name]
        rows = stratified_long_rows(w.N, stride, n_rand, seed=w.seed)
        assert len(rows) >= 256
    elif WORKLOAD_SAMPLES[name] is None:
        rows = np.arange(w.N)
    else:
        rows = sample_rows(inp["lengths"], w.N, WORKLOAD_SAMPLES[name], seed=w.seed)
    rt = torch.from_numpy(rows).cuda()
    ro, rl = oracle.attn_fwd(q.cpu(), k.cpu(), v.cpu(), inp["position_ids"].cpu(), rows=rows)
    assert ro.shape[1] == w.Hl
    assert_close("O", bf16_to_f64(o[rt]), ro)
    assert_close("LSE", lse[:, rt].double().cpu().numpy(), rl)


def test_fused_forward_llama8b_all_ranks():
    """The fused forward as the benchmark's fused step runs it on llama8b: every
    one of the 8 ranks reads its 4 query heads and 1 KV head straight out of the
    sequence-sharded Q/K/V (rows 8 KB and 2 KB apart) and writes its heads of
    O into the sequence layout. Sampled rows of every rank, all of its heads,
    against the oracle on that rank's head slice of the inputs."""
    import long_context_sequence_ulysses_b200 as U
    w = WORKLOADS["llama8b"]
    inp = make_inputs(w, device="cuda", with_grad_out=False)
    pos = inp["position_ids"]
    o_seq = torch.full_like(inp["q"], float("nan"))
    lse_all = torch.empty((w.H, w.N), dtype=torch.float32, device="cuda")
    for r in range(w.P):
        U.attn_fwd_fused(inp["q"], inp["k"], inp["v"], pos, w.P, r, out=o_seq,
                         lse=lse_all[r * w.Hl:(r + 1) * w.Hl])
    torch.cuda.synchronize()
    assert not torch.isnan(o_seq.float()).any()          # every rank wrote exactly its own heads
    qc, kc, vc, pc = inp["q"].cpu(), inp["k"].cpu(), inp["v"].cpu(), pos.cpu()
    for r in range(w.P):
        rows = sample_rows(inp["lengths"], w.N, 48, seed=100 + r)
        qs, ks = slice(r * w.Hl, (r + 1) * w.Hl), slice(r * w.Hkvl, (r + 1) * w.Hkvl)
        ro, rl = oracle.attn_fwd(qc[:, qs].contiguous(), kc[:, ks].contiguous(), vc[:, ks].contiguous(), pc,
                                 rows=rows)
        rt = torch.from_numpy(rows).cuda()
        assert_close(f"O rank {r}", bf16_to_f64(o_seq[rt][:, qs]), ro)
        assert_close(f"LSE rank {r}", lse_all[qs][:, rt].double().cpu().numpy(), rl)


def _irregular_ids(kind: str, N: int) -> torch.Tensor:
    """Position ids that break the 0, 1, 2, ... pattern in the ways the reading
    of the ids has to handle (a document starts at token 0 and at every 0;
    every other value is ignored)."""
    if kind == "first_not_zero":       # a shard boundary inside a document: ids start at 300
        ids = list(range(300, 300 + 700)) + list(range(N - 700))
    elif kind == "no_zero_at_all":     # one document, ids never 0
        ids = [7 + i for i in range(N)]
    else:                              # jumps, repeats and negative ids between the zeros
        ids = (list(range(100)) + list(range(500, 640)) + [3] * 40 + list(range(160)) + [-1] * 30
               + list(range(129)) + [9] * 3 + list(range(N - 602)))
    assert len(ids) == N
    return torch.tensor(ids, dtype=torch.int32)


@pytest.mark.parametrize("kind", ["first_not_zero", "no_zero_at_all", "jumps_repeats_negatives"])
@pytest.mark.parametrize("Hl,Hkvl,d", [(4, 2, 128), (3, 1, 64)])
def test_fwd_irregular_position_ids(kind, Hl, Hkvl, d):
    N = 1000
    c = random_case(N, Hl, Hkvl, d, [N], seed=61 + Hl, device="cuda")
    pos = _irregular_ids(kind, N)
    c["position_ids"] = pos.cuda()
    o, lse = _run(c)
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], pos)
    assert_close("O", bf16_to_f64(o), ro)
    assert_close("LSE", lse.double().cpu().numpy(), rl)


def test_fwd_beyond_1024_scan_blocks():
    """More than 1024 blocks of the document-start scan (N > 1048576), where
    each block's carry comes from a separate prefix over the block maxima: a
    document that starts in block 1020 and spans 40 more blocks, and short
    documents elsewhere; rows sampled across block and tile boundaries."""
    import long_context_sequence_ulysses_b200 as U
    N = 1024 * 1100
    start, long_len = 1020 * 1024 + 7, 40 * 1024 + 300
    lengths = [4096] * (start // 4096)
    if start > sum(lengths):
        lengths.append(start - sum(lengths))
    lengths.append(long_len)
    rest = N - sum(lengths)
    lengths += [4096] * (rest // 4096) + ([rest % 4096] if rest % 4096 else [])
    lengths = [L for L in lengths if L > 0]
    assert sum(lengths) == N
    c = random_case(N, 2, 1, 64, lengths, seed=81, device="cuda")
    o, lse = _run(c)
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([
        [start, start + 1, start + 1023, start + long_len - 1, N - 1, 1048575, 1048576],
        np.arange(1021 * 1024 - 2, 1021 * 1024 + 2), np.arange(1050 * 1024 - 2, 1050 * 1024 + 2),
        rng.integers(start, start + long_len, 48), rng.integers(0, N, 48)]))
    ro, rl = oracle.attn_fwd(c["q"].cpu(), c["k"].cpu(), c["v"].cpu(), c["position_ids"].cpu(), rows=rows)
    rt = torch.from_numpy(rows).cuda()
    assert_close("O", bf16_to_f64(o[rt]), ro)
    assert_close("LSE", lse[:, rt].double().cpu().numpy(), rl)
