"""Parity of the tensor-core attention backward (dQ, dK, dV) with the fp64
oracle's exact gradients of sum(dO * O).

The backward is fed the forward kernel's own O (bf16) and LSE (fp32), as in
training. Small cases are compared on every element; the training workload
(N = 65536, rank 0's 8 query heads and 2 KV heads, geometric document
lengths) is compared on whole documents, which the oracle computes on their
own (packed documents are independent, a property the oracle's pins check)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, assert_grad_close, bf16_to_f64
from workloads import WORKLOADS, make_inputs, random_case

pytestmark = pytest.mark.gpu


def _fwd_bwd(c, scale=None):
    import long_context_sequence_ulysses_b200 as U
    o, lse = U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"], scale=scale)
    dq, dk, dv = U.attn_bwd(c["q"], c["k"], c["v"], o, c["do"], lse, c["position_ids"], scale=scale)
    torch.cuda.synchronize()
    return o, lse, dq, dk, dv


CASES = [
    ([256], 2, 2, 32),
    ([128], 1, 1, 128),
    ([300], 2, 1, 128),                  # ragged tail
    ([700, 1, 300, 23], 4, 2, 128),
    ([129, 127, 384, 2], 4, 1, 64),
    ([5] * 40, 2, 2, 128),
    ([1000, 24], 8, 2, 128),
    ([513, 511], 2, 2, 32),
    ([600, 700, 29], 6, 2, 64),         # odd group size: three query heads per KV head
    ([1100, 3], 3, 1, 128),
    ([900, 100, 44], 8, 1, 64),         # group of 8: one dK/dV CTA sums eight heads
]


@pytest.mark.parametrize("lengths,Hl,Hkvl,d", CASES)
def test_bwd_matches_oracle(lengths, Hl, Hkvl, d):
    N = sum(lengths)
    c = random_case(N, Hl, Hkvl, d, lengths, seed=N + 3 * Hl + d, device="cuda", with_grad_out=True)
    _, _, dq, dk, dv = _fwd_bwd(c)
    rq, rk, rv, _, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"])
    assert_grad_close("dQ", bf16_to_f64(dq), rq)
    assert_grad_close("dK", bf16_to_f64(dk), rk)
    assert_grad_close("dV", bf16_to_f64(dv), rv)


def test_bwd_scale_and_determinism():
    import long_context_sequence_ulysses_b200 as U
    lengths = [333, 179]
    c = random_case(512, 4, 2, 128, lengths, seed=8, device="cuda", with_grad_out=True)
    o, lse, dq, dk, dv = _fwd_bwd(c, scale=0.07)
    rq, rk, rv, _, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"], scale=0.07)
    assert_grad_close("dQ", bf16_to_f64(dq), rq)
    assert_grad_close("dK", bf16_to_f64(dk), rk)
    assert_grad_close("dV", bf16_to_f64(dv), rv)
    dq2, dk2, dv2 = U.attn_bwd(c["q"], c["k"], c["v"], o, c["do"], lse, c["position_ids"], scale=0.07)
    torch.cuda.synchronize()
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)


def test_bwd_one_token_documents():
    # one key per row: P = 1, dS = 0, so dQ = dK = 0 and dV = the group's dO
    N, Hl, Hkvl, d = 256, 4, 2, 128
    c = random_case(N, Hl, Hkvl, d, [1] * N, seed=4, device="cuda", with_grad_out=True)
    _, _, dq, dk, dv = _fwd_bwd(c)
    assert dq.abs().max().item() <= 2e-2 and dk.abs().max().item() <= 2e-2
    ref = c["do"].double().view(N, Hkvl, Hl // Hkvl, d).sum(2).cpu().numpy()
    assert_grad_close("dV", bf16_to_f64(dv), ref)


def test_bwd_empty():
    import long_context_sequence_ulysses_b200 as U
    z = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 0), dtype=torch.float32, device="cuda")
    dq, dk, dv = U.attn_bwd(z, z[:, :1].contiguous(), z[:, :1].contiguous(), z, z, lse,
                            torch.empty(0, dtype=torch.int32, device="cuda"))
    assert dq.shape == (0, 2, 128)


def _train_rank0():
    import long_context_sequence_ulysses_b200 as U
    w = WORKLOADS["train"]
    inp = make_inputs(w, device="cuda", with_grad_out=True)
    q = U.seq_to_head(inp["q"], w.P, rank=0)
    k = U.seq_to_head(inp["k"], w.P, rank=0)
    v = U.seq_to_head(inp["v"], w.P, rank=0)
    do = U.seq_to_head(inp["do"], w.P, rank=0)
    pos = inp["position_ids"]
    o, lse = U.attn_fwd(q, k, v, pos)
    dq, dk, dv = U.attn_bwd(q, k, v, o, do, lse, pos)
    torch.cuda.synchronize()
    return w, inp, (q, k, v, do, pos), (dq, dk, dv)


def _doc_bounds(lengths):
    lengths = np.array(lengths)
    starts = np.concatenate([[0], np.cumsum(lengths)[:-1]])
    return lengths, starts


def test_train_workload_documents():
    """Rank 0 of the training workload, through the same launches the
    benchmark times; whole documents compared against the oracle."""
    w, inp, (q, k, v, do, pos), (dq, dk, dv) = _train_rank0()
    lengths, starts = _doc_bounds(inp["lengths"])
    # first, last-but-longest, shortest and a mid-length document, in full
    cand = [0, int(np.argmin(lengths))]
    order = np.argsort(lengths)
    cand.append(int(order[len(order) // 2]))
    picked = sorted({t for t in cand if lengths[t] <= 9000})
    assert len(picked) >= 3
    for t in picked:
        a, b = int(starts[t]), int(starts[t] + lengths[t])
        sl = slice(a, b)
        rq, rk, rv, _, _ = oracle.attn_bwd(q[sl].cpu(), k[sl].cpu(), v[sl].cpu(), do[sl].cpu(), pos[sl].cpu())
        assert_grad_close(f"dQ doc {t}", bf16_to_f64(dq[sl]), rq)
        assert_grad_close(f"dK doc {t}", bf16_to_f64(dk[sl]), rk)
        assert_grad_close(f"dV doc {t}", bf16_to_f64(dv[sl]), rv)


def test_train_longest_document():
    """The longest document of the training workload (18112 tokens): the dK/dV
    of its first 256 keys (the key tiles that every later query of the document
    reaches, the longest-running dK/dV work), of its last keys and of random
    keys, and the dQ of its last 128-row tile and random rows, against the
    oracle's exact gradients at those keys and rows."""
    w, inp, (q, k, v, do, pos), (dq, dk, dv) = _train_rank0()
    lengths, starts = _doc_bounds(inp["lengths"])
    t = int(np.argmax(lengths))
    a, L = int(starts[t]), int(lengths[t])
    assert L > 9000
    rng = np.random.default_rng(3)
    keys = np.unique(np.concatenate([np.arange(256), np.arange(L - 16, L), rng.integers(0, L, 48)]))
    rows = np.unique(np.concatenate([np.arange(8), np.arange(L - 128, L), rng.integers(0, L, 48)]))
    sl = slice(a, a + L)
    rq, rk, rv = oracle.attn_bwd_sampled(q[sl].cpu(), k[sl].cpu(), v[sl].cpu(), do[sl].cpu(), pos[sl].cpu(),
                                         rows, keys)
    kt, rt = torch.from_numpy(keys + a).cuda(), torch.from_numpy(rows + a).cuda()
    assert_grad_close("dK longest doc", bf16_to_f64(dk[kt]), rk)
    assert_grad_close("dV longest doc", bf16_to_f64(dv[kt]), rv)
    assert_grad_close("dQ longest doc", bf16_to_f64(dq[rt]), rq)


def test_train_fused_all_ranks():
    """The fused forward and backward as the benchmark's fused step runs them
    on the training workload: every one of the 4 ranks reads its 8 query heads
    and 2 KV heads straight out of the sequence-sharded buffers and writes O and
    dQ/dK/dV into the sequence layout. One document per rank (one straddling a
    128-token tile boundary, one long one on rank 1) against the oracle on that
    rank's head slice of the inputs."""
    import long_context_sequence_ulysses_b200 as U
    w = WORKLOADS["train"]
    inp = make_inputs(w, device="cuda", with_grad_out=True)
    pos = inp["position_ids"]
    nan = float("nan")
    o_seq = torch.full_like(inp["q"], nan)
    dq_s, dk_s, dv_s = (torch.full_like(inp[x], nan) for x in ("q", "k", "v"))
    lse_all = torch.empty((w.H, w.N), dtype=torch.float32, device="cuda")
    for r in range(w.P):
        U.attn_fwd_fused(inp["q"], inp["k"], inp["v"], pos, w.P, r, out=o_seq, lse=lse_all[r * w.Hl:(r + 1) * w.Hl])
    for r in range(w.P):
        U.attn_bwd_fused(inp["q"], inp["k"], inp["v"], o_seq, inp["do"], lse_all[r * w.Hl:(r + 1) * w.Hl], pos,
                         w.P, r, dq=dq_s, dk=dk_s, dv=dv_s)
    torch.cuda.synchronize()
    for x in (o_seq, dq_s, dk_s, dv_s):
        assert not torch.isnan(x.float()).any()          # the ranks together wrote every head
    lengths, starts = _doc_bounds(inp["lengths"])
    cpu = {x: inp[x].cpu() for x in ("q", "k", "v", "do")}
    pc = pos.cpu()
    full_docs = {0: 3, 2: 7, 3: 1}       # 240 tokens across a tile boundary, 1127, 1280
    for r in range(w.P):
        qs, ks = slice(r * w.Hl, (r + 1) * w.Hl), slice(r * w.Hkvl, (r + 1) * w.Hkvl)
        if r in full_docs:
            t = full_docs[r]
            a, b = int(starts[t]), int(starts[t] + lengths[t])
            sl = slice(a, b)
            rq, rk, rv, ro, rl = oracle.attn_bwd(cpu["q"][sl, qs].contiguous(), cpu["k"][sl, ks].contiguous(),
                                                 cpu["v"][sl, ks].contiguous(), cpu["do"][sl, qs].contiguous(), pc[sl])
            assert_close(f"O rank {r}", bf16_to_f64(o_seq[sl, qs]), ro)
            assert_close(f"LSE rank {r}", lse_all[qs, a:b].double().cpu().numpy(), rl)
            assert_grad_close(f"dQ fused rank {r}", bf16_to_f64(dq_s[sl, qs]), rq)
            assert_grad_close(f"dK fused rank {r}", bf16_to_f64(dk_s[sl, ks]), rk)
            assert_grad_close(f"dV fused rank {r}", bf16_to_f64(dv_s[sl, ks]), rv)
        else:
            t = 8                        # 9120 tokens: sampled keys and rows
            a, L = int(starts[t]), int(lengths[t])
            rng = np.random.default_rng(r)
            keys = np.unique(np.concatenate([np.arange(128), rng.integers(0, L, 32)]))
            rows = np.unique(np.concatenate([np.arange(L - 128, L), rng.integers(0, L, 32)]))
            sl = slice(a, a + L)
            rq, rk, rv = oracle.attn_bwd_sampled(cpu["q"][sl, qs].contiguous(), cpu["k"][sl, ks].contiguous(),
                                                 cpu["v"][sl, ks].contiguous(), cpu["do"][sl, qs].contiguous(),
                                                 pc[sl], rows, keys)
            kt, rt = torch.from_numpy(keys + a).cuda(), torch.from_numpy(rows + a).cuda()
            assert_grad_close(f"dK fused rank {r}", bf16_to_f64(dk_s[kt][:, ks]), rk)
            assert_grad_close(f"dV fused rank {r}", bf16_to_f64(dv_s[kt][:, ks]), rv)
            assert_grad_close(f"dQ fused rank {r}", bf16_to_f64(dq_s[rt][:, qs]), rq)


@pytest.mark.parametrize("kind", ["first_not_zero", "jumps_repeats_negatives"])
def test_bwd_irregular_position_ids(kind):
    from test_gpu_attn_fwd import _irregular_ids
    N, Hl, Hkvl, d = 1000, 4, 2, 128
    c = random_case(N, Hl, Hkvl, d, [N], seed=71, device="cuda", with_grad_out=True)
    pos = _irregular_ids(kind, N)
    c["position_ids"] = pos.cuda()
    _, _, dq, dk, dv = _fwd_bwd(c)
    rq, rk, rv, _, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], pos)
    assert_grad_close("dQ", bf16_to_f64(dq), rq)
    assert_grad_close("dK", bf16_to_f64(dk), rk)
    assert_grad_close("dV", bf16_to_f64(dv), rv)


def test_bwd_fused_equals_slice():
    """The fused backward (reading every rank's head slice straight from the
    sequence-sharded buffers and writing the gradients back into that layout)
    gives, bit for bit, the slice backward of each rank: the same kernels on the
    same values, only the addressing differs."""
    import long_context_sequence_ulysses_b200 as U
    lengths = [700, 1, 300, 23]
    N, P, H, Hkv, d = sum(lengths), 2, 8, 4, 128
    c = random_case(N, H, Hkv, d, lengths, seed=21, device="cuda", with_grad_out=True)
    Hl, Hkvl = H // P, Hkv // P
    dq_f = torch.zeros_like(c["q"]); dk_f = torch.zeros_like(c["k"]); dv_f = torch.zeros_like(c["v"])
    o_seq = torch.empty_like(c["q"])
    for r in range(P):
        qs, ks = slice(r * Hl, (r + 1) * Hl), slice(r * Hkvl, (r + 1) * Hkvl)
        q, k, v, do = (c["q"][:, qs].contiguous(), c["k"][:, ks].contiguous(), c["v"][:, ks].contiguous(),
                       c["do"][:, qs].contiguous())
        o, lse = U.attn_fwd(q, k, v, c["position_ids"])
        o_seq[:, qs] = o
        dq, dk, dv = U.attn_bwd(q, k, v, o, do, lse, c["position_ids"])
        U.attn_bwd_fused(c["q"], c["k"], c["v"], o_seq, c["do"], lse, c["position_ids"], P, r,
                         dq=dq_f, dk=dk_f, dv=dv_f)
        torch.cuda.synchronize()
        assert torch.equal(dq_f[:, qs], dq)
        assert torch.equal(dk_f[:, ks], dk)
        assert torch.equal(dv_f[:, ks], dv)


@pytest.mark.parametrize("P,H,Hkv,d,lengths", [
    (2, 6, 2, 64, [600, 700, 30]),      # group of 3: the forward pairs consecutive query tiles
    (4, 8, 4, 32, [500, 300, 200, 24]),
    (2, 4, 2, 128, [1000, 24]),
])
def test_fused_small_shapes_against_oracle(P, H, Hkv, d, lengths):
    """The fused forward and backward of every rank on small sequence-sharded
    buffers, every element of every rank's heads against the oracle on that
    rank's head slice (the fused path at group sizes and head dimensions the
    workload tests do not reach)."""
    import long_context_sequence_ulysses_b200 as U
    N = sum(lengths)
    c = random_case(N, H, Hkv, d, lengths, seed=N + H + d, device="cuda", with_grad_out=True)
    pos = c["position_ids"]
    Hl, Hkvl = H // P, Hkv // P
    nan = float("nan")
    o_seq = torch.full_like(c["q"], nan)
    dq_s, dk_s, dv_s = (torch.full_like(c[x], nan) for x in ("q", "k", "v"))
    lse_all = torch.empty((H, N), dtype=torch.float32, device="cuda")
    for r in range(P):
        U.attn_fwd_fused(c["q"], c["k"], c["v"], pos, P, r, out=o_seq, lse=lse_all[r * Hl:(r + 1) * Hl])
    for r in range(P):
        U.attn_bwd_fused(c["q"], c["k"], c["v"], o_seq, c["do"], lse_all[r * Hl:(r + 1) * Hl], pos, P, r,
                         dq=dq_s, dk=dk_s, dv=dv_s)
    torch.cuda.synchronize()
    for x in (o_seq, dq_s, dk_s, dv_s):
        assert not torch.isnan(x.float()).any()          # the ranks together wrote every head
    cpu = {x: c[x].cpu() for x in ("q", "k", "v", "do")}
    for r in range(P):
        qs, ks = slice(r * Hl, (r + 1) * Hl), slice(r * Hkvl, (r + 1) * Hkvl)
        rq, rk, rv, ro, rl = oracle.attn_bwd(cpu["q"][:, qs].contiguous(), cpu["k"][:, ks].contiguous(),
                                             cpu["v"][:, ks].contiguous(), cpu["do"][:, qs].contiguous(), pos.cpu())
        assert_close(f"O rank {r}", bf16_to_f64(o_seq[:, qs]), ro)
        assert_close(f"LSE rank {r}", lse_all[qs].double().cpu().numpy(), rl)
        assert_grad_close(f"dQ rank {r}", bf16_to_f64(dq_s[:, qs]), rq)
        assert_grad_close(f"dK rank {r}", bf16_to_f64(dk_s[:, ks]), rk)
        assert_grad_close(f"dV rank {r}", bf16_to_f64(dv_s[:, ks]), rv)
