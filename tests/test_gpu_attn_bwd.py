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
from helpers import assert_grad_close, bf16_to_f64
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


def test_train_workload_documents():
    """Rank 0 of the training workload, through the same launches the
    benchmark times; whole documents compared against the oracle."""
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
    lengths = np.array(inp["lengths"])
    starts = np.concatenate([[0], np.cumsum(lengths)[:-1]])
    # first, last, shortest and a mid-length document (skipping very long ones)
    cand = [0, len(lengths) - 1, int(np.argmin(lengths))]
    order = np.argsort(lengths)
    cand.append(int(order[len(order) // 2]))
    picked = sorted({t for t in cand if lengths[t] <= 9000})
    assert picked
    for t in picked:
        a, b = int(starts[t]), int(starts[t] + lengths[t])
        sl = slice(a, b)
        rq, rk, rv, _, _ = oracle.attn_bwd(q[sl].cpu(), k[sl].cpu(), v[sl].cpu(), do[sl].cpu(), pos[sl].cpu())
        assert_grad_close(f"dQ doc {t}", bf16_to_f64(dq[sl]), rq)
        assert_grad_close(f"dK doc {t}", bf16_to_f64(dk[sl]), rk)
        assert_grad_close(f"dV doc {t}", bf16_to_f64(dv[sl]), rv)


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
