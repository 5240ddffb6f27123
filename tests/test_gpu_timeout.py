"""Failure detection without a GPU fault: a bounded device-side wait that runs
out (a barrier that nothing arrives on, switched on by a host-side test flag)
makes the forward, or the backward, drain and return, ulysses_sync_status
reports ULYSSES_ERR_TIMEOUT, and the context stays usable: the next launch is
correct."""
import pytest
import torch

import oracle
from helpers import assert_close, assert_grad_close, bf16_to_f64
from workloads import random_case

pytestmark = pytest.mark.gpu


def test_forward_wait_runs_out_and_context_survives():
    import long_context_sequence_ulysses_b200 as U
    c = random_case(1024, 4, 2, 128, [700, 324], seed=13, device="cuda")
    ws = torch.empty(U.workspace_bytes(1024, 4, 2, 128), dtype=torch.uint8, device="cuda")
    U.set_wait_limit_ns(100_000_000)           # 0.1 s
    try:
        U.set_debug_flags(1)
        U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"], ws=ws)
        with pytest.raises(U.UlyssesError) as e:
            U.sync_status(ws)
        assert e.value.code == U.ULYSSES_ERR_TIMEOUT
    finally:
        U.set_debug_flags(0)
        U.set_wait_limit_ns(0)
    o, lse = U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"], ws=ws)
    U.sync_status(ws)
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert_close("O", bf16_to_f64(o), ro)
    assert_close("LSE", lse.double().cpu().numpy(), rl)


def test_backward_wait_runs_out_and_context_survives():
    """The same for the backward: the first dK/dV CTA's element-wise warps wait
    on a barrier nothing arrives on; every role of every CTA drains (the dQ
    kernel after it finds the status set), the status reports the timeout,
    and the next backward on the same workspace is correct."""
    import long_context_sequence_ulysses_b200 as U
    c = random_case(1024, 4, 2, 128, [700, 324], seed=17, device="cuda", with_grad_out=True)
    o, lse = U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    ws = torch.empty(U.workspace_bytes(1024, 4, 2, 128, backward=True), dtype=torch.uint8, device="cuda")
    U.set_wait_limit_ns(100_000_000)           # 0.1 s
    try:
        U.set_debug_flags(2)
        U.attn_bwd(c["q"], c["k"], c["v"], o, c["do"], lse, c["position_ids"], ws=ws)
        with pytest.raises(U.UlyssesError) as e:
            U.sync_status(ws)
        assert e.value.code == U.ULYSSES_ERR_TIMEOUT
    finally:
        U.set_debug_flags(0)
        U.set_wait_limit_ns(0)
    dq, dk, dv = U.attn_bwd(c["q"], c["k"], c["v"], o, c["do"], lse, c["position_ids"], ws=ws)
    U.sync_status(ws)
    rq, rk, rv, _, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"])
    assert_grad_close("dQ", bf16_to_f64(dq), rq)
    assert_grad_close("dK", bf16_to_f64(dk), rk)
    assert_grad_close("dV", bf16_to_f64(dv), rv)
