"""Parity of the projection GEMMs (QKV before the exchange, output after it,
each with the exchange's relayout fused in) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, bf16_to_f64
from workloads import WORKLOADS, normal_bf16, projection_inputs

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("N,P,H,Hkv,d,hidden", [
    (512, 2, 4, 2, 64, 256),      # 512 output columns: 256-wide tiles
    (300, 2, 4, 2, 64, 256),      # ragged last row tile
    (256, 2, 4, 4, 32, 128),      # the tiny workload's shape: 384 columns, 128-wide tiles
    (640, 4, 8, 4, 128, 1024),
    (1000, 8, 32, 8, 128, 512),   # llama8b heads, short hidden
])
def test_qkv_proj_matches_oracle(N, P, H, Hkv, d, hidden):
    import long_context_sequence_ulysses_b200 as U
    x = normal_bf16((N, hidden), seed=N, device="cuda", stream_id=11)
    w = normal_bf16(((H + 2 * Hkv) * d, hidden), seed=N, device="cuda", prescale=hidden ** -0.5, stream_id=12)
    q, k, v = U.qkv_proj(x, w, P, H, Hkv, d)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_proj(x, w, P, H, Hkv, d)
    assert_close("Q", bf16_to_f64(q), rq)
    assert_close("K", bf16_to_f64(k), rk)
    assert_close("V", bf16_to_f64(v), rv)


@pytest.mark.parametrize("N,P,H,d,hidden", [(512, 2, 4, 64, 256), (300, 2, 4, 128, 384), (640, 8, 32, 128, 1024)])
def test_out_proj_matches_oracle(N, P, H, d, hidden):
    import long_context_sequence_ulysses_b200 as U
    o = normal_bf16((P, N, H // P, d), seed=N + 1, device="cuda", stream_id=13)
    w = normal_bf16((hidden, H * d), seed=N + 1, device="cuda", prescale=(H * d) ** -0.5, stream_id=14)
    y = U.out_proj(o, w)
    torch.cuda.synchronize()
    assert_close("Y", bf16_to_f64(y), oracle.out_proj(o, w))


def test_identity_weights_give_the_exchanges_bit_exactly():
    """With identity weights the projections are exactly the two exchanges:
    qkv_proj = seq_to_head of x, out_proj = head_to_seq (bit for bit: each
    output is one product by 1.0, rounded back to the bf16 it came from)."""
    import long_context_sequence_ulysses_b200 as U
    N, P, H, d = 384, 4, 8, 64
    x = normal_bf16((N, H * d), seed=3, device="cuda", stream_id=15)
    eye = torch.eye(H * d, dtype=torch.bfloat16, device="cuda")
    q, k, v = U.qkv_proj(x, torch.cat([eye, eye, eye]), P, H, H, d)
    ref = U.seq_to_head(x.view(N, H, d), P)
    for t in (q, k, v):
        assert torch.equal(t.view(torch.int16), ref.view(torch.int16))
    y = U.out_proj(q, eye)
    assert torch.equal(y.view(torch.int16), x.view(torch.int16))


def test_projections_llama8b_size():
    """The llama8b layer shapes (32768 tokens, hidden 4096, 32 / 8 heads over
    8 ranks): sampled token rows of Q, K, V and of the output projection."""
    import long_context_sequence_ulysses_b200 as U
    w = WORKLOADS["llama8b"]
    inp = projection_inputs(w, device="cuda")
    q, k, v = U.qkv_proj(inp["x"], inp["w_qkv"], w.P, w.H, w.Hkv, w.d)
    o = normal_bf16((w.P, w.N, w.Hl, w.d), seed=9, device="cuda", stream_id=16)
    y = U.out_proj(o, inp["w_o"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, 127, 128, w.N - 129, w.N - 1], rng.integers(0, w.N, 120)]))
    rt = torch.from_numpy(rows).cuda()
    rq, rk, rv = oracle.qkv_proj(inp["x"].cpu(), inp["w_qkv"].cpu(), w.P, w.H, w.Hkv, w.d, rows=rows)
    assert_close("Q", bf16_to_f64(q[:, rt]), rq)
    assert_close("K", bf16_to_f64(k[:, rt]), rk)
    assert_close("V", bf16_to_f64(v[:, rt]), rv)
    assert_close("Y", bf16_to_f64(y[rt]), oracle.out_proj(o.cpu(), inp["w_o"].cpu(), rows=rows))
