"""Parity of the relayout kernels (the emulated all-to-alls) with the oracle:
bit-exact on every element."""
import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_inputs, normal_bf16

pytestmark = pytest.mark.gpu


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("N,P,Hx,d", [(256, 2, 4, 32), (384, 4, 8, 64), (640, 8, 8, 128), (1000, 2, 2, 128),
                                      (96, 1, 3, 32), (1024, 8, 32, 128), (64, 4, 4, 32), (200, 2, 64, 128)])
def test_seq_to_head_all_ranks_and_inverse(N, P, Hx, d):
    import long_context_sequence_ulysses_b200 as U
    x = normal_bf16((N, Hx, d), seed=N + P, device="cuda", stream_id=7)
    y = U.seq_to_head(x, P)
    ref = oracle.seq_to_head(x, N, P, Hx, d)
    assert np.array_equal(_u16(y), ref)
    back = U.head_to_seq(y, P)
    assert np.array_equal(_u16(back), _u16(x))
    assert np.array_equal(_u16(back), oracle.head_to_seq(ref, N, P, Hx, d).reshape(N, Hx, d))


@pytest.mark.parametrize("N,P,Hx,d", [(512, 4, 8, 128), (256, 2, 4, 32), (96, 8, 16, 64)])
def test_single_rank_slices(N, P, Hx, d):
    import long_context_sequence_ulysses_b200 as U
    x = normal_bf16((N, Hx, d), seed=3, device="cuda", stream_id=8)
    ref = oracle.seq_to_head(x, N, P, Hx, d)
    out = torch.full((N, Hx, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    for r in range(P):
        s = U.seq_to_head(x, P, rank=r)
        assert np.array_equal(_u16(s), ref[r])
        U.head_to_seq(s, P, rank=r, out=out)
    assert np.array_equal(_u16(out), _u16(x))


def test_empty_is_noop():
    import long_context_sequence_ulysses_b200 as U
    x = torch.empty((0, 8, 128), dtype=torch.bfloat16, device="cuda")
    assert U.seq_to_head(x, 4).shape == (4, 0, 2, 128)


@pytest.mark.parametrize("name", ["llama8b", "long131k", "train"])
def test_workload_relayouts_full_size(name):
    """Full-size exchanges of Q, K and V: every element checked against the
    oracle's index formula (K/V whole; Q whole for llama8b and train, by
    ranks for long131k)."""
    import long_context_sequence_ulysses_b200 as U
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda", with_grad_out=False)
    for key, Hx in (("k", w.Hkv), ("v", w.Hkv), ("q", w.H)):
        x = inp[key]
        y = U.seq_to_head(x, w.P)
        xh = _u16(x)
        ref = oracle.seq_to_head(xh, w.N, w.P, Hx, w.d)
        assert np.array_equal(_u16(y), ref), key
        back = U.head_to_seq(y, w.P)
        assert torch.equal(back.view(torch.int16), x.view(torch.int16)), key
        del y, back, ref, xh
    torch.cuda.empty_cache()


def test_million_relayout_properties():
    """Million-token workload, all 8 rank shards of Q, K and V: the result
    equals the tensor permutation [P][N/P][P][H/P][d] -> [P][P][N/P][H/P][d]
    and the inverse restores the input bit for bit; a sample of tokens is
    checked against the oracle's index formula."""
    import long_context_sequence_ulysses_b200 as U
    w = WORKLOADS["million"]
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    for Hx in (w.Hkv, w.H):
        x = torch.randint(-32768, 32767, (w.N, Hx, w.d), dtype=torch.int16, device="cuda", generator=g)
        xb = x.view(torch.bfloat16)
        y = U.seq_to_head(xb, w.P)
        perm = x.view(w.P, w.N // w.P, w.P, Hx // w.P, w.d).permute(2, 0, 1, 3, 4).reshape(w.P, w.N, Hx // w.P, w.d)
        assert torch.equal(y.view(torch.int16), perm)
        del perm
        back = U.head_to_seq(y, w.P)
        assert torch.equal(back.view(torch.int16), x)
        # sampled tokens through the oracle: a small problem made of the same
        # rows of every rank shard
        rng = np.random.default_rng(5)
        m = np.sort(rng.choice(w.N // w.P, 64, replace=False))
        sub = x.view(w.P, w.N // w.P, Hx, w.d)[:, torch.from_numpy(m).cuda()].contiguous()
        ref = oracle.seq_to_head(sub.cpu().numpy().view(np.uint16), w.P * len(m), w.P, Hx, w.d)
        got = y.view(torch.int16).view(w.P, w.P, w.N // w.P, Hx // w.P, w.d)[:, :, torch.from_numpy(m).cuda()]
        assert np.array_equal(got.reshape(w.P, w.P * len(m), Hx // w.P, w.d).cpu().numpy().view(np.uint16), ref)
        del x, y, back
        torch.cuda.empty_cache()


@pytest.mark.parametrize("N,P,row_heads,head0,Hx,d", [(256, 2, 8, 4, 4, 32), (384, 4, 32, 8, 8, 128),
                                                     (96, 1, 3, 1, 2, 64), (512, 8, 24, 16, 8, 128)])
def test_head_slice_exchanges(N, P, row_heads, head0, Hx, d):
    """The exchange of a slice of heads [head0, head0+Hx) of wider rows, read
    and written in place: equal to the oracle's exchange of that slice, and
    the unpack leaves the other heads of the destination untouched."""
    import long_context_sequence_ulysses_b200 as U
    x = normal_bf16((N, row_heads, d), seed=N + head0, device="cuda", stream_id=10)
    y = U.seq_to_head(x, P, heads=(head0, Hx))
    ref = oracle.seq_to_head(x[:, head0:head0 + Hx].contiguous(), N, P, Hx, d)
    assert np.array_equal(_u16(y), ref)
    out = torch.full_like(x, float("nan"))
    U.head_to_seq(y, P, out=out, head0=head0)
    assert np.array_equal(_u16(out[:, head0:head0 + Hx]), _u16(x[:, head0:head0 + Hx]))
    rest = torch.cat([out[:, :head0], out[:, head0 + Hx:]], dim=1)
    assert torch.isnan(rest.float()).all()
