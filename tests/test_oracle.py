"""Pins for the fp64 CPU oracle, checked against things other than itself.

No page prints a numeric worked example, so the oracle is pinned by
hand-derived fixtures (tests/golden), closed forms, brute force on tiny
inputs, a library routine (torch SDPA / autograd in fp64), finite
differences and the invariances the pages fix:

* relayout round trip (the second all-to-all restores sequence sharding,
  page "Hugging Face并行加速：10倍提升超长序列训练效率", section "Ulysses的工作原理",
  step 全体间通信复原);
* head independence: sharded output equals unsharded output (same section,
  closing paragraph: each head's attention is independent);
* packed documents behave as separate documents (page "Ulysses verteilt
  Millionen-Token-Kontexte auf mehrere GPUs", section "Integration in den
  Hugging-Face-Stack").
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import position_ids, random_case

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def f64(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float64).numpy()


def same_doc_mask(pos: np.ndarray) -> np.ndarray:
    """mask[i, j] is True iff j <= i and no document starts in (j, i].

    Written from the definition, independently of oracle.doc_start: a
    document starts at token t iff pos[t] == 0.
    """
    N = len(pos)
    m = np.zeros((N, N), dtype=bool)
    for i in range(N):
        for j in range(i + 1):
            m[i, j] = not any(pos[t] == 0 for t in range(j + 1, i + 1))
    return m


def brute_attention(q, k, v, pos, scale):
    """Full N x N scores, explicit boolean mask, row softmax (numpy fp64)."""
    N, Hl, d = q.shape
    G = Hl // k.shape[1]
    mask = same_doc_mask(np.asarray(pos))
    o = np.zeros((N, Hl, d))
    lse = np.zeros((Hl, N))
    for h in range(Hl):
        s = scale * (q[:, h, :] @ k[:, h // G, :].T)
        s = np.where(mask, s, -np.inf)
        mx = s.max(axis=1, keepdims=True)
        e = np.exp(s - mx)
        l = e.sum(axis=1, keepdims=True)
        o[:, h, :] = (e / l) @ v[:, h // G, :]
        lse[h] = (mx + np.log(l))[:, 0]
    return o, lse


# --------------------------------------------------------------------- relayout

def test_relayout_golden():
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "relayout_N4_P2_H4_d1.txt"))
            if ln.strip() and not ln.startswith("#")]
    src = np.array([[10 * t + h for h in range(4)] for t in range(4)], dtype=np.uint16).reshape(2, 2, 4, 1)
    dst = oracle.seq_to_head(src, N=4, P=2, Hx=4, d=1)
    for r, t, a, b in rows:
        assert dst[r, t, 0, 0] == a and dst[r, t, 1, 0] == b


@pytest.mark.parametrize("N,P,Hx,d", [(4, 2, 4, 1), (16, 1, 3, 8), (64, 4, 8, 32), (96, 8, 8, 16), (40, 2, 2, 128)])
def test_relayout_roundtrip_and_permutation(N, P, Hx, d):
    rng = np.random.default_rng(N * 7 + P)
    x = rng.integers(0, 65536, size=(P, N // P, Hx, d), dtype=np.uint16)
    y = oracle.seq_to_head(x, N, P, Hx, d)
    assert y.shape == (P, N, Hx // P, d)
    back = oracle.head_to_seq(y, N, P, Hx, d)
    assert np.array_equal(back, x)
    # the library's own reshape/transpose states the same exchange as a tensor permutation
    ref = np.transpose(x.reshape(P, N // P, P, Hx // P, d), (2, 0, 1, 3, 4)).reshape(P, N, Hx // P, d)
    assert np.array_equal(y, ref)


def test_relayout_moves_every_element_once():
    N, P, Hx, d = 32, 4, 8, 8     # 2048 distinct labels
    x = np.arange(N * Hx * d, dtype=np.uint16).reshape(P, N // P, Hx, d)
    y = oracle.seq_to_head(x, N, P, Hx, d)
    assert np.array_equal(np.sort(y.reshape(-1)), np.arange(N * Hx * d, dtype=np.uint16))


def test_relayout_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.seq_to_head(np.zeros(12, np.uint16), 6, 4, 4, 1)   # N % P != 0
    with pytest.raises(ValueError):
        oracle.seq_to_head(np.zeros(24, np.uint16), 8, 2, 3, 1)   # H % P != 0


# --------------------------------------------------------------------- doc starts

def test_doc_start_golden():
    lines = [ln.split(":", 1) for ln in open(os.path.join(GOLDEN, "doc_start.txt"))
             if ln.strip() and not ln.startswith("#")]
    for (ka, pa), (kb, sb) in zip(lines[0::2], lines[1::2]):
        assert ka == "pos" and kb == "start"
        pos = np.array(pa.split(), dtype=np.int32)
        assert list(oracle.doc_start(pos)) == [int(t) for t in sb.split()]


def test_doc_start_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(20):
        pos = rng.integers(0, 3, size=50).astype(np.int32)
        ref = [max([j for j in range(i + 1) if pos[j] == 0], default=0) for i in range(50)]
        assert list(oracle.doc_start(pos)) == ref


# --------------------------------------------------------------------- forward

def test_fwd_closed_form_golden():
    rows = [list(map(float, ln.split())) for ln in open(os.path.join(GOLDEN, "attn_closed_form.txt"))
            if ln.strip() and not ln.startswith("#")]
    q = torch.tensor([[[1.0]], [[1.0]]], dtype=torch.bfloat16)
    k = torch.tensor([[[0.0]], [[1.0]]], dtype=torch.bfloat16)
    v = torch.tensor([[[0.0]], [[2.0]]], dtype=torch.bfloat16)
    o, lse = oracle.attn_fwd(q, k, v, [0, 1], scale=1.0)
    for r, oo, ll in rows:
        assert o[int(r), 0, 0] == pytest.approx(oo, abs=1e-15)
        assert lse[0, int(r)] == pytest.approx(ll, abs=1e-15)


@pytest.mark.parametrize("lengths,H,Hkv,d", [
    ([16], 2, 2, 8), ([5, 11], 4, 2, 4), ([1, 3, 1, 7, 4], 4, 1, 16), ([9, 1, 6], 3, 3, 2)])
def test_fwd_matches_brute_force(lengths, H, Hkv, d):
    N = sum(lengths)
    c = random_case(N, H, Hkv, d, lengths, seed=N + H)
    scale = 0.37
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"], scale=scale)
    ob, lb = brute_attention(f64(c["q"]), f64(c["k"]), f64(c["v"]), c["position_ids"].numpy(), scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def test_fwd_lse_matches_torch_logsumexp():
    N, H, d = 24, 2, 8
    c = random_case(N, H, H, d, [N], seed=3)
    _, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    q, k = c["q"].double(), c["k"].double()
    for h in range(H):
        s = (q[:, h] @ k[:, h].T) / math.sqrt(d)
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
        np.testing.assert_allclose(lse[h], torch.logsumexp(s, dim=1).numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("H,Hkv", [(4, 4), (8, 2), (4, 1)])
def test_fwd_matches_sdpa_single_document(H, Hkv):
    N, d = 80, 32
    c = random_case(N, H, Hkv, d, [N], seed=H * 10 + Hkv)
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    G = H // Hkv
    q = c["q"].double().permute(1, 0, 2)[None]
    k = c["k"].double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    v = c["v"].double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)[0].permute(1, 0, 2)
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12, rtol=0)


def test_fwd_uniform_v_returns_v():
    lengths = [7, 1, 20, 4]
    N = sum(lengths)
    c = random_case(N, 4, 2, 16, lengths, seed=11)
    v = torch.full_like(c["v"], 0.0)
    v[..., :] = torch.linspace(-3, 3, 16).to(torch.bfloat16)
    o, _ = oracle.attn_fwd(c["q"], c["k"], v, c["position_ids"])
    ref = np.broadcast_to(f64(v[0, 0]), o.shape)
    np.testing.assert_allclose(o, ref, atol=1e-14, rtol=0)


def test_fwd_one_token_documents():
    N, H, Hkv, d = 12, 4, 2, 8
    c = random_case(N, H, Hkv, d, [1] * N, seed=2)
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    q, k, v = f64(c["q"]), f64(c["k"]), f64(c["v"])
    for i in range(N):
        for h in range(H):
            assert np.array_equal(o[i, h], v[i, h // 2])
            assert lse[h, i] == pytest.approx(np.dot(q[i, h], k[i, h // 2]) / math.sqrt(d), abs=1e-14)


def test_fwd_packed_equals_per_document_and_reorder():
    lengths = [6, 13, 1, 9]
    N, H, Hkv, d = sum(lengths), 4, 2, 16
    c = random_case(N, H, Hkv, d, lengths, seed=21)
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    starts = np.cumsum([0] + lengths)
    for a, b in zip(starts[:-1], starts[1:]):
        od, ld = oracle.attn_fwd(c["q"][a:b], c["k"][a:b], c["v"][a:b], c["position_ids"][a:b])
        assert np.array_equal(o[a:b], od) and np.array_equal(lse[:, a:b], ld)
    # reordering documents permutes the output the same way
    order = [2, 0, 3, 1]
    idx = np.concatenate([np.arange(starts[t], starts[t + 1]) for t in order])
    pos2 = position_ids([lengths[t] for t in order])
    o2, l2 = oracle.attn_fwd(c["q"][idx], c["k"][idx], c["v"][idx], pos2)
    assert np.array_equal(o2, o[idx]) and np.array_equal(l2, lse[:, idx])


def _as_u16(a: np.ndarray) -> np.ndarray:
    """View an fp64 [N][Hl][d] array as 16-bit words [N][Hl][4d] (pure data movement)."""
    return np.ascontiguousarray(a).view(np.uint16)


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_sharded_equals_unsharded(P):
    lengths = [40, 3, 21]
    N, H, Hkv, d = 64, 8, 8, 16
    c = random_case(N, H, Hkv, d, lengths, seed=77)
    # reference: one rank holding every head
    o_full, lse_full = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    # Ulysses: exchange to head slices, local attention per rank, exchange back
    qs = oracle.seq_to_head(c["q"], N, P, H, d)
    ks = oracle.seq_to_head(c["k"], N, P, Hkv, d)
    vs = oracle.seq_to_head(c["v"], N, P, Hkv, d)
    o_ranks = np.empty((P, N, H // P, d))
    lse_ranks = []
    for r in range(P):
        o_r, lse_r = oracle.attn_fwd(qs[r], ks[r], vs[r], c["position_ids"])
        o_ranks[r] = o_r
        lse_ranks.append(lse_r)
    back = oracle.head_to_seq(_as_u16(o_ranks), N, P, H, 4 * d).reshape(-1).view(np.float64)
    assert np.array_equal(back.reshape(N, H, d), o_full)
    assert np.array_equal(np.concatenate(lse_ranks, axis=0), lse_full)


def test_sharded_equals_unsharded_gqa():
    # GQA: 8 query heads over 4 KV heads, P = 2 -> each rank: 4 Q heads, 2 KV heads
    lengths = [30, 34]
    N, H, Hkv, d, P = 64, 8, 4, 8, 2
    c = random_case(N, H, Hkv, d, lengths, seed=78)
    o_full, _ = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    qs = oracle.seq_to_head(c["q"], N, P, H, d)
    ks = oracle.seq_to_head(c["k"], N, P, Hkv, d)
    vs = oracle.seq_to_head(c["v"], N, P, Hkv, d)
    for r in range(P):
        o_r, _ = oracle.attn_fwd(qs[r], ks[r], vs[r], c["position_ids"])
        assert np.array_equal(o_r, o_full[:, r * H // P:(r + 1) * H // P])


def test_fwd_row_subset_matches_full():
    lengths = [17, 30, 17]
    N = sum(lengths)
    c = random_case(N, 2, 1, 8, lengths, seed=4)
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    rows = [0, 16, 17, 40, 63]
    o2, l2 = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"], rows=rows)
    assert np.array_equal(o2, o[rows]) and np.array_equal(l2, lse[:, rows])


# --------------------------------------------------------------------- backward

def _torch_attention_f64(q, k, v, pos, scale):
    """Explicit masked attention in torch fp64 (for autograd)."""
    N, Hl, d = q.shape
    G = Hl // k.shape[1]
    mask = torch.from_numpy(same_doc_mask(np.asarray(pos)))
    outs = []
    for h in range(Hl):
        s = scale * (q[:, h] @ k[:, h // G].T)
        s = s.masked_fill(~mask, float("-inf"))
        outs.append(torch.softmax(s, dim=1) @ v[:, h // G])
    return torch.stack(outs, dim=1)


@pytest.mark.parametrize("lengths,H,Hkv,d", [([12], 2, 2, 8), ([5, 1, 10], 4, 2, 8), ([3, 9], 4, 1, 4)])
def test_bwd_matches_autograd(lengths, H, Hkv, d):
    N = sum(lengths)
    c = random_case(N, H, Hkv, d, lengths, seed=N * 3 + H, with_grad_out=True)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv, o, lse = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"])
    q = c["q"].double().requires_grad_()
    k = c["k"].double().requires_grad_()
    v = c["v"].double().requires_grad_()
    out = _torch_attention_f64(q, k, v, c["position_ids"].numpy(), scale)
    (out * c["do"].double()).sum().backward()
    np.testing.assert_allclose(o, out.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-11, rtol=0)


def test_bwd_finite_differences():
    lengths = [4, 6]
    N, H, Hkv, d = 10, 2, 1, 4
    c = random_case(N, H, Hkv, d, lengths, seed=9, with_grad_out=True)
    scale = 0.5
    dq, dk, dv, _, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"], scale=scale)
    q0, k0, v0, g = f64(c["q"]), f64(c["k"]), f64(c["v"]), f64(c["do"])
    pos = c["position_ids"].numpy()

    def loss(q, k, v):
        return float((brute_attention(q, k, v, pos, scale)[0] * g).sum())

    eps = 1e-6
    for name, base, grad in (("q", q0, dq), ("k", k0, dk), ("v", v0, dv)):
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args = {"q": q0, "k": k0, "v": v0}
            args[name] = plus
            lp = loss(args["q"], args["k"], args["v"])
            args[name] = minus
            lm = loss(args["q"], args["k"], args["v"])
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, atol=1e-7, rtol=0, err_msg=name)


def test_bwd_sum_rules_per_document():
    lengths = [33, 1, 30]
    N, H, Hkv, d = sum(lengths), 4, 2, 16
    c = random_case(N, H, Hkv, d, lengths, seed=31, with_grad_out=True)
    dq, dk, dv, o, lse = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"])
    g = f64(c["do"])
    starts = np.cumsum([0] + lengths)
    G = H // Hkv
    for a, b in zip(starts[:-1], starts[1:]):
        for kvh in range(Hkv):
            # rows of dS sum to zero, so the keys' dK sum to zero within a document
            np.testing.assert_allclose(dk[a:b, kvh].sum(axis=0), 0.0, atol=1e-11)
            # rows of P sum to one, so the keys' dV sum to the group's upstream gradient
            np.testing.assert_allclose(dv[a:b, kvh].sum(axis=0),
                                       g[a:b, kvh * G:(kvh + 1) * G].sum(axis=(0, 1)), atol=1e-11)
    o2, l2 = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)


# Position ids that do not count 0, 1, 2, ... from token 0: the first document
# starts at token 0 whatever its id, every later 0 starts a new document, and
# any other value (a jump, a repeat, a negative id) is ignored.
IRREGULAR_POS = [5, 6, 7, 0, 1, 9, 9, -3, 0, 2, 0, 1, 1, 4]


def test_bwd_sampled_matches_full():
    """The sampled backward equals the full backward on the rows and keys it is
    asked for (first and last keys of documents, a one-token document, GQA)."""
    lengths = [40, 1, 55, 32]
    N, H, Hkv, d = sum(lengths), 6, 2, 16
    c = random_case(N, H, Hkv, d, lengths, seed=17, with_grad_out=True)
    dq, dk, dv, _, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"])
    rows = [0, 3, 39, 40, 41, 95, 96, 127]
    keys = [0, 1, 39, 40, 41, 42, 94, 95, 96, 120, 127]
    sq, sk, sv = oracle.attn_bwd_sampled(c["q"], c["k"], c["v"], c["do"], c["position_ids"], rows, keys)
    assert np.array_equal(sq, dq[rows])
    assert np.array_equal(sk, dk[keys]) and np.array_equal(sv, dv[keys])


def test_bwd_sampled_matches_autograd_irregular_ids():
    """Against torch autograd of the explicit masked attention, with position
    ids that start above 0, jump, repeat and go negative."""
    pos = np.array(IRREGULAR_POS, dtype=np.int32)
    N, H, Hkv, d = len(pos), 4, 2, 8
    c = random_case(N, H, Hkv, d, [N], seed=23, with_grad_out=True)
    c["position_ids"] = torch.from_numpy(pos)
    scale = 1.0 / math.sqrt(d)
    q = c["q"].double().requires_grad_()
    k = c["k"].double().requires_grad_()
    v = c["v"].double().requires_grad_()
    out = _torch_attention_f64(q, k, v, pos, scale)
    (out * c["do"].double()).sum().backward()
    rows = list(range(N))
    sq, sk, sv = oracle.attn_bwd_sampled(c["q"], c["k"], c["v"], c["do"], c["position_ids"], rows, rows)
    np.testing.assert_allclose(sq, q.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(sk, k.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(sv, v.grad.numpy(), atol=1e-11, rtol=0)
    dq, dk, dv, o, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"])
    np.testing.assert_allclose(o, out.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-11, rtol=0)


def test_fwd_irregular_ids_match_brute_force():
    pos = np.array(IRREGULAR_POS, dtype=np.int32)
    N, H, Hkv, d = len(pos), 4, 1, 8
    c = random_case(N, H, Hkv, d, [N], seed=29)
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], pos)
    bo, bl = brute_attention(f64(c["q"]), f64(c["k"]), f64(c["v"]), pos, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(o, bo, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, bl, atol=1e-12, rtol=0)


# --------------------------------------------------------------------- ring steps

def _brute_window(q, k, v, pos, scale, kv_lo, kv_hi):
    """brute_attention with the keys further restricted to [kv_lo, kv_hi);
    rows that see no key get o = 0, lse = -inf."""
    N, Hl, d = q.shape
    G = Hl // k.shape[1]
    mask = same_doc_mask(np.asarray(pos))
    cols = np.arange(N)
    mask &= ((cols >= kv_lo) & (cols < kv_hi))[None, :]
    o = np.zeros((N, Hl, d))
    lse = np.full((Hl, N), -np.inf)
    for h in range(Hl):
        s = scale * (q[:, h, :] @ k[:, h // G, :].T)
        for i in range(N):
            if not mask[i].any():
                continue
            si = s[i][mask[i]]
            mx = si.max()
            e = np.exp(si - mx)
            o[i, h] = (e / e.sum()) @ v[mask[i], h // G, :]
            lse[h, i] = mx + np.log(e.sum())
    return o, lse


@pytest.mark.parametrize("kv_lo,kv_hi", [(0, 45), (8, 16), (13, 30), (20, 20), (44, 45), (0, 1)])
def test_window_matches_brute_force(kv_lo, kv_hi):
    lengths = [12, 1, 20, 12]
    N, H, Hkv, d = sum(lengths), 4, 2, 8
    c = random_case(N, H, Hkv, d, lengths, seed=37)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd_window(c["q"], c["k"], c["v"], c["position_ids"], kv_lo, kv_hi)
    bo, bl = _brute_window(f64(c["q"]), f64(c["k"]), f64(c["v"]), c["position_ids"].numpy(), scale, kv_lo, kv_hi)
    np.testing.assert_allclose(o, bo, atol=1e-12, rtol=0)
    assert np.array_equal(np.isinf(lse), np.isinf(bl))
    np.testing.assert_allclose(lse[np.isfinite(lse)], bl[np.isfinite(bl)], atol=1e-12, rtol=0)


def test_window_over_all_keys_equals_attention():
    lengths = [30, 2, 33]
    N = sum(lengths)
    c = random_case(N, 4, 1, 16, lengths, seed=41)
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    ow, lw = oracle.attn_fwd_window(c["q"], c["k"], c["v"], c["position_ids"], 0, N)
    assert np.array_equal(o, ow) and np.array_equal(lse, lw)


def test_merge_closed_form():
    """Two partials with sums e^a and e^b: the merged output is their average
    weighted by those sums, and the merged lse is log(e^a + e^b); a partial
    with lse = -inf contributes nothing; all -inf gives o = 0, lse = -inf."""
    a, b = 0.3, -1.7
    x = np.array([1.0, -2.0, 0.5])
    y = np.array([4.0, 0.25, -1.0])
    o_parts = np.zeros((3, 3, 1, 3))
    lse_parts = np.full((3, 1, 3), -np.inf)
    o_parts[0, 0, 0], o_parts[1, 0, 0], lse_parts[0, 0, 0], lse_parts[1, 0, 0] = x, y, a, b
    o_parts[1, 1, 0], lse_parts[1, 0, 1] = y, b          # row 1: only the second partial sees keys
    o, lse = oracle.merge(o_parts, lse_parts)
    ea, eb = math.exp(a), math.exp(b)
    np.testing.assert_allclose(o[0, 0], (ea * x + eb * y) / (ea + eb), atol=1e-15)
    assert lse[0, 0] == pytest.approx(math.log(ea + eb), abs=1e-15)
    np.testing.assert_allclose(o[1, 0], y, atol=1e-15)
    assert lse[0, 1] == pytest.approx(b, abs=1e-15)
    assert np.all(o[2] == 0.0) and lse[0, 2] == -np.inf


@pytest.mark.parametrize("bounds", [[0, 16, 32, 48, 65], [0, 5, 40, 65], [0, 65]])
def test_merged_windows_equal_attention(bounds):
    """Attention over disjoint key windows that cover every key, merged, is
    the attention over all keys: the identity a ring of chunk steps relies on."""
    lengths = [30, 2, 33]
    N = sum(lengths)
    c = random_case(N, 4, 2, 16, lengths, seed=43)
    o, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    parts = [oracle.attn_fwd_window(c["q"], c["k"], c["v"], c["position_ids"], lo, hi)
             for lo, hi in zip(bounds[:-1], bounds[1:])]
    om, lm = oracle.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(om, o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lm, lse, atol=1e-12, rtol=0)


# --------------------------------------------------------------------- projections

def _bf(shape, seed):
    from workloads import normal_bf16
    return normal_bf16(shape, seed)


def test_qkv_proj_identity_weights_is_the_exchange():
    """With w_qkv = [I; I; I] (hidden = H*d = Hkv*d), the projection returns x
    itself as Q, K and V, and the layout is exactly seq_to_head's."""
    N, P, H, d = 16, 2, 4, 8
    x = _bf((N, H * d), 3)
    eye = torch.eye(H * d, dtype=torch.bfloat16)
    w = torch.cat([eye, eye, eye], 0)
    q, k, v = oracle.qkv_proj(x, w, P, H, H, d)
    ref = oracle.seq_to_head(x.view(N, H, d), N, P, H, d)
    bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for t in (q, k, v):
        assert np.array_equal(bits(t), ref)


def test_qkv_proj_closed_form_and_head_order():
    """One token, hand-built weights: column block j of w_qkv picks x[j] times
    a known factor, so each head of Q, K, V holds a known value at a known
    rank and position."""
    P, H, Hkv, d = 2, 2, 2, 1          # hidden = 2, six output columns: q0 q1 k0 k1 v0 v1
    x = torch.tensor([[1.5, -2.0]], dtype=torch.bfloat16)
    w = torch.tensor([[1, 0], [0, 1], [2, 0], [0, 2], [1, 1], [1, -1]], dtype=torch.bfloat16)
    q, k, v = oracle.qkv_proj(x, w, P, H, Hkv, d)
    assert q.shape == (2, 1, 1, 1) and q[0, 0, 0, 0] == 1.5 and q[1, 0, 0, 0] == -2.0
    assert k[0, 0, 0, 0] == 3.0 and k[1, 0, 0, 0] == -4.0
    assert v[0, 0, 0, 0] == -0.5 and v[1, 0, 0, 0] == 3.5


def test_out_proj_identity_weights_is_the_inverse_exchange():
    P, N, Hl, d = 4, 8, 2, 4
    o = _bf((P, N, Hl, d), 5)
    y = oracle.out_proj(o, torch.eye(P * Hl * d, dtype=torch.bfloat16))
    back = oracle.head_to_seq(o, N, P, P * Hl, d).reshape(N, P * Hl * d)
    bits = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, back)


def test_projections_against_torch_matmul():
    N, P, H, Hkv, d, hidden = 12, 2, 4, 2, 8, 24
    x, w = _bf((N, hidden), 7), _bf(((H + 2 * Hkv) * d, hidden), 8)
    q, k, v = oracle.qkv_proj(x, w, P, H, Hkv, d)
    y = x.double() @ w.double().T
    np.testing.assert_allclose(q[1, :, 0], y[:, (H // P) * d:(H // P + 1) * d].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(v[1, :, 0], y[:, (H + Hkv + Hkv // P) * d:(H + Hkv + Hkv // P + 1) * d].numpy(),
                               rtol=0, atol=1e-12)
    rows = [0, 5, 11]
    qs, _, _ = oracle.qkv_proj(x, w, P, H, Hkv, d, rows=rows)
    assert np.array_equal(qs, q[:, rows])
    o = _bf((P, N, H // P, d), 9)
    wo = _bf((hidden, H * d), 10)
    seq = o.double().permute(1, 0, 2, 3).reshape(N, H * d)
    np.testing.assert_allclose(oracle.out_proj(o, wo), (seq @ wo.double().T).numpy(), rtol=0, atol=1e-12)


def test_thread_count_setting_leaves_results_unchanged():
    """The host thread count of the oracle's loops is a launch setting: the
    same inputs give bit-identical results with one thread and with all."""
    n0 = oracle.max_threads()
    c = random_case(300, 2, 1, 32, [200, 100], seed=5, device="cpu")
    try:
        oracle.set_num_threads(1)
        assert oracle.max_threads() == 1
        o1, l1 = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    finally:
        oracle.set_num_threads(n0)
    assert oracle.max_threads() == n0
    o2, l2 = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
