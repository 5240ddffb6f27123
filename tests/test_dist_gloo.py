"""The multi-GPU Ulysses exchange (long_context_sequence_ulysses_b200.dist),
run as world_size 2 and 4 gloo processes on the CPU with the oracle standing
in for the local kernels: the sharded result must equal the unsharded
oracle's attention bit for bit (after the same bf16 rounding), since the
exchange only moves data and heads are independent."""
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from workloads import random_case


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_world(world: int, case: dict):
    import dist_worker
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=dist_worker.worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            r, o, lse, pos, heads = q.get(timeout=90)
            assert not (isinstance(o, str) and o == "error"), f"rank {r}: {lse}"
            results[r] = (o, lse, pos, heads)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    return results


def _check_against_unsharded(world: int, case: dict, results: dict):
    c = random_case(case["N"], case["H"], case["Hkv"], case["d"], case["lengths"], seed=case["seed"])
    ref_o, ref_lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    ref_bits = torch.from_numpy(ref_o).to(torch.bfloat16).view(torch.int16).numpy()
    n_loc = case["N"] // world
    seen = []
    for r in range(world):
        o, lse, pos, heads = results[r]
        assert np.array_equal(o, ref_bits[r * n_loc:(r + 1) * n_loc])          # this rank's sequence shard
        assert np.array_equal(lse, ref_lse[heads])                             # this rank's heads
        assert np.array_equal(pos, c["position_ids"].numpy())
        seen += list(heads)
    assert sorted(seen) == list(range(case["H"]))                             # every head exactly once


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_exchange_matches_unsharded(world):
    case = {"N": 64, "H": 8, "Hkv": 4, "d": 32, "lengths": [23, 1, 40], "seed": 12}
    results = _run_world(world, case)
    for r in range(world):                                                   # contiguous head blocks
        assert list(results[r][3]) == list(range(r * case["H"] // world, (r + 1) * case["H"] // world))
    _check_against_unsharded(world, case, results)


@pytest.mark.parametrize("world,chunks", [(2, 2), (2, 1), (4, 2)])
def test_head_chunked_exchange_matches_unsharded(world, chunks):
    """Heads in chunks, the next chunk's exchange in flight while the current
    one is computed: the same result, each head on the rank the chunking
    assigns it to."""
    case = {"N": 64, "H": 16, "Hkv": 8, "d": 32, "lengths": [30, 2, 32], "seed": 5, "chunks": chunks}
    results = _run_world(world, case)
    _check_against_unsharded(world, case, results)


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_backward_exchange_matches_unsharded(world):
    """The backward across ranks: dO crosses the first exchange, each rank
    computes the gradients of its heads, dQ/dK/dV cross the second exchange
    back to sequence shards. Every rank's shards of dQ, dK and dV equal the
    unsharded oracle's gradients (rounded to bf16) bit for bit."""
    case = {"N": 64, "H": 8, "Hkv": 4, "d": 16, "lengths": [23, 1, 40], "seed": 19, "backward": True}
    results = _run_world(world, case)
    c = random_case(case["N"], case["H"], case["Hkv"], case["d"], case["lengths"], seed=case["seed"],
                    with_grad_out=True)
    rq, rk, rv, ro, _ = oracle.attn_bwd(c["q"], c["k"], c["v"], c["do"], c["position_ids"])
    bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy()
    n_loc = case["N"] // world
    for r in range(world):
        o, (dq, dk, dv), pos, _ = results[r]
        sl = slice(r * n_loc, (r + 1) * n_loc)
        assert np.array_equal(o, bits(ro)[sl])
        assert np.array_equal(dq, bits(rq)[sl])
        assert np.array_equal(dk, bits(rk)[sl])
        assert np.array_equal(dv, bits(rv)[sl])
