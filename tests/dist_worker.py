"""Worker for the multi-process (gloo, CPU) tests of the Ulysses exchange.

Each process holds one sequence shard, runs the library's exchange logic
(long_context_sequence_ulysses_b200.dist) with CPU stand-ins for the local
steps — the oracle's relayouts as pack/unpack and the oracle's attention —
and returns its shard of O and LSE through a queue."""
import os

import numpy as np
import torch
import torch.distributed as dist


def _bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def worker(rank: int, world: int, port: int, case: dict, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        _run(rank, world, case, out_q)
    except Exception as e:  # report instead of leaving the parent waiting
        out_q.put((rank, "error", repr(e), None, None))
        raise
    finally:
        dist.destroy_process_group()


def _run(rank, world, case, out_q):
    if True:
        import oracle
        from long_context_sequence_ulysses_b200 import dist as udist
        from workloads import random_case

        c = random_case(case["N"], case["H"], case["Hkv"], case["d"], case["lengths"], seed=case["seed"],
                        with_grad_out=bool(case.get("backward")))
        N, d = case["N"], case["d"]
        n_loc = N // world
        sl = slice(rank * n_loc, (rank + 1) * n_loc)

        def pack(x, G):
            n, Hx, dd = x.shape
            return _bits_to_bf16(oracle.seq_to_head(x, n, G, Hx, dd))

        def unpack(y, G):
            Gp, n, Hl, dd = y.shape
            return _bits_to_bf16(oracle.head_to_seq(y, n, G, Hl * G, dd)).view(n, Hl * G, dd)

        def attn(q, k, v, pos, scale=None):
            o, lse = oracle.attn_fwd(q, k, v, pos, scale=scale)
            return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse)

        args = (c["q"][sl].contiguous(), c["k"][sl].contiguous(), c["v"][sl].contiguous(),
                c["position_ids"][sl].contiguous())
        if case.get("backward"):
            def attn_bwd(q, k, v, o, g, lse, pos, scale=None):
                # the oracle recomputes O and LSE itself from q, k, v
                dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, g, pos, scale=scale)
                return tuple(torch.from_numpy(x).to(torch.bfloat16) for x in (dq, dk, dv))

            o_loc, lse, pos, saved = udist.attention_forward(*args, attn=attn, pack=pack, unpack=unpack,
                                                             keep_for_backward=True)
            dq, dk, dv = udist.attention_backward(saved, lse, pos, c["do"][sl].contiguous(), attn_bwd=attn_bwd,
                                                  pack=pack, unpack=unpack)
            out_q.put((rank, o_loc.view(torch.int16).numpy().copy(),
                       [x.view(torch.int16).numpy().copy() for x in (dq, dk, dv)], pos.numpy().copy(), None))
            dist.barrier()
            return
        if case.get("chunks"):
            o_loc, lse, pos, heads = udist.attention_forward_chunked(*args, case["chunks"], attn=attn, pack=pack,
                                                                     unpack=unpack)
            lse = lse.reshape(-1, N)
            heads = np.array([h for hc in heads for h in hc])
        else:
            o_loc, lse, pos = udist.attention_forward(*args, attn=attn, pack=pack, unpack=unpack)
            heads = np.arange(rank * (case["H"] // world), (rank + 1) * (case["H"] // world))
        out_q.put((rank, o_loc.view(torch.int16).numpy().copy(), lse.numpy().copy(), pos.numpy().copy(), heads))
        dist.barrier()
