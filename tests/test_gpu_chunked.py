"""The head-chunked Ulysses step (dist.attention_forward_chunked, the UPipe
variant of page "Ulysses 序列並行：百萬 Token 上下文訓練", section "競品分析") run
through the CUDA kernels on one GPU, as a one-rank NCCL group: each chunk's
heads are packed in place from the full shard, cross the (here one-rank)
all-to-all, run through the attention kernel and are unpacked in place into
the output. Compared with the oracle's attention of the whole problem; the
device memory a step allocates shrinks with the number of chunks."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, bf16_to_f64
from workloads import random_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def one_rank_group():
    import torch.distributed as dist
    if dist.is_initialized():
        yield dist
        return
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    import datetime
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield dist
    dist.destroy_process_group()


@pytest.mark.parametrize("chunks", [1, 2, 4])
def test_chunked_forward_matches_oracle(one_rank_group, chunks):
    from long_context_sequence_ulysses_b200 import dist as udist
    N, H, Hkv, d = 2048, 8, 4, 128
    c = random_case(N, H, Hkv, d, [1000, 1, 1047], seed=33, device="cuda")
    o, lse, pos, heads = udist.attention_forward_chunked(c["q"], c["k"], c["v"], c["position_ids"], chunks)
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
    assert_close("O", bf16_to_f64(o), ro)
    got_lse = lse.reshape(-1, N).double().cpu().numpy()
    order = [h for hc in heads for h in hc]
    assert sorted(order) == list(range(H))
    assert_close("LSE", got_lse, rl[order])


def test_chunked_forward_memory_shrinks(one_rank_group):
    """Device memory allocated during one step, beyond the resident inputs and
    output, for 1, 2 and 4 chunks: it falls as the chunk count rises."""
    from long_context_sequence_ulysses_b200 import dist as udist
    N, H, Hkv, d = 16384, 16, 8, 128
    c = random_case(N, H, Hkv, d, [N], seed=34, device="cuda")
    peaks = []
    for chunks in (1, 2, 4):
        udist.attention_forward_chunked(c["q"], c["k"], c["v"], c["position_ids"], chunks)
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        o, _, _, _ = udist.attention_forward_chunked(c["q"], c["k"], c["v"], c["position_ids"], chunks)
        torch.cuda.synchronize()
        peaks.append(torch.cuda.max_memory_allocated() - base)
        del o
    print("step peak bytes for 1, 2, 4 chunks:", peaks)
    assert peaks[0] > peaks[1] > peaks[2]
