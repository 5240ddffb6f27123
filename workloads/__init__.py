"""Seeded synthetic inputs for the Ulysses per-rank attention path.

This module holds input recipes only: shapes, seeds, document-length draws,
position ids and normally distributed bf16 tensors. It contains none of the
method's arithmetic, so both the CUDA path and the CPU oracle can use it
without sharing any computation.

Workloads (named by what they are):

* ``tiny``      N=256, P=2, H=4 = Hkv, d=32, one document.
* ``llama8b``   N=32768, P=8, H=32 / Hkv=8, d=128, packed documents with
                lengths uniform in [512, 8192], inputs scaled by 1/sqrt(d).
* ``long131k``  N=131072, P=4, H=32 / Hkv=8, d=128, one document.
* ``million``   N=1048576, P=8, H=32 / Hkv=8, d=128, one document.
* ``train``     N=65536, P=4, H=32 / Hkv=8, d=128, packed documents with
                geometric lengths (mean 4096), forward + backward.
* ``hybrid_kv2`` the llama8b shape with only 2 KV heads over P=8 ranks: fewer
                KV heads than ranks, so Ulysses alone cannot split it; run as
                the Ulysses x ring hybrid (2-way Ulysses, 4-way ring).

Sequence sharding follows the page "Hugging Face并行加速：10倍提升超长序列训练效率",
section "Ulysses的工作原理", step 序列分片: GPU i owns tokens [i*n/P, (i+1)*n/P).
Packing with position ids instead of a 4-D mask follows the page "Ulysses
verteilt Millionen-Token-Kontexte auf mehrere GPUs", section "Integration in
den Hugging-Face-Stack"; a new document starts wherever the id returns to 0.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int          # total tokens of the sequence (all ranks)
    P: int          # emulated sequence-parallel ranks
    H: int          # query heads (all ranks)
    Hkv: int        # key/value heads (all ranks)
    d: int          # head dimension
    docs: str       # "single" | "uniform" | "geometric"
    seed: int
    prescale: bool = False   # multiply Q/K/V by 1/sqrt(d) before the bf16 cast
    backward: bool = False   # the workload includes the backward pass
    ulysses: int = 0         # > 0: Ulysses x ring hybrid with this Ulysses degree (ring degree P / ulysses)

    @property
    def Hl(self) -> int:
        return self.H // self.P

    @property
    def Hkvl(self) -> int:
        return self.Hkv // self.P


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 256, 2, 4, 4, 32, "single", 0),
    "llama8b": Workload("llama8b", 32768, 8, 32, 8, 128, "uniform", 1, prescale=True),
    "long131k": Workload("long131k", 131072, 4, 32, 8, 128, "single", 2),
    "million": Workload("million", 1048576, 8, 32, 8, 128, "single", 3),
    "train": Workload("train", 65536, 4, 32, 8, 128, "geometric", 4, backward=True),
    "hybrid_kv2": Workload("hybrid_kv2", 32768, 8, 32, 2, 128, "uniform", 5, prescale=True, ulysses=2),
}


def doc_lengths(kind: str, N: int, seed: int) -> List[int]:
    """Document lengths that fill exactly N tokens.

    uniform:   integers uniform in [512, 8192], drawn until the sum reaches N;
               the last document is truncated to fit.
    geometric: support {1, 2, ...} with p = 1/4096 (mean 4096), drawn and
               truncated the same way.
    single:    one document of length N.
    """
    if N == 0:
        return []
    if kind == "single":
        return [N]
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out: List[int] = []
    total = 0
    while total < N:
        if kind == "uniform":
            L = int(torch.randint(512, 8193, (1,), generator=g).item())
        elif kind == "geometric":
            L = int(torch.empty(1, dtype=torch.float64).geometric_(1.0 / 4096.0, generator=g).item())
            L = max(L, 1)
        else:
            raise ValueError(f"unknown document-length kind {kind!r}")
        L = min(L, N - total)
        out.append(L)
        total += L
    return out


def position_ids(lengths: List[int]) -> torch.Tensor:
    """int32 position ids: 0..L-1 for each document, concatenated."""
    if not lengths:
        return torch.zeros(0, dtype=torch.int32)
    return torch.cat([torch.arange(L, dtype=torch.int32) for L in lengths])


def unmasked_pairs(lengths: List[int]) -> int:
    """Number of (query, key) pairs that causal document masking keeps."""
    return sum(L * (L + 1) // 2 for L in lengths)


def normal_bf16(shape, seed: int, device="cpu", prescale: Optional[float] = None,
                stream_id: int = 0) -> torch.Tensor:
    """Standard-normal fp32 draws cast to bf16 (round to nearest even).

    ``stream_id`` separates the Q/K/V/dO draws of one workload: each uses its
    own generator seeded with seed*16 + stream_id.
    """
    g = torch.Generator(device=device)
    g.manual_seed(seed * 16 + stream_id)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if prescale is not None:
        x.mul_(prescale)
    return x.to(torch.bfloat16)


STREAM_Q, STREAM_K, STREAM_V, STREAM_DO = 1, 2, 3, 4


def make_inputs(w: Workload, device="cpu", with_grad_out: Optional[bool] = None,
                N: Optional[int] = None) -> dict:
    """Sequence-sharded inputs of one workload.

    Q is [N][H][d], K and V are [N][Hkv][d]; viewed as [P][N/P][heads][d]
    they are the P rank buffers before the sequence-to-head exchange.
    dO (when requested) is [N][H][d] in the same layout as the output.
    ``N`` overrides the workload's length (for reduced-size test cases).
    """
    n = w.N if N is None else N
    lengths = doc_lengths(w.docs, n, w.seed)
    pos = position_ids(lengths)
    pre = (1.0 / math.sqrt(w.d)) if w.prescale else None
    out = {
        "lengths": lengths,
        "position_ids": pos.to(device),
        "q": normal_bf16((n, w.H, w.d), w.seed, device, pre, STREAM_Q),
        "k": normal_bf16((n, w.Hkv, w.d), w.seed, device, pre, STREAM_K),
        "v": normal_bf16((n, w.Hkv, w.d), w.seed, device, pre, STREAM_V),
    }
    if with_grad_out if with_grad_out is not None else w.backward:
        out["do"] = normal_bf16((n, w.H, w.d), w.seed, device, None, STREAM_DO)
    return out


def random_case(N: int, H: int, Hkv: int, d: int, lengths: List[int], seed: int,
                device="cpu", with_grad_out: bool = False) -> dict:
    """A free-form case (arbitrary shapes and document lengths) for tests."""
    assert sum(lengths) == N
    out = {
        "lengths": list(lengths),
        "position_ids": position_ids(list(lengths)).to(device),
        "q": normal_bf16((N, H, d), seed, device, None, STREAM_Q),
        "k": normal_bf16((N, Hkv, d), seed, device, None, STREAM_K),
        "v": normal_bf16((N, Hkv, d), seed, device, None, STREAM_V),
    }
    if with_grad_out:
        out["do"] = normal_bf16((N, H, d), seed, device, None, STREAM_DO)
    return out


STREAM_WQKV, STREAM_WO, STREAM_X = 5, 6, 7


def projection_inputs(w: Workload, device="cpu", N: Optional[int] = None) -> dict:
    """Synthetic layer inputs around the path: activations x [N][hidden] ~
    N(0, 1) and random-init weights w_qkv [(H+2Hkv)d][hidden], w_o [hidden][Hd]
    ~ N(0, 1/hidden) (hidden = H*d, as in the Llama-8B shape), all bf16."""
    n = w.N if N is None else N
    hidden = w.H * w.d
    sc = 1.0 / math.sqrt(hidden)
    return {
        "x": normal_bf16((n, hidden), w.seed, device, None, STREAM_X),
        "w_qkv": normal_bf16(((w.H + 2 * w.Hkv) * w.d, hidden), w.seed, device, sc, STREAM_WQKV),
        "w_o": normal_bf16((hidden, w.H * w.d), w.seed, device, sc, STREAM_WO),
    }
