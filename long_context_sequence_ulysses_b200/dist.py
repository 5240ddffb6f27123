"""Ulysses across G GPUs: one process per GPU, torch.distributed over NCCL.

Page "Hugging Face并行加速：10倍提升超长序列训练效率", section "Ulysses的工作原理":
GPU g holds tokens [g*N/G, (g+1)*N/G) (step 序列分片); an all-to-all gives every
GPU the whole sequence for H/G heads (step 全体间通信); attention runs locally
(本地注意力计算); a second all-to-all restores sequence shards (全体间通信复原).

The single-GPU relayout kernels are exactly the local halves of the exchange:
  pack    ulysses_seq_to_head(shard [N/G][H][d], N/G, P=G) -> [G][N/G][H/G][d],
          block r is what GPU r receives;
  all_to_all_single(recv, send) then leaves [G src][N/G][H/G][d] = [N][H/G][d],
          the head slice, with no unpacking;
  unpack  ulysses_head_to_seq(recv [G][N/G][H/G][d], N/G, P=G) -> [N/G][H][d]
          after the second exchange.
The exchange moves raw bytes (tensors are sent as uint8 views), so it is
dtype-agnostic and works on any backend that has all_to_all.

The local steps are parameters (defaulting to the CUDA library) so that the
host logic can be exercised with CPU stand-ins over gloo.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist


def _world(group) -> Tuple[int, int]:
    return dist.get_world_size(group), dist.get_rank(group)


def _cuda_pack(x: torch.Tensor, G: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    import long_context_sequence_ulysses_b200 as U
    return U.seq_to_head(x, G, out=out)


def _cuda_unpack(y: torch.Tensor, G: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    import long_context_sequence_ulysses_b200 as U
    return U.head_to_seq(y, G, out=out)


def seq_to_head(x_local: torch.Tensor, group=None,
                pack: Optional[Callable] = None, send: Optional[torch.Tensor] = None,
                recv: Optional[torch.Tensor] = None) -> torch.Tensor:
    """[N/G][Hx][d] sequence shard -> [N][Hx/G][d] head slice of this rank.
    ``send`` / ``recv`` are optional preallocated [G][N/G][Hx/G][d] buffers."""
    G, _ = _world(group)
    n_loc, Hx, d = x_local.shape
    if Hx % G or n_loc % G:
        raise ValueError(f"heads ({Hx}) and local tokens ({n_loc}) must be divisible by the group size {G}")
    if pack is None:
        send = _cuda_pack(x_local, G, out=send)                  # [G][N/G][Hx/G][d]
    else:
        send = pack(x_local, G)
    if recv is None:
        recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(torch.uint8), send.contiguous().view(torch.uint8), group=group)
    return recv.view(G * n_loc, Hx // G, d)


def head_to_seq(y: torch.Tensor, group=None,
                unpack: Optional[Callable] = None, recv: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """[N][Hx/G][d] head slice -> [N/G][Hx][d] sequence shard of this rank.
    ``recv`` ([G][N/G][Hx/G][d]) and ``out`` ([N/G][Hx][d]) may be preallocated."""
    G, _ = _world(group)
    N, Hl, d = y.shape
    if N % G:
        raise ValueError(f"N ({N}) must be divisible by the group size {G}")
    send = y.contiguous().view(G, N // G, Hl, d)                # block r goes to rank r
    if recv is None:
        recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(torch.uint8), send.view(torch.uint8), group=group)
    if unpack is None:
        return _cuda_unpack(recv, G, out=out)                    # [N/G][Hx][d]
    return unpack(recv, G)


def gather_position_ids(pos_local: torch.Tensor, group=None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """All ranks' position ids, in sequence order (each rank needs the whole
    sequence's document structure once it holds whole-sequence head slices)."""
    G, _ = _world(group)
    if out is not None and pos_local.is_cuda:
        dist.all_gather_into_tensor(out, pos_local.contiguous(), group=group)
        return out
    parts = [torch.empty_like(pos_local) for _ in range(G)]
    dist.all_gather(parts, pos_local.contiguous(), group=group)
    return torch.cat(parts)


def attention_forward(q_local: torch.Tensor, k_local: torch.Tensor, v_local: torch.Tensor,
                      pos_local: torch.Tensor, group=None, scale: Optional[float] = None,
                      attn: Optional[Callable] = None, pack=None, unpack=None, keep_for_backward: bool = False):
    """The Ulysses attention step of one rank: returns (o_local [N/G][H][d],
    lse [H/G][N] for this rank's heads, position ids of the whole sequence).
    With ``keep_for_backward`` a fourth item holds what the backward needs:
    this rank's head slices (q, k, v, o), each [N][heads/G][d]."""
    pos = gather_position_ids(pos_local, group)
    q = seq_to_head(q_local, group, pack)
    k = seq_to_head(k_local, group, pack)
    v = seq_to_head(v_local, group, pack)
    if attn is None:
        import long_context_sequence_ulysses_b200 as U
        attn = U.attn_fwd
    o, lse = attn(q, k, v, pos, scale=scale)
    o_local = head_to_seq(o, group, unpack)
    if keep_for_backward:
        return o_local, lse, pos, (q, k, v, o)
    return o_local, lse, pos


def attention_backward(saved, lse: torch.Tensor, pos: torch.Tensor, dout_local: torch.Tensor, group=None,
                       scale: Optional[float] = None, attn_bwd: Optional[Callable] = None, pack=None,
                       unpack=None):
    """The backward of the Ulysses attention step of one rank. The upstream
    gradient arrives sequence-sharded like O, so it crosses the first exchange
    (dO [N/G][H][d] -> [N][H/G][d]); the gradients of this rank's heads are
    computed locally, as in the forward (heads are independent); dQ, dK and dV
    cross the second exchange back to sequence shards. ``saved`` is the
    (q, k, v, o) head slices attention_forward keeps; lse and pos are its
    other outputs. Returns (dq_local [N/G][H][d], dk_local, dv_local
    [N/G][Hkv][d])."""
    q, k, v, o = saved
    g = seq_to_head(dout_local, group, pack)
    if attn_bwd is None:
        import long_context_sequence_ulysses_b200 as U
        attn_bwd = U.attn_bwd
    dq, dk, dv = attn_bwd(q, k, v, o, g, lse, pos, scale=scale)
    return head_to_seq(dq, group, unpack), head_to_seq(dk, group, unpack), head_to_seq(dv, group, unpack)


def attention_forward_chunked(q_local: torch.Tensor, k_local: torch.Tensor, v_local: torch.Tensor,
                              pos_local: torch.Tensor, chunks: int, group=None, scale: Optional[float] = None,
                              attn: Optional[Callable] = None, pack=None, unpack=None):
    """The Ulysses attention step of one rank with the heads taken in
    ``chunks`` groups, the head-chunked variant the pages list as UPipe (page
    "Ulysses 序列並行：百萬 Token 上下文訓練", section "競品分析"): chunk c's Q/K/V
    cross the first all-to-all while chunk c-1 is being computed, and only
    one chunk's head slices are resident at a time, so the activation memory
    of the exchange and of the attention inputs shrinks by ``chunks``.

    Chunk c holds query heads [c*H/chunks, (c+1)*H/chunks) and KV heads
    [c*Hkv/chunks, (c+1)*Hkv/chunks); each rank gets 1/G of both, which keeps
    every query head with its KV head as long as Hkv is divisible by
    chunks*G. Returns (o_local [N/G][H][d], lse [chunks][H/(chunks*G)][N],
    position ids of the whole sequence, heads) where heads[c][j] is the
    global query head of lse[c][j]."""
    G, rank = _world(group)
    n_loc, H, d = q_local.shape
    Hkv = k_local.shape[1]
    if chunks < 1 or H % (chunks * G) or Hkv % (chunks * G):
        raise ValueError(f"H={H} and Hkv={Hkv} must be divisible by chunks*G={chunks * G}")
    if n_loc % G:
        raise ValueError(f"local tokens ({n_loc}) must be divisible by the group size {G}")
    Hc, Hkvc = H // chunks, Hkv // chunks
    if attn is None:
        import long_context_sequence_ulysses_b200 as U
        attn = U.attn_fwd
    pos = gather_position_ids(pos_local, group)

    def start(c: int):
        """Pack chunk c's Q, K, V and start their all-to-alls (asynchronous).
        The CUDA pack reads the chunk's heads in place from the full shard."""
        inflight = []
        for x, h in ((q_local, Hc), (k_local, Hkvc), (v_local, Hkvc)):
            if pack is None:
                import long_context_sequence_ulysses_b200 as U
                send = U.seq_to_head(x, G, heads=(c * h, h))                # [G][N/G][h/G][d]
            else:
                send = pack(x[:, c * h:(c + 1) * h].contiguous(), G).contiguous()
            recv = torch.empty_like(send)
            work = dist.all_to_all_single(recv.view(torch.uint8), send.view(torch.uint8), group=group,
                                          async_op=True)
            inflight.append((work, recv, send))
        return inflight

    o_local = torch.empty_like(q_local)
    lses, heads = [], []
    pending = start(0)
    for c in range(chunks):
        current = pending
        pending = start(c + 1) if c + 1 < chunks else None
        for work, _, _ in current:
            work.wait()
        # the send buffers are free once their exchange is done; keep only the received slices
        recvs = [recv for _, recv, _ in current]
        del current
        q, k, v = (recv.view(G * n_loc, recv.shape[2], d) for recv in recvs)
        o, lse = attn(q, k, v, pos, scale=scale)
        if unpack is None:
            # second exchange, then the unpack writes this chunk's heads of o_local in place
            send = o.contiguous().view(G, n_loc, o.shape[1], d)
            recv = torch.empty_like(send)
            dist.all_to_all_single(recv.view(torch.uint8), send.view(torch.uint8), group=group)
            import long_context_sequence_ulysses_b200 as U
            U.head_to_seq(recv, G, out=o_local, head0=c * Hc)
        else:
            o_local[:, c * Hc:(c + 1) * Hc] = head_to_seq(o, group, unpack)
        lses.append(lse)
        heads.append([c * Hc + rank * (Hc // G) + j for j in range(Hc // G)])
        del recvs, q, k, v, o
    return o_local, torch.stack(lses), pos, heads
