"""Ulysses x ring hybrid, every rank emulated on one GPU.

Ulysses alone needs the KV heads to split over the P ranks; ring attention
does not (page "Ulysses 序列並行：百萬 Token 上下文訓練", section "競品分析"; page
"Ulysses verteilt Millionen-Token-Kontexte auf mehrere GPUs", section "Wann
Ulysses sinnvoll ist"). The hybrid factors P = U * R: U-way Ulysses over heads
inside each group of U ranks, R-way ring over sequence chunks across groups.
Rank (rho, u) holds, after the Ulysses exchange of its group, the query heads
[u*H/U, (u+1)*H/U) (KV heads [u*Hkv/U, ...)) for the sequence chunk rho of
N/R tokens; the ring then passes the chunks of keys and values around: at
step s the rank holds key chunk c = (rho - s) mod R and computes the partial
attention of its queries over that chunk; the partials merge through their
log-sum-exp into exact attention. A chunk that lies entirely after the rank's
queries (c > rho) holds no key any of them may see, so it is not computed.

On one GPU the P rank buffers are emulated as in the pure Ulysses path: the
U-way exchange is one relayout of the whole sequence (every group's slices at
once), a ring step is a key-window pass of the forward kernel
(ulysses_attn_fwd_window), and the merge is ulysses_attn_merge. Every step
runs in the library's kernels; this module only sequences the calls.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import attn_fwd_window, attn_merge, head_to_seq, seq_to_head


def split(P: int, H: int, Hkv: int, N: int, U: Optional[int] = None) -> Tuple[int, int]:
    """(U, R): the Ulysses degree (by default the largest divisor of P that
    also divides H and Hkv) and the ring degree R = P / U."""
    if U is None:
        U = max(u for u in range(1, P + 1) if P % u == 0 and H % u == 0 and Hkv % u == 0)
    if P % U or H % U or Hkv % U:
        raise ValueError(f"Ulysses degree {U} must divide P={P}, H={H} and Hkv={Hkv}")
    R = P // U
    if N % R:
        raise ValueError(f"N={N} must split into {R} ring chunks")
    return U, R


class HybridPlan:
    """Buffers of one emulated hybrid step (allocated once, reused)."""

    def __init__(self, N: int, H: int, Hkv: int, d: int, P: int, U: Optional[int], device):
        self.U, self.R = split(P, H, Hkv, N, U)
        self.N, self.H, self.Hkv, self.d, self.P = N, H, Hkv, d, P
        U_, R = self.U, self.R
        self.chunk = N // R
        bf = torch.bfloat16
        self.q_all = torch.empty((U_, N, H // U_, d), dtype=bf, device=device)
        self.k_all = torch.empty((U_, N, Hkv // U_, d), dtype=bf, device=device)
        self.v_all = torch.empty_like(self.k_all)
        self.o_all = torch.empty_like(self.q_all)
        self.lse = torch.empty((H, N), dtype=torch.float32, device=device)
        self.o_parts = torch.empty((R, self.chunk, H // U_, d), dtype=bf, device=device)
        self.lse_parts = torch.empty((R, H // U_, self.chunk), dtype=torch.float32, device=device)
        from . import workspace_bytes
        self.ws = torch.empty(workspace_bytes(N, H // U_, Hkv // U_, d, False), dtype=torch.uint8, device=device)

    def steps(self):
        """(rank, ring steps of that rank): rank = (rho, u); steps are the key
        chunks it computes, in ring order (its own chunk first)."""
        for u in range(self.U):
            for rho in range(self.R):
                yield (rho, u), [c for c in ((rho - s) % self.R for s in range(self.R)) if c <= rho]


def forward(q_seq: torch.Tensor, k_seq: torch.Tensor, v_seq: torch.Tensor, position_ids: torch.Tensor, P: int,
            U: Optional[int] = None, scale: Optional[float] = None, plan: Optional[HybridPlan] = None,
            out: Optional[torch.Tensor] = None, timed=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention of the whole sequence through the emulated U x R hybrid.
    q_seq [N][H][d], k_seq / v_seq [N][Hkv][d] (the P rank buffers, sequence
    sharded). Returns (o_seq [N][H][d], lse [H][N]). ``timed(kind, fn)``, if
    given, wraps each launch ("relayout", "attn_fwd", "merge") for timing."""
    run = timed if timed is not None else (lambda kind, fn: fn())
    N, H, d = q_seq.shape
    Hkv = k_seq.shape[1]
    if plan is None:
        plan = HybridPlan(N, H, Hkv, d, P, U, q_seq.device)
    Ud, ch, Hu = plan.U, plan.chunk, H // plan.U
    # Ulysses exchange inside every group of U ranks
    run("relayout", lambda: seq_to_head(q_seq, Ud, out=plan.q_all))
    run("relayout", lambda: seq_to_head(k_seq, Ud, out=plan.k_all))
    run("relayout", lambda: seq_to_head(v_seq, Ud, out=plan.v_all))
    for (rho, u), chunks in plan.steps():
        for s, c in enumerate(chunks):
            run("attn_fwd", lambda: attn_fwd_window(plan.q_all[u], plan.k_all[u], plan.v_all[u], position_ids,
                                                    rho * ch, (rho + 1) * ch, c * ch, (c + 1) * ch, scale=scale,
                                                    out=plan.o_parts[s], lse=plan.lse_parts[s], ws=plan.ws))
        run("merge", lambda: attn_merge(plan.o_parts[:len(chunks)], plan.lse_parts[:len(chunks)],
                                        out=plan.o_all[u, rho * ch:(rho + 1) * ch],
                                        lse=plan.lse[u * Hu:(u + 1) * Hu, rho * ch:(rho + 1) * ch]))
    o_seq = run("relayout", lambda: head_to_seq(plan.o_all, Ud, out=out))
    return o_seq, plan.lse
