#!/usr/bin/env python
"""Benchmark of the Ulysses per-rank attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|llama8b|...] [--chunks C]
    python bench.py --impl reference ...     # the fp64 CPU oracle, timed on host cores

By default the headline line is the llama8b workload and its "workloads"
object holds the same measurement of tiny, long131k, million and train.
One step = one pass of the whole hot path over the workload, for every
emulated rank r of P (rank 0 only for the million-token workload):
    seq_to_head(Q), seq_to_head(K), seq_to_head(V)   (rank r's head slice)
    attention forward (doc-bounds scan + tensor-core kernel) -> O, LSE
    [attention backward when the workload has one]
    head_to_seq(O)                                     (back to sequence shards)
The metric is attention TFLOP/s over the step (FLOPs counted over unmasked
pairs only: 4*d*H*pairs forward, 10*d*H*pairs backward), with the relayout
GB/s and the dominant kernel's roofline reported beside it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import WORKLOADS, make_inputs, unmasked_pairs  # noqa: E402

METRIC = "causal packed attn fwd/bwd TFLOP/s + relayout GB/s on 1 B200, % of roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.txt")


def fwd_launches(n):
    """Kernels of one forward call over n tokens: the document scan, the fix-up
    with the work order (one launch up to 2^20 tokens; past that a carry
    prefix, the fix-up and the order), the attention."""
    return 3 if n <= 1 << 20 else 5


def bwd_launches(n):
    """Kernels of one backward call: the document scan, its carry prefix (past
    2^20 tokens), the fix-up, the key-tile query ends, the two work orders, the
    delta prep, the dK/dV kernel and the dQ kernel."""
    return 8 + (n > 1 << 20)


# Workloads the default run measures after the headline one, with the steps
# each times (the million-token step lasts about a second: 3 are enough).
SUB_WORKLOADS = ("tiny", "long131k", "million", "train", "hybrid_kv2")
SUB_STEPS = {"million": 3}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# Sources a kernel's DRAM traffic depends on (its own file and the shared headers).
KERNEL_SOURCES = {
    "attn_fwd_kernel": ("attn_fwd.cu", "ptx.cuh", "ulysses_internal.cuh"),
    "attn_bwd_dkdv_kernel": ("attn_bwd.cu", "ptx.cuh", "ulysses_internal.cuh"),
    "attn_bwd_dq_kernel": ("attn_bwd.cu", "ptx.cuh", "ulysses_internal.cuh"),
    "proj_gemm_kernel": ("proj.cu", "ptx.cuh", "ulysses_internal.cuh"),
    "attn_merge_kernel": ("merge.cu", "ulysses_internal.cuh"),
}


def kernel_source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES.get(kernel, ("attn_fwd.cu", "attn_bwd.cu", "ptx.cuh", "ulysses_internal.cuh")):
        p = os.path.join(ROOT, "long_context_sequence_ulysses_b200", "csrc", name)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def lookup_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, valid only while the
    kernel's sources are unchanged since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    sha = kernel_source_sha(kernel)
    for ln in open(TRAFFIC_FILE):
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        parts = ln.split()
        if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload and parts[3] == sha:
            return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


def workload_work(w, lengths):
    pairs = unmasked_pairs(lengths)
    fwd = 4.0 * w.d * w.H * pairs
    bwd = 10.0 * w.d * w.H * pairs if w.backward else 0.0
    elem = 2
    # relayout bytes (read + write of every element moved): Q, K, V in; O out
    # (backward adds dO in and dQ, dK, dV out)
    qkv = (w.N * w.H * w.d + 2 * w.N * w.Hkv * w.d) * elem
    o = w.N * w.H * w.d * elem
    relayout = 2 * (qkv + o)
    if w.backward:
        relayout += 2 * (o + qkv)
    return pairs, fwd, bwd, relayout


# --------------------------------------------------------------------------- GPU arm

class Timer:
    """CUDA events around one kind of launch, on the launching (current)
    stream. With `external` the events are recorded as nodes of a CUDA graph
    being captured, and read after its replays (the last replay's times)."""

    def __init__(self, stream, enabled: bool):
        self.stream = stream
        self.enabled = enabled
        self.external = False
        self.ev = {"attn_fwd": [], "attn_bwd": [], "relayout": [], "exchange": [], "merge": []}

    def reset(self):
        for k in self.ev:
            self.ev[k] = []

    def __call__(self, kind, fn):
        if not self.enabled:
            return fn()
        a = torch.cuda.Event(enable_timing=True, external=self.external)
        b = torch.cuda.Event(enable_timing=True, external=self.external)
        s = torch.cuda.current_stream()
        a.record(s)
        r = fn()
        b.record(s)
        self.ev[kind].append((a, b))
        return r

    def stats(self, kind):
        xs = [a.elapsed_time(b) for a, b in self.ev[kind]]
        return ((sum(xs) / len(xs)) if xs else None), (sum(xs) if xs else None)


def build_single(U, w, inp, dev, timed, attn_ranks=None):
    """One GPU: the P ranks are emulated as P buffers, the exchanges are the
    relayout kernels. The attention runs for the ranks in ``attn_ranks``
    (default: all of them; the million-token workload times rank 0's).
    Returns (step, our kernel launches per step, workspace)."""
    P, N, d, Hl, Hkvl = w.P, w.N, w.d, w.Hl, w.Hkvl
    ranks = list(range(P)) if attn_ranks is None else list(attn_ranks)
    pos = inp["position_ids"]
    q_seq, k_seq, v_seq, do_seq = inp["q"], inp["k"], inp["v"], inp.get("do")
    q_all = torch.empty((P, N, Hl, d), dtype=torch.bfloat16, device=dev)
    k_all = torch.empty((P, N, Hkvl, d), dtype=torch.bfloat16, device=dev)
    v_all = torch.empty((P, N, Hkvl, d), dtype=torch.bfloat16, device=dev)
    o_all = torch.empty((P, N, Hl, d), dtype=torch.bfloat16, device=dev)
    lse_all = torch.empty((P * Hl, N), dtype=torch.float32, device=dev)
    o_seq = torch.empty_like(q_seq)
    ws = torch.empty(U.workspace_bytes(N, Hl, Hkvl, d, w.backward), dtype=torch.uint8, device=dev)
    if w.backward:
        do_all = torch.empty_like(q_all)
        dq_all, dk_all, dv_all = torch.empty_like(q_all), torch.empty_like(k_all), torch.empty_like(v_all)
        dq_seq, dk_seq, dv_seq = torch.empty_like(q_seq), torch.empty_like(k_seq), torch.empty_like(v_seq)

    def step():
        # first all-to-all: every rank's head slice of Q, K, V
        timed("relayout", lambda: U.seq_to_head(q_seq, P, out=q_all))
        timed("relayout", lambda: U.seq_to_head(k_seq, P, out=k_all))
        timed("relayout", lambda: U.seq_to_head(v_seq, P, out=v_all))
        for r in ranks:
            timed("attn_fwd", lambda: U.attn_fwd(q_all[r], k_all[r], v_all[r], pos, out=o_all[r],
                                                 lse=lse_all[r * Hl:(r + 1) * Hl], ws=ws))
        if w.backward:
            timed("relayout", lambda: U.seq_to_head(do_seq, P, out=do_all))
            for r in ranks:
                timed("attn_bwd", lambda: U.attn_bwd(q_all[r], k_all[r], v_all[r], o_all[r], do_all[r],
                                                     lse_all[r * Hl:(r + 1) * Hl], pos, ws=ws, dq=dq_all[r],
                                                     dk=dk_all[r], dv=dv_all[r]))
            timed("relayout", lambda: U.head_to_seq(dq_all, P, out=dq_seq))
            timed("relayout", lambda: U.head_to_seq(dk_all, P, out=dk_seq))
            timed("relayout", lambda: U.head_to_seq(dv_all, P, out=dv_seq))
        # second all-to-all: O back to sequence shards
        timed("relayout", lambda: U.head_to_seq(o_all, P, out=o_seq))

    launches = 3 + fwd_launches(w.N) * len(ranks) + 1 + ((1 + bwd_launches(w.N) * len(ranks) + 3) if w.backward else 0)
    return step, launches, ws


def build_hybrid(U, w, inp, dev, timed):
    """One GPU, the Ulysses x ring hybrid (fewer KV heads than ranks): the
    U-way exchange of Q, K, V, each rank's ring steps as key-window passes of
    the forward and their merge, the U-way exchange of O back. Returns (step,
    our kernel launches per step, workspace)."""
    from long_context_sequence_ulysses_b200 import hybrid
    plan = hybrid.HybridPlan(w.N, w.H, w.Hkv, w.d, w.P, w.ulysses, dev)
    pos = inp["position_ids"]
    o_seq = torch.empty_like(inp["q"])
    n_steps = sum(len(c) for _, c in plan.steps())
    n_ranks = plan.U * plan.R

    def step():
        hybrid.forward(inp["q"], inp["k"], inp["v"], pos, w.P, w.ulysses, plan=plan, out=o_seq, timed=timed)

    return step, 3 + fwd_launches(w.N) * n_steps + n_ranks + 1, plan.ws


def build_fused(U, w, inp, dev):
    """One GPU, fused exchanges: every emulated rank's attention reads its head
    slice straight from the sequence-sharded Q/K/V (and dO) and writes O (and
    dQ/dK/dV) straight back into that layout, so no relayout runs.
    Returns (step, our kernel launches per step, workspace)."""
    P, N, d, Hl, Hkvl = w.P, w.N, w.d, w.Hl, w.Hkvl
    pos = inp["position_ids"]
    q_seq, k_seq, v_seq, do_seq = inp["q"], inp["k"], inp["v"], inp.get("do")
    o_seq = torch.empty_like(q_seq)
    lse_all = torch.empty((P * Hl, N), dtype=torch.float32, device=dev)
    ws = torch.empty(U.workspace_bytes(N, Hl, Hkvl, d, w.backward), dtype=torch.uint8, device=dev)
    if w.backward:
        dq_seq, dk_seq, dv_seq = torch.empty_like(q_seq), torch.empty_like(k_seq), torch.empty_like(v_seq)

    def step():
        for r in range(P):
            U.attn_fwd_fused(q_seq, k_seq, v_seq, pos, P, r, out=o_seq, lse=lse_all[r * Hl:(r + 1) * Hl], ws=ws)
        if w.backward:
            for r in range(P):
                U.attn_bwd_fused(q_seq, k_seq, v_seq, o_seq, do_seq, lse_all[r * Hl:(r + 1) * Hl], pos, P, r,
                                 dq=dq_seq, dk=dk_seq, dv=dv_seq, ws=ws)

    return step, fwd_launches(w.N) * P + (bwd_launches(w.N) * P if w.backward else 0), ws


def time_fused(U, w, inp, dev, steps, total_flop, use_graph=True):
    """The step with the exchanges fused into the attention (see build_fused),
    replayed as a CUDA graph like the main step (or launched eagerly)."""
    step, launches, ws = build_fused(U, w, inp, dev)
    stream = torch.cuda.current_stream(dev)
    step()
    torch.cuda.synchronize()
    U.sync_status(ws)
    run_step = step
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph.replay()
        torch.cuda.synchronize()
        U.sync_status(ws)
        run_step = graph.replay
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        run_step()
    t1.record(stream)
    torch.cuda.synchronize()
    U.sync_status(ws)
    ms = t0.elapsed_time(t1) / steps
    return {"ms_per_step": round(ms, 4), "value": round(total_flop / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "gpu_launches": launches * steps,
            "step": "attn_fwd_fused per rank" + ("; attn_bwd_fused per rank" if w.backward else "")
                    + ": sequence-sharded Q/K/V in, O out, no relayout"}


def build_multi(U, w, inp, dev, timed, G, rank, chunks=1):
    """G GPUs: Ulysses with P = G real ranks. Each GPU holds tokens
    [rank*N/G, (rank+1)*N/G); the pack before and the unpack after each NCCL
    all-to-all are the relayout kernels; each GPU computes H/G heads. With
    chunks > 1 the forward takes the heads in that many chunks, the next
    chunk's all-to-alls in flight while the current chunk is computed."""
    from long_context_sequence_ulysses_b200 import dist as udist
    N, d = w.N, w.d
    if w.H % G or w.Hkv % G or N % (G * G):
        raise SystemExit(f"workload {w.name} cannot be split over {G} GPUs")
    n_loc, Hg, Hkvg = N // G, w.H // G, w.Hkv // G
    sl = slice(rank * n_loc, (rank + 1) * n_loc)
    q_loc, k_loc, v_loc = (inp[x][sl].contiguous() for x in ("q", "k", "v"))
    do_loc = inp["do"][sl].contiguous() if w.backward else None
    pos_loc = inp["position_ids"][sl].contiguous()
    buf = lambda h: torch.empty((G, n_loc, h, d), dtype=torch.bfloat16, device=dev)
    sq, rq, sk, rk, sv, rv = buf(Hg), buf(Hg), buf(Hkvg), buf(Hkvg), buf(Hkvg), buf(Hkvg)
    o_head, ro = torch.empty((N, Hg, d), dtype=torch.bfloat16, device=dev), buf(Hg)
    o_loc = torch.empty_like(q_loc)
    lse = torch.empty((Hg, N), dtype=torch.float32, device=dev)
    pos = torch.empty(N, dtype=torch.int32, device=dev)
    ws = torch.empty(U.workspace_bytes(N, Hg, Hkvg, d, w.backward), dtype=torch.uint8, device=dev)
    if w.backward:
        sdo, rdo = buf(Hg), buf(Hg)
        dq_h, dk_h, dv_h = (torch.empty((N, h, d), dtype=torch.bfloat16, device=dev) for h in (Hg, Hkvg, Hkvg))
        rdq, rdk, rdv = buf(Hg), buf(Hkvg), buf(Hkvg)
        dq_loc, dk_loc, dv_loc = torch.empty_like(q_loc), torch.empty_like(k_loc), torch.empty_like(v_loc)

    if chunks > 1:
        if w.backward:
            raise SystemExit("--chunks applies to the forward only")

        def step():
            o, _, _, _ = timed("attn_fwd", lambda: udist.attention_forward_chunked(q_loc, k_loc, v_loc, pos_loc,
                                                                                    chunks))
            o_loc.copy_(o)

        return step, chunks * (3 + fwd_launches(w.N) + 1), ws

    def step():
        udist.gather_position_ids(pos_loc, out=pos)
        q = timed("exchange", lambda: udist.seq_to_head(q_loc, send=sq, recv=rq))
        k = timed("exchange", lambda: udist.seq_to_head(k_loc, send=sk, recv=rk))
        v = timed("exchange", lambda: udist.seq_to_head(v_loc, send=sv, recv=rv))
        timed("attn_fwd", lambda: U.attn_fwd(q, k, v, pos, out=o_head, lse=lse, ws=ws))
        if w.backward:
            g = timed("exchange", lambda: udist.seq_to_head(do_loc, send=sdo, recv=rdo))
            timed("attn_bwd", lambda: U.attn_bwd(q, k, v, o_head, g, lse, pos, ws=ws, dq=dq_h, dk=dk_h, dv=dv_h))
            timed("exchange", lambda: udist.head_to_seq(dq_h, recv=rdq, out=dq_loc))
            timed("exchange", lambda: udist.head_to_seq(dk_h, recv=rdk, out=dk_loc))
            timed("exchange", lambda: udist.head_to_seq(dv_h, recv=rdv, out=dv_loc))
        timed("exchange", lambda: udist.head_to_seq(o_head, recv=ro, out=o_loc))

    launches = 3 + fwd_launches(w.N) + 1 + ((1 + bwd_launches(w.N) + 3) if w.backward else 0)
    return step, launches, ws


def measure(U, w, dev, args, steps, warmup, world, rank, dist, headline):
    """Time one workload: `warmup` untimed steps, then exactly `steps` steps
    between a barrier and synchronisation on both sides, on the device with
    CUDA events, clocks sampled meanwhile. Returns the JSON record of it (the
    headline record also gets e2e, the fused step and the CPU baseline)."""
    inp = make_inputs(w, device=dev)
    lengths = inp["lengths"]
    pairs, fwd_flop, bwd_flop, relayout_bytes = workload_work(w, lengths)
    stream = torch.cuda.current_stream(dev)
    timed = Timer(stream, False)
    attn_ranks = [0] if w.name == "million" else None
    if world == 1 and w.ulysses:
        step, launches_per_step, ws = build_hybrid(U, w, inp, dev, timed)
    elif world == 1:
        step, launches_per_step, ws = build_single(U, w, inp, dev, timed, attn_ranks)
    else:
        step, launches_per_step, ws = build_multi(U, w, inp, dev, timed, world, rank, args.chunks)
        for key in ("q", "k", "v", "do"):
            inp.pop(key, None)     # each rank keeps only its shard
        torch.cuda.empty_cache()
    n_attn = (1 if attn_ranks else w.P) if world == 1 else 1   # attention launches per step on this GPU
    frac_ranks = (n_attn / w.P) if world == 1 else 1.0         # share of the attention work one step does
    fwd_flop_step, bwd_flop_step = fwd_flop * frac_ranks, bwd_flop * frac_ranks

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    U.sync_status(ws)        # raises if a bounded device wait ran out
    timed.enabled = args.kernel_events
    # One GPU: the step is captured once as a CUDA graph (its launches, with
    # the per-kind timing events as graph nodes) and replayed; the launch
    # overhead between the step's kernels then stays off the GPU's timeline.
    graph = None
    if world == 1 and args.graph:
        timed.external = True
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        timed.external = False
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        U.sync_status(ws)
        run_step = graph.replay
    else:
        run_step = step

    sampler = ClockSampler(int(str(dev).split(":")[-1]) if ":" in str(dev) else 0)
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        run_step()
    t1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()
    ev_steps = 1 if graph is not None else steps   # steps the per-kind events cover
    U.sync_status(ws)
    ms_total = t0.elapsed_time(t1)
    if dist is not None:
        t = torch.tensor([ms_total], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_step = ms_total / steps

    fwd_avg, fwd_sum = timed.stats("attn_fwd")
    bwd_avg, bwd_sum = timed.stats("attn_bwd")
    _, rel_sum = timed.stats("relayout")
    _, exch_sum = timed.stats("exchange")
    _, merge_sum = timed.stats("merge")

    # the whole job: all ranks (all GPUs), all heads of the ranks that ran
    total_flop = fwd_flop_step + bwd_flop_step
    value = total_flop / (ms_step * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    # a kernel timed inside a step of a second or more runs at the sustained (power-capped) rate
    long_step = ms_step > 500.0
    bf16_peak = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    peak_source = "%s %s" % (peak_kind, "sustained" if long_step else "burst")
    n_fwd = len(timed.ev["attn_fwd"]) // ev_steps if timed.ev["attn_fwd"] else 1   # attention launches per step
    n_bwd = len(timed.ev["attn_bwd"]) // ev_steps if timed.ev["attn_bwd"] else 1
    fwd_flop_launch = fwd_flop_step / n_fwd
    bwd_flop_launch = bwd_flop_step / n_bwd
    # the attention work of a step over the time its launches took (launches of
    # equal size for Ulysses; the hybrid's ring steps differ in size)
    achieved = fwd_flop_step / (fwd_sum / ev_steps * 1e-3) / 1e12 if fwd_sum else None
    bwd_ach = bwd_flop_step / (bwd_sum / ev_steps * 1e-3) / 1e12 if bwd_sum else None
    traffic = lookup_traffic("attn_fwd_kernel", w.name) if world == 1 else None

    def roof(kernel, ach, flop_launch, traffic_b):
        return {"kernel": kernel, "bound": "tensor", "achieved": round(ach, 2) if ach else None, "peak": bf16_peak,
                "peak_source": peak_source, "unit": "TFLOP/s", "frac": round(ach / bf16_peak, 4) if ach else None,
                "frac_of_spec_2250": round(ach / SPEC_BF16_TFLOPS, 4) if ach else None, "traffic": traffic_b,
                "flop_per_launch": flop_launch}

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "strong" if world > 1 else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w.name, "N": w.N, "P": w.P if world == 1 else world, "H": w.H, "Hkv": w.Hkv, "d": w.d,
            "docs": w.docs, "documents": len(lengths), "unmasked_pairs": pairs, "backward": w.backward,
            "step": (("Ulysses x ring hybrid, U=%d x R=%d: seq_to_head(Q,K,V) over U; per rank its ring steps "
                      "(key-window attention) and their merge; head_to_seq(O) over U"
                      % (w.ulysses, w.P // w.ulysses)) if (w.ulysses and world == 1) else
                     ("seq_to_head(Q,K,V) for all P ranks; attn_fwd for "
                      + ("rank 0's head slice" if attn_ranks else "each rank's head slice")
                      + ("; seq_to_head(dO), attn_bwd per rank, head_to_seq(dQ,dK,dV)" if w.backward else "")
                      + "; head_to_seq(O) for all ranks") if world == 1 else
                     ("Ulysses over %d GPUs: pack + NCCL all-to-all of Q,K,V; attn_fwd on N x H/%d heads"
                      % (world, world) + ("; dO exchange, attn_bwd, dQ/dK/dV exchanges" if w.backward else "")
                      + "; O exchange + unpack"
                      + ("; heads in %d chunks, the next chunk's exchanges in flight" % args.chunks
                         if args.chunks > 1 else ""))),
            "step_flop": total_flop,
            "l2": "inputs larger than L2 (126 MB): Q alone is %d MiB" % (w.N * w.H * w.d * 2 >> 20)
                  if w.N * w.H * w.d * 2 > (126 << 20) else
                  "inputs smaller than L2; each step re-reads them from L2 (launch-latency bound, no roofline claim)",
        },
        "roofline": roof("attn_fwd_kernel (timed with the doc-bounds launch that precedes it)"
                         + ("; the hybrid's key-window passes, merges not included" if w.ulysses else ""),
                         achieved, fwd_flop_launch, traffic),
        "attn_fwd_ms_per_launch": round(fwd_avg, 4) if fwd_avg else None,
        "attn_bwd_ms_per_launch": round(bwd_avg, 4) if bwd_avg else None,
        "attn_bwd_tflops": round(bwd_ach, 2) if bwd_ach else None,
        "gpu_launches": launches_per_step * steps,
        "timing": ("the step captured once as a CUDA graph and replayed; per-kind kernel times from the "
                   "last replay's event nodes") if graph is not None else "eager launches",
        "clocks": clocks,
    }
    if bwd_avg:
        out["roofline_bwd"] = roof("attn_bwd (prep, dK/dV and dQ kernels with their doc-bounds launches)", bwd_ach,
                                   bwd_flop_launch, lookup_traffic("attn_bwd_dkdv_kernel", w.name))
    if rel_sum:
        rbytes = relayout_bytes
        rb = rbytes / (rel_sum / ev_steps * 1e-3) / 1e9
        out["relayout"] = {"bytes_per_step": rbytes, "ms_per_step": round(rel_sum / ev_steps, 4),
                           "achieved_gbs": round(rb, 1), "peak_gbs": peaks["hbm_gbs"],
                           "peak_source": peak_kind, "frac": round(rb / peaks["hbm_gbs"], 4),
                           "frac_of_spec_8000": round(rb / SPEC_HBM_GBS, 4)}
    if exch_sum:
        out["exchange_ms_per_step"] = round(exch_sum / ev_steps, 4)
    if merge_sum:
        out["merge_ms_per_step"] = round(merge_sum / ev_steps, 4)
    if world > 1:
        # device memory one step allocates beyond what is resident before it
        # (exchange buffers and head slices; smaller with more head chunks)
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        timed.enabled = False
        step()
        torch.cuda.synchronize()
        peak = torch.tensor([torch.cuda.max_memory_allocated(dev) - base], device=dev, dtype=torch.float64)
        dist.all_reduce(peak, op=dist.ReduceOp.MAX)
        out["step_peak_mem_bytes"] = int(peak.item())
        out["chunks"] = args.chunks
    if headline:
        out["e2e"] = run_e2e(U, w, inp, args, dev) if (args.e2e_steps > 0 and world == 1) else None
    if world == 1 and args.fused and not attn_ranks and not w.ulysses:
        out["fused_step"] = time_fused(U, w, inp, dev, steps, total_flop, args.graph)
    if headline and rank == 0 and not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(w, inp, args)
    del inp, step, ws
    torch.cuda.empty_cache()
    return out


def measure_layer(U, w, dev, args, steps, warmup):
    """The layer step around the path on one GPU, all P ranks: the QKV
    projection written straight into every rank's head slice (projection and
    first exchange in one kernel), the attention of each rank, and the output
    projection read straight from the head slices (second exchange and
    projection in one kernel). Synthetic activations and random-init weights
    of the workload's shape (hidden = H*d)."""
    from workloads import projection_inputs
    inp = make_inputs(w, device=dev)
    pin = projection_inputs(w, device=dev)
    pairs, fwd_flop, _, _ = workload_work(w, inp["lengths"])
    hidden = w.H * w.d
    qkv_flop = 2.0 * w.N * hidden * (w.H + 2 * w.Hkv) * w.d
    out_flop = 2.0 * w.N * (w.H * w.d) * hidden
    P, N, d, Hl, Hkvl = w.P, w.N, w.d, w.Hl, w.Hkvl
    q_all = torch.empty((P, N, Hl, d), dtype=torch.bfloat16, device=dev)
    k_all = torch.empty((P, N, Hkvl, d), dtype=torch.bfloat16, device=dev)
    v_all = torch.empty_like(k_all)
    o_all = torch.empty_like(q_all)
    lse_all = torch.empty((w.H, N), dtype=torch.float32, device=dev)
    y = torch.empty((N, hidden), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(U.workspace_bytes(N, Hl, Hkvl, d, False), dtype=torch.uint8, device=dev)
    pws = U.proj_workspace(dev)
    pos = inp["position_ids"]
    stream = torch.cuda.current_stream(dev)
    timed = Timer(stream, False)
    timed.ev["gemm_qkv"], timed.ev["gemm_out"] = [], []

    def step():
        timed("gemm_qkv", lambda: U.qkv_proj(pin["x"], pin["w_qkv"], P, w.H, w.Hkv, d, q_out=q_all, k_out=k_all,
                                             v_out=v_all, ws=pws))
        for r in range(P):
            timed("attn_fwd", lambda: U.attn_fwd(q_all[r], k_all[r], v_all[r], pos, out=o_all[r],
                                                 lse=lse_all[r * Hl:(r + 1) * Hl], ws=ws))
        timed("gemm_out", lambda: U.out_proj(o_all, pin["w_o"], out=y, ws=pws))

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    U.sync_status(ws)
    U.sync_status(pws)
    timed.enabled = args.kernel_events
    sampler = ClockSampler(int(str(dev).split(":")[-1]) if ":" in str(dev) else 0)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    U.sync_status(ws)
    U.sync_status(pws)
    ms = t0.elapsed_time(t1) / steps
    peaks, peak_kind = load_peaks()
    peak = peaks["bf16_tflops"]
    total = fwd_flop + qkv_flop + out_flop
    rec = {"value": round(total / (ms * 1e-3) / 1e12, 2), "ms_per_step": round(ms, 4), "steps": steps,
           "warmup": warmup, "config": {"workload": w.name + "_layer", "N": N, "P": P, "H": w.H, "Hkv": w.Hkv,
                                        "d": d, "hidden": hidden, "step_flop": total,
                                        "step": "qkv_proj into every rank's head slice (fused first exchange); "
                                                "attn_fwd per rank; out_proj from the head slices (fused second "
                                                "exchange)", "weights": "random-init, N(0, 1/hidden), seeded"},
           "clocks": clocks, "gpu_launches": (2 + fwd_launches(w.N) * P) * steps}
    for kind, flop, name in (("gemm_qkv", qkv_flop, "qkv_proj (proj_gemm_kernel<256>)"),
                             ("gemm_out", out_flop, "out_proj (proj_gemm_kernel<256>)")):
        avg, _ = timed.stats(kind)
        if avg:
            ach = flop / (avg * 1e-3) / 1e12
            rec["roofline_" + kind] = {"kernel": name, "bound": "tensor", "achieved": round(ach, 2), "peak": peak,
                                       "peak_source": peak_kind + " burst", "unit": "TFLOP/s",
                                       "frac": round(ach / peak, 4), "frac_of_spec_2250": round(ach / SPEC_BF16_TFLOPS, 4),
                                       "flop_per_launch": flop, "ms_per_launch": round(avg, 4),
                                       "traffic": lookup_traffic("proj_gemm_kernel",
                                                                 "layer_qkv" if kind == "gemm_qkv" else "layer_out")}
    fwd_avg, fwd_sum = timed.stats("attn_fwd")
    if fwd_sum:
        rec["attn_fwd_tflops"] = round(fwd_flop / (fwd_sum / steps * 1e-3) / 1e12, 2)
    del inp, pin, q_all, k_all, v_all, o_all, y
    torch.cuda.empty_cache()
    return rec


def run_gpu(args):
    import long_context_sequence_ulysses_b200 as U

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    if args.workload == "layer" and world == 1:
        # the layer step alone (projections with the exchanges fused in, attention per rank)
        out = measure_layer(U, WORKLOADS["llama8b"], dev, args, args.steps, args.warmup)
        out.update({"metric": METRIC, "unit": "TFLOP/s", "n_gpus": 1, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "bf16", "data": "synthetic"})
        print(json.dumps(out), flush=True)
        return
    name = "llama8b" if args.workload == "all" else args.workload
    out = measure(U, WORKLOADS[name], dev, args, args.steps, args.warmup, world, rank, dist, headline=True)
    if args.workload == "all" and world == 1:
        subs = {}
        for sub in SUB_WORKLOADS:
            k = SUB_STEPS.get(sub, args.steps)
            r = measure(U, WORKLOADS[sub], dev, args, k, max(3, args.warmup if sub != "million" else 3), world,
                        rank, dist, headline=False)
            for key in ("metric", "unit", "n_gpus", "higher_is_better", "scaling", "vs_baseline", "dtype", "data"):
                r.pop(key, None)
            subs[sub] = r
        subs["llama8b_layer"] = measure_layer(U, WORKLOADS["llama8b"], dev, args, args.steps, max(3, args.warmup))
        out["workloads"] = subs
        out["gpu_launches"] += sum(r["gpu_launches"] for r in subs.values())
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_e2e_pipelined(U, w, inp, args, dev):
    from cuda.bindings import runtime as cudart
    P, N, d, Hl, H, Hkvl, Hkv = w.P, w.N, w.d, w.Hl, w.H, w.Hkvl, w.Hkv
    pin = lambda t: t.cpu().pin_memory()
    hq, hk, hv, hpos = pin(inp["q"]), pin(inp["k"]), pin(inp["v"]), pin(inp["position_ids"])
    ho = torch.empty_like(hq).pin_memory()
    hlse = torch.empty((H, N), dtype=torch.float32).pin_memory()
    gq, gk, gv = torch.empty_like(inp["q"]), torch.empty_like(inp["k"]), torch.empty_like(inp["v"])
    gpos = torch.empty_like(inp["position_ids"])
    o_seq = torch.empty_like(gq)
    lse_all = torch.empty((H, N), dtype=torch.float32, device=dev)
    ws = torch.empty(U.workspace_bytes(N, Hl, w.Hkvl, d, False), dtype=torch.uint8, device=dev)
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    row, cols = H * d * 2, Hl * d * 2            # bytes per token row of Q / O; one rank's heads in it
    krow, kcols = Hkv * d * 2, Hkvl * d * 2      # the same for K and V
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2 + hpos.numel() * 4
    d2h = ho.numel() * 2 + hlse.numel() * 4
    ev_in = [torch.cuda.Event() for _ in range(P)]
    ev_cmp = [torch.cuda.Event() for _ in range(P)]
    ev_out = [torch.cuda.Event() for _ in range(P)]   # rank r's results read back
    ev_cdone = torch.cuda.Event()                     # a step's attention has read its inputs
    for e in ev_out:
        e.record(s_out)
    ev_cdone.record(s_cmp)
    H2D, D2H = cudart.cudaMemcpyKind.cudaMemcpyHostToDevice, cudart.cudaMemcpyKind.cudaMemcpyDeviceToHost

    def copy2d(dst, src, kind, stream, pitch=None, width=None):
        pitch, width = pitch or row, width or cols
        err, = cudart.cudaMemcpy2DAsync(dst, pitch, src, pitch, width, N, kind,
                                        cudart.cudaStream_t(stream.cuda_stream))
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaMemcpy2DAsync: {err}")

    def step():
        # Consecutive steps overlap: a step's inputs may land once the previous
        # step's attention has read its own (its results may still be going back),
        # and rank r's attention waits only for the previous step's rank r results
        # to have been read back from the output buffers it rewrites.
        s_in.wait_event(ev_cdone)
        with torch.cuda.stream(s_in):
            gpos.copy_(hpos, non_blocking=True)
            for r in range(P):
                # rank r's query heads and KV heads: one pitched copy each
                copy2d(gk.data_ptr() + r * kcols, hk.data_ptr() + r * kcols, H2D, s_in, krow, kcols)
                copy2d(gv.data_ptr() + r * kcols, hv.data_ptr() + r * kcols, H2D, s_in, krow, kcols)
                copy2d(gq.data_ptr() + r * cols, hq.data_ptr() + r * cols, H2D, s_in)
                ev_in[r].record(s_in)
        with torch.cuda.stream(s_cmp):
            for r in range(P):
                s_cmp.wait_event(ev_in[r])
                s_cmp.wait_event(ev_out[r])
                U.attn_fwd_fused(gq, gk, gv, gpos, P, r, out=o_seq, lse=lse_all[r * Hl:(r + 1) * Hl], ws=ws)
                ev_cmp[r].record(s_cmp)
            ev_cdone.record(s_cmp)
        with torch.cuda.stream(s_out):
            for r in range(P):
                s_out.wait_event(ev_cmp[r])
                copy2d(ho.data_ptr() + r * cols, o_seq.data_ptr() + r * cols, D2H, s_out)
                hlse[r * Hl:(r + 1) * Hl].copy_(lse_all[r * Hl:(r + 1) * Hl], non_blocking=True)
                ev_out[r].record(s_out)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(args.e2e_steps):
        step()
    b.record(s_out)
    torch.cuda.synchronize()
    U.sync_status(ws)
    ms = a.elapsed_time(b) / args.e2e_steps
    pairs, fwd_flop, bwd_flop, _ = workload_work(w, inp["lengths"])
    return {"value": round((fwd_flop + bwd_flop) / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": args.e2e_steps,
            "path": "pinned host -> device copies (ids, then each rank's K, V and query heads as pitched copies), "
                    "attn_fwd_fused per rank as its heads arrive, each rank's O columns and LSE back on a third "
                    "stream; a step's input copies start once the previous step's attention has read its inputs"}


def run_e2e(U, w, inp, args, dev):
    """The step through the public API from pinned HOST buffers, host<->device
    copies inside the timed region. A forward-only workload runs as a
    three-stream pipeline over the emulated ranks: the position ids first,
    then rank by rank its KV heads and query heads (pitched copies of those
    columns of every token row); rank r's fused attention (which reads its
    heads straight from the sequence layout) starts as soon as its heads have
    arrived, and its O columns and LSE rows go back to the host on a third
    stream while the later ranks still compute, so the two copy directions
    overlap each other and the compute (also across steps: the next step's
    inputs start as soon as this step's attention has read its own). A workload with a backward copies in
    everything, runs the step, and copies the results out."""
    if not w.backward:
        return run_e2e_pipelined(U, w, inp, args, dev)
    P, N, d, Hl, Hkvl = w.P, w.N, w.d, w.Hl, w.Hkvl
    pin = lambda t: t.cpu().pin_memory()
    hq, hk, hv, hpos = pin(inp["q"]), pin(inp["k"]), pin(inp["v"]), pin(inp["position_ids"])
    hdo = pin(inp["do"]) if w.backward else None
    ho = torch.empty_like(hq).pin_memory()
    hlse = torch.empty((w.H, N), dtype=torch.float32).pin_memory()
    gq, gk, gv = torch.empty_like(inp["q"]), torch.empty_like(inp["k"]), torch.empty_like(inp["v"])
    gpos = torch.empty_like(inp["position_ids"])
    q_all = torch.empty((P, N, Hl, d), dtype=torch.bfloat16, device=dev)
    k_all = torch.empty((P, N, Hkvl, d), dtype=torch.bfloat16, device=dev)
    v_all = torch.empty_like(k_all)
    o_all = torch.empty_like(q_all)
    lse_all = torch.empty((w.H, N), dtype=torch.float32, device=dev)
    o_seq = torch.empty_like(gq)
    ws = torch.empty(U.workspace_bytes(N, Hl, Hkvl, d, w.backward), dtype=torch.uint8, device=dev)
    if w.backward:
        gdo = torch.empty_like(gq)
        do_all, dq_all = torch.empty_like(q_all), torch.empty_like(q_all)
        dk_all, dv_all = torch.empty_like(k_all), torch.empty_like(k_all)
        dq_seq, dk_seq, dv_seq = torch.empty_like(gq), torch.empty_like(gk), torch.empty_like(gv)
        hdq, hdk, hdv = (torch.empty_like(hq).pin_memory(), torch.empty_like(hk).pin_memory(),
                         torch.empty_like(hv).pin_memory())
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2 + hpos.numel() * 4 + (hdo.numel() * 2 if w.backward else 0)
    d2h = ho.numel() * 2 + hlse.numel() * 4 + ((hq.numel() + hk.numel() + hv.numel()) * 2 if w.backward else 0)
    stream = torch.cuda.current_stream(dev)

    def step():
        gq.copy_(hq, non_blocking=True)
        gk.copy_(hk, non_blocking=True)
        gv.copy_(hv, non_blocking=True)
        gpos.copy_(hpos, non_blocking=True)
        U.seq_to_head(gq, P, out=q_all)
        U.seq_to_head(gk, P, out=k_all)
        U.seq_to_head(gv, P, out=v_all)
        for r in range(P):
            U.attn_fwd(q_all[r], k_all[r], v_all[r], gpos, out=o_all[r], lse=lse_all[r * Hl:(r + 1) * Hl], ws=ws)
        if w.backward:
            gdo.copy_(hdo, non_blocking=True)
            U.seq_to_head(gdo, P, out=do_all)
            for r in range(P):
                U.attn_bwd(q_all[r], k_all[r], v_all[r], o_all[r], do_all[r], lse_all[r * Hl:(r + 1) * Hl], gpos,
                           ws=ws, dq=dq_all[r], dk=dk_all[r], dv=dv_all[r])
            U.head_to_seq(dq_all, P, out=dq_seq)
            U.head_to_seq(dk_all, P, out=dk_seq)
            U.head_to_seq(dv_all, P, out=dv_seq)
            hdq.copy_(dq_seq, non_blocking=True)
            hdk.copy_(dk_seq, non_blocking=True)
            hdv.copy_(dv_seq, non_blocking=True)
        U.head_to_seq(o_all, P, out=o_seq)
        ho.copy_(o_seq, non_blocking=True)
        hlse.copy_(lse_all, non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.e2e_steps
    pairs, fwd_flop, bwd_flop, _ = workload_work(w, inp["lengths"])
    return {"value": round((fwd_flop + bwd_flop) / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": args.e2e_steps}


# --------------------------------------------------------------------------- CPU oracle

def _oracle_rows_sample(w, lengths, budget_pairs: float, seed: int):
    """Rows of rank 0 spread over the sequence, with about `budget_pairs`
    (query, key) pairs over rank 0's heads in total."""
    import numpy as np
    starts = np.cumsum([0] + list(lengths))[:-1]
    ds = np.repeat(starts, lengths)
    keys = np.arange(w.N) - ds + 1          # keys per row
    rng = np.random.default_rng(seed)
    order = rng.permutation(w.N)
    cum = np.cumsum(keys[order]) * w.Hl
    n = int(np.searchsorted(cum, budget_pairs)) + 1
    rows = np.sort(order[:max(1, min(n, w.N))])
    return rows, int(keys[rows].sum()) * w.Hl


def _oracle_slice(w, inp):
    q = inp["q"][:, :w.Hl].contiguous().cpu()
    k = inp["k"][:, :w.Hkvl].contiguous().cpu()
    v = inp["v"][:, :w.Hkvl].contiguous().cpu()
    return q, k, v, inp["position_ids"].cpu()


def _oracle_rate(w, inp, sl):
    """Query-key pairs per second of the oracle on a small calibration sample."""
    import oracle
    rows, pr = _oracle_rows_sample(w, inp["lengths"], 2e6, seed=1)
    t = time.perf_counter()
    oracle.attn_fwd(*sl, rows=rows)
    return pr / max(time.perf_counter() - t, 1e-3)


def _oracle_step(w, inp, sl, rate, seconds_target, seed):
    """One timed oracle run on about seconds_target of rank 0's rows.
    Returns (seconds, pairs, rows)."""
    import oracle
    rows, pr = _oracle_rows_sample(w, inp["lengths"], rate * seconds_target, seed=seed)
    t = time.perf_counter()
    oracle.attn_fwd(*sl, rows=rows)
    return time.perf_counter() - t, pr, len(rows)


def cpu_baseline(w, inp, args, seconds_target: float = 15.0):
    """The fp64 oracle timed on this host's cores on a bounded sample of rank
    0's rows; its rate is scaled to TFLOP/s with the same FLOP count per pair."""
    import oracle
    threads = oracle.max_threads()   # the threads its loops actually use
    sl = _oracle_slice(w, inp)
    dt, pr, nrows = _oracle_step(w, inp, sl, _oracle_rate(w, inp, sl), seconds_target, seed=2)
    flop = 4.0 * w.d * pr
    return {"value": round(flop / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": "forward attention of %d rows x %d heads of rank 0 (%d query-key pairs, %.1f s)"
                      % (nrows, w.Hl, pr, dt)}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, on this host's cores.
    Each step is a bounded sample of rank 0's rows of the workload (about
    --ref-seconds of work); value and ms_per_step are those of the sampled work
    actually timed, not an extrapolation to the whole step."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = WORKLOADS["llama8b" if args.workload == "all" else args.workload]
    inp = make_inputs(w, device="cpu")
    import oracle
    if world > 1:
        # the launcher gives every rank one host thread; the other ranks do no work
        oracle.set_num_threads(os.cpu_count() or 1)
    threads = oracle.max_threads()
    sl = _oracle_slice(w, inp)
    rate = _oracle_rate(w, inp, sl)
    times, pairs = [], []
    for i in range(args.warmup + args.steps):
        dt, pr, nrows = _oracle_step(w, inp, sl, rate, args.ref_seconds, seed=2 + i)
        if i >= args.warmup:
            times.append(dt)
            pairs.append(pr)
    flop = 4.0 * w.d * sum(pairs)
    value = flop / sum(times) / 1e12
    ms_step = sum(times) / len(times) * 1e3
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "N": w.N, "P": w.P, "H": w.H, "Hkv": w.Hkv, "d": w.d, "docs": w.docs,
                   "note": "each step times the fp64 CPU oracle on a bounded sample of rank 0's rows (about "
                           "%.0f s of host work, %d query-key pairs on average); value and ms_per_step are "
                           "those of the sampled work" % (args.ref_seconds, sum(pairs) // len(pairs))},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": "forward attention of rank 0's rows x %d heads, %d steps of about %.0f s "
                                   "(%d query-key pairs in all)" % (w.Hl, len(times), args.ref_seconds,
                                                                     sum(pairs))},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="all", choices=["all", "layer"] + sorted(WORKLOADS),
                    help="all (default): llama8b as the headline line, the other workloads in its 'workloads' "
                         "object; one workload alone; or layer: llama8b's layer step with the projections")
    ap.add_argument("--chunks", type=int, default=1,
                    help="multi-GPU forward with the heads in this many chunks (head-chunked Ulysses)")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fused", dest="fused", action="store_false",
                    help="skip the extra timing of the step with the exchanges fused into the attention")
    ap.add_argument("--no-kernel-events", dest="kernel_events", action="store_false")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch the step eagerly instead of replaying it as a CUDA graph (one GPU)")
    ap.add_argument("--ref-seconds", type=float, default=4.0,
                    help="host seconds of oracle work per reference-arm step")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "b200":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
