"""fp64 CPU oracle for the Ulysses per-rank attention path.

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library under
``long_context_sequence_ulysses_b200`` never does, and this package imports
nothing from it. The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP
over heads and rows); this module only builds it with gcc and marshals numpy
arrays through ctypes.

Parity status of each function (what pins it is listed in the tests):
  seq_to_head, head_to_seq  pinned (hand-derived golden permutation, inverse)
  doc_start                 pinned (hand-derived golden, definition by brute force)
  attn_fwd                  pinned (brute force, SDPA, closed forms, invariances)
  attn_bwd                  pinned (finite differences, autograd, sum rules)
  attn_bwd_sampled          pinned (equal to attn_bwd on the sampled rows and keys)
  attn_fwd_window           pinned (brute force with the window, whole window = attn_fwd)
  merge                     pinned (closed form; merged windows = attention over their union)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I64, I32, F64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.oracle_seq_to_head.argtypes = [P, P, I64, I32, I32, I32]
            lib.oracle_seq_to_head.restype = I32
            lib.oracle_head_to_seq.argtypes = [P, P, I64, I32, I32, I32]
            lib.oracle_head_to_seq.restype = I32
            lib.oracle_doc_start.argtypes = [P, I64, P]
            lib.oracle_doc_start.restype = None
            lib.oracle_set_num_threads.argtypes = [I32]
            lib.oracle_set_num_threads.restype = None
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = I32
            lib.oracle_attn_fwd_rows.argtypes = [P, P, P, P, I64, I32, I32, I32, F64, P, I64, P, P]
            lib.oracle_attn_fwd_rows.restype = I32
            lib.oracle_attn_bwd.argtypes = [P, P, P, P, P, I64, I32, I32, I32, F64, P, P, P, P, P]
            lib.oracle_attn_bwd.restype = I32
            lib.oracle_attn_bwd_sampled.argtypes = [P, P, P, P, P, I64, I32, I32, I32, F64, P, I64, P, I64, P, P, P]
            lib.oracle_attn_bwd_sampled.restype = I32
            lib.oracle_attn_fwd_window_rows.argtypes = [P, P, P, P, I64, I32, I32, I32, F64, I64, I64, P, I64, P, P]
            lib.oracle_attn_fwd_window_rows.restype = I32
            lib.oracle_merge.argtypes = [P, P, I32, I64, I32, I32, P, P]
            lib.oracle_merge.restype = None
            _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array of its bits."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16, x.dtype
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16, a.dtype
    return a


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def seq_to_head(src, N: int, P: int, Hx: int, d: int) -> np.ndarray:
    """[P][N/P][Hx][d] -> [P][N][Hx/P][d] on raw 16-bit patterns."""
    s = _bits(src).reshape(-1)
    dst = np.empty(P * N * (Hx // P) * d if P else 0, dtype=np.uint16)
    rc = _load().oracle_seq_to_head(_ptr(s), _ptr(dst), N, P, Hx, d)
    if rc != 0:
        raise ValueError("oracle_seq_to_head: invalid arguments")
    return dst.reshape(P, N, Hx // P, d)


def head_to_seq(src, N: int, P: int, Hx: int, d: int) -> np.ndarray:
    """[P][N][Hx/P][d] -> [P][N/P][Hx][d] on raw 16-bit patterns."""
    s = _bits(src).reshape(-1)
    dst = np.empty(N * Hx * d, dtype=np.uint16)
    rc = _load().oracle_head_to_seq(_ptr(s), _ptr(dst), N, P, Hx, d)
    if rc != 0:
        raise ValueError("oracle_head_to_seq: invalid arguments")
    return dst.reshape(P, N // P, Hx, d)


def doc_start(pos) -> np.ndarray:
    p = _i32(pos)
    out = np.empty(p.shape[0], dtype=np.int32)
    _load().oracle_doc_start(_ptr(p), p.shape[0], _ptr(out))
    return out


def attn_fwd(q, k, v, pos, scale: Optional[float] = None,
             rows: Optional[Sequence[int]] = None):
    """Exact forward attention of one rank's head slice.

    q [N][Hl][d], k/v [N][Hkvl][d] (bf16), pos [N] int.
    Returns (o, lse): o [N or len(rows)][Hl][d] fp64, lse [Hl][N or len(rows)].
    ``scale`` defaults to 1/sqrt(d).
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    N, Hl, d = qb.shape
    Hkvl = kb.shape[1]
    p = _i32(pos)
    assert p.shape[0] == N
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nr = r.shape[0]
    o = np.empty((Hl, nr, d), dtype=np.float64)
    lse = np.empty((Hl, nr), dtype=np.float64)
    rc = _load().oracle_attn_fwd_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(p), N, Hl, Hkvl, d,
                                      float(scale), _ptr(r), nr, _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_rows failed ({rc})")
    return np.ascontiguousarray(o.transpose(1, 0, 2)), lse


def attn_bwd(q, k, v, dout, pos, scale: Optional[float] = None):
    """Exact gradients (dq, dk, dv) of sum(dO * O), plus (o, lse), in fp64."""
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    N, Hl, d = qb.shape
    Hkvl = kb.shape[1]
    p = _i32(pos)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq = np.empty((N, Hl, d), dtype=np.float64)
    dk = np.empty((N, Hkvl, d), dtype=np.float64)
    dv = np.empty((N, Hkvl, d), dtype=np.float64)
    o = np.empty((N, Hl, d), dtype=np.float64)
    lse = np.empty((Hl, N), dtype=np.float64)
    rc = _load().oracle_attn_bwd(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _ptr(p), N, Hl, Hkvl, d,
                                 float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd failed ({rc})")
    return dq, dk, dv, o, lse


def attn_bwd_sampled(q, k, v, dout, pos, rows: Sequence[int], keys: Sequence[int], scale: Optional[float] = None):
    """The exact gradients of sum(dO * O) only where asked: dq [len(rows)][Hl][d]
    for the query rows ``rows`` and dk, dv [len(keys)][Hkvl][d] for the keys
    ``keys``, in fp64 (same formulas as attn_bwd)."""
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    N, Hl, d = qb.shape
    Hkvl = kb.shape[1]
    p = _i32(pos)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    kk = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
    dq = np.empty((r.shape[0], Hl, d), dtype=np.float64)
    dk = np.empty((kk.shape[0], Hkvl, d), dtype=np.float64)
    dv = np.empty((kk.shape[0], Hkvl, d), dtype=np.float64)
    rc = _load().oracle_attn_bwd_sampled(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _ptr(p), N, Hl, Hkvl, d,
                                         float(scale), _ptr(r), r.shape[0], _ptr(kk), kk.shape[0], _ptr(dq),
                                         _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd_sampled failed ({rc})")
    return dq, dk, dv


def attn_fwd_window(q, k, v, pos, kv_lo: int, kv_hi: int, scale: Optional[float] = None,
                    rows: Optional[Sequence[int]] = None):
    """Attention of one rank's head slice over the keys [kv_lo, kv_hi) only
    (one ring step's partial result). Returns (o [rows][Hl][d], lse [Hl][rows])
    in fp64; a row that sees no key gets o = 0, lse = -inf."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    N, Hl, d = qb.shape
    Hkvl = kb.shape[1]
    p = _i32(pos)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nr = r.shape[0]
    o = np.empty((Hl, nr, d), dtype=np.float64)
    lse = np.empty((Hl, nr), dtype=np.float64)
    rc = _load().oracle_attn_fwd_window_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(p), N, Hl, Hkvl, d, float(scale),
                                             int(kv_lo), int(kv_hi), _ptr(r), nr, _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_window_rows failed ({rc})")
    return np.ascontiguousarray(o.transpose(1, 0, 2)), lse


def merge(o_parts, lse_parts):
    """Merge partial results over disjoint key sets: o_parts [R][M][Hl][d],
    lse_parts [R][Hl][M] (fp64) -> (o [M][Hl][d], lse [Hl][M])."""
    op = np.ascontiguousarray(o_parts, dtype=np.float64)
    lp = np.ascontiguousarray(lse_parts, dtype=np.float64)
    R, M, Hl, d = op.shape
    assert lp.shape == (R, Hl, M)
    o = np.empty((M, Hl, d), dtype=np.float64)
    lse = np.empty((Hl, M), dtype=np.float64)
    _load().oracle_merge(_ptr(op), _ptr(lp), R, M, Hl, d, _ptr(o), _ptr(lse))
    return o, lse


# ---------------------------------------------------------------- projections
# The steps either side of the path (page "Hugging Face并行加速：10倍提升超长序列训练效率",
# section "Ulysses的工作原理", steps QKV投影 and 输出投影; page "DeepSpeed Ulysses
# 详解", section "DeepSpeed-Ulysses 的核心机制", items 2 and 6): every rank
# projects its own tokens with the full weights. The product is numpy's fp64
# matmul of the exactly widened bf16 values (a library primitive used as a
# step); the exchange layout is the pinned seq_to_head / head_to_seq above.

def _f64(x) -> np.ndarray:
    b = _bits(x)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def qkv_proj(x, w_qkv, P: int, H: int, Hkv: int, d: int, rows: Optional[Sequence[int]] = None):
    """x [N][hidden] (the P sequence shards), w_qkv [(H+2Hkv)*d][hidden] ->
    fp64 (q, k, v) in every rank's head-slice layout [P][N][H/P][d] and
    [P][N][Hkv/P][d]: y = x w_qkv^T, columns [0, H*d) are Q's heads, then K's,
    then V's, each head's d columns contiguous. With ``rows``, only those
    tokens: [P][len(rows)][heads/P][d]."""
    xf = _f64(x)
    if rows is not None:
        xf = xf[np.asarray(rows, dtype=np.int64)]
    y = xf @ _f64(w_qkv).T
    n = y.shape[0]
    out = []
    for lo, heads in ((0, H), (H * d, Hkv), ((H + Hkv) * d, Hkv)):
        part = y[:, lo:lo + heads * d].reshape(n, heads, d)
        # the exchange: rank r holds heads [r*heads/P, (r+1)*heads/P) of every token
        out.append(np.ascontiguousarray(part.reshape(n, P, heads // P, d).transpose(1, 0, 2, 3)))
    return tuple(out)


def out_proj(o_heads, w_o, rows: Optional[Sequence[int]] = None):
    """o_heads [P][N][H/P][d] (every rank's head slice of the attention output),
    w_o [hidden][H*d] -> y [N][hidden] fp64: the second exchange back to the
    sequence layout [N][H*d] (head r*H/P + h at columns (r*H/P + h)*d ...), then
    y = o w_o^T. With ``rows``, only those tokens."""
    of = _f64(o_heads)
    P, N, Hl, d = of.shape
    seq = of.transpose(1, 0, 2, 3).reshape(N, P * Hl * d)
    if rows is not None:
        seq = seq[np.asarray(rows, dtype=np.int64)]
    return seq @ _f64(w_o).T


def set_num_threads(n: int) -> None:
    """Host threads of the oracle's loops (no effect on its arithmetic)."""
    _load().oracle_set_num_threads(int(n))


def max_threads() -> int:
    """Threads the oracle's loops use."""
    return int(_load().oracle_max_threads())
