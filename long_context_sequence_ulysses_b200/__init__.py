"""Ulysses sequence-parallel attention hot path for one B200 (sm_100a).

Thin ctypes binding over ``libulysses.so`` (declared in ``include/ulysses.h``).
The functions here only marshal arguments: they check tensor shapes and
dtypes, allocate outputs and workspace through torch (device memory and
streams are torch's job), and call the C ABI on the current CUDA stream.
Every step of the computation runs in the library's CUDA kernels; there is no
fallback, and importing the package fails if the library has not been built
(``python long_context_sequence_ulysses_b200/build.py``).

The method (page "Hugging Face并行加速：10倍提升超长序列训练效率", section
"Ulysses的工作原理"): N tokens are split over P ranks; an all-to-all gives each
rank the whole sequence for H/P heads; each rank runs attention for its heads;
a second all-to-all restores sequence sharding. On one GPU the ranks are
emulated as P buffers and the all-to-alls as in-HBM permutations.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "UlyssesError", "library_path", "seq_to_head", "head_to_seq", "workspace_bytes", "attn_fwd",
    "attn_fwd_fused", "attn_bwd", "attn_bwd_fused", "attn_fwd_window", "attn_merge", "qkv_proj",
    "out_proj", "proj_workspace", "sync_status",
    "set_wait_limit_ns", "set_debug_flags", "version",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libulysses.so")

ULYSSES_OK = 0
ULYSSES_ERR_INVALID = -1
ULYSSES_ERR_UNSUPPORTED = -2
ULYSSES_ERR_CUDA = -3
ULYSSES_ERR_TIMEOUT = -4
ULYSSES_ERR_WORKSPACE = -5


class UlyssesError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python long_context_sequence_ulysses_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, I32, SZ, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    lib.ulysses_last_error.restype = ctypes.c_char_p
    lib.ulysses_version.restype = ctypes.c_char_p
    lib.ulysses_seq_to_head.argtypes = [P, P, I64, I32, I32, I32, I32, P]
    lib.ulysses_head_to_seq.argtypes = [P, P, I64, I32, I32, I32, I32, P]
    lib.ulysses_seq_to_head_heads.argtypes = [P, P, I64, I32, I32, I32, I32, I32, I32, P]
    lib.ulysses_head_to_seq_heads.argtypes = [P, P, I64, I32, I32, I32, I32, I32, I32, P]
    lib.ulysses_attn_workspace_bytes.argtypes = [I64, I32, I32, I32, I32]
    lib.ulysses_attn_workspace_bytes.restype = SZ
    lib.ulysses_attn_fwd.argtypes = [P, P, P, P, I64, I32, I32, I32, F32, P, P, P, SZ, P]
    lib.ulysses_attn_fwd_fused.argtypes = [P, P, P, P, I64, I32, I32, I32, I32, I32, F32, P, P, P, SZ, P]
    lib.ulysses_attn_bwd.argtypes = [P, P, P, P, P, P, P, I64, I32, I32, I32, F32, P, P, P, P, SZ, P]
    lib.ulysses_attn_bwd_fused.argtypes = [P, P, P, P, P, P, P, I64, I32, I32, I32, I32, I32, F32, P, P, P, P, SZ,
                                           P]
    lib.ulysses_attn_fwd_window.argtypes = [P, P, P, P, I64, I32, I32, I32, I64, I64, I64, I64, F32, P, P, P, SZ,
                                            P]
    lib.ulysses_attn_merge.argtypes = [P, P, I32, I64, I32, I32, P, P, I64, P]
    lib.ulysses_proj_workspace_bytes.argtypes = []
    lib.ulysses_proj_workspace_bytes.restype = SZ
    lib.ulysses_qkv_proj.argtypes = [P, P, I64, I32, I32, I32, I32, I32, P, P, P, P, SZ, P]
    lib.ulysses_out_proj.argtypes = [P, P, I64, I32, I32, I32, I32, P, P, SZ, P]
    lib.ulysses_sync_status.argtypes = [P, P]
    lib.ulysses_set_wait_limit_ns.argtypes = [I64]
    lib.ulysses_set_wait_limit_ns.restype = None
    lib.ulysses_set_debug_flags.argtypes = [ctypes.c_uint32]
    lib.ulysses_set_debug_flags.restype = None
    for name in ("ulysses_seq_to_head", "ulysses_head_to_seq", "ulysses_seq_to_head_heads",
                 "ulysses_head_to_seq_heads", "ulysses_attn_fwd", "ulysses_attn_fwd_fused",
                 "ulysses_attn_bwd", "ulysses_attn_bwd_fused", "ulysses_attn_fwd_window", "ulysses_attn_merge",
                 "ulysses_qkv_proj", "ulysses_out_proj", "ulysses_sync_status"):
        getattr(lib, name).restype = I32
    return lib


_lib = _load()


def library_path() -> str:
    return _LIB_PATH


def version() -> str:
    return _lib.ulysses_version().decode()


def _check(rc: int) -> None:
    if rc != ULYSSES_OK:
        raise UlyssesError(rc, _lib.ulysses_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _spec(name: str, t, shape, dtype=torch.bfloat16) -> None:
    """Shape, dtype and contiguity of a buffer the C call reads or writes.

    The C ABI derives every size from N, the head counts and d, so a buffer
    smaller than that would be read or written past its end: every tensor is
    checked against the exact shape the call implies. Raised as ValueError
    (TypeError if it is not a tensor); the device is checked separately."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_cuda(*named) -> None:
    """Every tensor on one CUDA device."""
    dev = None
    for name, t in named:
        if not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")


def _dims(name: str, t, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")
    return tuple(t.shape)


def _pos32(pos: torch.Tensor, N: int) -> torch.Tensor:
    if not isinstance(pos, torch.Tensor) or pos.dim() != 1 or pos.shape[0] != N:
        raise ValueError("position_ids must be a 1-D tensor of length N")
    if pos.dtype not in (torch.int32, torch.int64):
        raise ValueError("position_ids must be int32 or int64")
    if not pos.is_cuda:
        raise TypeError("position_ids must be a CUDA tensor")
    if pos.dtype != torch.int32:
        pos = pos.to(torch.int32)   # argument marshalling: the ABI takes int32 ids
    return pos.contiguous()


def seq_to_head(src: torch.Tensor, P: int, rank: int = -1, out: Optional[torch.Tensor] = None,
                heads: Optional[Tuple[int, int]] = None) -> torch.Tensor:
    """[N][Hx][d] (= P rank buffers [P][N/P][Hx][d]) -> [P][N][Hx/P][d], or
    rank r's slice [N][Hx/P][d] when ``rank >= 0``. With ``heads=(head0, n)``
    only heads [head0, head0+n) of src's rows are exchanged (read in place)."""
    N, row_heads, d = _dims("src", src, 3)
    _spec("src", src, (N, row_heads, d))
    head0, Hx = (0, row_heads) if heads is None else (int(heads[0]), int(heads[1]))
    if head0 < 0 or Hx < 1 or head0 + Hx > row_heads:
        raise ValueError(f"heads [{head0}, {head0 + Hx}) outside the {row_heads} heads of src")
    if P < 1 or Hx % P:
        raise ValueError(f"head count {Hx} must be divisible by P={P}")
    shape = (P, N, Hx // P, d) if rank < 0 else (N, Hx // P, d)
    if out is not None:
        _spec("out", out, shape)
        _same_cuda(("src", src), ("out", out))
    else:
        _same_cuda(("src", src))
        out = torch.empty(shape, dtype=src.dtype, device=src.device)
    if heads is None:
        _check(_lib.ulysses_seq_to_head(_ptr(src), _ptr(out), N, P, Hx, d, rank, _stream(src)))
    else:
        _check(_lib.ulysses_seq_to_head_heads(_ptr(src), _ptr(out), N, P, Hx, d, rank, row_heads, head0,
                                              _stream(src)))
    return out


def head_to_seq(src: torch.Tensor, P: int, rank: int = -1, out: Optional[torch.Tensor] = None,
                head0: Optional[int] = None) -> torch.Tensor:
    """[P][N][Hx/P][d] -> [N][Hx][d]; with ``rank >= 0`` src is rank r's slice
    [N][Hx/P][d] and only its heads of ``out`` are written. With ``head0`` the
    result goes to heads [head0, head0+Hx) of ``out`` [N][row_heads][d] (the
    other heads are kept)."""
    if rank < 0:
        Pp, N, Hl, d = _dims("src", src, 4)
        if Pp != P:
            raise ValueError("src.shape[0] must equal P")
        _spec("src", src, (P, N, Hl, d))
    else:
        N, Hl, d = _dims("src", src, 3)
        _spec("src", src, (N, Hl, d))
    Hx = Hl * P
    if head0 is not None:
        if out is None:
            raise ValueError("head_to_seq with head0 needs `out`")
        row_heads = _dims("out", out, 3)[1]
        if head0 < 0 or head0 + Hx > row_heads:
            raise ValueError(f"heads [{head0}, {head0 + Hx}) outside the {row_heads} heads of out")
        _spec("out", out, (N, row_heads, d))
        _same_cuda(("src", src), ("out", out))
        _check(_lib.ulysses_head_to_seq_heads(_ptr(src), _ptr(out), N, P, Hx, d, rank, row_heads, int(head0),
                                              _stream(src)))
        return out
    shape = (N, Hx, d)
    if out is not None:
        _spec("out", out, shape)
        _same_cuda(("src", src), ("out", out))
    else:
        if rank >= 0:
            raise ValueError("head_to_seq with rank >= 0 needs `out` (other ranks' heads are kept)")
        _same_cuda(("src", src))
        out = torch.empty(shape, dtype=src.dtype, device=src.device)
    _check(_lib.ulysses_head_to_seq(_ptr(src), _ptr(out), N, P, Hx, d, rank, _stream(src)))
    return out


def workspace_bytes(N: int, Hl: int, Hkvl: int, d: int, backward: bool = False) -> int:
    return int(_lib.ulysses_attn_workspace_bytes(N, Hl, Hkvl, d, 1 if backward else 0))


def _workspace(ws: Optional[torch.Tensor], nbytes: int, device) -> torch.Tensor:
    """The caller's workspace if it is a large enough uint8 buffer on the
    device, else a fresh one."""
    if ws is not None:
        if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or not ws.is_contiguous():
            raise ValueError("ws must be a contiguous uint8 tensor")
        if ws.device != device:
            raise ValueError(f"ws is on {ws.device}, expected {device}")
        if ws.numel() >= nbytes:
            return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _heads_ok(Hl: int, Hkvl: int) -> None:
    if Hl < 1 or Hkvl < 1 or Hl % Hkvl:
        raise ValueError(f"query heads ({Hl}) must be a positive multiple of KV heads ({Hkvl})")


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, position_ids: torch.Tensor,
             scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
             lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None
             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Causal document-masked GQA attention of one rank's head slice.

    q [N][Hl][d], k/v [N][Hkvl][d] bf16; position_ids [N]. Returns
    (o [N][Hl][d] bf16, lse [Hl][N] fp32)."""
    N, Hl, d = _dims("q", q, 3)
    Hkvl = _dims("k", k, 3)[1]
    _spec("q", q, (N, Hl, d))
    _spec("k", k, (N, Hkvl, d))
    _spec("v", v, (N, Hkvl, d))
    _heads_ok(Hl, Hkvl)
    if out is not None:
        _spec("out", out, (N, Hl, d))
    if lse is not None:
        _spec("lse", lse, (Hl, N), torch.float32)
    pos = _pos32(position_ids, N)
    _same_cuda(("q", q), ("k", k), ("v", v), *((("out", out),) if out is not None else ()),
               *((("lse", lse),) if lse is not None else ()))
    _same_cuda(("q", q), ("position_ids", pos))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hl, N), dtype=torch.float32, device=q.device)
    nbytes = workspace_bytes(N, Hl, Hkvl, d, False)
    ws = _workspace(ws, nbytes, q.device)
    sc = 0.0 if scale is None else float(scale)
    _check(_lib.ulysses_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), N, Hl, Hkvl, d, sc, _ptr(out), _ptr(lse),
                                 _ptr(ws), ws.numel(), _stream(q)))
    return out, lse


def attn_fwd_window(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, position_ids: torch.Tensor,
                    q_lo: int, q_hi: int, kv_lo: int, kv_hi: int, scale: Optional[float] = None,
                    out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One ring step: the attention of rows [q_lo, q_hi) of the head slice
    q [N][Hl][d] over the keys [kv_lo, kv_hi) of k/v [N][Hkvl][d] only.
    Returns (o [q_hi-q_lo][Hl][d] bf16, lse [Hl][q_hi-q_lo] fp32); rows that
    see no key get o = 0, lse = -inf."""
    N, Hl, d = _dims("q", q, 3)
    Hkvl = _dims("k", k, 3)[1]
    _spec("q", q, (N, Hl, d))
    _spec("k", k, (N, Hkvl, d))
    _spec("v", v, (N, Hkvl, d))
    _heads_ok(Hl, Hkvl)
    if not (0 <= q_lo <= q_hi <= N and 0 <= kv_lo <= kv_hi <= N):
        raise ValueError(f"windows [{q_lo}, {q_hi}) and [{kv_lo}, {kv_hi}) must lie in [0, {N}]")
    M = q_hi - q_lo
    if out is not None:
        _spec("out", out, (M, Hl, d))
    if lse is not None:
        _spec("lse", lse, (Hl, M), torch.float32)
    pos = _pos32(position_ids, N)
    _same_cuda(("q", q), ("k", k), ("v", v), ("position_ids", pos), *((("out", out),) if out is not None else ()),
               *((("lse", lse),) if lse is not None else ()))
    if out is None:
        out = torch.empty((M, Hl, d), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((Hl, M), dtype=torch.float32, device=q.device)
    ws = _workspace(ws, workspace_bytes(N, Hl, Hkvl, d, False), q.device)
    sc = 0.0 if scale is None else float(scale)
    _check(_lib.ulysses_attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), N, Hl, Hkvl, d, int(q_lo), int(q_hi),
                                        int(kv_lo), int(kv_hi), sc, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                        _stream(q)))
    return out, lse


def attn_merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Merge R partial results over disjoint key sets: o_parts [R][M][Hl][d]
    bf16, lse_parts [R][Hl][M] fp32 -> (o [M][Hl][d], lse [Hl][M]). ``lse`` may
    be a column slice of a wider [Hl][*] fp32 tensor (rows contiguous)."""
    R, M, Hl, d = _dims("o_parts", o_parts, 4)
    _spec("o_parts", o_parts, (R, M, Hl, d))
    _spec("lse_parts", lse_parts, (R, Hl, M), torch.float32)
    if out is not None:
        _spec("out", out, (M, Hl, d))
    ld = M
    if lse is not None:
        if not isinstance(lse, torch.Tensor) or lse.dtype != torch.float32 or tuple(lse.shape) != (Hl, M) \
                or lse.stride(1) != 1 or (Hl > 1 and lse.stride(0) < M):
            raise ValueError(f"lse must be fp32 [{Hl}][{M}] with contiguous rows")
        ld = lse.stride(0) if Hl > 1 else M
    _same_cuda(("o_parts", o_parts), ("lse_parts", lse_parts), *((("out", out),) if out is not None else ()),
               *((("lse", lse),) if lse is not None else ()))
    if out is None:
        out = torch.empty((M, Hl, d), dtype=o_parts.dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty((Hl, M), dtype=torch.float32, device=o_parts.device)
    _check(_lib.ulysses_attn_merge(_ptr(o_parts), _ptr(lse_parts), R, M, Hl, d, _ptr(out), _ptr(lse), ld,
                                   _stream(o_parts)))
    return out, lse


def proj_workspace(device) -> torch.Tensor:
    """Workspace of the projection calls (a status word)."""
    return torch.zeros(int(_lib.ulysses_proj_workspace_bytes()), dtype=torch.uint8, device=device)


def qkv_proj(x: torch.Tensor, w_qkv: torch.Tensor, P: int, H: int, Hkv: int, d: int,
             q_out: Optional[torch.Tensor] = None, k_out: Optional[torch.Tensor] = None,
             v_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None
             ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """QKV projection of the P sequence shards x [N][hidden] with w_qkv
    [(H+2Hkv)*d][hidden], written straight into every rank's head slice:
    returns q [P][N][H/P][d], k and v [P][N][Hkv/P][d]."""
    N, hidden = _dims("x", x, 2)
    _spec("x", x, (N, hidden))
    _spec("w_qkv", w_qkv, ((H + 2 * Hkv) * d, hidden))
    if P < 1 or H % P or Hkv % P:
        raise ValueError(f"H={H} and Hkv={Hkv} must be divisible by P={P}")
    shapes = ((P, N, H // P, d), (P, N, Hkv // P, d), (P, N, Hkv // P, d))
    outs = []
    for name, t, shp in (("q_out", q_out, shapes[0]), ("k_out", k_out, shapes[1]), ("v_out", v_out, shapes[2])):
        if t is not None:
            _spec(name, t, shp)
        outs.append(t)
    _same_cuda(("x", x), ("w_qkv", w_qkv), *((n, t) for n, t in zip(("q_out", "k_out", "v_out"), outs)
                                             if t is not None))
    outs = [torch.empty(shp, dtype=torch.bfloat16, device=x.device) if t is None else t
            for t, shp in zip(outs, shapes)]
    ws = proj_workspace(x.device) if ws is None else ws
    _check(_lib.ulysses_qkv_proj(_ptr(x), _ptr(w_qkv), N, hidden, P, H, Hkv, d, _ptr(outs[0]), _ptr(outs[1]),
                                 _ptr(outs[2]), _ptr(ws), ws.numel(), _stream(x)))
    return tuple(outs)


def out_proj(o_heads: torch.Tensor, w_o: torch.Tensor, out: Optional[torch.Tensor] = None,
             ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Output projection read straight from every rank's head slice of the
    attention output o_heads [P][N][H/P][d], with w_o [hidden][H*d]:
    returns y [N][hidden] in the sequence layout."""
    P, N, Hl, d = _dims("o_heads", o_heads, 4)
    _spec("o_heads", o_heads, (P, N, Hl, d))
    hidden = _dims("w_o", w_o, 2)[0]
    _spec("w_o", w_o, (hidden, P * Hl * d))
    if out is not None:
        _spec("out", out, (N, hidden))
    _same_cuda(("o_heads", o_heads), ("w_o", w_o), *((("out", out),) if out is not None else ()))
    if out is None:
        out = torch.empty((N, hidden), dtype=torch.bfloat16, device=o_heads.device)
    ws = proj_workspace(o_heads.device) if ws is None else ws
    _check(_lib.ulysses_out_proj(_ptr(o_heads), _ptr(w_o), N, hidden, P, P * Hl, d, _ptr(out), _ptr(ws), ws.numel(),
                                 _stream(o_heads)))
    return out


def _rank_heads(H: int, Hkv: int, P: int, rank: int) -> Tuple[int, int]:
    if P < 1 or H % P or Hkv % P:
        raise ValueError(f"H={H} and Hkv={Hkv} must be divisible by P={P}")
    if not 0 <= rank < P:
        raise ValueError(f"rank={rank} outside [0, {P})")
    _heads_ok(H // P, Hkv // P)
    return H // P, Hkv // P


def attn_fwd_fused(q_seq: torch.Tensor, k_seq: torch.Tensor, v_seq: torch.Tensor, position_ids: torch.Tensor,
                   P: int, rank: int, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                   lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None
                   ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention of rank ``rank``'s heads read straight from the
    sequence-sharded buffers q_seq [N][H][d], k_seq/v_seq [N][Hkv][d]; O is
    written into ``out`` [N][H][d] (only this rank's heads)."""
    N, H, d = _dims("q_seq", q_seq, 3)
    Hkv = _dims("k_seq", k_seq, 3)[1]
    _spec("q_seq", q_seq, (N, H, d))
    _spec("k_seq", k_seq, (N, Hkv, d))
    _spec("v_seq", v_seq, (N, Hkv, d))
    Hl, Hkvl = _rank_heads(H, Hkv, P, rank)
    if out is not None:
        _spec("out", out, (N, H, d))
    if lse is not None:
        _spec("lse", lse, (Hl, N), torch.float32)
    pos = _pos32(position_ids, N)
    _same_cuda(("q_seq", q_seq), ("k_seq", k_seq), ("v_seq", v_seq),
               *((("out", out),) if out is not None else ()), *((("lse", lse),) if lse is not None else ()))
    _same_cuda(("q_seq", q_seq), ("position_ids", pos))
    if out is None:
        out = torch.empty_like(q_seq)
    if lse is None:
        lse = torch.empty((Hl, N), dtype=torch.float32, device=q_seq.device)
    nbytes = workspace_bytes(N, Hl, Hkvl, d, False)
    ws = _workspace(ws, nbytes, q_seq.device)
    sc = 0.0 if scale is None else float(scale)
    _check(_lib.ulysses_attn_fwd_fused(_ptr(q_seq), _ptr(k_seq), _ptr(v_seq), _ptr(pos), N, P, H, Hkv, d, rank,
                                       sc, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(q_seq)))
    return out, lse


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, dout: torch.Tensor,
             lse: torch.Tensor, position_ids: torch.Tensor, scale: Optional[float] = None,
             ws: Optional[torch.Tensor] = None, dq: Optional[torch.Tensor] = None,
             dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None
             ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients (dq, dk, dv) of sum(dout * o) for one rank's head slice."""
    N, Hl, d = _dims("q", q, 3)
    Hkvl = _dims("k", k, 3)[1]
    qshape, kshape = (N, Hl, d), (N, Hkvl, d)
    for name, t, shp in (("q", q, qshape), ("k", k, kshape), ("v", v, kshape), ("o", o, qshape),
                         ("dout", dout, qshape)):
        _spec(name, t, shp)
    _spec("lse", lse, (Hl, N), torch.float32)
    _heads_ok(Hl, Hkvl)
    named = [("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("lse", lse)]
    for name, t, shp in (("dq", dq, qshape), ("dk", dk, kshape), ("dv", dv, kshape)):
        if t is not None:
            _spec(name, t, shp)
            named.append((name, t))
    pos = _pos32(position_ids, N)
    _same_cuda(*named)
    _same_cuda(("q", q), ("position_ids", pos))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = workspace_bytes(N, Hl, Hkvl, d, True)
    ws = _workspace(ws, nbytes, q.device)
    sc = 0.0 if scale is None else float(scale)
    _check(_lib.ulysses_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(pos), N, Hl, Hkvl,
                                 d, sc, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream(q)))
    return dq, dk, dv


def sync_status(ws: torch.Tensor) -> None:
    """Synchronise the current stream; raise UlyssesError(ULYSSES_ERR_TIMEOUT)
    if a bounded device-side wait of the last call that used ``ws`` ran out."""
    _check(_lib.ulysses_sync_status(_ptr(ws), _stream(ws)))


def set_wait_limit_ns(ns: int) -> None:
    _lib.ulysses_set_wait_limit_ns(int(ns))


def set_debug_flags(flags: int) -> None:
    """Test hook: bit 0 makes later forward launches, bit 1 later backward
    launches, run one bounded wait out."""
    _lib.ulysses_set_debug_flags(int(flags))


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def attn_bwd_fused(q_seq: torch.Tensor, k_seq: torch.Tensor, v_seq: torch.Tensor, o_seq: torch.Tensor,
                   dout_seq: torch.Tensor, lse: torch.Tensor, position_ids: torch.Tensor, P: int, rank: int,
                   scale: Optional[float] = None, dq: Optional[torch.Tensor] = None,
                   dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients of rank ``rank``'s heads read straight from the sequence-sharded
    buffers (q/o/dout [N][H][d], k/v [N][Hkv][d]) and written into dq [N][H][d],
    dk / dv [N][Hkv][d] (only this rank's heads); lse is [H/P][N]."""
    N, H, d = _dims("q_seq", q_seq, 3)
    Hkv = _dims("k_seq", k_seq, 3)[1]
    qshape, kshape = (N, H, d), (N, Hkv, d)
    for name, t, shp in (("q_seq", q_seq, qshape), ("k_seq", k_seq, kshape), ("v_seq", v_seq, kshape),
                         ("o_seq", o_seq, qshape), ("dout_seq", dout_seq, qshape)):
        _spec(name, t, shp)
    Hl, Hkvl = _rank_heads(H, Hkv, P, rank)
    _spec("lse", lse, (Hl, N), torch.float32)
    named = [("q_seq", q_seq), ("k_seq", k_seq), ("v_seq", v_seq), ("o_seq", o_seq), ("dout_seq", dout_seq),
             ("lse", lse)]
    for name, t, shp in (("dq", dq, qshape), ("dk", dk, kshape), ("dv", dv, kshape)):
        if t is not None:
            _spec(name, t, shp)
            named.append((name, t))
    pos = _pos32(position_ids, N)
    _same_cuda(*named)
    _same_cuda(("q_seq", q_seq), ("position_ids", pos))
    dq = torch.empty_like(q_seq) if dq is None else dq
    dk = torch.empty_like(k_seq) if dk is None else dk
    dv = torch.empty_like(v_seq) if dv is None else dv
    nbytes = workspace_bytes(N, Hl, Hkvl, d, True)
    ws = _workspace(ws, nbytes, q_seq.device)
    sc = 0.0 if scale is None else float(scale)
    _check(_lib.ulysses_attn_bwd_fused(_ptr(q_seq), _ptr(k_seq), _ptr(v_seq), _ptr(o_seq), _ptr(dout_seq), _ptr(lse),
                                       _ptr(pos), N, P, H, Hkv, d, rank, sc, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                       ws.numel(), _stream(q_seq)))
    return dq, dk, dv
