"""ulysses_attn_fwd_noalloc: the forward for callers that cannot allocate
device memory (for example a plugin whose host framework owns every device
buffer and hands over only inputs and outputs). Its scratch lives in a static
device array inside the library. Called here through the C ABI and compared
with ulysses_attn_fwd (which takes a caller-provided workspace) on three calls
in a row (two whose schedule pairs heads, then one whose schedule pairs query
tiles), so stale scratch left by one call would show up in the next.
Collected last on purpose."""
import ctypes

import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS
from workloads import random_case

pytestmark = pytest.mark.gpu


def _fn():
    import long_context_sequence_ulysses_b200 as U
    lib = ctypes.CDLL(U.library_path())
    f = lib.ulysses_attn_fwd_noalloc
    P = ctypes.c_void_p
    f.argtypes = [P, P, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, P, P, P]
    f.restype = ctypes.c_int
    return U, lib, f


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_attn_fwd_on_consecutive_calls():
    U, lib, f = _fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        random_case(3000, 4, 2, 128, [1200, 1, 1799], seed=41, device="cuda"),
        random_case(1536, 2, 1, 64, [700, 300, 536], seed=42, device="cuda"),
        # odd group size: the schedule holds pairs of query tiles (a different
        # layout of the same scratch), N not a multiple of 256
        random_case(2000, 3, 1, 128, [1500, 2, 498], seed=43, device="cuda"),
    ]
    for c in cases:
        N, Hl, d = c["q"].shape
        Hkvl = c["k"].shape[1]
        o = torch.empty_like(c["q"])
        lse = torch.empty((Hl, N), dtype=torch.float32, device="cuda")
        rc = f(_ptr(c["q"]), _ptr(c["k"]), _ptr(c["v"]), _ptr(c["position_ids"]), N, Hl, Hkvl, d,
               ctypes.c_float(0.0), _ptr(o), _ptr(lse), stream)
        assert rc == 0, lib.ulysses_last_error()
        ref_o, ref_lse = U.attn_fwd(c["q"], c["k"], c["v"], c["position_ids"])
        torch.cuda.synchronize()
        do = (o.float() - ref_o.float()).abs()
        dl = (lse - ref_lse).abs()
        assert do.max().item() <= MAX_ABS and do.mean().item() <= MEAN_ABS
        assert dl.max().item() <= MAX_ABS and dl.mean().item() <= MEAN_ABS


def test_noalloc_rejects_sequences_beyond_its_scratch():
    U, lib, f = _fn()
    fake = ctypes.c_void_p(0x10000)
    lib.ulysses_last_error.restype = ctypes.c_char_p
    rc = f(fake, fake, fake, fake, 131073, 4, 1, 128, ctypes.c_float(0.0), fake, fake, None)
    assert rc == -2
    assert b"131072" in lib.ulysses_last_error()
