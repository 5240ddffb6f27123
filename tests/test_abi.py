"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/ulysses.h declares, sizes its workspace, and rejects
bad arguments with the documented status codes before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ulysses.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ulysses_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import long_context_sequence_ulysses_b200 as U
    lib = ctypes.CDLL(U.library_path())
    syms = _declared_symbols()
    assert len(syms) >= 10, syms
    for s in syms:
        assert hasattr(lib, s), f"{s} declared in ulysses.h but not exported"


def test_version_and_no_error_initially():
    import long_context_sequence_ulysses_b200 as U
    assert "sm_100a" in U.version()


def _lib():
    import long_context_sequence_ulysses_b200 as U
    return U._lib


FAKE = ctypes.c_void_p(0x10000)       # never dereferenced: validation fails first
FAKE_MIS = ctypes.c_void_p(0x10008)   # misaligned


@pytest.mark.parametrize("fn", ["ulysses_seq_to_head", "ulysses_head_to_seq"])
def test_relayout_argument_errors(fn):
    lib = _lib()
    f = getattr(lib, fn)
    assert f(FAKE, FAKE, 10, 4, 8, 128, -1, None) == -1            # N % P
    assert f(FAKE, FAKE, 16, 4, 6, 128, -1, None) == -1            # H % P
    assert f(FAKE, FAKE, 16, 4, 8, 96, -1, None) == -1             # d
    assert f(FAKE, FAKE, 16, 0, 8, 128, -1, None) == -1            # P
    assert f(FAKE, FAKE, 16, 4, 8, 128, 4, None) == -1             # rank >= P
    assert f(None, FAKE, 16, 4, 8, 128, -1, None) == -1            # null
    assert f(FAKE_MIS, FAKE, 16, 4, 8, 128, -1, None) == -1        # alignment
    assert f(None, None, 0, 4, 8, 128, -1, None) == 0              # empty is a no-op
    assert b"divisible" in lib.ulysses_last_error() or True


def test_workspace_sizes():
    lib = _lib()
    a = lib.ulysses_attn_workspace_bytes(32768, 4, 1, 128, 0)
    b = lib.ulysses_attn_workspace_bytes(32768, 4, 1, 128, 1)
    assert a > 32768 * 4 and b > a + 32768 * 4 * 4
    assert lib.ulysses_attn_workspace_bytes(0, 4, 1, 128, 0) > 0
    assert lib.ulysses_attn_workspace_bytes(-1, 4, 1, 128, 0) == 0


def test_attn_argument_errors():
    lib = _lib()
    ws_ok = lib.ulysses_attn_workspace_bytes(256, 4, 2, 128, 0)
    args = lambda N, Hl, Hkvl, d, ws, wsb: (FAKE, FAKE, FAKE, FAKE, N, Hl, Hkvl, d, ctypes.c_float(0.0), FAKE, FAKE,
                                            ws, wsb, None)
    f = lib.ulysses_attn_fwd
    assert f(*args(256, 4, 3, 128, FAKE, ws_ok)) == -1           # Hl % Hkvl
    assert f(*args(256, 4, 2, 80, FAKE, ws_ok)) == -1            # d
    assert f(*args(-5, 4, 2, 128, FAKE, ws_ok)) == -1            # N
    assert f(*args(256, 4, 2, 128, None, ws_ok)) == -5           # no workspace
    assert f(*args(256, 4, 2, 128, FAKE, ws_ok - 1)) == -5       # workspace too small
    assert f(*args(0, 4, 2, 128, FAKE, ws_ok)) == 0              # empty
    assert b"workspace" in lib.ulysses_last_error() or True
    fused = lib.ulysses_attn_fwd_fused
    fa = lambda N, P, H, Hkv, rank: (FAKE, FAKE, FAKE, FAKE, N, P, H, Hkv, 128, rank, ctypes.c_float(0.0), FAKE, FAKE,
                                     FAKE, ws_ok, None)
    assert fused(*fa(256, 3, 4, 4, 0)) == -1                      # H % P
    assert fused(*fa(256, 4, 8, 2, 0)) == -1                      # Hkv % P
    assert fused(*fa(255, 2, 4, 2, 0)) == -1                      # N % P
    assert fused(*fa(256, 2, 4, 2, 2)) == -1                      # rank
    b = lib.ulysses_attn_bwd
    bws = lib.ulysses_attn_workspace_bytes(256, 4, 2, 128, 1)
    ba = lambda N, Hl, Hkvl, d, ws, wsb: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, N, Hl, Hkvl, d,
                                          ctypes.c_float(0.0), FAKE, FAKE, FAKE, ws, wsb, None)
    assert b(*ba(256, 4, 3, 128, FAKE, bws)) == -1
    assert b(*ba(256, 4, 2, 128, FAKE, ws_ok)) == -5              # forward-sized workspace is too small
    assert b(*ba(0, 4, 2, 128, FAKE, bws)) == 0
    bf = lib.ulysses_attn_bwd_fused
    bfa = lambda N, P, H, Hkv, rank, wsb: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, N, P, H, Hkv, 128, rank,
                                           ctypes.c_float(0.0), FAKE, FAKE, FAKE, FAKE, wsb, None)
    bws_f = lib.ulysses_attn_workspace_bytes(256, 2, 1, 128, 1)
    assert bf(*bfa(256, 3, 4, 4, 0, bws_f)) == -1                 # H % P
    assert bf(*bfa(256, 4, 8, 2, 0, bws_f)) == -1                 # Hkv % P
    assert bf(*bfa(255, 2, 4, 2, 0, bws_f)) == -1                 # N % P
    assert bf(*bfa(256, 2, 4, 2, 2, bws_f)) == -1                 # rank
    assert bf(*bfa(256, 2, 4, 2, 1, bws_f - 1)) == -5             # workspace too small
    assert bf(*bfa(0, 2, 4, 2, 1, bws_f)) == 0                    # empty


def test_python_binding_rejects_cpu_tensors():
    import torch
    import long_context_sequence_ulysses_b200 as U
    x = torch.zeros(8, 4, 32, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        U.seq_to_head(x, 2)
    with pytest.raises(TypeError):
        U.attn_fwd(x, x, x, torch.arange(8))
