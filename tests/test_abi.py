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

    def rejects(args, code, text):
        assert f(*args) == code
        assert text in lib.ulysses_last_error(), lib.ulysses_last_error()

    rejects((FAKE, FAKE, 10, 4, 8, 128, -1, None), -1, b"N=10 not divisible by P=4")
    rejects((FAKE, FAKE, 16, 4, 6, 128, -1, None), -1, b"heads 6 not divisible by P=4")
    rejects((FAKE, FAKE, 16, 4, 8, 96, -1, None), -1, b"d=96 not in {32,64,128}")
    rejects((FAKE, FAKE, 16, 0, 8, 128, -1, None), -1, b"P=0 < 1")
    rejects((FAKE, FAKE, 16, 4, 8, 128, 4, None), -1, b"rank=4 >= P=4")
    rejects((None, FAKE, 16, 4, 8, 128, -1, None), -1, b"null pointer")
    rejects((FAKE_MIS, FAKE, 16, 4, 8, 128, -1, None), -1, b"16-byte aligned")
    assert f(None, None, 0, 4, 8, 128, -1, None) == 0              # empty is a no-op
    assert lib.ulysses_last_error() == b""                         # a success clears the message


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

    def rejects(f, args, code, text):
        assert f(*args) == code
        assert text in lib.ulysses_last_error(), lib.ulysses_last_error()

    args = lambda N, Hl, Hkvl, d, ws, wsb: (FAKE, FAKE, FAKE, FAKE, N, Hl, Hkvl, d, ctypes.c_float(0.0), FAKE, FAKE,
                                            ws, wsb, None)
    f = lib.ulysses_attn_fwd
    rejects(f, args(256, 4, 3, 128, FAKE, ws_ok), -1, b"Hl=4 not divisible by Hkvl=3")
    rejects(f, args(256, 4, 2, 80, FAKE, ws_ok), -1, b"d=80")
    rejects(f, args(-5, 4, 2, 128, FAKE, ws_ok), -1, b"N=-5 < 0")
    rejects(f, args(256, 4, 2, 128, None, ws_ok), -5, b"workspace is null")
    rejects(f, args(256, 4, 2, 128, FAKE, ws_ok - 1), -5, b"required")
    rejects(f, args(256, 4, 2, 128, FAKE_MIS, ws_ok), -1, b"workspace must be 16-byte aligned")
    assert f(*args(0, 4, 2, 128, FAKE, ws_ok)) == 0              # empty
    fused = lib.ulysses_attn_fwd_fused
    fa = lambda N, P, H, Hkv, rank: (FAKE, FAKE, FAKE, FAKE, N, P, H, Hkv, 128, rank, ctypes.c_float(0.0), FAKE, FAKE,
                                     FAKE, ws_ok, None)
    rejects(fused, fa(256, 3, 4, 4, 0), -1, b"divisible by P=3")      # H % P
    rejects(fused, fa(256, 4, 8, 2, 0), -1, b"divisible by P=4")      # Hkv % P
    rejects(fused, fa(255, 2, 4, 2, 0), -1, b"N=255 not divisible")   # N % P
    rejects(fused, fa(256, 2, 4, 2, 2), -1, b"rank=2 outside")        # rank
    b = lib.ulysses_attn_bwd
    bws = lib.ulysses_attn_workspace_bytes(256, 4, 2, 128, 1)
    ba = lambda N, Hl, Hkvl, d, ws, wsb: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, N, Hl, Hkvl, d,
                                          ctypes.c_float(0.0), FAKE, FAKE, FAKE, ws, wsb, None)
    rejects(b, ba(256, 4, 3, 128, FAKE, bws), -1, b"not divisible by Hkvl=3")
    rejects(b, ba(256, 4, 2, 128, FAKE, ws_ok), -5, b"required")      # forward-sized workspace is too small
    assert b(*ba(0, 4, 2, 128, FAKE, bws)) == 0
    bf = lib.ulysses_attn_bwd_fused
    bfa = lambda N, P, H, Hkv, rank, wsb: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, N, P, H, Hkv, 128, rank,
                                           ctypes.c_float(0.0), FAKE, FAKE, FAKE, FAKE, wsb, None)
    bws_f = lib.ulysses_attn_workspace_bytes(256, 2, 1, 128, 1)
    rejects(bf, bfa(256, 3, 4, 4, 0, bws_f), -1, b"divisible by P=3")     # H % P
    rejects(bf, bfa(256, 4, 8, 2, 0, bws_f), -1, b"divisible by P=4")     # Hkv % P
    rejects(bf, bfa(255, 2, 4, 2, 0, bws_f), -1, b"N=255 not divisible")  # N % P
    rejects(bf, bfa(256, 2, 4, 2, 2, bws_f), -1, b"rank=2 outside")       # rank
    rejects(bf, bfa(256, 2, 4, 2, 1, bws_f - 1), -5, b"required")         # workspace too small
    assert bf(*bfa(0, 2, 4, 2, 1, bws_f)) == 0                            # empty


def test_python_binding_rejects_cpu_tensors():
    import torch
    import long_context_sequence_ulysses_b200 as U
    x = torch.zeros(8, 4, 32, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        U.seq_to_head(x, 2)
    with pytest.raises(TypeError):
        U.attn_fwd(x, x, x, torch.arange(8))


# ---------------------------------------------------------------- binding shape checks
# The C ABI derives every size from N, the head counts and d, so a wrongly
# shaped buffer would be read or written past its end on the device. The
# binding checks every tensor against the exact shape the call implies, before
# it looks at the device, so these run without a GPU.

def _bf(*shape):
    import torch
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _f32(*shape):
    import torch
    return torch.zeros(*shape, dtype=torch.float32)


N_, HL, HKVL, D_ = 16, 4, 2, 32


def _fwd_ok():
    import torch
    return dict(q=_bf(N_, HL, D_), k=_bf(N_, HKVL, D_), v=_bf(N_, HKVL, D_), position_ids=torch.arange(N_))


@pytest.mark.parametrize("field,bad", [
    ("k", _bf(N_, HKVL, 64)), ("v", _bf(N_ + 1, HKVL, D_)), ("v", _bf(N_, HKVL + 1, D_)),
    ("out", _bf(N_ - 1, HL, D_)), ("out", _bf(N_, HL, D_).float()), ("lse", _f32(HL, N_ - 1)),
    ("lse", _f32(N_, HL)), ("position_ids", __import__("torch").arange(N_ - 1)),
])
def test_attn_fwd_rejects_wrong_shapes(field, bad):
    import long_context_sequence_ulysses_b200 as U
    kw = _fwd_ok()
    kw[field] = bad
    with pytest.raises(ValueError):
        U.attn_fwd(**kw)


def _bwd_ok():
    import torch
    return dict(q=_bf(N_, HL, D_), k=_bf(N_, HKVL, D_), v=_bf(N_, HKVL, D_), o=_bf(N_, HL, D_),
                dout=_bf(N_, HL, D_), lse=_f32(HL, N_), position_ids=torch.arange(N_))


@pytest.mark.parametrize("field,bad", [
    ("k", _bf(N_, HKVL, 64)), ("v", _bf(N_, HKVL + 1, D_)), ("o", _bf(N_, HL - 1, D_)), ("dout", _bf(N_ - 1, HL, D_)),
    ("lse", _f32(HL, N_ + 1)), ("dq", _bf(N_, HL - 1, D_)), ("dk", _bf(N_, HKVL, D_ // 2)),
    ("dv", _bf(N_ - 2, HKVL, D_)), ("dq", _f32(N_, HL, D_)),
])
def test_attn_bwd_rejects_wrong_shapes(field, bad):
    import long_context_sequence_ulysses_b200 as U
    kw = _bwd_ok()
    kw[field] = bad
    with pytest.raises(ValueError):
        U.attn_bwd(**kw)


P_, H_, HKV_ = 2, 4, 2


def _fused_ok():
    import torch
    return dict(q_seq=_bf(N_, H_, D_), k_seq=_bf(N_, HKV_, D_), v_seq=_bf(N_, HKV_, D_),
                position_ids=torch.arange(N_), P=P_, rank=1)


@pytest.mark.parametrize("field,bad", [
    ("k_seq", _bf(N_, HKV_, 64)), ("v_seq", _bf(N_ - 1, HKV_, D_)), ("v_seq", _bf(N_, HKV_ + 2, D_)),
    ("out", _bf(N_, H_ // P_, D_)), ("lse", _f32(H_, N_)), ("P", 3), ("rank", 2),
])
def test_attn_fwd_fused_rejects_wrong_shapes(field, bad):
    import long_context_sequence_ulysses_b200 as U
    kw = _fused_ok()
    kw[field] = bad
    with pytest.raises(ValueError):
        U.attn_fwd_fused(**kw)


@pytest.mark.parametrize("field,bad", [
    ("k_seq", _bf(N_, HKV_, 64)), ("o_seq", _bf(N_, H_ // P_, D_)), ("dout_seq", _bf(N_ + 2, H_, D_)),
    ("lse", _f32(H_, N_)), ("dq", _bf(N_, H_ // P_, D_)), ("dk", _bf(N_, HKV_ // P_, D_)),
    ("dv", _bf(N_, HKV_, 2 * D_)), ("rank", -1),
])
def test_attn_bwd_fused_rejects_wrong_shapes(field, bad):
    import long_context_sequence_ulysses_b200 as U
    kw = _fused_ok()
    kw.update(o_seq=_bf(N_, H_, D_), dout_seq=_bf(N_, H_, D_), lse=_f32(H_ // P_, N_))
    kw[field] = bad
    with pytest.raises(ValueError):
        U.attn_bwd_fused(**kw)


@pytest.mark.parametrize("call", ["seq_to_head", "head_to_seq_all", "head_to_seq_rank"])
def test_relayout_binding_rejects_wrong_out(call):
    import long_context_sequence_ulysses_b200 as U
    with pytest.raises(ValueError):
        if call == "seq_to_head":
            U.seq_to_head(_bf(N_, H_, D_), P_, out=_bf(P_, N_, H_, D_))
        elif call == "head_to_seq_all":
            U.head_to_seq(_bf(P_, N_, H_ // P_, D_), P_, out=_bf(N_, H_ // P_, D_))
        else:
            U.head_to_seq(_bf(N_, H_ // P_, D_), P_, rank=0, out=_bf(N_ - 1, H_, D_))


def test_binding_checks_shapes_before_device():
    """Correct shapes on CPU tensors reach the device check (TypeError), so the
    ValueErrors above are shape errors, not device errors."""
    import long_context_sequence_ulysses_b200 as U
    with pytest.raises(TypeError):
        U.attn_fwd(**_fwd_ok())
    with pytest.raises(TypeError):
        U.attn_bwd(**_bwd_ok())
    with pytest.raises(TypeError):
        U.attn_fwd_fused(**_fused_ok())


def test_window_and_merge_argument_errors():
    lib = _lib()
    ws_ok = lib.ulysses_attn_workspace_bytes(256, 4, 2, 128, 0)

    def rejects(f, args, code, text):
        assert f(*args) == code
        assert text in lib.ulysses_last_error(), lib.ulysses_last_error()

    f = lib.ulysses_attn_fwd_window
    wa = lambda ql, qh, kl, kh: (FAKE, FAKE, FAKE, FAKE, 256, 4, 2, 128, ql, qh, kl, kh, ctypes.c_float(0.0), FAKE,
                                 FAKE, FAKE, ws_ok, None)
    rejects(f, wa(-1, 10, 0, 256), -1, b"query window [-1, 10)")
    rejects(f, wa(10, 5, 0, 256), -1, b"query window [10, 5)")
    rejects(f, wa(0, 257, 0, 256), -1, b"query window [0, 257)")
    rejects(f, wa(0, 256, 100, 50), -1, b"key window [100, 50)")
    rejects(f, wa(0, 256, 0, 300), -1, b"key window [0, 300)")
    assert f(*wa(64, 64, 0, 256)) == 0                            # empty query window: nothing to do
    m = lib.ulysses_attn_merge
    ma = lambda R, M, Hl, d, ld: (FAKE, FAKE, R, M, Hl, d, FAKE, FAKE, ld, None)
    rejects(m, ma(0, 16, 4, 128, 16), -1, b"R=0 outside [1, 64]")
    rejects(m, ma(65, 16, 4, 128, 16), -1, b"R=65")
    rejects(m, ma(2, 16, 4, 96, 16), -1, b"d=96")
    rejects(m, ma(2, 16, 4, 128, 15), -1, b"lse_ld=15 < M=16")
    rejects(m, (FAKE_MIS, FAKE, 2, 16, 4, 128, FAKE, FAKE, 16, None), -1, b"16-byte aligned")
    assert m(*ma(2, 0, 4, 128, 0)) == 0                           # no rows
