"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol the header declares,
and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import exact_io_aware_76_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

FAKE = 0x10000  # aligned, never dereferenced: validation fails first
MISALIGNED = 0x10008


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    assert {"fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_status_string", "fa_device_status"} <= names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(fa.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, 7):
        s = fa.status_string(code)
        assert isinstance(s, str) and s


def fwd_call(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Sq=128, Sk=128, H=1, D=64, causal=0, scale=0.0, dtype=0):
    return fa.lib().fa_fwd(q, k, v, o, lse, B, Sq, Sk, H, D, causal, scale, dtype, None)


@pytest.mark.parametrize("kw", [dict(q=None), dict(k=None), dict(v=None), dict(o=None), dict(lse=None),
                                dict(q=MISALIGNED), dict(o=MISALIGNED), dict(lse=MISALIGNED), dict(B=0), dict(Sq=0),
                                dict(Sk=-1), dict(H=0), dict(D=0), dict(scale=float("nan")),
                                dict(scale=float("inf")), dict(scale=float("-inf")), dict(dtype=2)])
def test_fwd_rejects_invalid(kw):
    assert fwd_call(**kw) == -1


@pytest.mark.parametrize("scale", [-0.5, -1e-30, -0.0, -300.0])
def test_negative_scale_passes_validation(scale):
    # any finite scale is used as given: a negative one gets past the argument checks and the call fails only
    # at the (later) head-dim check, before anything touches a device
    assert fwd_call(scale=scale, D=96) == -2
    assert bwd_call(scale=scale, D=96) == -2


@pytest.mark.parametrize("D", [32, 96, 256])
def test_fwd_unsupported_head_dim(D):
    assert fwd_call(D=D) == -2


def bwd_call(ptr=FAKE, ws=FAKE, ws_bytes=1 << 30, B=1, Sq=128, Sk=128, H=1, D=64, scale=0.0, dtype=0, **over):
    args = dict(q=ptr, k=ptr, v=ptr, o=ptr, lse=ptr, do=ptr, dq=ptr, dk=ptr, dv=ptr)
    args.update(over)
    return fa.lib().fa_bwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["do"], args["dq"],
                           args["dk"], args["dv"], B, Sq, Sk, H, D, 1, scale, dtype, ws, ws_bytes, None)


@pytest.mark.parametrize("kw", [dict(q=None), dict(dq=None), dict(dk=MISALIGNED), dict(B=0), dict(scale=float("nan")),
                                dict(dtype=5)])
def test_bwd_rejects_invalid(kw):
    assert bwd_call(**kw) == -1


def test_bwd_workspace_checks():
    need = fa.workspace_size(2, 300, 3, 64)
    assert need > 0
    assert bwd_call(B=2, Sq=300, H=3, ws=None) == -5
    assert bwd_call(B=2, Sq=300, H=3, ws_bytes=need - 1) == -5
    assert bwd_call(B=2, Sq=300, H=3, ws=FAKE + 16) == -5  # not 256-byte aligned


def test_workspace_size_invalid_is_zero():
    assert fa.workspace_size(0, 128, 1, 64) == 0
    assert fa.workspace_size(1, 128, 1, 96) == 0


def fwd_fp8_call(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Sq=128, Sk=128, H=2, Hkv=1, D=128, causal=0,
                 left=-1, right=-1, scale=0.0, qd=1.0, kd=1.0, vd=1.0):
    return fa.lib().fa_fwd_fp8(q, k, v, o, lse, B, Sq, Sk, H, Hkv, D, causal, left, right, scale, qd, kd, vd, None)


@pytest.mark.parametrize("kw", [dict(q=None), dict(v=MISALIGNED), dict(lse=None), dict(Hkv=0), dict(Hkv=3),
                                dict(B=0), dict(Sq=0), dict(scale=float("nan")), dict(qd=0.0), dict(kd=-1.0),
                                dict(vd=float("inf")), dict(qd=float("nan"))])
def test_fwd_fp8_rejects_invalid(kw):
    assert fwd_fp8_call(**kw) == -1


@pytest.mark.parametrize("D", [32, 96, 256])
def test_fwd_fp8_unsupported_head_dim(D):
    assert fwd_fp8_call(D=D) == -2


def fwd_drop_call(p, B=1, Sq=128, Sk=128, H=1, Hkv=1, D=64):
    return fa.lib().fa_fwd_dropout(FAKE, FAKE, FAKE, FAKE, FAKE, B, Sq, Sk, H, Hkv, D, 0, -1, -1, 0.0, 0, p, 1, 0, None)


@pytest.mark.parametrize("p", [-0.1, 1.0, 1.5, 0.999, float("nan"), float("inf")])
def test_dropout_rejects_bad_probability(p):
    # 0.999 rounds to t = 256 (everything dropped): rejected like p >= 1
    assert fwd_drop_call(p) == -1
    assert fa.lib().fa_bwd_dropout(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, 1, 1, 64, 0, -1,
                                   -1, 0.0, 0, p, 1, 0, FAKE, 1 << 30, None) == -1


def test_dropout_rejects_bad_shapes_first():
    assert fwd_drop_call(0.1, B=0) == -1
    assert fwd_drop_call(0.1, D=96) == -2


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    # No fallback: without the built library the binding raises instead of computing anything elsewhere.
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setattr(fa, "LIB_PATH", str(tmp_path / "libfa.so"))
    with pytest.raises(ImportError):
        fa.lib()


@pytest.mark.parametrize("H,Hkv", [(6, 4), (6, 0), (0, 1), (4, -1)])
def test_grouped_entry_points_reject_bad_head_groups(H, Hkv):
    # H must be a positive multiple of Hkv >= 1; checked before anything touches a device
    L = fa.lib()
    assert L.fa_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, H, Hkv, 64, 0, -1, -1, 0.0, 1, None) == -1
    assert L.fa_bwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, H, Hkv, 64, 0, -1, -1, 0.0,
                       1, FAKE, 1 << 30, None) == -1
    assert L.fa_fwd_dropout(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, H, Hkv, 64, 0, -1, -1, 0.0, 1, 0.1, 1, 0,
                            None) == -1
    assert L.fa_bwd_dropout(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, H, Hkv, 64, 0, -1, -1,
                            0.0, 1, 0.1, 1, 0, FAKE, 1 << 30, None) == -1


def test_noalloc_host_checks():
    # sizes are validated, and problems whose workspace exceeds the fixed scratch rejected, before any device
    # lookup (the scratch's address is only looked up for calls that can run)
    L = fa.lib()
    L.fa_bwd_noalloc.restype = ctypes.c_int
    L.fa_bwd_noalloc.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_int,
                                                                               ctypes.c_void_p]
    args = [FAKE] * 9
    assert L.fa_bwd_noalloc(*args, 0, 128, 128, 1, 64, 1, 0.0, 1, None) == -1
    assert L.fa_bwd_noalloc(*args, 1, 128, 128, 1, 64, 1, float("nan"), 1, None) == -1
    assert L.fa_bwd_noalloc(*args, 1, 128, 128, 1, 96, 1, 0.0, 1, None) == -2
    B, S, H, D = 1, 8192, 32, 128
    assert fa.workspace_size(B, S, H, D) > (64 << 20)
    assert L.fa_bwd_noalloc(*args, B, S, S, H, D, 1, 0.0, 1, None) == -5
