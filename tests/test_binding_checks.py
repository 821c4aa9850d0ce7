"""The Python binding's operand checks, on the CPU: every input and caller-passed output is checked against
the shapes, dtypes and device the C ABI assumes, and a mismatch raises before the library is called; the call
itself runs with q's device current. Tensors are stand-ins that carry only the attributes the binding reads,
placed on a CUDA device by name, so nothing touches a GPU and nothing is launched."""
import contextlib

import pytest
import torch

import exact_io_aware_76_b200 as fa

BF16, F16, F32 = torch.bfloat16, torch.float16, torch.float32


class T:
    """A tensor stand-in: shape, dtype, device, contiguity, a fake aligned address."""

    def __init__(self, shape, dtype=BF16, device="cuda:0", contiguous=True):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self._contig = contiguous

    def is_contiguous(self):
        return self._contig

    def data_ptr(self):
        return 0x10000

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def element_size(self):
        return torch.tensor([], dtype=self.dtype).element_size()


B, Sq, Sk, H, Hkv, D = 2, 100, 120, 4, 2, 64


def good_fwd(**over):
    a = dict(q=T((B, Sq, H, D)), k=T((B, Sk, Hkv, D)), v=T((B, Sk, Hkv, D)), out=T((B, Sq, H, D)),
             lse=T((B, H, Sq), F32))
    a.update(over)
    return a


class FakeLib:
    """Records the calls it gets and the device that was current at the time; returns FA_OK."""

    def __init__(self, current):
        self.calls = []
        self.current = current

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, self.current[-1] if self.current else None))
            return 0
        return call


@pytest.fixture
def fake_lib(monkeypatch):
    current = []

    @contextlib.contextmanager
    def device_ctx(dev):
        current.append(dev)
        try:
            yield
        finally:
            current.pop()

    lib = FakeLib(current)
    monkeypatch.setattr(fa, "lib", lambda: lib)
    monkeypatch.setattr(fa, "_device", device_ctx)
    monkeypatch.setattr(fa, "_stream", lambda stream, dev: None)
    monkeypatch.setattr(fa, "workspace_size", lambda *a: 1024)
    return lib


def test_well_formed_call_reaches_the_library_on_qs_device(fake_lib):
    a = good_fwd(**{n: T(t.shape, t.dtype, "cuda:1") for n, t in good_fwd().items()})
    fa.fwd(a["q"], a["k"], a["v"], out=a["out"], lse=a["lse"])
    assert fake_lib.calls == [("fa_fwd_ex", torch.device("cuda:1"))]


@pytest.mark.parametrize("over", [
    dict(k=T((B, Sk, Hkv, 128))),                      # head dim differs from q's
    dict(k=T((B + 1, Sk, Hkv, D))),                    # batch differs
    dict(v=T((B, Sk - 1, Hkv, D))),                    # shorter v
    dict(v=T((B, Sk, Hkv, D), F16)),                   # dtype differs
    dict(k=T((B, Sk, 3, D)), v=T((B, Sk, 3, D))),      # 3 K/V heads do not divide 4 query heads
    dict(k=T((B, Sk, 0, D)), v=T((B, Sk, 0, D))),      # no K/V head
    dict(k=T((B, Sk, Hkv, D), device="cuda:1")),       # another device
    dict(q=T((B, Sq, H, D), device="cpu")),            # not on a GPU
    dict(q=T((B, Sq, H, D), contiguous=False)),        # strided
    dict(q=T((B, Sq, H, D), F32)),                     # fp32 input
    dict(q=T((Sq, H, D))),                             # wrong rank
    dict(out=T((B, Sq, H, D), F16)),                   # output dtype
    dict(out=T((B, Sq, H + 1, D))),                    # output shape
    dict(lse=T((B, Sq, H), F32)),                      # lse in the wrong order
    dict(lse=T((B, H, Sq), F16)),                      # lse not fp32
    dict(lse=T((B, H, Sq), F32, device="cuda:1")),     # lse on another device
])
def test_fwd_rejects_mismatched_operands_before_any_call(fake_lib, over):
    a = good_fwd(**over)
    with pytest.raises((ValueError, TypeError)):
        fa.fwd(a["q"], a["k"], a["v"], out=a["out"], lse=a["lse"])
    assert fake_lib.calls == []


def good_bwd(**over):
    a = good_fwd()
    a.update(dout=T((B, Sq, H, D)), dq=T((B, Sq, H, D)), dk=T((B, Sk, Hkv, D)), dv=T((B, Sk, Hkv, D)),
             workspace=T((4096,), torch.uint8))
    a.update(over)
    return a


def call_bwd(a, **kw):
    return fa.bwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], dq=a["dq"], dk=a["dk"], dv=a["dv"],
                  workspace=a["workspace"], **kw)


def test_well_formed_backward_reaches_the_library(fake_lib):
    call_bwd(good_bwd())
    assert [c[0] for c in fake_lib.calls] == ["fa_bwd_ex"]


@pytest.mark.parametrize("over", [
    dict(dout=T((B, Sq, H, D), F16)), dict(dout=T((B, Sq - 1, H, D))), dict(dq=T((B, Sq, H, D), F16)),
    dict(dk=T((B, Sk, H, D))), dict(dv=T((B, Sk, Hkv, D), device="cuda:1")), dict(out=T((B, Sq, H, 128))),
    dict(lse=T((B, H, Sq + 1), F32)), dict(workspace=T((16,), torch.uint8)),
    dict(workspace=T((4096,), torch.uint8, device="cuda:1")),
])
def test_bwd_rejects_mismatched_operands_before_any_call(fake_lib, over):
    with pytest.raises((ValueError, TypeError)):
        call_bwd(good_bwd(**over))
    assert fake_lib.calls == []


def test_single_stages_only_for_plain_attention(fake_lib):
    with pytest.raises(ValueError):
        call_bwd(good_bwd(), stage=1)  # grouped heads (Hkv = 2 < H = 4)
    assert fake_lib.calls == []


def test_fp8_checks(fake_lib):
    e4 = torch.float8_e4m3fn
    q, k, v = T((B, Sq, H, 128), e4), T((B, Sk, Hkv, 128), e4), T((B, Sk, Hkv, 128), e4)
    fa.fwd_fp8(q, k, v, out=T((B, Sq, H, 128)), lse=T((B, H, Sq), F32))
    assert [c[0] for c in fake_lib.calls] == ["fa_fwd_fp8"]
    for bad in (dict(out=T((B, Sq, H, 128), F16)), dict(q=T((B, Sq, H, 128)))):
        a = dict(q=q, out=T((B, Sq, H, 128)))
        a.update(bad)
        with pytest.raises((ValueError, TypeError)):
            fa.fwd_fp8(a["q"], k, v, out=a["out"], lse=T((B, H, Sq), F32))
    assert len(fake_lib.calls) == 1


def test_noalloc_checks(fake_lib):
    a = good_bwd(k=T((B, Sk, H, D)), v=T((B, Sk, H, D)), dk=T((B, Sk, H, D)), dv=T((B, Sk, H, D)))
    fa.bwd_noalloc(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], dq=a["dq"], dk=a["dk"], dv=a["dv"])
    assert [c[0] for c in fake_lib.calls] == ["fa_bwd_noalloc"]
    with pytest.raises((ValueError, TypeError)):
        fa.bwd_noalloc(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], dq=a["dq"], dk=a["dk"],
                       dv=T((B, Sk, H, D), F16))
    assert len(fake_lib.calls) == 1
