"""B200-native (sm_100a) exact IO-aware attention: a thin Python binding over the C ABI of ``libfa.so``.

Every step of the computation runs in the library's CUDA kernels; this module only marshals arguments
(PyTorch tensors -> device pointers, sizes and a CUDA stream) and turns status codes into exceptions. There is
no fallback: if the library is missing or fails to load, every call raises.

    fwd(q, k, v, causal=False, scale=None, window=(-1, -1)) -> (out, lse)
    bwd(q, k, v, out, lse, dout, causal=False, scale=None, window=(-1, -1)) -> (dq, dk, dv)

Layouts follow the C header (include/fa.h): q/out/dout [B, Sq, H, D], k/v [B, Sk, Hkv, D] (Hkv divides H:
grouped or multi-query K/V heads), fp16 or bf16, contiguous, on one CUDA device; lse is fp32 [B, H, Sq].
``scale=None`` means 1/sqrt(D); ``window=(left, right)`` limits each query to keys within left before and
right after its aligned key (-1 = unbounded side).

Every operand (inputs and caller-passed outputs alike) is checked against these shapes, dtypes and the
device of ``q`` before anything is launched; a mismatch raises ``ValueError`` or ``TypeError``. Each call
runs with ``q``'s device current and, unless a stream is given, on that device's current stream.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa.so")

FA_F16, FA_BF16 = 0, 1
FA_OK = 0
STATUS_NAMES = {0: "FA_OK", -1: "FA_ERR_INVALID", -2: "FA_ERR_UNSUPPORTED", -3: "FA_ERR_CUDA",
                -4: "FA_ERR_TIMEOUT", -5: "FA_ERR_WORKSPACE"}
EXPORTS = ("fa_fwd", "fa_fwd_ex", "fa_fwd_fp8", "fa_fwd_dropout", "fa_bwd_dropout", "fa_bwd", "fa_bwd_ex",
           "fa_bwd_stage", "fa_bwd_noalloc", "fa_bwd_workspace_size", "fa_status_string", "fa_device_status")

_lib = None


class FAError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s: %s (%s)" % (what, status_string(status), STATUS_NAMES.get(status, status)))


def lib():
    """The loaded ``libfa.so`` (ctypes.CDLL). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libfa.so not found at %s; build it with `python -m exact_io_aware_76_b200.build`"
                          % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    u32, u64 = ctypes.c_uint32, ctypes.c_uint64
    L.fa_fwd.restype = i
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
    L.fa_bwd.restype = i
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, sz, vp]
    L.fa_bwd_stage.restype = i
    L.fa_bwd_stage.argtypes = [i] + L.fa_bwd.argtypes
    L.fa_bwd_noalloc.restype = i
    L.fa_bwd_noalloc.argtypes = [vp] * 9 + [i] * 6 + [f, i, vp]
    L.fa_fwd_ex.restype = i
    L.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, i, vp]
    L.fa_fwd_fp8.restype = i
    L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, f, f, f, vp]
    L.fa_fwd_dropout.restype = i
    L.fa_fwd_dropout.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, i, f, u64, u32, vp]
    L.fa_bwd_dropout.restype = i
    L.fa_bwd_dropout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, i, f, u64, u32,
                                 vp, sz, vp]
    L.fa_bwd_ex.restype = i
    L.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, i, vp, sz, vp]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_status_string.argtypes = [i]
    L.fa_device_status.restype = i
    L.fa_device_status.argtypes = [i]
    _lib = L
    return L


def status_string(status):
    return lib().fa_status_string(int(status)).decode()


# ------------------------------------------------------------------------------------------ operand checks
def _dtype_code(t):
    import torch

    if t.dtype == torch.float16:
        return FA_F16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise TypeError("expected float16 or bfloat16, got %s" % t.dtype)


def _check(name, t, dev, shape=None, dtype=None):
    """``t`` must be a contiguous tensor on the CUDA device ``dev`` (and have ``shape`` / ``dtype`` if given)."""
    d = getattr(t, "device", None)
    if d is None or d.type != "cuda" or d != dev:
        raise ValueError("%s must be a CUDA tensor on %s, got %s" % (name, dev, d))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def check_qkv(q, k, v, dtypes):
    """Shapes of the inputs: q [B, Sq, H, D], k and v [B, Sk, Hkv, D] with Hkv >= 1 dividing H, one dtype (from
    ``dtypes``) for all three, one CUDA device. Returns (B, Sq, Sk, H, Hkv, D, device)."""
    dev = getattr(q, "device", None)
    if dev is None or dev.type != "cuda":
        raise ValueError("q must be a CUDA tensor, got device %s" % dev)
    if len(q.shape) != 4:
        raise ValueError("q must be a [B, Sq, H, D] tensor, got shape %s" % (tuple(q.shape),))
    if q.dtype not in dtypes:
        raise TypeError("q must be one of %s, got %s" % (tuple(str(x) for x in dtypes), q.dtype))
    _check("q", q, dev)
    B, Sq, H, D = q.shape
    if len(k.shape) != 4 or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k must be [B=%d, Sk, Hkv, D=%d], got %s" % (B, D, tuple(k.shape)))
    Sk, Hkv = k.shape[1], k.shape[2]
    if Hkv < 1 or H % Hkv != 0:
        raise ValueError("the K/V head count %d must divide the query head count %d" % (Hkv, H))
    _check("k", k, dev, dtype=q.dtype)
    _check("v", v, dev, shape=k.shape, dtype=q.dtype)
    return B, Sq, Sk, H, Hkv, D, dev


def check_fwd_outputs(out, lse, B, Sq, H, D, dev, out_dtype):
    import torch

    _check("out", out, dev, shape=(B, Sq, H, D), dtype=out_dtype)
    _check("lse", lse, dev, shape=(B, H, Sq), dtype=torch.float32)


def check_bwd_operands(q, k, out, lse, dout, dq, dk, dv, workspace, ws_bytes, B, Sq, H, D, dev):
    check_fwd_outputs(out, lse, B, Sq, H, D, dev, q.dtype)
    _check("dout", dout, dev, shape=q.shape, dtype=q.dtype)
    _check("dq", dq, dev, shape=q.shape, dtype=q.dtype)
    _check("dk", dk, dev, shape=k.shape, dtype=q.dtype)
    _check("dv", dv, dev, shape=k.shape, dtype=q.dtype)
    if workspace is not None:
        _check("workspace", workspace, dev)
        if workspace.numel() * workspace.element_size() < ws_bytes:
            raise ValueError("workspace must hold at least %d bytes" % ws_bytes)


def _stream(stream, dev):
    import torch

    s = torch.cuda.current_stream(dev) if stream is None else stream
    if s.device != dev:
        raise ValueError("stream is on %s but the tensors are on %s" % (s.device, dev))
    return ctypes.c_void_p(s.cuda_stream)


def _device(dev):
    import torch

    return torch.cuda.device(dev)


# ------------------------------------------------------------------------------------------ entry points
def fwd(q, k, v, causal=False, scale=None, out=None, lse=None, stream=None, window=(-1, -1), dropout_p=0.0, seed=0,
        offset=0):
    """Forward attention. Returns (out [B,Sq,H,D] in q's dtype, lse fp32 [B,H,Sq]).

    ``dropout_p`` > 0 drops attention probabilities with the Philox mask of ``fa_fwd_dropout`` (include/fa.h),
    keyed by ``seed`` (64-bit) and ``offset`` (32-bit); the backward must get the same three values."""
    import torch

    B, Sq, Sk, H, Hkv, D, dev = check_qkv(q, k, v, (torch.float16, torch.bfloat16))
    with _device(dev):
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
        check_fwd_outputs(out, lse, B, Sq, H, D, dev, q.dtype)
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Sq, Sk, H, Hkv, D,
                int(bool(causal)), int(window[0]), int(window[1]), float(0.0 if scale is None else scale),
                _dtype_code(q))
        if dropout_p:
            rc = lib().fa_fwd_dropout(*args, float(dropout_p), int(seed), int(offset), _stream(stream, dev))
        else:
            rc = lib().fa_fwd_ex(*args, _stream(stream, dev))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_dropout" if dropout_p else "fa_fwd_ex")
    return out, lse


def fwd_fp8(q, k, v, causal=False, scale=None, descale=(1.0, 1.0, 1.0), out=None, lse=None, stream=None,
            window=(-1, -1)):
    """Forward attention on float8_e4m3fn inputs (D = 64 or 128). The real inputs are q * descale[0],
    k * descale[1], v * descale[2]. Returns (out bf16 [B,Sq,H,D], lse fp32 [B,H,Sq])."""
    import torch

    B, Sq, Sk, H, Hkv, D, dev = check_qkv(q, k, v, (torch.float8_e4m3fn,))
    with _device(dev):
        if out is None:
            out = torch.empty((B, Sq, H, D), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
        check_fwd_outputs(out, lse, B, Sq, H, D, dev, torch.bfloat16)
        rc = lib().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Sq, Sk,
                              H, Hkv, D, int(bool(causal)), int(window[0]), int(window[1]),
                              float(0.0 if scale is None else scale), float(descale[0]), float(descale[1]),
                              float(descale[2]), _stream(stream, dev))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_fp8")
    return out, lse


def workspace_size(B, Sq, H, D):
    return int(lib().fa_bwd_workspace_size(B, Sq, H, D))


def bwd(q, k, v, out, lse, dout, causal=False, scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None,
        stage=-1, window=(-1, -1), dropout_p=0.0, seed=0, offset=0):
    """Backward attention (P recomputed from lse). Returns (dq, dk, dv) in q's dtype.

    ``stage`` selects one of the three launches (0 preprocess, 1 main, 2 dQ conversion; -1 all), see
    ``fa_bwd_stage`` in include/fa.h; a caller running the stages separately must pass the same workspace."""
    import torch

    B, Sq, Sk, H, Hkv, D, dev = check_qkv(q, k, v, (torch.float16, torch.bfloat16))
    if stage != -1 and (dropout_p or Hkv != H or tuple(window) != (-1, -1)):
        raise ValueError("single backward stages are available for plain attention only")
    with _device(dev):
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        ws_bytes = workspace_size(B, Sq, H, D)
        check_bwd_operands(q, k, out, lse, dout, dq, dk, dv, workspace, ws_bytes, B, Sq, H, D, dev)
        if workspace is None:
            workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
        sc = float(0.0 if scale is None else scale)
        ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
        ws_args = (workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream, dev))
        if dropout_p:
            rc = lib().fa_bwd_dropout(*ptrs, B, Sq, Sk, H, Hkv, D, int(bool(causal)), int(window[0]), int(window[1]),
                                      sc, _dtype_code(q), float(dropout_p), int(seed), int(offset), *ws_args)
        elif stage == -1:
            rc = lib().fa_bwd_ex(*ptrs, B, Sq, Sk, H, Hkv, D, int(bool(causal)), int(window[0]), int(window[1]), sc,
                                 _dtype_code(q), *ws_args)
        else:
            rc = lib().fa_bwd_stage(int(stage), *ptrs, B, Sq, Sk, H, D, int(bool(causal)), sc, _dtype_code(q),
                                    *ws_args)
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd")
    return dq, dk, dv


def bwd_noalloc(q, k, v, out, lse, dout, causal=False, scale=None, dq=None, dk=None, dv=None, stream=None):
    """``fa_bwd_noalloc``: the plain backward with the library's fixed device scratch instead of a workspace
    (problems up to FA_NOALLOC_SCRATCH_BYTES of workspace; see include/fa.h). Returns (dq, dk, dv)."""
    import torch

    B, Sq, Sk, H, Hkv, D, dev = check_qkv(q, k, v, (torch.float16, torch.bfloat16))
    if Hkv != H:
        raise ValueError("the no-alloc backward takes as many K/V heads as query heads")
    with _device(dev):
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        check_bwd_operands(q, k, out, lse, dout, dq, dk, dv, None, 0, B, Sq, H, D, dev)
        rc = lib().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Sq, Sk, H, D,
                                  int(bool(causal)), float(0.0 if scale is None else scale), _dtype_code(q),
                                  _stream(stream, dev))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_noalloc")
    return dq, dk, dv


def device_status(reset=False, device=None):
    """The device-side sticky status word (FA_OK, or FA_ERR_TIMEOUT after a kernel gave up on a wait) of
    ``device`` (default: the current device)."""
    import torch

    if device is None:
        return int(lib().fa_device_status(int(bool(reset))))
    with torch.cuda.device(device):
        return int(lib().fa_device_status(int(bool(reset))))
