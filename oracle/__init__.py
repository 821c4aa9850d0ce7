"""fp64 CPU oracle for exact scaled dot-product attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and ``--impl reference``
legs) may import this package. The product library (``exact_io_aware_76_b200``) never imports it, and this
package imports nothing from the product.

What it computes is the plain definition of standard attention written out in fp64 (page "Flash Attention —
長い系列を扱う Transformer の学習と推論を速くする", Workflow 1 Step 2: ``softmax(q @ k^T / sqrt(d_k)) @ v``),
with the causal flag of the same page's quick start, and the chain-rule backward. The C source
``fa_oracle.c`` documents each step and the readings taken where the pages are silent.

Array convention (numpy, float64, C-contiguous), one entry per attention head:
    q, dout: [n_q_heads, Sq, D]    k, v: [n_kv_heads, Sk, D]   (q head h reads K/V head h // (n_q / n_kv))
    rows:    [n_q_heads, n_rows] int64 query rows to evaluate (default: all rows)
    window:  (left, right) sliding window around the key aligned with each query; -1 = unbounded side
    dropout: (dropout_p, seed, offset) attention dropout with a Philox4x32-10 mask (None = no dropout);
             head_index[h] is listed head h's head number b * H + h in the mask's counter (default: h)
Outputs:
    fwd -> out [n_q_heads, n_rows, D], lse [n_q_heads, n_rows]   (natural-log LSE, scale included)
    bwd -> dq [n_q_heads, n_rows, D], dk/dv [n_kv_heads, Sk, D] (contributions of the listed rows, summed
           over each group of q heads)

Parity: pinned by tests/test_oracle_pins.py (closed forms, invariants, finite differences, hand-worked
examples under tests/golden/, and a float64 PyTorch SDPA cross-check on tiny shapes).
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_F64P = ctypes.POINTER(ctypes.c_double)
_I64P = ctypes.POINTER(ctypes.c_int64)


def default_scale(D):
    """``softmax_scale=None`` means 1/sqrt(head_dim) (skill page, Workflow 2 Step 2, "Auto-scale")."""
    return 1.0 / math.sqrt(D)


class Oracle:
    """ctypes handle on one compiled oracle library (the default one, or a test's modified copy)."""

    def __init__(self, libpath=None):
        if libpath is None:
            libpath = _build.ensure_built()
        self.libpath = libpath
        lib = ctypes.CDLL(libpath)
        lib.oracle_attn_fwd.restype = ctypes.c_int
        i64 = ctypes.c_int64
        lib.oracle_attn_fwd.argtypes = [_F64P, _F64P, _F64P, i64, i64, i64, i64, i64, ctypes.c_int, i64, i64,
                                        ctypes.c_double, _I64P, i64, _F64P, _F64P]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [_F64P, _F64P, _F64P, _F64P, i64, i64, i64, i64, i64, ctypes.c_int, i64,
                                        i64, ctypes.c_double, _I64P, i64, _F64P, _F64P, _F64P]
        u32, u64, dbl = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double
        lib.oracle_attn_fwd_dropout.restype = ctypes.c_int
        lib.oracle_attn_fwd_dropout.argtypes = [_F64P, _F64P, _F64P, i64, i64, i64, i64, i64, ctypes.c_int, i64, i64,
                                                dbl, dbl, u64, u32, _I64P, _I64P, i64, _F64P, _F64P]
        lib.oracle_attn_bwd_dropout.restype = ctypes.c_int
        lib.oracle_attn_bwd_dropout.argtypes = [_F64P, _F64P, _F64P, _F64P, i64, i64, i64, i64, i64, ctypes.c_int,
                                                i64, i64, dbl, dbl, u64, u32, _I64P, _I64P, i64, _F64P, _F64P,
                                                _F64P]
        lib.oracle_philox4x32_10.restype = None
        lib.oracle_philox4x32_10.argtypes = [ctypes.POINTER(u32), ctypes.POINTER(u32), ctypes.POINTER(u32)]
        lib.oracle_dropout_mask.restype = ctypes.c_int
        lib.oracle_dropout_mask.argtypes = [dbl, u64, u32, i64, i64, i64, ctypes.POINTER(ctypes.c_uint8)]
        lib.oracle_set_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        self.lib = lib

    def set_threads(self, n):
        """Use n OpenMP threads from the calling thread on (n < 1: unchanged); returns the count in effect."""
        return int(self.lib.oracle_set_threads(int(n)))

    @staticmethod
    def _prep(q, k, v, rows):
        q = np.ascontiguousarray(q, dtype=np.float64)
        k = np.ascontiguousarray(k, dtype=np.float64)
        v = np.ascontiguousarray(v, dtype=np.float64)
        if (q.ndim != 3 or k.ndim != 3 or v.shape != k.shape or q.shape[0] % k.shape[0] != 0
                or q.shape[2] != k.shape[2]):
            raise ValueError("expected q [n_q_heads,Sq,D], k/v [n_kv_heads,Sk,D] with n_kv_heads dividing n_q_heads")
        nh, Sq, D = q.shape
        if rows is None:
            rows = np.broadcast_to(np.arange(Sq, dtype=np.int64), (nh, Sq))
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        if rows.ndim == 1:
            rows = np.ascontiguousarray(np.broadcast_to(rows, (nh, rows.shape[0])))
        if rows.shape[0] != nh:
            raise ValueError("rows must be [n_heads, n_rows]")
        return q, k, v, rows

    @staticmethod
    def _heads(head_index, nh):
        if head_index is None:
            head_index = np.arange(nh, dtype=np.int64)
        head_index = np.ascontiguousarray(head_index, dtype=np.int64)
        if head_index.shape != (nh,):
            raise ValueError("head_index must have one entry per q head")
        return head_index

    def philox4x32_10(self, ctr, key):
        """Philox4x32-10 of one 4-word counter under a 2-word key (both unsigned 32-bit words)."""
        c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
        kk = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
        out = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(c, kk, out)
        return [int(x) for x in out]

    def dropout_mask(self, dropout_p, seed, offset, bh, Sq, Sk):
        """Keep mask (bool [Sq, Sk]) of head number bh."""
        keep = np.zeros((Sq, Sk), np.uint8)
        rc = self.lib.oracle_dropout_mask(float(dropout_p), int(seed), int(offset), int(bh), int(Sq), int(Sk),
                                          keep.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
        if rc != 0:
            raise ValueError("oracle_dropout_mask rejected its arguments")
        return keep.astype(bool)

    def fwd(self, q, k, v, causal=False, scale=None, rows=None, window=(-1, -1), dropout=None, head_index=None):
        q, k, v, rows = self._prep(q, k, v, rows)
        nh, Sq, D = q.shape
        nkv, Sk = k.shape[0], k.shape[1]
        if scale is None:
            scale = default_scale(D)
        nr = rows.shape[1]
        out = np.zeros((nh, nr, D), np.float64)
        lse = np.zeros((nh, nr), np.float64)
        if dropout is None:
            rc = self.lib.oracle_attn_fwd(q.ctypes.data_as(_F64P), k.ctypes.data_as(_F64P),
                                          v.ctypes.data_as(_F64P), nh, nkv, Sq, Sk, D, int(bool(causal)),
                                          int(window[0]), int(window[1]), float(scale),
                                          rows.ctypes.data_as(_I64P), nr, out.ctypes.data_as(_F64P),
                                          lse.ctypes.data_as(_F64P))
        else:
            hi = self._heads(head_index, nh)
            rc = self.lib.oracle_attn_fwd_dropout(q.ctypes.data_as(_F64P), k.ctypes.data_as(_F64P),
                                                  v.ctypes.data_as(_F64P), nh, nkv, Sq, Sk, D, int(bool(causal)),
                                                  int(window[0]), int(window[1]), float(scale),
                                                  float(dropout[0]), int(dropout[1]), int(dropout[2]),
                                                  hi.ctypes.data_as(_I64P), rows.ctypes.data_as(_I64P), nr,
                                                  out.ctypes.data_as(_F64P), lse.ctypes.data_as(_F64P))
        if rc != 0:
            raise ValueError("oracle_attn_fwd rejected its arguments")
        return out, lse

    def bwd(self, q, k, v, dout, causal=False, scale=None, rows=None, window=(-1, -1), dropout=None,
            head_index=None):
        q, k, v, rows = self._prep(q, k, v, rows)
        dout = np.ascontiguousarray(dout, dtype=np.float64)
        if dout.shape != q.shape:
            raise ValueError("dout must have q's shape")
        nh, Sq, D = q.shape
        nkv, Sk = k.shape[0], k.shape[1]
        if scale is None:
            scale = default_scale(D)
        nr = rows.shape[1]
        dq = np.zeros((nh, nr, D), np.float64)
        dk = np.zeros((nkv, Sk, D), np.float64)
        dv = np.zeros((nkv, Sk, D), np.float64)
        if dropout is None:
            rc = self.lib.oracle_attn_bwd(q.ctypes.data_as(_F64P), k.ctypes.data_as(_F64P),
                                          v.ctypes.data_as(_F64P), dout.ctypes.data_as(_F64P), nh, nkv, Sq, Sk, D,
                                          int(bool(causal)), int(window[0]), int(window[1]), float(scale),
                                          rows.ctypes.data_as(_I64P), nr, dq.ctypes.data_as(_F64P),
                                          dk.ctypes.data_as(_F64P), dv.ctypes.data_as(_F64P))
        else:
            hi = self._heads(head_index, nh)
            rc = self.lib.oracle_attn_bwd_dropout(q.ctypes.data_as(_F64P), k.ctypes.data_as(_F64P),
                                                  v.ctypes.data_as(_F64P), dout.ctypes.data_as(_F64P), nh, nkv, Sq,
                                                  Sk, D, int(bool(causal)), int(window[0]), int(window[1]),
                                                  float(scale), float(dropout[0]), int(dropout[1]),
                                                  int(dropout[2]), hi.ctypes.data_as(_I64P),
                                                  rows.ctypes.data_as(_I64P), nr, dq.ctypes.data_as(_F64P),
                                                  dk.ctypes.data_as(_F64P), dv.ctypes.data_as(_F64P))
        if rc != 0:
            raise ValueError("oracle_attn_bwd rejected its arguments")
        return dq, dk, dv


_default = None


def _get():
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def attn_fwd(q, k, v, causal=False, scale=None, rows=None, window=(-1, -1), dropout=None, head_index=None):
    """O and LSE of the listed query rows (all rows by default). See the module docstring for layouts."""
    return _get().fwd(q, k, v, causal=causal, scale=scale, rows=rows, window=window, dropout=dropout,
                      head_index=head_index)


def attn_bwd(q, k, v, dout, causal=False, scale=None, rows=None, window=(-1, -1), dropout=None, head_index=None):
    """dQ of the listed rows and their dK/dV contributions. See the module docstring for layouts."""
    return _get().bwd(q, k, v, dout, causal=causal, scale=scale, rows=rows, window=window, dropout=dropout,
                      head_index=head_index)


def philox4x32_10(ctr, key):
    return _get().philox4x32_10(ctr, key)


def set_threads(n):
    return _get().set_threads(n)


def dropout_mask(dropout_p, seed, offset, bh, Sq, Sk):
    return _get().dropout_mask(dropout_p, seed, offset, bh, Sq, Sk)


def bshd_heads(x, b, h):
    """Slice one head of a [B, S, H, D] CPU tensor/array into a float64 [S, D] array (exact upcast)."""
    a = x[b, :, h, :]
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)
