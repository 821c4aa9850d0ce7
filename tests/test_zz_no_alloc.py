"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory (a caller inside a framework
that owns all device memory, or one that cannot afford the synchronisation cudaMalloc may cause). It uses a
fixed scratch array inside the library instead of a caller workspace. Checked through the C ABI against
fa_bwd with a caller-owned workspace (dK and dV bit for bit, dQ up to the order of its fp32 reductions) and
against the fp64 oracle, on two calls in a row with different problems, so that the second call also proves
that stale scratch contents from the first one are cleared.

This file is named to be collected last: the scratch is shared by every call in the process, so it must pass
both alone in a fresh process and after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_io_aware_76_b200 as fa
from exact_io_aware_76_b200.inputs import make_inputs
from parity_util import all_heads, check_grad, gather_rows, half_ulp, heads_f64, oracle_bwd

SCRATCH_BYTES = 64 << 20


def _noalloc(q, k, v, out, lse, do, causal):
    L = fa.lib()
    L.fa_bwd_noalloc.restype = ctypes.c_int
    L.fa_bwd_noalloc.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_int,
                                                                               ctypes.c_void_p]
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = L.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), do.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Sq, Sk, H, D, int(causal), 0.0,
                          1 if q.dtype == torch.bfloat16 else 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, dq, dk, dv


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_twice():
    # bigger problem first, then a smaller one: the second call finds the first one's contents in the scratch
    problems = [(2, 1000, 1000, 4, 128, "bf16", True, 71), (1, 700, 900, 6, 64, "f16", False, 72)]
    for (B, Sq, Sk, H, D, dt, causal, seed) in problems:
        assert fa.workspace_size(B, Sq, H, D) <= SCRATCH_BYTES
        q, k, v, do = make_inputs(B, Sq, Sk, H, D, dt, seed=seed, with_dout=True)
        out, lse = fa.fwd(q, k, v, causal=causal)
        ref = fa.bwd(q, k, v, out, lse, do, causal=causal)
        rc, dq, dk, dv = _noalloc(q, k, v, out, lse, do, causal)
        torch.cuda.synchronize()
        assert rc == 0, fa.status_string(rc)
        assert fa.device_status() == 0
        # The same kernels on the same inputs: dK and dV accumulate in a fixed order (bit for bit equal); dQ's
        # fp32 reductions may land in another order, so it may differ by rounding only.
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
        a, b = dq.double().cpu().numpy(), ref[0].double().cpu().numpy()
        assert np.all(np.abs(a - b) <= 2 * half_ulp(b, q.dtype))  # at most one output ulp apart
        check_grad(heads_f64(dq, all_heads(B, H)), heads_f64(ref[0], all_heads(B, H)), "dQ vs fa_bwd", rtol=1e-3)
        # and both against the oracle, head by head and element by element
        heads = all_heads(B, H)
        dq_r, dk_r, dv_r = oracle_bwd(q, k, v, do, causal, None, heads)
        print(check_grad(gather_rows(dq, heads), dq_r, "dQ", elementwise=True),
              check_grad(gather_rows(dk, heads), dk_r, "dK", elementwise=True),
              check_grad(gather_rows(dv, heads), dv_r, "dV", elementwise=True))


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_the_scratch():
    B, S, H, D = 1, 8192, 32, 128
    assert fa.workspace_size(B, S, H, D) > SCRATCH_BYTES
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    L = fa.lib()
    L.fa_bwd_noalloc.restype = ctypes.c_int
    L.fa_bwd_noalloc.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_int,
                                                                               ctypes.c_void_p]
    p = t.data_ptr()
    rc = L.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, S, S, H, D, 1, 0.0, 1, None)
    assert rc == -5
