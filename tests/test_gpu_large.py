"""Tensors of 2^32 elements (B=512, S=512, H=128, D=128 bf16 causal: 8.6 GB per tensor, a 17 GB fp32 dQ
accumulator), so that element offsets pass 2^31: every global index in the kernels is 64-bit. Forward O/LSE and
backward dQ/dK/dV of whole heads at the start, in the middle and at the very end of the tensors are compared
with the oracle. About 100 GB of device memory at the peak."""
import numpy as np
import pytest
import torch

import exact_io_aware_76_b200 as fa
from exact_io_aware_76_b200.inputs import make_inputs
from parity_util import check_grad, check_lse, check_out, gather_lse, gather_rows, oracle_bwd, oracle_fwd

pytestmark = pytest.mark.gpu


def test_more_than_2_31_elements_per_tensor():
    B, S, H, D = 512, 512, 128, 128
    assert B * S * H * D == 2 ** 32
    q, k, v, do = make_inputs(B, S, S, H, D, "bf16", 4242, device="cuda", with_dout=True)
    out, lse = fa.fwd(q, k, v, causal=True)
    dq, dk, dv = fa.bwd(q, k, v, out, lse, do, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    heads = [(0, 0), (257, 64), (B - 1, H - 1)]
    o_ref, l_ref = oracle_fwd(q, k, v, True, None, heads)
    print(check_out(gather_rows(out, heads), o_ref, q.dtype), check_lse(gather_lse(lse, heads), l_ref))
    dq_r, dk_r, dv_r = oracle_bwd(q, k, v, do, True, None, heads)
    print(check_grad(gather_rows(dq, heads), dq_r, "dQ"), check_grad(gather_rows(dk, heads), dk_r, "dK"),
          check_grad(gather_rows(dv, heads), dv_r, "dV"))
    del q, k, v, do, out, lse, dq, dk, dv
    torch.cuda.empty_cache()
