"""The usage shown for callers of the pages' flash_attn_func (forward, backward, grouped K/V heads with a
window, dropout, e4m3), at small sizes: every call returns, the outputs are finite, and the variants agree with
the plain forward where they should."""
import pytest
import torch

import exact_io_aware_76_b200 as fa

pytestmark = pytest.mark.gpu


def test_usage_example():
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    q = torch.randn(2, 1024, 8, 128, device="cuda", dtype=torch.bfloat16, generator=g)
    k, v = (torch.randn(q.shape, device="cuda", dtype=torch.bfloat16, generator=g) for _ in range(2))
    out, lse = fa.fwd(q, k, v, causal=True)
    dq, dk, dv = fa.bwd(q, k, v, out, lse, torch.randn_like(q), causal=True)
    kg, vg = (torch.randn(2, 1024, 2, 128, device="cuda", dtype=torch.bfloat16, generator=g) for _ in range(2))
    out_g, _ = fa.fwd(q, kg, vg, causal=True, window=(256, 0))
    out_d0, lse_d0 = fa.fwd(q, k, v, causal=True, dropout_p=0.0, seed=1234, offset=0)
    out_d, lse_d = fa.fwd(q, k, v, causal=True, dropout_p=0.1, seed=1234, offset=0)
    out8, lse8 = fa.fwd_fp8(*(t.to(torch.float8_e4m3fn) for t in (q, k, v)), causal=True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for t in (out, lse, dq, dk, dv, out_g, out_d, lse_d, out8, lse8):
        assert torch.isfinite(t.float()).all()
    assert torch.equal(out_d0, out) and torch.equal(lse_d0, lse)   # dropout_p = 0 is the plain forward
    # dropout leaves the LSE unchanged (up to the order of the fp32 row sum, which the dropout loop forms in
    # groups of 16 keys)
    assert (lse_d - lse).abs().max() <= 1e-5
    assert (out_d.float() - out.float()).abs().max() > 0            # but not the output
    assert (lse8 - lse).abs().max() < 0.5                           # e4m3 inputs: the same scores, rounded
