"""Backward parity: dQ, dK, dV from the CUDA path (through the C ABI) against the fp64 oracle.

Small and ragged shapes: every row, every head. Mid shapes: every row of four heads. GPT-style workload
(4x32x8192x128 bf16 causal, seeded dO): dQ on 512 sampled rows of the real run; dK and dV from a second GPU
backward with dO zeroed outside the sampled rows, which makes them exactly the sampled rows' contributions
(what the oracle computes for a row subset); plus invariants of the full real-run dK/dV
(sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head).
"""
import numpy as np
import pytest
import torch

import exact_io_aware_76_b200 as fa
from exact_io_aware_76_b200.inputs import make_inputs
from exact_io_aware_76_b200.workloads import WORKLOADS, make_workload_inputs
from parity_util import all_heads, check_grad, gather_rows, oracle_bwd

pytestmark = pytest.mark.gpu


def run_bwd(q, k, v, do, causal, scale=None):
    out, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa.bwd(q, k, v, out, lse, do, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return out, lse, dq, dk, dv


def check_full(q, k, v, do, causal, heads, scale=None, chunk=8, elementwise=False):
    """Every row of ``heads``: each gradient's relative Frobenius error per head (and, with ``elementwise``,
    element by element; see parity_util.check_grad)."""
    _, _, dq, dk, dv = run_bwd(q, k, v, do, causal, scale)
    info = []
    for c0 in range(0, len(heads), chunk):
        sub = heads[c0:c0 + chunk]
        dq_r, dk_r, dv_r = oracle_bwd(q, k, v, do, causal, scale, sub)
        info.append(check_grad(gather_rows(dq, sub), dq_r, "dQ", elementwise=elementwise))
        info.append(check_grad(gather_rows(dk, sub), dk_r, "dK", elementwise=elementwise))
        info.append(check_grad(gather_rows(dv, sub), dv_r, "dV", elementwise=elementwise))
    return info


@pytest.mark.parametrize("B,Sq,Sk,H,D,causal,dtype", [
    (1, 128, 128, 2, 64, False, "f16"), (2, 512, 512, 8, 64, True, "f16"), (2, 512, 512, 8, 64, False, "f16"),
    (2, 512, 512, 4, 128, True, "bf16"), (2, 512, 512, 4, 128, False, "bf16"),
])
def test_small_full(B, Sq, Sk, H, D, causal, dtype):
    q, k, v, do = make_inputs(B, Sq, Sk, H, D, dtype, seed=500 + Sq + D, with_dout=True)
    print(check_full(q, k, v, do, causal, all_heads(B, H), elementwise=True))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("sigma", [1.0, 4.0])
def test_mid_four_heads(D, dtype, sigma):
    q, k, v, do = make_inputs(2, 2048, 2048, 16, D, dtype, seed=1002, sigma=sigma, with_dout=True)
    print(check_full(q, k, v, do, True, [(0, 0), (0, 9), (1, 4), (1, 15)]))


@pytest.mark.parametrize("B,Sq,Sk,H,D,causal", [
    (1, 1, 1, 1, 64, False), (1, 1, 1, 1, 128, True), (2, 300, 300, 3, 64, True), (2, 300, 300, 3, 128, False),
    (1, 200, 333, 2, 64, True), (1, 333, 200, 2, 128, True), (1, 257, 129, 2, 64, False), (3, 130, 700, 5, 128, True),
    (1, 5, 1000, 1, 64, True), (1, 1000, 5, 1, 128, True), (2, 191, 449, 2, 128, False), (1, 384, 384, 4, 64, True),
])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_ragged_and_degenerate(B, Sq, Sk, H, D, causal, dtype):
    q, k, v, do = make_inputs(B, Sq, Sk, H, D, dtype, seed=900 + Sq + 3 * Sk + D, with_dout=True)
    print(check_full(q, k, v, do, causal, all_heads(B, H), elementwise=True))


def test_explicit_scale():
    q, k, v, do = make_inputs(1, 256, 256, 2, 128, "bf16", seed=31, with_dout=True)
    print(check_full(q, k, v, do, True, all_heads(1, 2), scale=0.2))


@pytest.mark.parametrize("B,S,H,D,causal,scale,dtype", [
    (1, 300, 2, 128, True, -0.09, "bf16"), (2, 257, 2, 64, False, -0.125, "f16"), (1, 200, 3, 128, False, -1.0, "f16"),
])
def test_negative_scale(B, S, H, D, causal, scale, dtype):
    """Any finite softmax_scale is used as given, negative ones included (the largest s*c of a row is then c
    times its smallest score)."""
    q, k, v, do = make_inputs(B, S, S, H, D, dtype, seed=77 + S + D, with_dout=True)
    print(check_full(q, k, v, do, causal, all_heads(B, H), scale=scale, elementwise=True))


def test_gpt_workload_sampled_rows_and_invariants():
    w = WORKLOADS["gpt"]
    q, k, v, do = make_workload_inputs(w, with_dout=True)
    out, lse, dq, dk, dv = run_bwd(q, k, v, do, True)
    heads = all_heads(w.B, w.H)
    r = np.random.default_rng(4)
    # 512 sampled rows, 4 per (b, h): the first row, the last row and both sides of the first tile edge on
    # even heads; four random rows on odd heads.
    rows = np.stack([np.array([0, w.Sq - 1, 127, 128], np.int64) if t % 2 == 0
                     else np.sort(r.choice(w.Sq, 4, replace=False)).astype(np.int64) for t in range(len(heads))])
    # dK/dV contributions of the sampled rows: rerun with dO zeroed elsewhere.
    mask = torch.zeros(w.B, w.Sq, w.H, 1, dtype=do.dtype, device=do.device)
    for t, (b, h) in enumerate(heads):
        mask[b, torch.as_tensor(rows[t], device=do.device), h] = 1
    _, dk_m, dv_m = fa.bwd(q, k, v, out, lse, do * mask, causal=True)
    torch.cuda.synchronize()
    for c0 in range(0, len(heads), 16):
        sub = heads[c0:c0 + 16]
        dq_r, dk_r, dv_r = oracle_bwd(q, k, v, do, True, None, sub, rows[c0:c0 + 16])
        check_grad(gather_rows(dq, sub, rows[c0:c0 + 16]), dq_r, "dQ sampled rows", per_head=False)
        check_grad(gather_rows(dk_m, sub), dk_r, "dK of sampled rows", per_head=False)
        check_grad(gather_rows(dv_m, sub), dv_r, "dV of sampled rows", per_head=False)
    # Invariants of the real run over every key: sum_j dK_j = 0, sum_j dV_j = sum_i dO_i (per head).
    sdk = dk.double().sum(dim=1)
    adk = dk.double().abs().sum(dim=1)
    assert (sdk.abs() <= 1e-2 * adk + 1e-3).all(), float((sdk.abs() / (adk + 1e-30)).max())
    sdv = dv.double().sum(dim=1)
    sdo = do.double().sum(dim=1)
    adv = dv.double().abs().sum(dim=1)
    assert ((sdv - sdo).abs() <= 1e-2 * adv + 1e-2).all(), float(((sdv - sdo).abs() / (adv + 1e-30)).max())
