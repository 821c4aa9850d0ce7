"""Attention dropout (the dropout_p argument of the skill page's flash_attn_func call) on the GPU, through the C
ABI (fa_fwd_dropout / fa_bwd_dropout), against the oracle's Philox4x32-10 mask.

* The mask itself is compared exactly: with Sk = D and V = I the output row is P o Z, so its zero pattern is the
  dropped (or invisible) set, element by element, and its values are P / (1 - t/256).
* O, LSE and dQ/dK/dV are compared with the bounds of the plain path (tests/parity_util.py), the O bound scaled
  by 1/(1 - t/256) because every kept probability is.
* dropout_p = 0 is the plain kernel, bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_76_b200 as fa
import oracle
from exact_io_aware_76_b200.inputs import draw
from exact_io_aware_76_b200.workloads import WORKLOADS, make_workload_inputs
from parity_util import (all_heads, check_grad, check_lse, check_out, gather_lse, gather_rows, heads_f64, kv_heads)

pytestmark = pytest.mark.gpu


def make(B, Sq, Sk, H, Hkv, D, dtype, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    dt = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    q = draw((B, Sq, H, D), dt, g, "cuda")
    k = draw((B, Sk, Hkv, D), dt, g, "cuda")
    v = draw((B, Sk, Hkv, D), dt, g, "cuda")
    do = draw((B, Sq, H, D), dt, g, "cuda")
    return q, k, v, do


def rescale(p):
    return 1.0 / (1.0 - math.floor(256 * p + 0.5) / 256)


def head_numbers(heads, H):
    return np.array([b * H + h for (b, h) in heads], np.int64)


@pytest.mark.parametrize("causal,p,seed,offset", [(False, 0.1, 1, 0), (True, 0.5, 0xDEADBEEF12345678, 7),
                                                  (False, 0.9, 42, 0xFFFFFFFF)])
def test_mask_is_exact(causal, p, seed, offset):
    B, Sq, Sk, H, D = 2, 200, 128, 3, 128
    g = torch.Generator(device="cuda")
    g.manual_seed(91)
    q = draw((B, Sq, H, D), torch.bfloat16, g, "cuda")
    k = draw((B, Sk, H, D), torch.bfloat16, g, "cuda")
    v = torch.eye(Sk, dtype=torch.bfloat16, device="cuda")[None, :, None, :].expand(B, Sk, H, D).contiguous()
    out, lse = fa.fwd(q, k, v, causal=causal, dropout_p=p, seed=seed, offset=offset)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    heads = all_heads(B, H)
    o = gather_rows(out, heads)
    P, _ = oracle.attn_fwd(heads_f64(q, heads), heads_f64(k, heads), heads_f64(v, heads), causal=causal)
    for t, (b, h) in enumerate(heads):
        keep = oracle.dropout_mask(p, seed, offset, b * H + h, Sq, Sk)
        expect_nonzero = keep & (P[t] > 0)
        got_nonzero = o[t] != 0
        bad = np.argwhere(expect_nonzero != got_nonzero)
        assert bad.size == 0, "head %d: %d mask mismatches, first (row, key) %s" % (t, len(bad), bad[:4].tolist())
    o_ref = P * np.stack([oracle.dropout_mask(p, seed, offset, b * H + h, Sq, Sk) for (b, h) in heads]) * rescale(p)
    print(check_out(o, o_ref, torch.bfloat16, sigma=rescale(p)))


CASES = [
    # B, Sq, Sk, H, Hkv, D, causal, window, dtype, p
    (1, 256, 256, 2, 2, 128, False, (-1, -1), "bf16", 0.1),
    (2, 333, 517, 4, 2, 128, True, (-1, -1), "bf16", 0.25),
    (1, 300, 300, 2, 1, 64, True, (-1, -1), "f16", 0.5),
    (2, 200, 129, 3, 3, 64, False, (-1, -1), "bf16", 0.2),
    (1, 640, 640, 4, 2, 128, True, (200, 0), "f16", 0.15),
    (1, 1, 1, 1, 1, 128, False, (-1, -1), "bf16", 0.5),          # one query, one key
    (1, 129, 1, 2, 2, 128, True, (-1, -1), "f16", 0.2),          # one key: rows 0..127 see none
    (1, 517, 333, 2, 1, 64, True, (100, -1), "bf16", 0.3),       # MQA, left bound, rows without keys
    (2, 384, 384, 8, 1, 128, True, (-1, -1), "bf16", 0.1),       # MQA, group 8: the backward walks 8 heads
    (1, 256, 300, 2, 2, 64, False, (-1, -1), "f16", 0.9),        # t = 230: scale 1/(1 - 230/256)
]


@pytest.mark.parametrize("B,Sq,Sk,H,Hkv,D,causal,window,dtype,p", CASES)
def test_forward(B, Sq, Sk, H, Hkv, D, causal, window, dtype, p):
    q, k, v, _ = make(B, Sq, Sk, H, Hkv, D, dtype, 8000 + Sq)
    seed, offset = 1000 + Sk, 3
    out, lse = fa.fwd(q, k, v, causal=causal, window=window, dropout_p=p, seed=seed, offset=offset)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    heads = all_heads(B, H)
    kv = kv_heads(q, k, heads)
    o_ref, l_ref = oracle.attn_fwd(heads_f64(q, heads), heads_f64(k, kv), heads_f64(v, kv), causal=causal,
                                   window=window, dropout=(p, seed, offset), head_index=head_numbers(heads, H))
    print(check_out(gather_rows(out, heads), o_ref, q.dtype, sigma=rescale(p)),
          check_lse(gather_lse(lse, heads), l_ref))


@pytest.mark.parametrize("B,Sq,Sk,H,Hkv,D,causal,window,dtype,p", CASES)
def test_backward(B, Sq, Sk, H, Hkv, D, causal, window, dtype, p):
    q, k, v, do = make(B, Sq, Sk, H, Hkv, D, dtype, 9000 + Sq)
    seed, offset = 77 + Sq, 11
    kw = dict(causal=causal, window=window, dropout_p=p, seed=seed, offset=offset)
    out, lse = fa.fwd(q, k, v, **kw)
    dq, dk, dv = fa.bwd(q, k, v, out, lse, do, **kw)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    group = H // Hkv
    for b in range(B):
        for h_kv in range(Hkv):
            qh = [(b, h_kv * group + g) for g in range(group)]
            dq_r, dk_r, dv_r = oracle.attn_bwd(heads_f64(q, qh), heads_f64(k, [(b, h_kv)]), heads_f64(v, [(b, h_kv)]),
                                               heads_f64(do, qh), causal=causal, window=window,
                                               dropout=(p, seed, offset), head_index=head_numbers(qh, H))
            check_grad(heads_f64(dq, qh), dq_r, "dQ")
            check_grad(heads_f64(dk, [(b, h_kv)]), dk_r, "dK")
            check_grad(heads_f64(dv, [(b, h_kv)]), dv_r, "dV")


def test_zero_probability_is_the_plain_kernel():
    q, k, v, do = make(1, 300, 300, 2, 2, 128, "bf16", 8500)
    L = fa.lib()
    o1, l1 = fa.fwd(q, k, v, causal=True)
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    rc = L.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(), 1, 300, 300, 2, 2,
                          128, 1, -1, -1, 0.0, 1, 0.0, 5, 0, None)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_gpt_workload_sampled_rows():
    """The GPT-shaped workload (4x32x8192x128 bf16 causal) with dropout 0.1: O and LSE on 4 sampled rows of every
    head; dQ of those rows and their dK/dV contributions (a second backward with dO zeroed on every other row,
    which removes exactly the other rows' terms)."""
    w = WORKLOADS["gpt"]
    q, k, v, do = make_workload_inputs(w, with_dout=True)
    p, seed, offset = 0.1, 20240601, 17
    kw = dict(causal=True, dropout_p=p, seed=seed, offset=offset)
    out, lse = fa.fwd(q, k, v, **kw)
    heads = all_heads(w.B, w.H)
    r = np.random.default_rng(5)
    rows = np.stack([np.array([0, w.Sq - 1, 127, 128], np.int64) if t % 2 == 0
                     else np.sort(r.choice(w.Sq, 4, replace=False)).astype(np.int64) for t in range(len(heads))])
    mask = torch.zeros(w.B, w.Sq, w.H, 1, dtype=do.dtype, device=do.device)
    for t, (b, h) in enumerate(heads):
        mask[b, torch.as_tensor(rows[t], device=do.device), h] = 1
    dq, _, _ = fa.bwd(q, k, v, out, lse, do, **kw)
    _, dk_m, dv_m = fa.bwd(q, k, v, out, lse, do * mask, **kw)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for c0 in range(0, len(heads), 16):
        sub = heads[c0:c0 + 16]
        sr = rows[c0:c0 + 16]
        hi = head_numbers(sub, w.H)
        args = (heads_f64(q, sub), heads_f64(k, sub), heads_f64(v, sub))
        o_ref, l_ref = oracle.attn_fwd(*args, causal=True, rows=sr, dropout=(p, seed, offset), head_index=hi)
        check_out(gather_rows(out, sub, sr), o_ref, q.dtype, sigma=rescale(p))
        check_lse(gather_lse(lse, sub, sr), l_ref)
        dq_r, dk_r, dv_r = oracle.attn_bwd(*args, heads_f64(do, sub), causal=True, rows=sr,
                                           dropout=(p, seed, offset), head_index=hi)
        check_grad(gather_rows(dq, sub, sr), dq_r, "dQ sampled rows", per_head=False)
        check_grad(gather_rows(dk_m, sub), dk_r, "dK of sampled rows", per_head=False)
        check_grad(gather_rows(dv_m, sub), dv_r, "dV of sampled rows", per_head=False)
