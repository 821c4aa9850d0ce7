"""Grouped/multi-query K/V heads and the sliding window (skill page, Workflow 2 Steps 2-3) on the GPU, through
the C ABI (fa_fwd_ex / fa_bwd_ex), against the oracle's grouped-head and windowed path."""
import pytest
import torch

import exact_io_aware_76_b200 as fa
from exact_io_aware_76_b200.inputs import draw
from parity_util import (all_heads, check_grad, check_lse, check_out, gather_lse, gather_rows, heads_f64,
                         oracle_bwd_grouped, oracle_fwd)

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


CASES = [
    # B, Sq, Sk, H, Hkv, D, causal, window, dtype
    (2, 384, 384, 8, 2, 128, True, (-1, -1), "bf16"),       # GQA, group 4
    (1, 300, 500, 4, 1, 64, False, (-1, -1), "f16"),        # MQA, Sq != Sk
    (1, 1000, 1000, 2, 2, 64, True, (256, 0), "bf16"),      # causal sliding window
    (1, 700, 700, 2, 2, 128, False, (256, 256), "f16"),     # symmetric window (the skill page's example)
    (2, 333, 517, 4, 2, 128, False, (5, 3), "bf16"),        # tiny window, ragged, Sq != Sk
    (1, 517, 333, 2, 1, 64, True, (100, -1), "f16"),        # left bound only, rows without keys
    (1, 400, 400, 2, 2, 128, False, (-1, 40), "bf16"),      # right bound only
    (2, 640, 640, 6, 3, 128, True, (300, 0), "bf16"),       # GQA + window
    (1, 1000, 1000, 4, 2, 64, True, (256, 256), "bf16"),    # the skill page's call as written: causal + (256, 256)
    (1, 517, 700, 2, 2, 128, True, (100, 50), "f16"),       # causal with a positive right bound (capped at 0)
]


@pytest.mark.parametrize("B,Sq,Sk,H,Hkv,D,causal,window,dtype", CASES)
def test_forward(B, Sq, Sk, H, Hkv, D, causal, window, dtype):
    q, k, v, _ = make(B, Sq, Sk, H, Hkv, D, dtype, 4000 + Sq + Hkv)
    out, lse = fa.fwd(q, k, v, causal=causal, window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    heads = all_heads(B, H)
    o_ref, l_ref = oracle_fwd(q, k, v, causal, None, heads, window=window)
    print(check_out(gather_rows(out, heads), o_ref, q.dtype), check_lse(gather_lse(lse, heads), l_ref))


@pytest.mark.parametrize("B,Sq,Sk,H,Hkv,D,causal,window,dtype", CASES)
def test_backward(B, Sq, Sk, H, Hkv, D, causal, window, dtype):
    q, k, v, do = make(B, Sq, Sk, H, Hkv, D, dtype, 5000 + Sq + Hkv)
    out, lse = fa.fwd(q, k, v, causal=causal, window=window)
    dq, dk, dv = fa.bwd(q, k, v, out, lse, do, causal=causal, window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    group = H // Hkv
    for b in range(B):
        for h_kv in range(Hkv):
            dq_r, dk_r, dv_r = oracle_bwd_grouped(q, k, v, do, causal, None, b, h_kv, window=window)
            qh = [(b, h_kv * group + g) for g in range(group)]
            check_grad(heads_f64(dq, qh), dq_r, "dQ")
            check_grad(heads_f64(dk, [(b, h_kv)]), dk_r, "dK")
            check_grad(heads_f64(dv, [(b, h_kv)]), dv_r, "dV")


def test_ex_entry_points_reject_bad_groups():
    t = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    L = fa.lib()
    assert L.fa_fwd_ex(p, p, p, p, p, 1, 128, 128, 6, 4, 64, 0, -1, -1, 0.0, 1, None) == -1
    assert L.fa_fwd_ex(p, p, p, p, p, 1, 128, 128, 6, 0, 64, 0, -1, -1, 0.0, 1, None) == -1


def test_several_key_tiles_per_cta():
    """A shape large enough that the head-dim-128 backward gives each CTA two key tiles (32 K/V heads x 64 key
    tiles: 1024 CTAs, about seven full waves), with grouped heads, Sq != Sk and a causal window that leaves the
    first twelve key tiles without any query, so that CTAs also meet key tiles with nothing to do; dQ/dK/dV of
    two whole K/V head groups against the oracle, and exact zeros for the keys no query sees."""
    B, Sq, Sk, H, Hkv, D, window = 1, 6144, 8192, 64, 32, 128, (512, 0)
    q, k, v, do = make(B, Sq, Sk, H, Hkv, D, "bf16", 6001)
    out, lse = fa.fwd(q, k, v, causal=True, window=window)
    dq, dk, dv = fa.bwd(q, k, v, out, lse, do, causal=True, window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    unseen = Sk - Sq - window[0]  # key j is seen by rows r <= j - (Sk - Sq) + left
    assert dk[:, :unseen].abs().max().item() == 0 and dv[:, :unseen].abs().max().item() == 0
    assert dk[:, unseen:].abs().max().item() > 0
    group = H // Hkv
    for h_kv in (0, Hkv - 1):
        dq_r, dk_r, dv_r = oracle_bwd_grouped(q, k, v, do, True, None, 0, h_kv, window=window)
        qh = [(0, h_kv * group + g) for g in range(group)]
        check_grad(heads_f64(dq, qh), dq_r, "dQ")
        check_grad(heads_f64(dk, [(0, h_kv)]), dk_r, "dK")
        check_grad(heads_f64(dv, [(0, h_kv)]), dv_r, "dV")
