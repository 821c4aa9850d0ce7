"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Small workloads are compared element by element over every row; the GPT-style (4x32x8192x128) and long-context
(1x32x131072x128) workloads on sampled rows (first row, last row, both sides of a tile edge, random rows),
which the oracle computes one by one. Ragged and degenerate shapes cover partial tiles, Sq != Sk causal
alignment, fully masked rows and single keys.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_76_b200 as fa
from exact_io_aware_76_b200.inputs import make_inputs
from exact_io_aware_76_b200.workloads import WORKLOADS, make_workload_inputs
from parity_util import all_heads, check_lse, check_out, gather_lse, gather_rows, oracle_fwd

pytestmark = pytest.mark.gpu


def run_and_check(q, k, v, causal, scale, sigma, heads=None, rows=None, chunk=16):
    """Run the CUDA forward once, then compare ``heads`` (rows ``rows``) with the oracle, ``chunk`` heads at a
    time so that the fp64 host copies stay small."""
    B, Sq, H, D = q.shape
    out, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    heads = heads or all_heads(B, H)
    info = []
    for c0 in range(0, len(heads), chunk):
        sub = heads[c0:c0 + chunk]
        sub_rows = None if rows is None else rows[c0:c0 + chunk]
        o_ref, l_ref = oracle_fwd(q, k, v, causal, scale, sub, sub_rows)
        info.append(check_out(gather_rows(out, sub, sub_rows), o_ref, q.dtype, sigma))
        info.append(check_lse(gather_lse(lse, sub, sub_rows), l_ref))
    return info


def sampled_rows(S, heads, per_head, seed):
    """Rows 0 and S-1, both sides of the first 128-row tile edge, and random rows, per head."""
    r = np.random.default_rng(seed)
    base = [0, S - 1, min(127, S - 1), min(128, S - 1)]
    rows = []
    for _ in heads:
        extra = r.choice(S, size=max(0, per_head - len(base)), replace=False)
        rows.append(np.array((base + list(extra))[:per_head], dtype=np.int64))
    return np.stack(rows)


@pytest.mark.parametrize("name", ["tiny", "small_causal", "small_noncausal"])
def test_small_workloads_full(name):
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    print(run_and_check(q, k, v, w.causal, None, w.sigma))


@pytest.mark.parametrize("name", sorted(n for n in WORKLOADS if n.startswith("mid_")))
def test_mid_workloads(name):
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    heads = [(0, 0), (0, 7), (1, 3), (1, 15)]  # full rows of 4 heads; every head's rows via the sampled test below
    print(run_and_check(q, k, v, w.causal, None, w.sigma, heads=heads))
    hs = all_heads(w.B, w.H)
    print(run_and_check(q, k, v, w.causal, None, w.sigma, heads=hs, rows=sampled_rows(w.Sq, hs, 6, 5)))


@pytest.mark.parametrize("B,Sq,Sk,H,D,causal", [
    (1, 1, 1, 1, 64, False), (1, 1, 1, 1, 128, True), (2, 300, 300, 3, 64, True), (2, 300, 300, 3, 128, False),
    (1, 200, 333, 2, 64, True), (1, 333, 200, 2, 128, True), (1, 257, 129, 2, 64, False), (3, 130, 700, 5, 128, True),
    (1, 5, 1000, 1, 64, True), (1, 1000, 5, 1, 128, True), (2, 511, 513, 2, 64, False), (1, 384, 384, 4, 128, True),
])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_ragged_and_degenerate(B, Sq, Sk, H, D, causal, dtype):
    q, k, v = make_inputs(B, Sq, Sk, H, D, dtype, seed=11 + Sq + 7 * Sk + D)
    print(run_and_check(q, k, v, causal, None, 1.0))


@pytest.mark.parametrize("scale", [0.05, 0.3, -0.05, -0.3])
def test_explicit_scale(scale):
    q, k, v = make_inputs(1, 256, 256, 2, 64, "bf16", seed=3)
    print(run_and_check(q, k, v, True, scale, 1.0))


@pytest.mark.parametrize("B,Sq,Sk,H,D,causal,scale,dtype", [
    (1, 333, 200, 2, 128, True, -0.088, torch.bfloat16),   # rows without keys under a negative scale
    (2, 300, 517, 3, 64, False, -1.5, torch.float16),     # large negative scale: exponents far below the max
    (1, 1000, 1000, 2, 128, True, -0.2, torch.float16),   # many key tiles: the running extremum moves
])
def test_negative_scale(B, Sq, Sk, H, D, causal, scale, dtype):
    """Any finite scale is used as given: with scale < 0 the row maximum of s * scale is scale times the
    row's smallest score, and masked scores must carry no weight either way."""
    q, k, v = make_inputs(B, Sq, Sk, H, D, dtype, seed=41 + Sq + D)
    print(run_and_check(q, k, v, causal, scale, 1.0))


def test_single_key_closed_form():
    """Sk = 1: every row's output is v_0 exactly and LSE is scale * q . k_0."""
    q, k, v = make_inputs(2, 300, 1, 3, 128, "bf16", seed=21)
    out, lse = fa.fwd(q, k, v, causal=False)
    torch.cuda.synchronize()
    assert torch.equal(out, v.expand(2, 300, 3, 128))
    ref = torch.einsum("bshd,bhd->bhs", q.double(), k[:, 0].double()) / math.sqrt(128)
    assert (lse.double() - ref).abs().max().item() <= 1e-3


def test_gpt_workload_sampled_rows():
    w = WORKLOADS["gpt"]
    q, k, v = make_workload_inputs(w)
    hs = all_heads(w.B, w.H)
    print(run_and_check(q, k, v, w.causal, None, w.sigma, heads=hs, rows=sampled_rows(w.Sq, hs, 4, 1)))


def test_skill_timing_sampled_rows():
    """The skill page's timing shape (Workflow 1 Step 4: batch 4, seqlen 4096, 32 heads, head dim 64, fp16, no
    mask), which runs the head-dim-64 forward with P handed over in two halves; sampled rows of every head."""
    w = WORKLOADS["skill_timing"]
    q, k, v = make_workload_inputs(w)
    hs = all_heads(w.B, w.H)
    print(run_and_check(q, k, v, w.causal, None, w.sigma, heads=hs, rows=sampled_rows(w.Sq, hs, 6, 3)))


def test_long_context_sampled_rows():
    w = WORKLOADS["long"]
    q, k, v = make_workload_inputs(w)
    hs = all_heads(w.B, w.H)
    print(run_and_check(q, k, v, w.causal, None, w.sigma, heads=hs, rows=sampled_rows(w.Sq, hs, 8, 2), chunk=4))


def test_pages_accuracy_check():
    """The skill page's accuracy snippet (Workflow 1, Step 4) compares flash attention with standard attention
    (no mask) in fp16 on (batch 1, heads 8, seqlen 512, headdim 64) and expects a maximum absolute difference
    below 1e-3; the same check against the fp64 oracle. (With a causal mask the first rows average few values
    of |v| up to ~4, where half an fp16 ulp is already ~1e-3: those rows are held to the bounds of the parity
    tests above, which include the output rounding.)"""
    q, k, v = make_inputs(1, 512, 512, 8, 64, "f16", 1158)
    out, _ = fa.fwd(q, k, v, causal=False)
    torch.cuda.synchronize()
    heads = all_heads(1, 8)
    o_ref, _ = oracle_fwd(q, k, v, False, None, heads)
    err = float(np.abs(gather_rows(out, heads) - o_ref).max())
    print("max abs diff %.3e" % err)
    assert err < 1e-3


# Mid-sized problems of between one and two waves of CTAs (148 < CTAs <= 296 on a 148-SM B200, a CTA taking 256
# query rows of one (batch, head)): ragged lengths, Sq != Sk, grouped heads, a window, rows without keys and a
# negative scale, each checked on every row of three heads and on sampled rows of all heads.
@pytest.mark.parametrize("B,Sq,Sk,H,Hkv,D,causal,window,dtype,scale", [
    (1, 5000, 5000, 10, 10, 128, True, (-1, -1), torch.bfloat16, None),   # 20 query blocks x 10 heads, ragged
    (2, 2500, 3000, 8, 2, 64, True, (-1, -1), torch.float16, None),       # Sq != Sk, grouped heads
    (1, 4100, 4100, 12, 4, 128, False, (300, 200), torch.float16, None),  # window, non-causal, ragged tail
    (3, 1700, 900, 8, 8, 128, True, (-1, -1), torch.bfloat16, None),      # Sq > Sk: rows without keys
    (1, 4000, 4000, 10, 10, 64, True, (-1, -1), torch.bfloat16, -0.1),    # negative scale
])
def test_mid_size_forward_shapes(B, Sq, Sk, H, Hkv, D, causal, window, dtype, scale):
    n_units = ((Sq + 255) // 256) * B * H
    assert 148 < n_units <= 296, n_units
    g = torch.Generator(device="cuda")
    g.manual_seed(600 + Sq + H)
    from exact_io_aware_76_b200.inputs import draw
    q = draw((B, Sq, H, D), dtype, g, "cuda")
    k = draw((B, Sk, Hkv, D), dtype, g, "cuda")
    v = draw((B, Sk, Hkv, D), dtype, g, "cuda")
    out, lse = fa.fwd(q, k, v, causal=causal, scale=scale, window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    hs = all_heads(B, H)
    # every row of three heads, sampled rows of all heads
    for heads, rows in ((hs[:1] + hs[len(hs) // 2:len(hs) // 2 + 1] + hs[-1:], None),
                        (hs, sampled_rows(Sq, hs, 6, 9))):
        o_ref, l_ref = oracle_fwd(q, k, v, causal, scale, heads, rows, window=window)
        print(check_out(gather_rows(out, heads, rows), o_ref, dtype), check_lse(gather_lse(lse, heads, rows), l_ref))
