"""Host logic behind the numbers the benchmark reports: the visible-pair count of the FLOP convention (closed
form against brute-force counting of the mask) and the e4m3 input recipe."""
import dataclasses

import numpy as np
import pytest
import torch

from exact_io_aware_76_b200.inputs import draw_e4m3
from exact_io_aware_76_b200.workloads import WORKLOADS


def brute_pairs(Sq, Sk, causal):
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    return int(((j <= i + (Sk - Sq)) if causal else np.ones((Sq, Sk), bool)).sum())


@pytest.mark.parametrize("Sq", [1, 2, 5, 64, 127, 128, 129, 300])
@pytest.mark.parametrize("Sk", [1, 3, 64, 128, 200, 517])
@pytest.mark.parametrize("causal", [False, True])
def test_pairs_closed_form_matches_the_mask(Sq, Sk, causal):
    w = dataclasses.replace(WORKLOADS["tiny"], Sq=Sq, Sk=Sk, causal=causal)
    assert w.pairs() == brute_pairs(Sq, Sk, causal)


def test_flop_figures_of_the_full_size_workloads():
    gpt, long_ = WORKLOADS["gpt"], WORKLOADS["long"]
    assert gpt.pairs() == 8192 * 8193 // 2 and long_.pairs() == 131072 * 131073 // 2
    assert gpt.fwd_flops() == 4 * 4 * 32 * 128 * gpt.pairs()          # 2199 GFLOP
    assert gpt.bwd_flops() == 10 * 4 * 32 * 128 * gpt.pairs()         # 5498 GFLOP
    assert round(gpt.fwd_flops() / 1e9) == 2199 and round(gpt.bwd_flops() / 1e9) == 5498
    assert round(long_.fwd_flops() / 1e9) == 140739                 # ≈ 140,740 GFLOP


def test_only_the_gpt_workload_is_a_training_step():
    # the benchmark plan: tiny, small, mid and long context are forward passes (O and LSE); the GPT-style
    # workload is a forward plus the recomputation backward
    assert [n for n, w in WORKLOADS.items() if w.backward] == ["gpt"]
    assert len([n for n in WORKLOADS if n.startswith("mid_")]) == 8


def test_e4m3_inputs():
    g = torch.Generator()
    g.manual_seed(0)
    x, d = draw_e4m3((64, 128), g, "cpu")
    assert x.dtype == torch.float8_e4m3fn and d == 1.0
    g.manual_seed(0)
    xs, ds = draw_e4m3((64, 128), g, "cpu", sigma=3.0, per_tensor_scale=True)
    # the largest magnitude lands on e4m3's largest finite value; x * descale recovers the draw to e4m3 precision
    assert float(xs.float().abs().max()) == 448.0
    g.manual_seed(0)
    ref = torch.randn((64, 128), generator=g) * 3.0
    assert abs(ds - float(ref.abs().max()) / 448.0) < 1e-12
    err = (xs.float() * ds - ref).abs() / ref.abs().clamp_min(ds * 2.0 ** -6)
    assert float(err.max()) <= 2.0 ** -4 + 1e-6
