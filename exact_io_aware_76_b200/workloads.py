"""Workload table and FLOP counting for the benchmark and the tests.

The five workloads follow the benchmark plan: tiny (1x2x128x64 fp16 non-causal), small (2x8x512x64 fp16,
causal and non-causal), mid (2x16x2048, D 64/128, fp16/bf16, causal, inputs scaled by 1 and 4), GPT-style
training (4x32x8192x128 bf16 causal) and long context (1x32x131072x128 bf16 causal). The GPT-style step is a
forward and a backward; the others are forward passes (O and LSE). A sixth, skill_timing, is the timing shape
of the skill page's Workflow 1 Step 4 (4x32x4096x64 fp16, non-causal), a forward pass.

FLOP convention: forward 4*B*H*D*pairs (QK^T and PV), backward 10*B*H*D*pairs (five matrix products, the
recomputation of QK^T included), where ``pairs`` counts only the (query, key) pairs the mask leaves visible.
"""
from dataclasses import dataclass

from .inputs import DTYPES


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, mask flag and input scale."""

    name: str
    B: int
    H: int
    Sq: int
    Sk: int
    D: int
    dtype: str
    causal: bool
    sigma: float = 1.0
    seed: int = 1000
    backward: bool = False  # a training step (forward + backward) rather than a forward pass

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    def pairs(self):
        """Number of (query, key) pairs visible under the mask (causal: bottom-right aligned, key j visible
        to query i iff j <= i + Sk - Sq). Row i sees min(Sk, max(0, i + Sk - Sq + 1)) keys."""
        if not self.causal:
            return self.Sq * self.Sk
        off = self.Sk - self.Sq
        i_lo = max(0, -off)                 # first row that sees at least one key
        i_full = max(0, self.Sk - off - 1)  # first row that sees every key
        hi = min(i_full, self.Sq)
        partial = sum_range(i_lo + off + 1, hi + off) if hi > i_lo else 0
        full = max(0, self.Sq - max(i_full, i_lo)) * self.Sk
        return partial + full

    def fwd_flops(self):
        return 4 * self.B * self.H * self.D * self.pairs()

    def bwd_flops(self):
        return 10 * self.B * self.H * self.D * self.pairs()


def sum_range(first, last):
    """Sum of the integers first..last inclusive."""
    if last < first:
        return 0
    return (first + last) * (last - first + 1) // 2


# The five workloads of the benchmark plan (seed 1000 + index). The mid workload is a sweep; its members
# are listed individually.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 128, 64, "f16", False, 1.0, 1000),
    "small_causal": Workload("small_causal", 2, 8, 512, 512, 64, "f16", True, 1.0, 1001),
    "small_noncausal": Workload("small_noncausal", 2, 8, 512, 512, 64, "f16", False, 1.0, 1001),
    "gpt": Workload("gpt", 4, 32, 8192, 8192, 128, "bf16", True, 1.0, 1003, backward=True),
    "long": Workload("long", 1, 32, 131072, 131072, 128, "bf16", True, 1.0, 1004),
}
for _D in (64, 128):
    for _dt in ("f16", "bf16"):
        for _sig in (1.0, 4.0):
            _n = "mid_d%d_%s_x%d" % (_D, _dt, int(_sig))
            WORKLOADS[_n] = Workload(_n, 2, 16, 2048, 2048, _D, _dt, True, _sig, 1002)
# The skill page's own timing shape (Workflow 1, Step 4: flash_attn_func on (4, 4096, 32, 64) fp16 tensors,
# no causal flag), as a forward workload for `bench.py --workload skill_timing`.
WORKLOADS["skill_timing"] = Workload("skill_timing", 4, 32, 4096, 4096, 64, "f16", False, 1.0, 1005)


def make_workload_inputs(w, device="cuda", with_dout=False):
    from .inputs import make_inputs
    return make_inputs(w.B, w.Sq, w.Sk, w.H, w.D, w.dtype, w.seed, w.sigma, device, with_dout)
