"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws q, k, v (and the upstream gradient dO) as iid
N(0, 1) samples, multiplies them by ``sigma`` and rounds them to the requested dtype, in the
``[batch, seqlen, nheads, headdim]`` layout of the skill page's ``flash_attn_func`` examples (page "Flash
Attention — 長い系列を扱う Transformer の学習と推論を速くする", quick start and Workflow 2 Step 2).

Recipe: one ``torch.Generator`` on the target device seeded with ``seed``; tensors drawn in the order
q, k, v, dO as float32 ``randn``; each multiplied by ``sigma`` and then rounded (round-to-nearest-even) to
fp16 or bf16. The rounded tensors are what both the CUDA path and the oracle consume.
"""
import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


def draw(shape, dtype, generator, device, sigma=1.0):
    """One N(0,1)*sigma tensor drawn in float32, rounded to ``dtype``."""
    x = torch.randn(shape, generator=generator, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(dtype)


def make_inputs(B, Sq, Sk, H, D, dtype, seed, sigma=1.0, device="cuda", with_dout=False):
    """q [B,Sq,H,D], k/v [B,Sk,H,D] (and dO [B,Sq,H,D]) drawn in that order from one seeded generator."""
    if isinstance(dtype, str):
        dtype = DTYPES[dtype]
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = draw((B, Sq, H, D), dtype, g, device, sigma)
    k = draw((B, Sk, H, D), dtype, g, device, sigma)
    v = draw((B, Sk, H, D), dtype, g, device, sigma)
    if not with_dout:
        return q, k, v
    do = draw((B, Sq, H, D), dtype, g, device, 1.0)
    return q, k, v, do


def draw_e4m3(shape, generator, device, sigma=1.0, per_tensor_scale=False):
    """One N(0,1)*sigma float32 tensor stored as float8_e4m3fn plus its descale factor, the FP8 input form of
    the skill page's Workflow 3. Without ``per_tensor_scale`` the samples are rounded to e4m3 directly (descale
    1); with it they are first divided by amax/448 so that the largest magnitude lands on e4m3's largest
    finite value (448), and the descale is amax/448. The real input is ``x_e4m3 * descale``."""
    x = torch.randn(shape, generator=generator, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    descale = 1.0
    if per_tensor_scale:
        descale = float(x.abs().max()) / 448.0
        x.div_(descale)
    return x.to(torch.float8_e4m3fn), descale
