"""FP8 (e4m3) forward (skill page, Workflow 3: a forward-only path on float8_e4m3fn inputs) on the GPU, through
the C ABI (fa_fwd_fp8), against the oracle run on the dequantized inputs.

The forward rounds each probability to e4m3 before the P V product (the tensor core's 8-bit operand), so O is
not the exact attention of the dequantized inputs. The bound below follows from that one rounding (the e4m3
inputs themselves reach the oracle exactly):
  * a probability p' >= 2^-6 (e4m3's smallest normal) is off by at most 2^-4 p' (4 significant bits, round to
    nearest); a smaller one by at most 2^-10 (half the subnormal spacing 2^-9);
  * the kernel exponentiates against a running maximum that never exceeds the row's true maximum m, so its
    normaliser is l' >= l = sum_j exp(s_j - m) >= 1 in the same units, and
        |O_i - O_ref,i| <= 2^-4 (P |V|)_i + 2^-10 sum_{j visible} |v_j| / l_i
    plus half a bf16 ulp for the output and a term for fp32 arithmetic: the normaliser l is a sum of at most
    n_i + 128 fp32 probabilities (n_i visible keys, padded to whole 128-key tiles), O a chain of fewer fp32
    accumulations (one per 32-key MMA step), and a few more roundings come from the exponentials (ex2.approx,
    a few ulps), the lazy rescales and the final scaling; each rounding is at most 2^-24 relative, so
        (n_i + 256) * 2^-23 * (P |V|)_i
    covers them with a factor of two to spare (the deterministic worst case; the observed error is far below).
LSE comes from unrounded probabilities and keeps the 1e-3 bound of the 16-bit path.

A second, sharp case makes every probability a power of two inside e4m3's exact range (q.k an integer in
[-4, 4] and scale * q_descale * k_descale = ln 2), so the rounding is exact and O must match the oracle to
fp32 accumulation and the final bf16 rounding.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_76_b200 as fa
import oracle
from exact_io_aware_76_b200.inputs import draw_e4m3
from exact_io_aware_76_b200.workloads import WORKLOADS, make_workload_inputs
from parity_util import all_heads, check_lse, gather_lse, gather_rows, half_ulp

pytestmark = pytest.mark.gpu


def deq(x, d, b, h):
    return x[b, :, h, :].to("cpu", torch.float64).numpy() * d


def visible_mask(Sq, Sk, causal, window, rows=None):
    i = (np.arange(Sq) if rows is None else np.asarray(rows))[:, None]
    j = np.arange(Sk)[None, :]
    c = i + (Sk - Sq)
    left, right = window
    if causal:
        right = 0 if right < 0 else min(right, 0)
    vis = np.ones((i.shape[0], Sk), bool)
    if left >= 0:
        vis &= j >= c - left
    if right >= 0:
        vis &= j <= c + right
    return vis


def oracle_heads(qs, ks, vs, causal, scale, window):
    o, l = oracle.attn_fwd(np.stack(qs), np.stack(ks), np.stack(vs), causal=causal, scale=scale, window=window)
    return o, l


def bound(qh, kh, vh, causal, scale, window, rows=None):
    """Per-element bound on |O - O_ref| from rounding the probabilities to e4m3 (see the module docstring), for
    every row of qh or only the listed rows."""
    Sq, Sk = qh.shape[0], kh.shape[0]
    vis = visible_mask(Sq, Sk, causal, window, rows)
    s = scale * ((qh if rows is None else qh[rows]) @ kh.T)
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    has = np.isfinite(m)
    e = np.where(vis & has, np.exp(s - np.where(has, m, 0.0)), 0.0)
    l = e.sum(axis=1, keepdims=True)
    lsafe = np.where(l > 0, l, 1.0)
    p_absv = (e / lsafe) @ np.abs(vh)
    tail = (vis.astype(np.float64) @ np.abs(vh)) * 2.0 ** -10 / lsafe
    return 2.0 ** -4 * p_absv + tail + accumulation(vis, p_absv)


def accumulation(vis, p_absv):
    """fp32 arithmetic term of the bound: (n_i + 256) * 2^-23 * (P |V|)_i, n_i the visible keys of row i."""
    n = vis.sum(axis=1, keepdims=True).astype(np.float64)
    return (n + 256.0) * 2.0 ** -23 * p_absv


CASES = [
    # B, Sq, Sk, H, Hkv, causal, window, per_tensor_scale
    (1, 256, 256, 2, 2, False, (-1, -1), False),
    (2, 333, 517, 4, 2, True, (-1, -1), True),
    (1, 700, 700, 4, 1, False, (128, 128), False),
    (1, 1000, 1000, 2, 2, True, (256, 0), True),
    (1, 517, 333, 2, 1, True, (100, -1), False),   # rows without keys
    (1, 1, 1, 1, 1, False, (-1, -1), False),       # one query, one key
    (1, 5, 1000, 2, 2, True, (-1, -1), True),      # short query block at the end of a long key range
    (1, 1000, 5, 2, 1, True, (-1, -1), False),     # five keys: all but the last five rows see none
]


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("B,Sq,Sk,H,Hkv,causal,window,scaled", CASES)
def test_fp8_forward_within_rounding_bound(B, Sq, Sk, H, Hkv, causal, window, scaled, D):
    g = torch.Generator(device="cuda")
    g.manual_seed(7000 + Sq + H + D)
    q, dq_ = draw_e4m3((B, Sq, H, D), g, "cuda", per_tensor_scale=scaled)
    k, dk_ = draw_e4m3((B, Sk, Hkv, D), g, "cuda", per_tensor_scale=scaled)
    v, dv_ = draw_e4m3((B, Sk, Hkv, D), g, "cuda", per_tensor_scale=scaled)
    scale = 1.0 / math.sqrt(D)
    out, lse = fa.fwd_fp8(q, k, v, causal=causal, scale=scale, descale=(dq_, dk_, dv_), window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    grp = H // Hkv
    heads = [(b, h) for b in range(B) for h in range(H)]
    qs = [deq(q, dq_, b, h) for (b, h) in heads]
    ks = [deq(k, dk_, b, h // grp) for (b, h) in heads]
    vs = [deq(v, dv_, b, h // grp) for (b, h) in heads]
    o_ref, l_ref = oracle_heads(qs, ks, vs, causal, scale, window)
    o = gather_rows(out, heads)
    worst = 0.0
    for t in range(len(heads)):
        bd = bound(qs[t], ks[t], vs[t], causal, scale, window) + half_ulp(o_ref[t], torch.bfloat16)
        err = np.abs(o[t] - o_ref[t])
        worst = max(worst, float((err / bd).max()))
        assert np.all(err <= bd), "head %d: max err/bound %.3f" % (t, float((err / bd).max()))
    rel = np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref)
    print("O: max err/bound %.3f, rel Frobenius %.3e;" % (worst, rel), check_lse(gather_lse(lse, heads), l_ref))


def vis_and_pv(qh, kh, vh, causal, scale, window):
    """The visibility mask and (P |V|) of every row (fp64)."""
    Sq, Sk = qh.shape[0], kh.shape[0]
    vis = visible_mask(Sq, Sk, causal, window)
    s = np.where(vis, scale * (qh @ kh.T), -np.inf)
    m = s.max(axis=1, keepdims=True)
    has = np.isfinite(m)
    e = np.where(vis & has, np.exp(s - np.where(has, m, 0.0)), 0.0)
    l = e.sum(axis=1, keepdims=True)
    return vis, (e / np.where(l > 0, l, 1.0)) @ np.abs(vh)


def sparse_pm1(shape, nnz, g):
    """e4m3 tensor with exactly ``nnz`` entries of +-1 per head-dim row, the rest 0."""
    idx = torch.rand(shape, generator=g, device="cuda").argsort(dim=-1)[..., :nnz]
    sign = torch.randint(0, 2, shape[:-1] + (nnz,), generator=g, device="cuda").float() * 2 - 1
    x = torch.zeros(shape, device="cuda")
    x.scatter_(-1, idx, sign)
    return x.to(torch.float8_e4m3fn)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("causal,window,dq_", [(False, (-1, -1), 1.0), (True, (-1, -1), 0.5),
                                                (False, (64, 200), 2.0)])
def test_fp8_forward_exact_when_probabilities_are_powers_of_two(causal, window, dq_, D):
    B, Sq, Sk, H = 1, 384, 640, 2
    g = torch.Generator(device="cuda")
    g.manual_seed(7100 + int(causal) + D)
    q = sparse_pm1((B, Sq, H, D), 4, g)
    k = sparse_pm1((B, Sk, H, D), 4, g)
    v, dv_ = draw_e4m3((B, Sk, H, D), g, "cuda")
    dk_ = 1.0
    scale = math.log(2.0) / (dq_ * dk_)
    out, lse = fa.fwd_fp8(q, k, v, causal=causal, scale=scale, descale=(dq_, dk_, dv_), window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    heads = [(0, h) for h in range(H)]
    qs = [deq(q, dq_, b, h) for (b, h) in heads]
    ks = [deq(k, dk_, b, h) for (b, h) in heads]
    vs = [deq(v, dv_, b, h) for (b, h) in heads]
    o_ref, l_ref = oracle_heads(qs, ks, vs, causal, scale, window)
    o = gather_rows(out, heads)
    err = np.abs(o - o_ref)
    # every probability is exact in e4m3, so only the output rounding and fp32 arithmetic remain
    acc = np.stack([accumulation(*vis_and_pv(qs[t], ks[t], vs[t], causal, scale, window)) for t in range(H)])
    bd = half_ulp(o_ref, torch.bfloat16) + acc
    assert np.all(err <= bd), "max err %.3e, max err/bound %.3f" % (float(err.max()), float((err / bd).max()))
    print("O: max err %.3e, max err/bound %.3f;" % (float(err.max()), float((err / bd).max())),
          check_lse(gather_lse(lse, heads), l_ref))


@pytest.mark.parametrize("name,n_heads,per_head", [("gpt", 128, 4), ("long", 8, 4)])
def test_fp8_full_size_sampled_rows(name, n_heads, per_head):
    """The GPT-shaped (4x32x8192x128) and long-context (1x32x131072x128) workloads in e4m3, on sampled rows
    (first, last, both sides of the first tile edge and random) of n_heads evenly spaced heads."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    q8, k8, v8 = (x.to(torch.float8_e4m3fn) for x in (q, k, v))
    del q, k, v
    out, lse = fa.fwd_fp8(q8, k8, v8, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    heads = all_heads(w.B, w.H)
    heads = heads[::max(1, len(heads) // n_heads)][:n_heads]
    r = np.random.default_rng(11)
    scale = 1.0 / math.sqrt(w.D)
    worst = 0.0
    for (b, h) in heads:
        rows = np.array([0, w.Sq - 1, 127, 128] + list(r.choice(w.Sq, per_head, replace=False)), np.int64)
        qh, kh, vh = deq(q8, 1.0, b, h), deq(k8, 1.0, b, h), deq(v8, 1.0, b, h)
        o_ref, l_ref = oracle.attn_fwd(qh[None], kh[None], vh[None], causal=w.causal, scale=scale, rows=rows[None])
        bd = bound(qh, kh, vh, w.causal, scale, (-1, -1), rows) + half_ulp(o_ref[0], torch.bfloat16)
        o = gather_rows(out, [(b, h)], [rows])[0]
        err = np.abs(o - o_ref[0])
        worst = max(worst, float((err / bd).max()))
        assert np.all(err <= bd), "head (%d,%d): max err/bound %.3f" % (b, h, float((err / bd).max()))
        check_lse(gather_lse(lse, [(b, h)], [rows]), l_ref)
    print("max err/bound %.3f over %d heads" % (worst, len(heads)))


def test_fp8_skill_page_workflow3_shape():
    """The skill page's only FP8 call (Workflow 3, Step 3): [2, 4096, 32, 64] tensors cast to float8_e4m3fn,
    causal. Every row of two heads and 8 sampled rows (first, last, both sides of a tile edge, random) of every
    other head, against the oracle on the dequantized inputs under the rounding bound."""
    B, S, H, D = 2, 4096, 32, 64
    g = torch.Generator(device="cuda")
    g.manual_seed(7300)
    q8, k8, v8 = (torch.randn((B, S, H, D), generator=g, device="cuda").to(torch.float8_e4m3fn) for _ in range(3))
    out, lse = fa.fwd_fp8(q8, k8, v8, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    scale = 1.0 / math.sqrt(D)
    r = np.random.default_rng(12)
    worst = 0.0
    for (b, h) in all_heads(B, H):
        full = (b, h) in ((0, 0), (1, 31))
        rows = np.arange(S, dtype=np.int64) if full else \
            np.array([0, S - 1, 127, 128] + list(r.choice(S, 4, replace=False)), np.int64)
        qh, kh, vh = deq(q8, 1.0, b, h), deq(k8, 1.0, b, h), deq(v8, 1.0, b, h)
        o_ref, l_ref = oracle.attn_fwd(qh[None], kh[None], vh[None], causal=True, scale=scale, rows=rows[None])
        bd = bound(qh, kh, vh, True, scale, (-1, -1), rows) + half_ulp(o_ref[0], torch.bfloat16)
        o = gather_rows(out, [(b, h)], [rows])[0]
        err = np.abs(o - o_ref[0])
        worst = max(worst, float((err / bd).max()))
        assert np.all(err <= bd), "head (%d,%d): max err/bound %.3f" % (b, h, float((err / bd).max()))
        check_lse(gather_lse(lse, [(b, h)], [rows]), l_ref)
    print("max err/bound %.3f over %d heads" % (worst, B * H))
