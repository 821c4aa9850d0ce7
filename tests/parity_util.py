"""Helpers shared by the GPU parity tests: move [B, S, H, D] tensors into the oracle's per-head fp64 layout,
run the oracle on selected heads/rows, and apply the parity bounds.

Parity bounds (the tolerance of the benchmark plan, with the reading for outputs the 16-bit format cannot
represent that closely):
  * O: |O - O_ref| <= tol * sigma + ulp(O_ref) / 2, tol = 1e-2 (bf16) or 2e-3 (fp16), sigma the input scale
    (O is linear in V, so the bound scales with it), plus half a unit in the last place of the output format
    at |O_ref| for the final rounding to 16 bits, which no implementation can avoid.
  * LSE: |LSE - LSE_ref| <= 1e-3 where LSE_ref is finite; rows with no visible key must be -inf on both sides.
  * dQ, dK, dV: ||G - G_ref||_F / ||G_ref||_F <= 2e-2 per tensor over the checked set and for every head on
    its own; on small shapes also element by element against 2e-2 of the head's largest gradient (plus the
    16-bit output rounding), so that an error confined to one row or tile edge cannot hide inside a norm.
"""
import numpy as np
import torch

import oracle

O_TOL = {torch.bfloat16: 1e-2, torch.float16: 2e-3}
LSE_TOL = 1e-3
GRAD_RTOL = 2e-2
MANT_BITS = {torch.bfloat16: 8, torch.float16: 11}  # significand bits incl. the implicit one


def heads_f64(x, heads):
    """x [B, S, H, D] (any device) -> float64 numpy [len(heads), S, D] for the (b, h) pairs in ``heads``."""
    parts = [x[b, :, h, :].detach().to("cpu", torch.float64) for (b, h) in heads]
    return torch.stack(parts).numpy()


def all_heads(B, H):
    return [(b, h) for b in range(B) for h in range(H)]


def kv_heads(q, k, heads):
    """The K/V head each query head of ``heads`` reads (grouped heads: h // (Hq / Hkv))."""
    group = q.shape[2] // k.shape[2]
    return [(b, h // group) for (b, h) in heads]


def oracle_fwd(q, k, v, causal, scale, heads, rows=None, window=(-1, -1)):
    kv = kv_heads(q, k, heads)
    return oracle.attn_fwd(heads_f64(q, heads), heads_f64(k, kv), heads_f64(v, kv), causal=causal,
                           scale=scale, rows=rows, window=window)


def oracle_bwd(q, k, v, do, causal, scale, heads, rows=None, window=(-1, -1)):
    kv = kv_heads(q, k, heads)
    return oracle.attn_bwd(heads_f64(q, heads), heads_f64(k, kv), heads_f64(v, kv), heads_f64(do, heads),
                           causal=causal, scale=scale, rows=rows, window=window)


def oracle_bwd_grouped(q, k, v, do, causal, scale, b, h_kv, window=(-1, -1)):
    """dQ of the whole group of query heads of K/V head (b, h_kv), and that K/V head's dK/dV summed over the
    group (the oracle's grouped-head path)."""
    group = q.shape[2] // k.shape[2]
    qh = [(b, h_kv * group + g) for g in range(group)]
    return oracle.attn_bwd(heads_f64(q, qh), heads_f64(k, [(b, h_kv)]), heads_f64(v, [(b, h_kv)]),
                           heads_f64(do, qh), causal=causal, scale=scale, window=window)


def gather_rows(x, heads, rows=None):
    """x [B, S, H, D] -> float64 [n_heads, n_rows, D] (all rows if rows is None)."""
    out = []
    for t, (b, h) in enumerate(heads):
        xs = x[b, :, h, :] if rows is None else x[b, torch.as_tensor(rows[t], device=x.device), h, :]
        out.append(xs.detach().to("cpu", torch.float64))
    return torch.stack(out).numpy()


def gather_lse(lse, heads, rows=None):
    out = []
    for t, (b, h) in enumerate(heads):
        ls = lse[b, h, :] if rows is None else lse[b, h, torch.as_tensor(rows[t], device=lse.device)]
        out.append(ls.detach().to("cpu", torch.float64))
    return torch.stack(out).numpy()


def half_ulp(ref, dtype):
    """Half a unit in the last place of ``dtype`` at |ref| (normal range)."""
    a = np.maximum(np.abs(ref), 2.0 ** -14)
    return 0.5 * 2.0 ** (np.floor(np.log2(a)) - (MANT_BITS[dtype] - 1))


def check_out(o, o_ref, dtype, sigma=1.0, what="O"):
    o = np.asarray(o, np.float64)
    err = np.abs(o - o_ref)
    bound = O_TOL[dtype] * sigma + half_ulp(o_ref, dtype)
    bad = ~(err <= bound)
    ulps = err / (2 * half_ulp(o_ref, dtype))
    # The bare tolerance (tol * sigma, without the half ulp of the output rounding): how many elements need the
    # rounding allowance at all. For sigma = 1 workloads these are elements with |O_ref| large enough that half
    # an ulp of the 16-bit output exceeds the tolerance.
    bare = int((err > O_TOL[dtype] * sigma).sum())
    big = int((np.abs(o_ref) >= (4.0 if dtype == torch.bfloat16 else 8.0)).sum())
    info = "%s: max err %.3e, max err/bound %.3f, max err %.2f ulp, %d/%d over; %d above the bare %.0e (%d with |O_ref| where half an ulp exceeds it)" % (
        what, float(err.max()) if err.size else 0.0, float((err / bound).max()) if err.size else 0.0,
        float(ulps.max()) if ulps.size else 0.0, int(bad.sum()), err.size, bare, O_TOL[dtype] * sigma, big)
    assert not bad.any(), info
    return info


def check_lse(lse, lse_ref, what="LSE"):
    lse = np.asarray(lse, np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lse), ~fin), what + ": -inf rows differ"
    err = np.abs(lse[fin] - lse_ref[fin])
    info = "%s: max err %.3e" % (what, float(err.max()) if err.size else 0.0)
    assert err.size == 0 or err.max() <= LSE_TOL, info
    return info


def check_grad(g, g_ref, what, per_head=True, elementwise=False, rtol=GRAD_RTOL):
    """Relative Frobenius error of the whole set and (``per_head``) of every head on its own, each <= rtol.
    With ``elementwise`` every element must also satisfy |G - G_ref| <= rtol * max|G_ref of its head| plus two
    ulps of the 16-bit output at |G_ref|, so a wrong row or tile edge cannot hide inside a norm.

    ``per_head`` is for checked sets of whole heads. On a few sampled rows per head it only reports the worst
    head (``per_head=False``): there one row can dominate a head's norm, e.g. dQ of a causal first row, exactly
    0, which the kernel obtains as the small difference dP - D with D_i = dO_i . O_i taken from the 16-bit O."""
    g = np.asarray(g, np.float64)
    g_ref = np.asarray(g_ref, np.float64)
    assert np.all(np.isfinite(g)), what + ": non-finite values"

    def rel(a, b):
        den = np.linalg.norm(b)
        return np.linalg.norm(a - b) / den if den > 0 else np.linalg.norm(a - b)

    whole = rel(g, g_ref)
    info = "%s: rel Frobenius err %.3e" % (what, whole)
    assert whole <= rtol, info
    if g.ndim == 3:
        per = [rel(g[t], g_ref[t]) for t in range(g.shape[0])]
        worst = int(np.argmax(per))
        info += ", worst head %.3e (head %d of %d)" % (per[worst], worst, len(per))
        assert not per_head or per[worst] <= rtol, info
    if elementwise:
        hm = np.abs(g_ref).reshape(g_ref.shape[0], -1).max(axis=1) if g_ref.ndim == 3 else np.abs(g_ref).max()
        hm = hm.reshape((-1,) + (1,) * (g_ref.ndim - 1)) if g_ref.ndim == 3 else hm
        bound = rtol * hm + 4 * half_ulp(g_ref, torch.bfloat16)
        err = np.abs(g - g_ref)
        info += ", max abs err %.3e (max err/bound %.3f)" % (float(err.max()), float((err / bound).max()))
        assert np.all(err <= bound), info
    return info
