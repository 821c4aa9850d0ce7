"""Checks that pin the fp64 oracle to facts fixed outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` instance and raises AssertionError on a mismatch. The
same functions run against the real oracle (tests/test_oracle_pins.py) and against copies of it with a
planted mistake (tests/test_oracle_mutants.py), which must each fail at least one pin.

What pins it:
  * closed forms of special cases: a single key (O = v_0, LSE = s_00, dQ = dK = 0, dV_0 = sum_i dO_i);
    identical keys (O_i = mean of the visible v_j, LSE_i = s + ln |J(i)|); the first causal row (O_0 = v_0);
    V = ones gives O = 1 because every softmax row sums to 1;
  * hand-worked examples with their derivations (tests/golden/hand_examples.json);
  * invariants: joint permutation of (K, V) rows leaves a non-causal result unchanged; sum_j dK_j = 0 and
    sum_j dV_j = sum_i dO_i per head; keys hidden from a row by the mask have no influence on it, whatever
    they hold (scores beyond exp's range included), and receive no gradient from it;
  * central finite differences of L = sum dO * O in fp64 on tiny shapes (the backward has no formula on
    the pages, so the gradient of the oracle's own forward is the definition it must match);
  * a library routine the definition reduces to: torch's scaled_dot_product_attention on the CPU in
    float64, with autograd for the gradients (the skill page names SDPA in its quick start);
  * the causal reading for Sq != Sk (bottom-right aligned) and fully masked rows (O = 0, LSE = -inf);
  * the default scale 1/sqrt(d): the skill page divides by 8.0 for d = 64 (Workflow 1, Step 3 and 4);
  * grouped K/V heads (skill page, Workflow 2 Step 3): the same as repeating each K/V head over its group
    (dK/dV summed over the group), finite differences through the shared heads, and torch SDPA with
    enable_gqa; the sliding window (Workflow 2 Steps 2-3, window_size=(left, right)): a window wider than the
    sequence changes nothing, (0, 0) keeps only the aligned key, finite differences, SDPA with a band mask;
  * dropout (the dropout_p argument of the skill page's call): Philox4x32-10 against its published
    known-answer vectors and a keep block derived by hand from one of them (tests/golden/philox_dropout.json);
    dropout_p = 0 is the plain path; the keep rate matches 1 - t/256; O averaged over many seeds converges to
    the undropped O (the 1/(1 - p) rescale) with LSE unchanged; with V = I the output is P o Z itself; finite
    differences with the mask held fixed (and heads numbered as in a larger batch); hand-derived cases of the
    probability's resolution t = floor(256 p + 1/2) and its rejections; the counter layout of the
    dropout stream applied to the pinned generator on blocks whose row and key indices differ;
  * linearity in V: sum_j v_j . dV_j equals the loss sum_i dO_i . O_i, with and without dropout.
"""
import json
import math
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
TOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol * max(1.0, float(np.max(np.abs(b))) if b.size else 1.0), (what, err)


def pin_single_key(orc):
    r = _rng(1)
    for causal in (False, True):
        q = r.standard_normal((2, 5, 4)) if not causal else r.standard_normal((2, 1, 4))
        k = r.standard_normal((2, 1, 4))
        v = r.standard_normal((2, 1, 4))
        do = r.standard_normal(q.shape)
        out, lse = orc.fwd(q, k, v, causal=causal, scale=0.7)
        Sq = q.shape[1]
        _close(out, np.broadcast_to(v, (2, Sq, 4)), what="O = v0")
        _close(lse, 0.7 * np.einsum("hid,hd->hi", q, k[:, 0]), what="LSE = s00")
        dq, dk, dv = orc.bwd(q, k, v, do, causal=causal, scale=0.7)
        _close(dq, np.zeros_like(dq), what="dQ = 0")
        _close(dk, np.zeros_like(dk), what="dK = 0")
        _close(dv[:, 0], do.sum(axis=1), what="dV0 = sum dO")


def pin_identical_keys(orc):
    r = _rng(2)
    S, D = 7, 3
    q = r.standard_normal((1, S, D))
    kk = r.standard_normal(D)
    k = np.broadcast_to(kk, (1, S, D)).copy()
    v = r.standard_normal((1, S, D))
    out, lse = orc.fwd(q, k, v, causal=False, scale=0.3)
    _close(out[0], np.broadcast_to(v[0].mean(axis=0), (S, D)), what="mean of V")
    _close(lse[0], 0.3 * q[0] @ kk + math.log(S), what="LSE identical keys")
    out, lse = orc.fwd(q, k, v, causal=True, scale=0.3)
    for i in range(S):
        _close(out[0, i], v[0, : i + 1].mean(axis=0), what="causal prefix mean")
        _close(lse[0, i], 0.3 * q[0, i] @ kk + math.log(i + 1), what="causal LSE")


def pin_first_causal_row(orc):
    r = _rng(3)
    q, k, v = (r.standard_normal((3, 6, 5)) for _ in range(3))
    out, lse = orc.fwd(q, k, v, causal=True, scale=0.9, rows=np.zeros((3, 1), np.int64))
    _close(out[:, 0], v[:, 0], what="O_0 = v_0")
    _close(lse[:, 0], 0.9 * np.einsum("hd,hd->h", q[:, 0], k[:, 0]), what="LSE_0 = s_00")


def pin_rows_sum_to_one(orc):
    r = _rng(4)
    for causal in (False, True):
        q = r.standard_normal((2, 9, 4)) * 3
        k = r.standard_normal((2, 9, 4)) * 3
        v = np.ones((2, 9, 4))
        out, _ = orc.fwd(q, k, v, causal=causal, scale=0.5)
        _close(out, np.ones_like(out), tol=1e-14, what="softmax rows sum to 1")


def pin_key_permutation(orc):
    r = _rng(5)
    q, k, v = (r.standard_normal((2, 8, 4)) for _ in range(3))
    perm = r.permutation(8)
    o1, l1 = orc.fwd(q, k, v, causal=False, scale=0.4)
    o2, l2 = orc.fwd(q, k[:, perm], v[:, perm], causal=False, scale=0.4)
    _close(o1, o2, what="perm O")
    _close(l1, l2, what="perm LSE")


def pin_masked_keys_have_no_influence(orc):
    # A masked (query, key) pair takes no part in the row, whatever the key holds: rows 0-2 of a 6 x 6 problem
    # see none of keys 3-5 (causal, and a window (1, 0) without the causal flag), which are replaced by vectors
    # whose scores exceed every visible score of row 2 by far more than exp's range and by huge values. O, LSE,
    # dQ and the rows' dK/dV contributions stay bit for bit the same, and keys 3-5 receive exactly zero.
    r = _rng(40)
    q, k, v, do = (r.standard_normal((1, 6, 3)) for _ in range(4))
    k2, v2 = k.copy(), v.copy()
    k2[0, 3:] = 1e4 * q[0, 2]
    v2[0, 3:] = 1e6
    rows = np.array([[0, 1, 2]], np.int64)
    for causal, window in ((True, (-1, -1)), (False, (1, 0))):
        kw = dict(causal=causal, scale=0.5, rows=rows, window=window)
        for a, b in zip(orc.fwd(q, k, v, **kw), orc.fwd(q, k2, v2, **kw)):
            assert np.array_equal(a, b), ("masked keys change the forward", causal, window)
        (dq1, dk1, dv1), (dq2, dk2, dv2) = orc.bwd(q, k, v, do, **kw), orc.bwd(q, k2, v2, do, **kw)
        assert np.array_equal(dq1, dq2), ("masked keys change dQ", causal, window)
        for g1, g2 in ((dk1, dk2), (dv1, dv2)):
            assert np.array_equal(g1[:, :3], g2[:, :3]), ("masked keys change dK/dV", causal, window)
            assert not g1[:, 3:].any() and not g2[:, 3:].any(), ("masked keys receive gradient", causal, window)


def _loss(orc, q, k, v, do, causal, scale):
    out, _ = orc.fwd(q, k, v, causal=causal, scale=scale)
    return float(np.sum(out * do))


def pin_finite_differences(orc):
    r = _rng(6)
    h = 1e-6
    for (Sq, Sk, D, causal) in ((4, 4, 3, False), (5, 5, 2, True), (3, 6, 2, True), (6, 4, 3, True), (3, 5, 4, False)):
        q = r.standard_normal((1, Sq, D))
        k = r.standard_normal((1, Sk, D))
        v = r.standard_normal((1, Sk, D))
        do = r.standard_normal((1, Sq, D))
        dq, dk, dv = orc.bwd(q, k, v, do, causal=causal, scale=0.8)
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp = x.copy()
                xp[idx] += h
                xm = x.copy()
                xm[idx] -= h
                args_p = {"q": q, "k": k, "v": v}
                args_m = dict(args_p)
                args_p[name] = xp
                args_m[name] = xm
                num[idx] = (_loss(orc, args_p["q"], args_p["k"], args_p["v"], do, causal, 0.8)
                            - _loss(orc, args_m["q"], args_m["k"], args_m["v"], do, causal, 0.8)) / (2 * h)
            err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
            zero_ok = np.linalg.norm(num) < 1e-9 and np.linalg.norm(g) < 1e-9
            assert zero_ok or err <= 1e-6, ("finite differences d" + name, Sq, Sk, causal, err)


def pin_grad_invariants(orc):
    r = _rng(7)
    for causal in (False, True):
        q, k, v, do = (r.standard_normal((2, 10, 4)) for _ in range(4))
        _, dk, dv = orc.bwd(q, k, v, do, causal=causal, scale=0.6)
        _close(dk.sum(axis=1), np.zeros((2, 4)), tol=1e-13, what="sum_j dK_j = 0")
        _close(dv.sum(axis=1), do.sum(axis=1), tol=1e-13, what="sum_j dV_j = sum_i dO_i")


def pin_row_subset(orc):
    """dK/dV for a row subset equal the full gradient with dO zeroed outside the subset."""
    r = _rng(8)
    q, k, v, do = (r.standard_normal((2, 9, 3)) for _ in range(4))
    rows = np.array([[0, 4, 8], [2, 3, 7]], np.int64)
    dq_s, dk_s, dv_s = orc.bwd(q, k, v, do, causal=True, scale=0.5, rows=rows)
    do_m = np.zeros_like(do)
    for hh in range(2):
        do_m[hh, rows[hh]] = do[hh, rows[hh]]
    dq_f, dk_f, dv_f = orc.bwd(q, k, v, do_m, causal=True, scale=0.5)
    _close(dk_s, dk_f, what="subset dK")
    _close(dv_s, dv_f, what="subset dV")
    for hh in range(2):
        _close(dq_s[hh], dq_f[hh, rows[hh]], what="subset dQ")
    o_s, l_s = orc.fwd(q, k, v, causal=True, scale=0.5, rows=rows)
    o_f, l_f = orc.fwd(q, k, v, causal=True, scale=0.5)
    for hh in range(2):
        _close(o_s[hh], o_f[hh, rows[hh]], what="subset O")
        _close(l_s[hh], l_f[hh, rows[hh]], what="subset LSE")


def _sdpa(q, k, v, do, mask, scale):
    import torch

    tq = torch.tensor(q[None], dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k[None], dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v[None], dtype=torch.float64, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    o.backward(torch.tensor(do[None], dtype=torch.float64))
    return (o.detach()[0].numpy(), tq.grad[0].numpy(), tk.grad[0].numpy(), tv.grad[0].numpy())


def pin_sdpa_crosscheck(orc):
    """float64 CPU SDPA ([B,H,S,D] after transposing; one batch of heads) with an explicit boolean mask."""
    import torch

    r = _rng(9)
    for (Sq, Sk, D, causal) in ((16, 16, 8, False), (16, 16, 8, True), (5, 12, 4, True), (12, 12, 16, True),
                                (7, 3, 4, False)):
        H = 3
        q = r.standard_normal((H, Sq, D))
        k = r.standard_normal((H, Sk, D))
        v = r.standard_normal((H, Sk, D))
        do = r.standard_normal((H, Sq, D))
        scale = 1.0 / math.sqrt(D)
        mask = None
        if causal:
            # the bottom-right aligned reading, written as a boolean mask for SDPA
            mask = torch.ones(Sq, Sk, dtype=torch.bool).tril(diagonal=Sk - Sq)
        o_ref, dq_ref, dk_ref, dv_ref = _sdpa(q, k, v, do, mask, scale)
        out, lse = orc.fwd(q, k, v, causal=causal, scale=None)
        dq, dk, dv = orc.bwd(q, k, v, do, causal=causal, scale=None)
        _close(out, o_ref, what="SDPA O")
        _close(dq, dq_ref, what="SDPA dQ")
        _close(dk, dk_ref, what="SDPA dK")
        _close(dv, dv_ref, what="SDPA dV")
        # LSE against torch.logsumexp of the masked scores
        s = torch.tensor(np.einsum("hid,hjd->hij", q, k) * scale)
        if mask is not None:
            s = s.masked_fill(~mask, float("-inf"))
        _close(lse, torch.logsumexp(s, dim=-1).numpy(), what="logsumexp")


def pin_negative_scale_sdpa(orc):
    """Any finite scale is used as given, negative ones included: float64 CPU SDPA with the same negative
    scale, causal and not. The scale of -200 puts the scores far beyond exp's range, so a row maximum taken
    the wrong way round (the largest q.k instead of the largest scale * q.k) overflows and is caught."""
    import torch

    r = _rng(19)
    for (Sq, Sk, D, causal, scale) in ((9, 9, 8, True, -0.7), (6, 11, 4, False, -0.35), (8, 8, 4, True, -200.0),
                                       (5, 7, 8, False, -200.0)):
        H = 2
        q = r.standard_normal((H, Sq, D))
        k = r.standard_normal((H, Sk, D))
        v = r.standard_normal((H, Sk, D))
        do = r.standard_normal((H, Sq, D))
        mask = torch.ones(Sq, Sk, dtype=torch.bool).tril(diagonal=Sk - Sq) if causal else None
        o_ref, dq_ref, dk_ref, dv_ref = _sdpa(q, k, v, do, mask, scale)
        out, lse = orc.fwd(q, k, v, causal=causal, scale=scale)
        dq, dk, dv = orc.bwd(q, k, v, do, causal=causal, scale=scale)
        big = max(1.0, abs(scale))
        _close(out, o_ref, what="negative scale O")
        _close(dq, dq_ref, tol=TOL * big, what="negative scale dQ")
        _close(dk, dk_ref, tol=TOL * big, what="negative scale dK")
        _close(dv, dv_ref, what="negative scale dV")
        s_ = torch.tensor(np.einsum("hid,hjd->hij", q, k) * scale)
        if mask is not None:
            s_ = s_.masked_fill(~mask, float("-inf"))
        _close(lse, torch.logsumexp(s_, dim=-1).numpy(), tol=TOL * big, what="negative scale logsumexp")


def pin_causal_alignment(orc):
    r = _rng(10)
    # Sq < Sk: the last query sees every key, like the non-causal result; row i sees i + Sk - Sq + 1 keys.
    q = r.standard_normal((1, 3, 4))
    k = r.standard_normal((1, 7, 4))
    v = r.standard_normal((1, 7, 4))
    oc, lc = orc.fwd(q, k, v, causal=True, scale=0.5)
    on, ln_ = orc.fwd(q, k, v, causal=False, scale=0.5)
    _close(oc[0, 2], on[0, 2], what="last row sees all keys")
    o5, l5 = orc.fwd(q[:, :1], k[:, :5], v[:, :5], causal=False, scale=0.5)
    _close(oc[0, 0], o5[0, 0], what="row 0 sees keys 0..4")
    _close(lc[0, 0], l5[0, 0], what="row 0 LSE")
    # Sq > Sk: the first Sq - Sk rows see no key at all.
    q = r.standard_normal((1, 6, 4))
    k = r.standard_normal((1, 2, 4))
    v = r.standard_normal((1, 2, 4))
    do = r.standard_normal((1, 6, 4))
    out, lse = orc.fwd(q, k, v, causal=True, scale=0.5)
    assert np.all(out[0, :4] == 0.0) and np.all(np.isneginf(lse[0, :4])), "fully masked rows"
    _close(out[0, 4], v[0, 0], what="first visible row sees key 0 only")
    dq, dk, dv = orc.bwd(q, k, v, do, causal=True, scale=0.5)
    assert np.all(dq[0, :4] == 0.0), "fully masked rows have zero dQ"


def pin_default_scale(orc):
    r = _rng(11)
    q, k, v = (r.standard_normal((1, 4, 64)) for _ in range(3))
    o_def, l_def = orc.fwd(q, k, v, scale=None)
    o_8, l_8 = orc.fwd(q, k, v, scale=1.0 / 8.0)
    _close(o_def, o_8, tol=0.0, what="default scale is 1/8 for d=64")
    _close(l_def, l_8, tol=0.0, what="default scale LSE")


def _parse(x):
    if isinstance(x, list):
        return [_parse(e) for e in x]
    if isinstance(x, str):
        coef, _, arg = x.partition("ln")
        c = float(coef) if coef not in ("", "-") else (-1.0 if coef == "-" else 1.0)
        return c * math.log(float(arg))
    return float(x)


def pin_golden_hand_examples(orc):
    with open(os.path.join(HERE, "golden", "hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v, do = (np.array(_parse(c[n]))[None] for n in ("q", "k", "v", "dout"))
        win = tuple(c.get("window", (-1, -1)))
        out, lse = orc.fwd(q, k, v, causal=c["causal"], scale=c["scale"], window=win)
        dq, dk, dv = orc.bwd(q, k, v, do, causal=c["causal"], scale=c["scale"], window=win)
        _close(out[0], _parse(c["out"]), tol=1e-14, what=c["name"] + " O")
        _close(lse[0], _parse(c["lse"]), tol=1e-14, what=c["name"] + " LSE")
        _close(dq[0], _parse(c["dq"]), tol=1e-14, what=c["name"] + " dQ")
        _close(dk[0], _parse(c["dk"]), tol=1e-14, what=c["name"] + " dK")
        _close(dv[0], _parse(c["dv"]), tol=1e-14, what=c["name"] + " dV")


def _repeat_heads(x, group):
    return np.repeat(x, group, axis=0)


def pin_gqa_matches_repeated_kv(orc):
    r = _rng(12)
    for causal, window in ((False, (-1, -1)), (True, (-1, -1)), (True, (2, 0)), (False, (1, 2))):
        nq, nkv, Sq, Sk, D = 6, 2, 7, 9, 4
        q = r.standard_normal((nq, Sq, D))
        k = r.standard_normal((nkv, Sk, D))
        v = r.standard_normal((nkv, Sk, D))
        do = r.standard_normal((nq, Sq, D))
        g = nq // nkv
        o1, l1 = orc.fwd(q, k, v, causal=causal, scale=0.6, window=window)
        o2, l2 = orc.fwd(q, _repeat_heads(k, g), _repeat_heads(v, g), causal=causal, scale=0.6, window=window)
        _close(o1, o2, what="GQA O")
        _close(l1, l2, what="GQA LSE")
        dq1, dk1, dv1 = orc.bwd(q, k, v, do, causal=causal, scale=0.6, window=window)
        dq2, dk2, dv2 = orc.bwd(q, _repeat_heads(k, g), _repeat_heads(v, g), do, causal=causal, scale=0.6,
                                window=window)
        _close(dq1, dq2, what="GQA dQ")
        _close(dk1, dk2.reshape(nkv, g, Sk, D).sum(axis=1), what="GQA dK = group sum")
        _close(dv1, dv2.reshape(nkv, g, Sk, D).sum(axis=1), what="GQA dV = group sum")


def _fd_check(orc, q, k, v, do, causal, scale, window, what):
    h = 1e-6
    dq, dk, dv = orc.bwd(q, k, v, do, causal=causal, scale=scale, window=window)

    def loss(qq, kk, vv):
        out, _ = orc.fwd(qq, kk, vv, causal=causal, scale=scale, window=window)
        return float(np.sum(out * do))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args = {"q": q, "k": k, "v": v}
            xp = x.copy()
            xp[idx] += h
            xm = x.copy()
            xm[idx] -= h
            ap = dict(args, **{name: xp})
            am = dict(args, **{name: xm})
            num[idx] = (loss(ap["q"], ap["k"], ap["v"]) - loss(am["q"], am["k"], am["v"])) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
        zero_ok = np.linalg.norm(num) < 1e-9 and np.linalg.norm(g) < 1e-9
        assert zero_ok or err <= 1e-6, (what, "d" + name, err)


def pin_gqa_and_window_finite_differences(orc):
    r = _rng(13)
    cases = [(4, 2, 4, 4, 2, False, (-1, -1)), (3, 1, 5, 5, 2, True, (-1, -1)), (2, 2, 6, 6, 2, True, (1, 0)),
             (2, 1, 4, 6, 2, False, (1, 1)), (4, 2, 6, 4, 2, True, (2, -1))]
    for (nq, nkv, Sq, Sk, D, causal, window) in cases:
        q = r.standard_normal((nq, Sq, D))
        k = r.standard_normal((nkv, Sk, D))
        v = r.standard_normal((nkv, Sk, D))
        do = r.standard_normal((nq, Sq, D))
        _fd_check(orc, q, k, v, do, causal, 0.7, window, (nq, nkv, Sq, Sk, causal, window))


def pin_window_limits(orc):
    r = _rng(14)
    q = r.standard_normal((2, 6, 3))
    k = r.standard_normal((2, 8, 3))
    v = r.standard_normal((2, 8, 3))
    for causal in (False, True):
        o1, l1 = orc.fwd(q, k, v, causal=causal, scale=0.5)
        o2, l2 = orc.fwd(q, k, v, causal=causal, scale=0.5, window=(100, 100))
        _close(o1, o2, what="wide window = no window")
        _close(l1, l2, what="wide window LSE")
    # (0, 0): only the aligned key c = i + Sk - Sq is visible
    o, l = orc.fwd(q, k, v, causal=False, scale=0.5, window=(0, 0))
    for i in range(6):
        c = i + 2
        _close(o[:, i], v[:, c], what="window (0,0) picks the aligned key")
        _close(l[:, i], 0.5 * np.einsum("hd,hd->h", q[:, i], k[:, c]), what="window (0,0) LSE")
    # rows whose window lies entirely outside the keys see nothing
    o, l = orc.fwd(q[:, :1], k[:, :3], v[:, :3], causal=False, scale=0.5, window=(0, 0))  # c = 0 + 3 - 1 = 2
    _close(o[:, 0], v[:, 2], what="window at the last key")
    qq = r.standard_normal((1, 4, 3))
    o, l = orc.fwd(qq, k[:1, :2], v[:1, :2], causal=True, scale=0.5, window=(0, 0))  # c = i - 2
    assert np.all(o[0, :2] == 0) and np.all(np.isneginf(l[0, :2])), "window before the first key sees nothing"


def pin_window_gqa_sdpa_crosscheck(orc):
    import torch

    r = _rng(15)
    for (nq, nkv, Sq, Sk, D, causal, window) in ((4, 2, 12, 12, 8, True, (3, 0)), (4, 4, 10, 14, 4, False, (2, 3)),
                                                  (6, 3, 9, 9, 4, True, (-1, -1)), (2, 1, 7, 5, 4, False, (1, -1))):
        q = r.standard_normal((nq, Sq, D))
        k = r.standard_normal((nkv, Sk, D))
        v = r.standard_normal((nkv, Sk, D))
        do = r.standard_normal((nq, Sq, D))
        i = torch.arange(Sq)[:, None]
        j = torch.arange(Sk)[None, :]
        c = i + (Sk - Sq)
        mask = torch.ones(Sq, Sk, dtype=torch.bool)
        if causal:
            mask &= j <= c
        if window[0] >= 0:
            mask &= j >= c - window[0]
        if window[1] >= 0:
            mask &= j <= c + window[1]
        tq = torch.tensor(q[None], requires_grad=True)
        tk = torch.tensor(k[None], requires_grad=True)
        tv = torch.tensor(v[None], requires_grad=True)
        o_ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, enable_gqa=True)
        o_ref.backward(torch.tensor(do[None]))
        rows_ok = mask.any(dim=1).numpy()
        out, _ = orc.fwd(q, k, v, causal=causal, window=window)
        dq, dk, dv = orc.bwd(q, k, v, do, causal=causal, window=window)
        _close(out[:, rows_ok], o_ref.detach()[0].numpy()[:, rows_ok], what="SDPA GQA/window O")
        if rows_ok.all():
            _close(dq, tq.grad[0].numpy(), what="SDPA GQA/window dQ")
            _close(dk, tk.grad[0].numpy(), what="SDPA GQA/window dK")
            _close(dv, tv.grad[0].numpy(), what="SDPA GQA/window dV")


def _golden_philox():
    with open(os.path.join(HERE, "golden", "philox_dropout.json")) as f:
        return json.load(f)


def pin_philox_known_answers(orc):
    g = _golden_philox()
    for case in g["philox4x32_10"]:
        ctr = [int(x, 16) for x in case["ctr"]]
        key = [int(x, 16) for x in case["key"]]
        out = orc.philox4x32_10(ctr, key)
        assert out == [int(x, 16) for x in case["out"]], ("Philox4x32-10 known answer", case["ctr"], out)


def pin_dropout_keep_block(orc):
    kb = _golden_philox()["keep_block"]
    keep = orc.dropout_mask(kb["dropout_p"], kb["seed"], kb["offset"], kb["bh"], 4, 4)
    assert np.array_equal(keep, np.array(kb["keep"], bool)), ("hand-derived keep block", keep.astype(int))


def pin_dropout_counter_layout(orc):
    # The published known answers reach only block (0, 0), where the row-block and key-block counter words are
    # equal, so the layout itself (the reading of the dropout stream: word i mod 4, byte j mod 4 of the
    # generator's output for counter (i / 4, j / 4, head number, offset) under key (seed low, seed high)) is
    # checked against the generator, which the known answers pin separately, on a ragged 10 x 19 mask whose
    # blocks have unequal row and key indices.
    p, seed, offset, bh = 0.3, 0x0123456789ABCDEF, 5, 6
    t = math.floor(256 * p + 0.5)
    key = (seed & 0xFFFFFFFF, seed >> 32)
    keep = orc.dropout_mask(p, seed, offset, bh, 10, 19)
    for i in range(10):
        for j in range(19):
            word = orc.philox4x32_10((i // 4, j // 4, bh, offset), key)[i % 4]
            expect = ((word >> (8 * (j % 4))) & 0xFF) >= t
            assert keep[i, j] == expect, ("dropout counter layout", i, j)


def pin_dropout_probability_resolution(orc):
    # Hand-derived cases of the probability's resolution (tests/golden/philox_dropout.json): with V = I the
    # output is P o Z, so every kept element is the undropped P times the case's scale 256 / (256 - t) and
    # every dropped one is 0; probabilities that round to t = 256, or lie outside [0, 1), are rejected.
    res = _golden_philox()["probability_resolution"]
    r = _rng(41)
    S = 32
    q, k = 0.3 * r.standard_normal((1, S, S)), 0.3 * r.standard_normal((1, S, S))  # head dim S, so V = I fits
    eye = np.eye(S)[None]
    plain, _ = orc.fwd(q, k, eye, causal=False, scale=0.5)
    for case in res["cases"]:
        p = case["dropout_p"]
        out, _ = orc.fwd(q, k, eye, causal=False, scale=0.5, dropout=(p, 11, 0))
        keep = orc.dropout_mask(p, 11, 0, 0, S, S)
        assert keep.any(), ("no element kept", p)
        _close(out[0][keep], plain[0][keep] * case["scale"], what="kept scale at p = %g" % p)
        assert not out[0][~keep].any(), ("dropped elements not zero", p)
        if case["t"] == 0:
            assert keep.all(), "t = 0 drops nothing"
    for case in res["rejected"]:
        for call in (lambda: orc.dropout_mask(case["dropout_p"], 11, 0, 0, S, S),
                     lambda: orc.fwd(q, k, eye, causal=False, scale=0.5, dropout=(case["dropout_p"], 11, 0))):
            try:
                call()
            except ValueError:
                continue
            raise AssertionError(("dropout probability accepted", case["dropout_p"]))


def pin_dropout_zero_is_plain(orc):
    r = _rng(16)
    q, k, v, do = (r.standard_normal((2, 7, 3)) for _ in range(4))
    for causal in (False, True):
        o1, l1 = orc.fwd(q, k, v, causal=causal, scale=0.6)
        o2, l2 = orc.fwd(q, k, v, causal=causal, scale=0.6, dropout=(0.0, 99, 3))
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2), "dropout_p = 0 changes the forward"
        g1 = orc.bwd(q, k, v, do, causal=causal, scale=0.6)
        g2 = orc.bwd(q, k, v, do, causal=causal, scale=0.6, dropout=(0.0, 99, 3))
        for a, b in zip(g1, g2):
            assert np.array_equal(a, b), "dropout_p = 0 changes the backward"


def pin_dropout_keep_rate(orc):
    # keep fraction of a 256 x 512 mask within 5 binomial standard deviations of 1 - t/256, for several p;
    # two different seeds, offsets or head numbers agree only as often as independent masks would
    n = 256 * 512
    for p in (0.1, 0.3, 0.5, 0.9):
        t = math.floor(256 * p + 0.5)
        keep_p = 1 - t / 256
        m = orc.dropout_mask(p, 1234, 7, 3, 256, 512)
        assert abs(m.mean() - keep_p) <= 5 * math.sqrt(keep_p * (1 - keep_p) / n), ("keep rate", p, m.mean())
        agree_p = keep_p ** 2 + (1 - keep_p) ** 2
        for other in (orc.dropout_mask(p, 1235, 7, 3, 256, 512), orc.dropout_mask(p, 1234, 8, 3, 256, 512),
                      orc.dropout_mask(p, 1234, 7, 4, 256, 512)):
            agree = (m == other).mean()
            assert abs(agree - agree_p) <= 5 * math.sqrt(agree_p * (1 - agree_p) / n), ("independent masks", p)


def pin_dropout_unbiased(orc):
    # E_seed[O_dropout] = O: each kept probability is scaled by 1 / (1 - p'); LSE ignores dropout
    r = _rng(17)
    q, k, v = (r.standard_normal((1, 3, 2)) for _ in range(3))
    p = 0.25
    pe = math.floor(256 * p + 0.5) / 256
    o_ref, l_ref = orc.fwd(q, k, v, scale=0.9)
    n = 3000
    acc = np.zeros_like(o_ref)
    for seed in range(n):
        o, l = orc.fwd(q, k, v, scale=0.9, dropout=(p, seed, 0))
        assert np.array_equal(l, l_ref), "LSE depends on dropout"
        acc += o
    # variance of one O element: sum_j P_ij^2 v_jd^2 p'/(1-p') <= sum_j P_ij v_jd^2 p'/(1-p'), the latter being
    # the plain forward with V replaced by v_jd^2
    var = np.zeros_like(o_ref)
    for d in range(2):
        vd = np.zeros((1, 3, 2))
        vd[0, :, 0] = v[0, :, d] ** 2
        od, _ = orc.fwd(q, k, vd, scale=0.9)
        var[0, :, d] = od[0, :, 0] * pe / (1 - pe)
    tol = 6 * np.sqrt(np.maximum(var, 0.0) / n) + 1e-12
    assert np.all(np.abs(acc / n - o_ref) <= tol), ("dropout mean", np.abs(acc / n - o_ref).max(), tol.max())


def pin_dropout_identity_values(orc):
    # With Sk = D and V = I, O = (P o Z) itself: P from the plain forward, Z from the exported mask
    r = _rng(18)
    Sq, Sk = 9, 6
    q = r.standard_normal((2, Sq, Sk))
    k = r.standard_normal((2, Sk, Sk))
    eye = np.broadcast_to(np.eye(Sk), (2, Sk, Sk)).copy()
    p = 0.3
    pe = math.floor(256 * p + 0.5) / 256
    for causal in (False, True):
        P, _ = orc.fwd(q, k, eye, causal=causal, scale=0.5)
        heads = np.array([5, 11])
        O, _ = orc.fwd(q, k, eye, causal=causal, scale=0.5, dropout=(p, 42, 9), head_index=heads)
        for h in range(2):
            keep = orc.dropout_mask(p, 42, 9, heads[h], Sq, Sk)
            _close(O[h], P[h] * keep / (1 - pe), what="O = P o Z with V = I")


def pin_dropout_finite_differences(orc):
    r = _rng(19)
    h = 1e-6
    # the second case numbers its heads 7 and 3 (as head b * H + h of a larger batch would be): the backward must
    # regenerate the forward's mask for those head numbers
    for (nq, nkv, Sq, Sk, D, causal, window, p, heads) in ((2, 1, 5, 6, 2, False, (-1, -1), 0.3, None),
                                                            (2, 2, 6, 6, 3, True, (2, 0), 0.5, [7, 3])):
        hidx = None if heads is None else np.array(heads, np.int64)
        q = r.standard_normal((nq, Sq, D))
        k = r.standard_normal((nkv, Sk, D))
        v = r.standard_normal((nkv, Sk, D))
        do = r.standard_normal((nq, Sq, D))
        drop = (p, 77, 1)
        dq, dk, dv = orc.bwd(q, k, v, do, causal=causal, scale=0.7, window=window, dropout=drop, head_index=hidx)

        def loss(qq, kk, vv):
            out, _ = orc.fwd(qq, kk, vv, causal=causal, scale=0.7, window=window, dropout=drop, head_index=hidx)
            return float(np.sum(out * do))

        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                args = {"q": q, "k": k, "v": v}
                xp = x.copy()
                xp[idx] += h
                xm = x.copy()
                xm[idx] -= h
                ap = dict(args, **{name: xp})
                am = dict(args, **{name: xm})
                num[idx] = (loss(ap["q"], ap["k"], ap["v"]) - loss(am["q"], am["k"], am["v"])) / (2 * h)
            err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
            assert err <= 1e-6, ("dropout finite differences d" + name, err)


def pin_value_linearity(orc):
    # O is linear in V, so L = sum_i dO_i . O_i equals sum_j v_j . dV_j exactly (with or without dropout,
    # grouped heads or a window): the gradient reaching V is the one that reproduces the loss.
    r = _rng(20)
    for (nq, nkv, Sq, Sk, D, causal, window, drop) in ((2, 2, 7, 9, 3, False, (-1, -1), None),
                                                       (4, 2, 9, 9, 4, True, (3, 0), None),
                                                       (2, 1, 8, 11, 3, False, (-1, -1), (0.3, 5, 2)),
                                                       (2, 2, 10, 10, 2, True, (4, -1), (0.6, 9, 0))):
        q = r.standard_normal((nq, Sq, D))
        k = r.standard_normal((nkv, Sk, D))
        v = r.standard_normal((nkv, Sk, D))
        do = r.standard_normal((nq, Sq, D))
        out, _ = orc.fwd(q, k, v, causal=causal, scale=0.6, window=window, dropout=drop)
        _, _, dv = orc.bwd(q, k, v, do, causal=causal, scale=0.6, window=window, dropout=drop)
        loss = float(np.sum(out * do))
        _close(float(np.sum(v * dv)), loss, tol=1e-10 * max(1.0, abs(loss)), what="sum v.dV = L")


ALL_PINS = [pin_single_key, pin_identical_keys, pin_first_causal_row, pin_rows_sum_to_one, pin_key_permutation,
            pin_masked_keys_have_no_influence,
            pin_finite_differences, pin_grad_invariants, pin_row_subset, pin_sdpa_crosscheck, pin_negative_scale_sdpa,
            pin_causal_alignment, pin_default_scale, pin_golden_hand_examples, pin_gqa_matches_repeated_kv,
            pin_gqa_and_window_finite_differences, pin_window_limits, pin_window_gqa_sdpa_crosscheck,
            pin_philox_known_answers, pin_dropout_keep_block, pin_dropout_counter_layout,
            pin_dropout_probability_resolution, pin_dropout_zero_is_plain,
            pin_dropout_keep_rate, pin_dropout_unbiased, pin_dropout_identity_values, pin_dropout_finite_differences,
            pin_value_linearity]
