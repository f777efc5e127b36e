"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test checks the oracle against a closed form, an invariant of the exact
attention definition, a hand-worked example (tests/golden/hand_worked.json),
brute-force finite differences, or a library special case.  A plausible bug
(a dropped term, a wrong sign or index, a transposed operand, a wrong head
map, an off-by-one mask) fails at least one of them; ``test_mutants_are_caught``
plants such bugs in copies of the oracle and checks that.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def fwd(q, k, v, causal, scale):
    return oracle.attention_fwd(q, k, v, causal, scale)


# ---------------------------------------------------------------- golden


def test_hand_worked_examples():
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        q = np.array(c["q"])[None, None]
        k = np.array(c["k"])[None, None]
        v = np.array(c["v"])[None, None]
        for causal, ok, lk in ((False, "o", "lse"), (True, "o_causal", "lse_causal")):
            o, lse = fwd(q, k, v, causal, c["scale"])
            np.testing.assert_allclose(o[0, 0], np.array(c[ok]), rtol=0, atol=1e-14)
            np.testing.assert_allclose(lse[0, 0], np.array(c[lk]), rtol=0, atol=1e-14)
        if "backward" in c:
            bw = c["backward"]
            do = np.array(bw["do"])[None, None]
            dq, dk, dv = oracle.attention_bwd(q, k, v, do, False, c["scale"])
            np.testing.assert_allclose(dq[0, 0], np.array(bw["dq"]), atol=1e-14)
            np.testing.assert_allclose(dk[0, 0], np.array(bw["dk"]), atol=1e-14)
            np.testing.assert_allclose(dv[0, 0], np.array(bw["dv"]), atol=1e-14)


# ---------------------------------------------------------------- forward


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    q, k = rnd((7, 5), 1), rnd((7, 5), 2)
    s = oa._scores(q, k, np.arange(7), causal, 0.4)
    p, _ = oracle.softmax_probs(s)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    if causal:
        assert np.all(p[np.triu_indices(7, 1)] == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_values(causal):
    n, d = 11, 6
    q = np.zeros((1, 1, n, d))
    k, v = rnd((1, 1, n, d), 3) * 4, rnd((1, 1, n, d), 4)
    o, lse = fwd(q, k, v, causal, 0.7)
    if causal:
        expect = np.cumsum(v[0, 0], axis=0) / np.arange(1, n + 1)[:, None]
        expect_lse = np.log(np.arange(1, n + 1))
    else:
        expect = np.broadcast_to(v[0, 0].mean(axis=0), (n, d))
        expect_lse = np.full(n, math.log(n))
    np.testing.assert_allclose(o[0, 0], expect, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], expect_lse, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_one_hot_keys_closed_form(causal):
    # Q_i = e_i, K_j = alpha e_j (N <= D): s_ij = a if i == j else 0 with a = alpha*scale.
    n, d, alpha, scale = 5, 8, 7.0, 0.5
    a = alpha * scale
    q = np.zeros((1, 1, n, d))
    k = np.zeros((1, 1, n, d))
    for i in range(n):
        q[0, 0, i, i] = 1.0
        k[0, 0, i, i] = alpha
    v = rnd((1, 1, n, d), 5)
    o, lse = fwd(q, k, v, causal, scale)
    for i in range(n):
        allowed = range(i + 1) if causal else range(n)
        ni = len(allowed)
        num = math.exp(a) * v[0, 0, i] + sum(v[0, 0, j] for j in allowed if j != i)
        np.testing.assert_allclose(o[0, 0, i], num / (math.exp(a) + ni - 1), atol=1e-13)
        assert abs(lse[0, 0, i] - math.log(math.exp(a) + ni - 1)) < 1e-13
    # a large a selects a single value row
    k2 = k * 60.0
    o2, _ = fwd(q, k2, v, causal, scale)
    np.testing.assert_allclose(o2[0, 0], v[0, 0], atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_value_shift_and_key_shift(causal):
    b, h, n, d, scale = 2, 3, 9, 4, 0.6
    q, k, v = rnd((b, h, n, d), 6), rnd((b, h, n, d), 7), rnd((b, h, n, d), 8)
    o, lse = fwd(q, k, v, causal, scale)
    w = rnd((d,), 9)
    o_w, lse_w = fwd(q, k, v + w, causal, scale)
    np.testing.assert_allclose(o_w, o + w, atol=1e-12)
    np.testing.assert_allclose(lse_w, lse, atol=1e-12)
    u = rnd((d,), 10)
    o_u, lse_u = fwd(q, k + u, v, causal, scale)
    np.testing.assert_allclose(o_u, o, atol=1e-12)
    np.testing.assert_allclose(lse_u, lse + scale * np.einsum("bhnd,d->bhn", q, u), atol=1e-12)


def test_key_permutation_invariance_noncausal():
    n, d = 13, 5
    q, k, v = rnd((1, 2, n, d), 11), rnd((1, 2, n, d), 12), rnd((1, 2, n, d), 13)
    perm = np.random.default_rng(14).permutation(n)
    o, lse = fwd(q, k, v, False, 0.3)
    o_p, lse_p = fwd(q, k[:, :, perm], v[:, :, perm], False, 0.3)
    np.testing.assert_allclose(o_p, o, atol=1e-12)
    np.testing.assert_allclose(lse_p, lse, atol=1e-12)
    # causal is NOT permutation invariant: guards against a mask that is ignored
    o_c, _ = fwd(q, k, v, True, 0.3)
    o_cp, _ = fwd(q, k[:, :, perm], v[:, :, perm], True, 0.3)
    assert np.max(np.abs(o_c - o_cp)) > 1e-3


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_returns_value(causal):
    q, k, v = rnd((2, 2, 1, 3), 15), rnd((2, 2, 1, 3), 16), rnd((2, 2, 1, 3), 17)
    o, lse = fwd(q, k, v, causal, 0.9)
    np.testing.assert_allclose(o, v, atol=1e-15)
    np.testing.assert_allclose(lse, 0.9 * np.sum(q * k, axis=-1), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_mha_with_repeated_heads(causal):
    b, hq, hkv, n, d = 2, 6, 2, 10, 4
    q = rnd((b, hq, n, d), 18)
    k, v = rnd((b, hkv, n, d), 19), rnd((b, hkv, n, d), 20)
    do = rnd((b, hq, n, d), 21)
    g = hq // hkv
    # contiguous groups: query head h reads key/value head h // g
    k_rep, v_rep = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    o, lse = fwd(q, k, v, causal, 0.5)
    o_r, lse_r = fwd(q, k_rep, v_rep, causal, 0.5)
    np.testing.assert_allclose(o, o_r, atol=1e-13)
    np.testing.assert_allclose(lse, lse_r, atol=1e-13)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, 0.5)
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k_rep, v_rep, do, causal, 0.5)
    np.testing.assert_allclose(dq, dq_r, atol=1e-12)
    np.testing.assert_allclose(dk, dk_r.reshape(b, hkv, g, n, d).sum(axis=2), atol=1e-12)
    np.testing.assert_allclose(dv, dv_r.reshape(b, hkv, g, n, d).sum(axis=2), atol=1e-12)


def test_rows_helper_matches_full():
    q, k, v = rnd((1, 4, 40, 8), 22), rnd((1, 2, 40, 8), 23), rnd((1, 2, 40, 8), 24)
    for causal in (False, True):
        o, lse = fwd(q, k, v, causal, 0.35)
        rows = [0, 7, 39, 21]
        o_r, lse_r = oracle.attention_fwd_rows(q, k, v, causal, 0.35, 0, 3, rows)
        np.testing.assert_allclose(o_r, o[0, 3, rows], atol=1e-13)
        np.testing.assert_allclose(lse_r, lse[0, 3, rows], atol=1e-13)


def test_matches_torch_sdpa_fp64_second_opinion():
    # library special case on the single-head fp32 workload shape (N=256, D=64)
    from exact_tiled_attention_37_b200.inputs import make_inputs, workload
    w = workload(0)
    q, k, v = make_inputs(w, with_do=False)
    for causal in (False, True):
        o, _ = fwd(q.numpy(), k.numpy(), v.numpy(), causal, w.scale)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.double(), k.double(), v.double(), is_causal=causal, scale=w.scale)
        np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)


# ---------------------------------------------------------------- backward


def _loss(q, k, v, do, causal, scale):
    o, _ = fwd(q, k, v, causal, scale)
    return float(np.sum(o * do))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(1, 1), (2, 1)])
def test_backward_matches_finite_differences(causal, hq, hkv):
    n, d, scale, h = 6, 3, 0.8, 1e-6
    q, k, v = rnd((1, hq, n, d), 30), rnd((1, hkv, n, d), 31), rnd((1, hkv, n, d), 32)
    do = rnd((1, hq, n, d), 33)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, scale)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (_loss(**args_p, do=do, causal=causal, scale=scale)
                       - _loss(**args_m, do=do, causal=causal, scale=scale)) / (2 * h)
        err = np.max(np.abs(fd - g)) / max(np.max(np.abs(g)), 1e-30)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_column_sums(causal):
    # rows of dS sum to zero => sum_j dK_j = 0; sum_j dV_j = sum_i dO_i
    q, k, v, do = (rnd((2, 2, 12, 5), s) for s in (40, 41, 42, 43))
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, 0.45)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-12)


def test_backward_head_subset():
    q, do = rnd((2, 4, 9, 3), 50), rnd((2, 4, 9, 3), 51)
    k, v = rnd((2, 2, 9, 3), 52), rnd((2, 2, 9, 3), 53)
    full = oracle.attention_bwd(q, k, v, do, True, 0.5)
    part = oracle.attention_bwd(q, k, v, do, True, 0.5, heads=[(1, 0)])
    for f, p in zip(full[:1], part[:1]):
        np.testing.assert_allclose(p[1, 0:2], f[1, 0:2], atol=1e-14)
    for f, p in zip(full[1:], part[1:]):
        np.testing.assert_allclose(p[1, 0], f[1, 0], atol=1e-14)
        assert np.isnan(p[0, 0]).all()


# ---------------------------------------------------------------- mutants


def _run_pins():
    """A quick subset of the pins above; returns the names that fail."""
    failed = []
    checks = {
        "golden": test_hand_worked_examples,
        "zero_q_causal": lambda: test_zero_query_gives_mean_of_values(True),
        "one_hot": lambda: test_one_hot_keys_closed_form(False),
        "gqa": lambda: test_gqa_equals_mha_with_repeated_heads(True),
        "fd": lambda: test_backward_matches_finite_differences(True, 2, 1),
        "colsum": lambda: test_backward_column_sums(False),
    }
    for name, fn in checks.items():
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


def test_mutants_are_caught(monkeypatch):
    assert _run_pins() == []

    def off_by_one_mask(q_rows, k_all, row_ids, causal, scale, window=None, block_mask=None,
                        block=128):
        s = scale * (q_rows @ k_all.T)
        if causal:
            cols = np.arange(k_all.shape[0])
            s = np.where(cols[None, :] >= row_ids[:, None], -np.inf, s)
            s[:, 0] = np.where(np.isinf(s[:, 0]), 0.0, s[:, 0])
        return s

    def dropped_scale(q_rows, k_all, row_ids, causal, scale, window=None, block_mask=None,
                      block=128):
        return oa.__dict__["_orig_scores"](q_rows, k_all, row_ids, causal, 1.0, window,
                                           block_mask, block)

    def lse_without_max(s):
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        z = np.sum(e, axis=1, keepdims=True)
        return e / z, np.log(z)[:, 0]

    oa.__dict__["_orig_scores"] = oa._scores
    try:
        for name, attr, mutant in (("mask", "_scores", off_by_one_mask),
                                   ("scale", "_scores", dropped_scale),
                                   ("lse", "softmax_probs", lse_without_max)):
            with monkeypatch.context() as mp:
                mp.setattr(oa, attr, mutant)
                assert _run_pins(), f"mutant {name} not caught"
    finally:
        del oa.__dict__["_orig_scores"]


def test_mutant_backward_without_row_term(monkeypatch):
    src_bwd = oa.attention_bwd

    def bwd_no_row_term(q, k, v, do, causal, scale, heads=None):
        # same as the oracle but dS = P * dP (row term dropped)
        q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
        g = q.shape[1] // k.shape[1]
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for b in range(q.shape[0]):
            for h in range(q.shape[1]):
                hk = h // g
                rows = np.arange(q.shape[2])
                p, _ = oracle.softmax_probs(oa._scores(q[b, h], k[b, hk], rows, causal, scale))
                dp = do[b, h] @ v[b, hk].T
                ds = p * dp
                dv[b, hk] += p.T @ do[b, h]
                dq[b, h] = scale * ds @ k[b, hk]
                dk[b, hk] += scale * ds.T @ q[b, h]
        return dq, dk, dv

    monkeypatch.setattr(oracle, "attention_bwd", bwd_no_row_term)
    failed = _run_pins()
    assert "fd" in failed or "colsum" in failed
    monkeypatch.setattr(oracle, "attention_bwd", src_bwd)


# ---------------------------------------------------------------- local windows


def _brute_window(q, k, v, wl, wr, scale):
    """Explicit loops over (i, j) for one head: the window definition written out."""
    n = q.shape[0]
    o = np.zeros_like(v)
    lse = np.zeros(n)
    for i in range(n):
        js = [j for j in range(n) if (wl < 0 or j >= i - wl) and (wr < 0 or j <= i + wr)]
        sc = np.array([scale * float(q[i] @ k[j]) for j in js])
        w = np.exp(sc - sc.max())
        o[i] = sum(wj * v[j] for wj, j in zip(w, js)) / w.sum()
        lse[i] = sc.max() + math.log(w.sum())
    return o, lse


@pytest.mark.parametrize("wl,wr", [(0, 0), (2, 0), (3, 1), (-1, 2), (1, -1), (100, 100)])
def test_window_matches_explicit_loops(wl, wr):
    q, k, v = rnd((9, 4), 60), rnd((9, 4), 61), rnd((9, 4), 62)
    o, lse = oracle.attention_fwd(q[None, None], k[None, None], v[None, None], False, 0.7,
                                  window=(wl, wr))
    o_b, lse_b = _brute_window(q, k, v, wl, wr, 0.7)
    np.testing.assert_allclose(o[0, 0], o_b, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], lse_b, atol=1e-13)


def test_window_special_cases():
    q, k, v = rnd((1, 2, 12, 5), 63), rnd((1, 2, 12, 5), 64), rnd((1, 2, 12, 5), 65)
    full, lf = fwd(q, k, v, False, 0.4)
    caus, lc = fwd(q, k, v, True, 0.4)
    for win, (o_ref, l_ref) in (((-1, -1), (full, lf)), ((12, 12), (full, lf)),
                                ((-1, 0), (caus, lc)), ((11, 0), (caus, lc))):
        o, l = oracle.attention_fwd(q, k, v, False, 0.4, window=win)
        np.testing.assert_allclose(o, o_ref, atol=1e-13)
        np.testing.assert_allclose(l, l_ref, atol=1e-13)
    # a zero-width window: every query sees only its own key
    o, l = oracle.attention_fwd(q, k, v, False, 0.4, window=(0, 0))
    np.testing.assert_allclose(o, v, atol=1e-14)
    np.testing.assert_allclose(l, 0.4 * np.sum(q * k, axis=-1), atol=1e-13)


def test_zero_query_window_mean():
    # Q = 0: O_i is the mean of V over the window [max(0, i - w), i]; lse = log(count)
    n, d, w = 10, 3, 3
    v = rnd((1, 1, n, d), 66)
    o, l = oracle.attention_fwd(np.zeros((1, 1, n, d)), rnd((1, 1, n, d), 67), v, True, 0.5,
                                window=(w, 0))
    for i in range(n):
        lo = max(0, i - w)
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, lo:i + 1].mean(axis=0), atol=1e-13)
        assert abs(l[0, 0, i] - math.log(i + 1 - lo)) < 1e-13


@pytest.mark.parametrize("window", [(2, 0), (1, 2)])
def test_window_backward_finite_differences(window):
    n, d, scale, h = 6, 3, 0.8, 1e-6
    q, k, v, do = (rnd((1, 2, n, d), s) for s in (70, 71, 72, 73))
    k, v = k[:, :1], v[:, :1]
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, False, scale, window=window)

    def loss(qq, kk, vv):
        o, _ = oracle.attention_fwd(qq, kk, vv, False, scale, window=window)
        return float(np.sum(o * do))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(args_p["q"], args_p["k"], args_p["v"])
                       - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
        err = np.max(np.abs(fd - g)) / max(np.max(np.abs(g)), 1e-30)
        assert err < 1e-6, (name, err)


# ---------------------------------------------------------------- block-sparse masks


def _brute_block(q, k, v, bm, blk, scale, causal):
    """Explicit loops over (i, j) for one head: the block-mask definition written out."""
    n = q.shape[0]
    o = np.zeros_like(v)
    lse = np.full(n, -np.inf)
    for i in range(n):
        js = [j for j in range(n) if bm[i // blk][j // blk] and (not causal or j <= i)]
        if not js:
            continue  # no visible key: O = 0, lse = -inf
        sc = [scale * float(q[i] @ k[j]) for j in js]
        mx = max(sc)
        w = [math.exp(x - mx) for x in sc]
        tot = sum(w)
        o[i] = sum(wj * v[j] for wj, j in zip(w, js)) / tot
        lse[i] = mx + math.log(tot)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_matches_explicit_loops(causal):
    n, d, blk = 10, 4, 3  # 4 x 4 tiles, ragged last tile
    q, k, v = rnd((n, d), 80), rnd((n, d), 81), rnd((n, d), 82)
    bm = np.array([[1, 0, 1, 0], [0, 1, 0, 0], [1, 1, 0, 1], [0, 0, 0, 1]], dtype=np.uint8)
    o, lse = oracle.attention_fwd(q[None, None], k[None, None], v[None, None], causal, 0.6,
                                  block_mask=bm[None, None], block=blk)
    o_b, lse_b = _brute_block(q, k, v, bm, blk, 0.6, causal)
    np.testing.assert_allclose(o[0, 0], o_b, atol=1e-13)
    np.testing.assert_array_equal(np.isinf(lse[0, 0]), np.isinf(lse_b))
    fin = np.isfinite(lse_b)
    np.testing.assert_allclose(lse[0, 0][fin], lse_b[fin], atol=1e-13)


def test_block_mask_special_cases():
    b, h, n, d, blk = 1, 2, 12, 5, 4
    q, k, v = rnd((b, h, n, d), 83), rnd((b, h, n, d), 84), rnd((b, h, n, d), 85)
    t = n // blk
    full, lf = fwd(q, k, v, False, 0.45)
    caus, lc = fwd(q, k, v, True, 0.45)
    ones = np.ones((b, h, t, t), np.uint8)
    lower = np.broadcast_to(np.tril(np.ones((t, t), np.uint8)), (b, h, t, t))
    for causal, bm, (o_ref, l_ref) in ((False, ones, (full, lf)), (True, ones, (caus, lc)),
                                       (True, lower, (caus, lc))):
        o, l = oracle.attention_fwd(q, k, v, causal, 0.45, block_mask=bm, block=blk)
        np.testing.assert_allclose(o, o_ref, atol=1e-13)
        np.testing.assert_allclose(l, l_ref, atol=1e-13)
    # block-diagonal mask = independent attention on each tile of rows
    diag = np.broadcast_to(np.eye(t, dtype=np.uint8), (b, h, t, t))
    o, l = oracle.attention_fwd(q, k, v, False, 0.45, block_mask=diag, block=blk)
    for s in range(t):
        sl = slice(s * blk, (s + 1) * blk)
        o_s, l_s = fwd(q[:, :, sl], k[:, :, sl], v[:, :, sl], False, 0.45)
        np.testing.assert_allclose(o[:, :, sl], o_s, atol=1e-13)
        np.testing.assert_allclose(l[:, :, sl], l_s, atol=1e-13)


def test_block_mask_empty_rows():
    # query tile 1 sees no key tile: O = 0, lse = -inf, no gradient through it
    b, h, n, d, blk = 1, 1, 8, 3, 4
    q, k, v, do = (rnd((b, h, n, d), s) for s in (86, 87, 88, 89))
    bm = np.array([[[[1, 1], [0, 0]]]], np.uint8)
    o, l = oracle.attention_fwd(q, k, v, False, 0.5, block_mask=bm, block=blk)
    assert np.all(o[0, 0, 4:] == 0.0) and np.all(l[0, 0, 4:] == -np.inf)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, False, 0.5, block_mask=bm, block=blk)
    assert np.all(dq[0, 0, 4:] == 0.0)
    # the other rows are plain attention over all keys, unaffected by dO of empty rows
    do2 = do.copy()
    do2[0, 0, 4:] = 17.0
    dq2, dk2, dv2 = oracle.attention_bwd(q, k, v, do2, False, 0.5, block_mask=bm, block=blk)
    np.testing.assert_allclose(dk2, dk, atol=1e-14)
    np.testing.assert_allclose(dv2, dv, atol=1e-14)
    o_full, _ = fwd(q, k, v, False, 0.5)
    np.testing.assert_allclose(o[0, 0, :4], o_full[0, 0, :4], atol=1e-13)


def test_block_mask_backward_finite_differences():
    n, d, scale, h, blk = 6, 3, 0.8, 1e-6, 2
    q, k, v, do = (rnd((1, 2, n, d), s) for s in (90, 91, 92, 93))
    k, v = k[:, :1], v[:, :1]
    bm = np.array([[[[1, 0, 1], [1, 1, 0], [0, 1, 1]], [[0, 1, 0], [1, 0, 1], [1, 1, 1]]]],
                  np.uint8)
    kw = dict(block_mask=bm, block=blk)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, False, scale, **kw)

    def loss(qq, kk, vv):
        o, _ = oracle.attention_fwd(qq, kk, vv, False, scale, **kw)
        return float(np.sum(o * do))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(args_p["q"], args_p["k"], args_p["v"])
                       - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
        err = np.max(np.abs(fd - g)) / max(np.max(np.abs(g)), 1e-30)
        assert err < 1e-6, (name, err)


def test_block_mask_transposed_mutant_is_caught(monkeypatch):
    orig = oa._scores

    def transposed(q_rows, k_all, row_ids, causal, scale, window=None, block_mask=None,
                   block=128):
        bm = None if block_mask is None else np.asarray(block_mask).T
        return orig(q_rows, k_all, row_ids, causal, scale, window, bm, block)

    monkeypatch.setattr(oa, "_scores", transposed)
    with pytest.raises(AssertionError):
        test_block_mask_matches_explicit_loops(False)


# ---------------------------------------------------------------- paged decode


def _paged(k, v, page, seed):
    """Scatter contiguous [B, Hkv, L, D] keys/values into a shuffled page pool."""
    b_, hkv, n, d = k.shape
    npg = (n + page - 1) // page
    total = b_ * npg + 3  # a few unused pages in the pool
    perm = np.random.default_rng(seed).permutation(total)
    kp = rnd((total, page, hkv, d), seed + 1)  # garbage in unused rows
    vp = rnd((total, page, hkv, d), seed + 2)
    table = np.zeros((b_, npg), np.int64)
    for b in range(b_):
        for p in range(npg):
            pg = perm[b * npg + p]
            table[b, p] = pg
            rows = np.arange(p * page, min(n, (p + 1) * page))
            kp[pg, rows - p * page] = k[b][:, rows].transpose(1, 0, 2)
            vp[pg, rows - p * page] = v[b][:, rows].transpose(1, 0, 2)
    return kp, vp, table


@pytest.mark.parametrize("causal", [False, True])
def test_decode_full_prefill_equals_attention(causal):
    # Sq = L: every token is new; bottom-right alignment is then top-left
    b_, hq, hkv, n, d, page = 2, 4, 2, 11, 5, 4
    q, k, v = rnd((b_, hq, n, d), 100), rnd((b_, hkv, n, d), 101), rnd((b_, hkv, n, d), 102)
    kp, vp, table = _paged(k, v, page, 103)
    o, l = oracle.attention_decode(q, kp, vp, table, [n] * b_, causal, 0.55, page=page)
    o_r, l_r = fwd(q, k, v, causal, 0.55)
    np.testing.assert_allclose(o, o_r, atol=1e-13)
    np.testing.assert_allclose(l, l_r, atol=1e-13)


def test_decode_last_tokens_bottom_right_aligned():
    # Sq newest tokens of length-L sequences = rows L-Sq .. L-1 of full causal attention
    b_, hq, hkv, d, page, sq = 3, 2, 1, 4, 5, 3
    lens = [13, 7, 3]
    n = max(lens)
    qfull, k, v = rnd((b_, hq, n, d), 110), rnd((b_, hkv, n, d), 111), rnd((b_, hkv, n, d), 112)
    kp, vp, table = _paged(k, v, page, 113)
    q = np.zeros((b_, hq, sq, d))
    for b, L in enumerate(lens):
        q[b] = qfull[b, :, L - sq:L]
    o, l = oracle.attention_decode(q, kp, vp, table, lens, True, 0.7, page=page)
    for b, L in enumerate(lens):
        for h in range(hq):
            o_r, l_r = oracle.attention_fwd_rows(qfull[b:b + 1, :, :L], k[b:b + 1, :, :L],
                                                 v[b:b + 1, :, :L], True, 0.7, 0, h,
                                                 np.arange(L - sq, L))
            np.testing.assert_allclose(o[b, h], o_r, atol=1e-13)
            np.testing.assert_allclose(l[b, h], l_r, atol=1e-13)


def test_decode_single_token_explicit_loops_and_empty():
    b_, hq, hkv, d, page = 2, 2, 2, 3, 4
    lens = [6, 0]
    k, v = rnd((b_, hkv, 6, d), 120), rnd((b_, hkv, 6, d), 121)
    q = rnd((b_, hq, 1, d), 122)
    kp, vp, table = _paged(k, v, page, 123)
    for causal in (False, True):
        o, l = oracle.attention_decode(q, kp, vp, table, lens, causal, 0.9, page=page)
        for h in range(hq):
            sc = [0.9 * float(q[0, h, 0] @ k[0, h, j]) for j in range(6)]
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            np.testing.assert_allclose(o[0, h, 0], sum(wj * k_ for wj, k_ in zip(w, v[0, h])) / sum(w),
                                       atol=1e-13)
            assert abs(l[0, h, 0] - (mx + math.log(sum(w)))) < 1e-13
        # an empty sequence: no key, O = 0, lse = -inf
        assert np.all(o[1] == 0.0) and np.all(l[1] == -np.inf)


def test_decode_gqa_and_page_order():
    b_, hq, hkv, n, d, page, sq = 2, 6, 2, 9, 4, 4, 2
    q, k, v = rnd((b_, hq, sq, d), 130), rnd((b_, hkv, n, d), 131), rnd((b_, hkv, n, d), 132)
    kp, vp, table = _paged(k, v, page, 133)
    kp2, vp2, table2 = _paged(k, v, page, 140)  # another page shuffle
    o, l = oracle.attention_decode(q, kp, vp, table, [n, n - 2], True, 0.6, page=page)
    o2, l2 = oracle.attention_decode(q, kp2, vp2, table2, [n, n - 2], True, 0.6, page=page)
    np.testing.assert_allclose(o, o2, atol=1e-14)
    np.testing.assert_allclose(l, l2, atol=1e-14)
    g = hq // hkv
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    kp3, vp3, table3 = _paged(kr, vr, page, 133)
    o3, l3 = oracle.attention_decode(q, kp3, vp3, table3, [n, n - 2], True, 0.6, page=page)
    np.testing.assert_allclose(o, o3, atol=1e-13)
    np.testing.assert_allclose(l, l3, atol=1e-13)


def test_decode_top_left_mutant_is_caught(monkeypatch):
    src = oa.attention_decode

    def top_left(q, k_pool, v_pool, block_table, seqlens, causal, scale, page=128):
        # wrong alignment: query token i at position i instead of L - Sq + i
        sq = np.asarray(q).shape[2]
        o, l = src(q, k_pool, v_pool, block_table, [sq] * len(seqlens), causal, scale, page)
        return o, l

    monkeypatch.setattr(oracle, "attention_decode", top_left)
    with pytest.raises(AssertionError):
        test_decode_last_tokens_bottom_right_aligned()
