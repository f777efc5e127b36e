"""Forward parity of the CTA-pair kernel (2-CTA tensor-core products,
tcgen05 .cta_group::2) for bf16 inputs with D = 128: against the fp64 oracle
on seeded inputs, and against the single-CTA kernel on the same inputs.

The pair is two query heads of one GQA group when the group size is even,
else two adjacent query tiles of one head; the cases below cover both, with
an odd number of query tiles (the second CTA of the last pair lies past N),
both masks, local windows, forced rescales and the named workloads."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_37_b200 import (attn_fwd, device_status, set_debug_flags,
                                           set_fwd_variant, set_wait_limit_ns)
from exact_tiled_attention_37_b200.inputs import make_inputs, make_random, workload

from ._util import TOL_LSE, TOL_REL, abs_err, rel_err, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128


@pytest.fixture(autouse=True)
def pair_variant():
    set_fwd_variant(2)
    yield
    set_fwd_variant(0)


def fwd(q, k, v, **kw):
    o, lse = attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
    torch.cuda.synchronize()
    code, where = device_status()
    assert code == 0, f"device status {code} at wait site {where}"
    return o, lse


def check(q, k, v, causal=False, window=None, scale=None):
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o, lse = fwd(q, k, v, causal=causal, window=window, scale=scale)
    o_ref, l_ref = oracle.attention_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                        causal, scale, window=window)
    eo, el = rel_err(to_np(o), o_ref), abs_err(to_np(lse), l_ref)
    assert eo <= TOL_REL and el <= TOL_LSE, (eo, el)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 64, 128, 200, 256, 300, 640, 1000])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (6, 2), (8, 2)])
def test_small_shapes(causal, N, hq, hkv):
    # (2, 2): tile pairs; (4, 2), (8, 2): head pairs; (6, 2): group of 3, tile pairs
    q, k, v = make_random(2, hq, hkv, N, D, "bf16", seed=N * 13 + hq + causal, with_do=False)
    check(q, k, v, causal)


@pytest.mark.parametrize("window", [(111, 0), (0, 0), (200, 200), (64, 300), (300, -1),
                                    (-1, 50), (5, 7)])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2)])
def test_windows(window, hq, hkv):
    q, k, v = make_random(1, hq, hkv, 1000, D, "bf16", seed=window[0] + 3 * hq, with_do=False)
    check(q, k, v, window=window)


def test_sharp_softmax_forces_rescales():
    q, k, v = make_random(1, 2, 2, 1000, D, "bf16", seed=77, k_mult=6.0, with_do=False)
    for causal in (False, True):
        check(q, k, v, causal, scale=0.3)


def test_strided_views():
    B, H, N = 2, 4, 300
    g = torch.Generator().manual_seed(5)
    base = [torch.randn(B, N, H, D, generator=g).to(torch.bfloat16) for _ in range(3)]
    q, k, v = (t.to(DEV).transpose(1, 2) for t in base)
    for causal in (False, True):
        o, lse = fwd(q, k, v, causal=causal)
        o_ref, l_ref = oracle.attention_fwd(*(to_np(t) for t in (q, k, v)), causal,
                                            1 / math.sqrt(D))
        assert rel_err(to_np(o), o_ref) <= TOL_REL
        assert abs_err(to_np(lse), l_ref) <= TOL_LSE


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_agrees_with_single_cta_kernel(hq, hkv):
    """Same products per row, same order of key tiles: the pair kernel's
    results match the single-CTA kernel's to rounding (both stay within the
    oracle tolerance); repeated pair runs agree bit for bit."""
    q, k, v = (t.to(DEV) for t in make_random(2, hq, hkv, 777, D, "bf16", seed=9,
                                              with_do=False))
    for causal in (False, True):
        o2, l2 = fwd(q, k, v, causal=causal)
        set_fwd_variant(1)
        o1, l1 = fwd(q, k, v, causal=causal)
        set_fwd_variant(2)
        assert float((o1.float() - o2.float()).abs().max()) <= 2e-2 * float(o1.float().abs().max())
        assert float((l1 - l2).abs().max()) <= 1e-4
        for _ in range(3):
            o3, l3 = fwd(q, k, v, causal=causal)
            assert torch.equal(o2, o3) and torch.equal(l2, l3)


def test_dropped_load_times_out_and_recovers():
    """Both CTAs of every pair skip their half of the first V tile: the
    leader's wait for it runs out, the status word reports it, both CTAs leave
    through the final cluster barrier, and the next call is correct."""
    q, k, v = (t.to(DEV) for t in make_random(1, 2, 2, 384, D, "bf16", seed=4, with_do=False))
    assert device_status()[0] == 0
    set_wait_limit_ns(50_000_000)
    set_debug_flags(1)
    try:
        attn_fwd(q, k, v, causal=False)
        code, where = device_status()
    finally:
        set_debug_flags(0)
        set_wait_limit_ns(0)
    assert code == 6, (code, where)
    o, lse = fwd(q, k, v, causal=False)
    o_ref, _ = oracle.attention_fwd(to_np(q), to_np(k), to_np(v), False, 1 / math.sqrt(D))
    assert rel_err(to_np(o), o_ref) <= TOL_REL


@pytest.mark.parametrize("causal", [False, True])
def test_workload_mha_2048(causal):
    q, k, v = make_inputs(workload(1), with_do=False)
    check(q, k, v, causal)


def _sampled(w, causal, heads, nrows, seed):
    q, k, v = make_inputs(w, with_do=False)
    o, lse = fwd(q, k, v, causal=causal)
    rng = np.random.default_rng(seed)
    worst_o, worst_l = 0.0, 0.0
    for (b, h) in heads:
        rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, w.N - 1],
                                         rng.integers(0, w.N, nrows)]))
        o_ref, l_ref = oracle.attention_fwd_rows(q.float().numpy(), k.float().numpy(),
                                                 v.float().numpy(), causal, w.scale, b, h, rows)
        idx = torch.as_tensor(rows, device=DEV)
        worst_o = max(worst_o, rel_err(to_np(o[b, h, idx]), o_ref))
        worst_l = max(worst_l, abs_err(to_np(lse[b, h, idx]), l_ref))
    assert worst_o <= TOL_REL and worst_l <= TOL_LSE, (worst_o, worst_l)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_workload_mha_4096_causal():
    _sampled(workload(2), True, [(0, 0), (1, 15), (0, 7)], 200, 1)


def test_workload_long_context_gqa():
    _sampled(workload(3), True, [(0, 0), (0, 1), (0, 4), (0, 31)], 96, 2)
