"""Block-sparse attention: the CUDA kernels (through the C ABI) against the
fp64 oracle with the same 128 x 128 tile mask, forward and backward, on
seeded inputs and seeded masks; plus the all-ones mask against the dense path
and repeated runs against each other."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_37_b200 import attn_bwd, attn_fwd, device_status
from exact_tiled_attention_37_b200.inputs import make_random

from ._util import TOL_LSE, TOL_REL, rel_err, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def make_mask(B, H, N, density, seed, empty_row=None):
    """Seeded [B, H, T, T] uint8 tile mask; `empty_row` clears one query tile row."""
    t = (N + 127) // 128
    g = np.random.default_rng(seed)
    m = (g.random((B, H, t, t)) < density).astype(np.uint8)
    if empty_row is not None:
        m[:, :, empty_row, :] = 0
    return m


def check_lse(got, ref):
    g, r = to_np(got), np.asarray(ref)
    assert np.array_equal(np.isneginf(g), np.isneginf(r)), "rows without keys differ"
    fin = np.isfinite(r)
    assert np.all(np.isfinite(g[fin]))
    if fin.any():
        assert float(np.max(np.abs(g[fin] - r[fin]))) <= TOL_LSE


def run(q, k, v, do, causal, window, mask, D, store_ds=True):
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    bm = torch.from_numpy(mask).to(DEV)
    o, lse = attn_fwd(qd, kd, vd, causal=causal, window=window, block_mask=bm)
    dq, dk, dv = attn_bwd(qd, kd, vd, o, lse, dod, causal=causal, window=window, block_mask=bm,
                          store_ds=store_ds)
    torch.cuda.synchronize()
    code, where = device_status()
    assert code == 0, f"device status {code} at wait site {where}"
    return o, lse, dq, dk, dv


def check_all(q, k, v, do, causal, window, mask, D, store_ds=True):
    o, lse, dq, dk, dv = run(q, k, v, do, causal, window, mask, D, store_ds)
    args = [t.float().numpy() for t in (q, k, v)]
    scale = 1 / math.sqrt(D)
    o_ref, l_ref = oracle.attention_fwd(*args, causal, scale, window=window, block_mask=mask)
    assert rel_err(to_np(o), o_ref) <= TOL_REL
    check_lse(lse, l_ref)
    ref = oracle.attention_bwd(*args, do.float().numpy(), causal, scale, window=window,
                               block_mask=mask)
    for got, r in zip((dq, dk, dv), ref):
        g = to_np(got)
        e = rel_err(g, r) if np.max(np.abs(r)) > 1e-6 else float(np.max(np.abs(g)))
        assert e <= TOL_REL


@pytest.mark.parametrize("D,store_ds", [(64, True), (128, True), (128, False)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,density", [(700, 0.5), (1000, 0.3), (1024, 0.8)])
def test_random_masks(D, causal, N, density, store_ds):
    q, k, v, do = make_random(1, 4, 2, N, D, "bf16", seed=N + D + causal)
    mask = make_mask(1, 4, N, density, seed=N * 3 + D, empty_row=1)
    check_all(q, k, v, do, causal, None, mask, D, store_ds)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window", [(200, 0), (64, 300)])
def test_masks_with_windows(D, window):
    N = 900
    q, k, v, do = make_random(2, 2, 1, N, D, "bf16", seed=D + window[0])
    mask = make_mask(2, 2, N, 0.6, seed=D + 7)
    check_all(q, k, v, do, False, window, mask, D)


def test_single_tile_pairs_and_empty_heads():
    # every query tile computes exactly one key tile (a permutation), one head none
    N, D = 640, 128
    q, k, v, do = make_random(1, 3, 3, N, D, "bf16", seed=41)
    t = (N + 127) // 128
    mask = np.zeros((1, 3, t, t), np.uint8)
    perm = np.random.default_rng(42).permutation(t)
    mask[0, 0, np.arange(t), perm] = 1
    mask[0, 1, np.arange(t), np.arange(t)] = 1
    check_all(q, k, v, do, False, None, mask, D)


@pytest.mark.parametrize("D", [64, 128])
def test_all_ones_mask_equals_dense(D):
    N = 777
    q, k, v, do = (t.to(DEV) for t in make_random(2, 4, 2, N, D, "bf16", seed=50 + D))
    t = (N + 127) // 128
    ones = torch.ones(2, 4, t, t, dtype=torch.uint8, device=DEV)
    for causal in (False, True):
        o1, l1 = attn_fwd(q, k, v, causal=causal)
        o2, l2 = attn_fwd(q, k, v, causal=causal, block_mask=ones)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        g1 = attn_bwd(q, k, v, o1, l1, do, causal=causal)
        g2 = attn_bwd(q, k, v, o1, l1, do, causal=causal, block_mask=ones)
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)


def test_repeated_runs_agree():
    N, D = 1500, 128
    q, k, v, do = (t.to(DEV) for t in make_random(1, 4, 1, N, D, "bf16", seed=60))
    bm = torch.from_numpy(make_mask(1, 4, N, 0.4, seed=61, empty_row=2)).to(DEV)
    o, lse = attn_fwd(q, k, v, causal=True, block_mask=bm)
    first = [t.clone() for t in attn_bwd(q, k, v, o, lse, do, causal=True, block_mask=bm)]
    for _ in range(3):
        o2, l2 = attn_fwd(q, k, v, causal=True, block_mask=bm)
        assert torch.equal(o, o2) and torch.equal(lse, l2)
        again = attn_bwd(q, k, v, o, lse, do, causal=True, block_mask=bm)
        for a, b in zip(first, again):
            assert torch.equal(a, b)


def test_long_sequence_sampled_rows():
    # local band of tiles plus a strided set of global tiles, N = 8192
    B, H, N, D = 1, 2, 8192, 128
    q, k, v, _ = make_random(B, H, H, N, D, "bf16", seed=70)
    t = N // 128
    i = np.arange(t)[:, None]
    j = np.arange(t)[None, :]
    mask = ((np.abs(i - j) <= 2) | (j % 8 == 0)).astype(np.uint8)
    mask = np.broadcast_to(mask, (B, H, t, t)).copy()
    bm = torch.from_numpy(mask).to(DEV)
    o, lse = attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, block_mask=bm)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    rows = np.array([0, 1, 127, 128, 1000, 4095, 4096, 8000, 8191])
    for h in range(H):
        o_ref, l_ref = oracle.attention_fwd_rows(q.float().numpy(), k.float().numpy(),
                                                 v.float().numpy(), True, 1 / math.sqrt(D), 0, h,
                                                 rows, block_mask=mask)
        assert rel_err(to_np(o[0, h, torch.as_tensor(rows, device=DEV)]), o_ref) <= TOL_REL
        check_lse(lse[0, h, torch.as_tensor(rows, device=DEV)], l_ref)
