"""Decode against a paged key/value cache: the CUDA kernels (through the C
ABI) against the fp64 oracle on seeded pools, shuffled page tables and mixed
sequence lengths (empty, within one page, page boundaries, long)."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_37_b200 import attn_decode, device_status

from ._util import TOL_LSE, TOL_REL, rel_err, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
PAGE = 128


def make_case(B, Hq, Hkv, Sq, D, lens, seed, extra_pages=5):
    """Seeded bf16 query and page pools, and a shuffled page table covering `lens`."""
    g = torch.Generator().manual_seed(seed)
    max_pages = max(1, max((n + PAGE - 1) // PAGE for n in lens))
    P = B * max_pages + extra_pages
    q = torch.randn(B, Hq, Sq, D, generator=g).to(torch.bfloat16)
    kp = torch.randn(P, PAGE, Hkv, D, generator=g).to(torch.bfloat16)
    vp = torch.randn(P, PAGE, Hkv, D, generator=g).to(torch.bfloat16)
    perm = torch.randperm(P, generator=g)
    table = perm[:B * max_pages].reshape(B, max_pages).to(torch.int32)
    seqlens = torch.tensor(lens, dtype=torch.int32)
    return q, kp, vp, table, seqlens


def run_and_check(q, kp, vp, table, seqlens, causal, scale=None):
    D = q.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o, lse = attn_decode(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), seqlens.to(DEV),
                         causal=causal, scale=scale)
    torch.cuda.synchronize()
    code, where = device_status()
    assert code == 0, f"device status {code} at wait site {where}"
    o_ref, l_ref = oracle.attention_decode(q.float().numpy(), kp.float().numpy(),
                                           vp.float().numpy(), table.numpy(), seqlens.numpy(),
                                           causal, scale, page=PAGE)
    assert rel_err(to_np(o), o_ref) <= TOL_REL
    lg = to_np(lse)
    assert np.array_equal(np.isneginf(lg), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    if fin.any():
        assert float(np.max(np.abs(lg[fin] - l_ref[fin]))) <= TOL_LSE
    return o, lse


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq", [1, 4])
def test_mixed_lengths(D, causal, Sq):
    lens = [0, 1, 127, 128, 129, 700, 2 * PAGE + 5, 3]
    q, kp, vp, table, seqlens = make_case(len(lens), 8, 2, Sq, D, lens, seed=D + Sq + causal)
    run_and_check(q, kp, vp, table, seqlens, causal)


@pytest.mark.parametrize("G,Sq", [(1, 1), (8, 1), (8, 16), (32, 4), (2, 64)])
def test_group_and_token_packing(G, Sq):
    # the M = G * Sq rows of a CTA's query tile pack the group's heads and tokens
    Hkv = 2
    lens = [300, 1000, 40]
    q, kp, vp, table, seqlens = make_case(len(lens), G * Hkv, Hkv, Sq, 128, lens, seed=G * 7 + Sq)
    run_and_check(q, kp, vp, table, seqlens, True)


def test_contiguous_cache_as_identity_pages():
    # a [B, L, Hkv, D] cache is a pool of B * L/128 pages with an identity table
    B, Hq, Hkv, L, D = 2, 4, 2, 512, 128
    g = torch.Generator().manual_seed(80)
    k = torch.randn(B, L, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, Hkv, D, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, 1, D, generator=g).to(torch.bfloat16)
    kp, vp = k.reshape(B * L // PAGE, PAGE, Hkv, D), v.reshape(B * L // PAGE, PAGE, Hkv, D)
    table = torch.arange(B * L // PAGE, dtype=torch.int32).reshape(B, L // PAGE)
    seqlens = torch.tensor([L, L - 77], dtype=torch.int32)
    run_and_check(q, kp, vp, table, seqlens, True)


def test_repeated_runs_agree():
    lens = [5000, 20, 128 * 9]
    q, kp, vp, table, seqlens = make_case(3, 16, 4, 2, 128, lens, seed=90)
    args = [t.to(DEV) for t in (q, kp, vp, table, seqlens)]
    o1, l1 = attn_decode(*args, causal=True)
    for _ in range(3):
        o2, l2 = attn_decode(*args, causal=True)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_long_context_batch():
    # B=4 sequences up to 32768 keys, Hq=32, Hkv=8, one new token (sampled heads)
    B, Hq, Hkv, D = 4, 32, 8, 128
    lens = [32768, 20000, 1, 32768 - 100]
    q, kp, vp, table, seqlens = make_case(B, Hq, Hkv, 1, D, lens, seed=99, extra_pages=0)
    o, lse = attn_decode(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), seqlens.to(DEV),
                         causal=True)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    for h in (0, 7, 8, 31):
        hk = h // (Hq // Hkv)
        o_h, l_h = oracle.attention_decode(q[:, h:h + 1].float().numpy(),
                                           kp[:, :, hk:hk + 1].float().numpy(),
                                           vp[:, :, hk:hk + 1].float().numpy(), table.numpy(),
                                           seqlens.numpy(), True, 1 / math.sqrt(D), page=PAGE)
        assert rel_err(to_np(o[:, h:h + 1]), o_h) <= TOL_REL
        assert float(np.max(np.abs(to_np(lse[:, h:h + 1]) - l_h))) <= TOL_LSE


def test_lengths_outside_the_table_are_clamped():
    """A length beyond what the block-table row holds (128 * max_pages) is taken
    as that maximum, for keys and query positions alike, and a negative length
    as 0 (no key: O = 0, lse = -inf): the result equals the call with the
    clamped lengths."""
    lens = [3 * PAGE, 2 * PAGE - 5]
    q, kp, vp, table, seqlens = make_case(len(lens), 8, 2, 2, 128, lens, seed=123)
    cap = table.shape[1] * PAGE
    args = [t.to(DEV) for t in (q, kp, vp, table)]
    for causal in (False, True):
        clamped = torch.tensor([cap, 0], dtype=torch.int32)
        wild = torch.tensor([cap + 1000, -7], dtype=torch.int32)
        o_c, l_c = attn_decode(*args, clamped.to(DEV), causal=causal)
        o_w, l_w = attn_decode(*args, wild.to(DEV), causal=causal)
        torch.cuda.synchronize()
        assert device_status()[0] == 0
        assert torch.equal(o_c, o_w)
        assert torch.equal(l_c, l_w)
        assert torch.all(o_w[1] == 0) and torch.all(torch.isneginf(l_w[1]))
        run_and_check(q, kp, vp, table, clamped, causal)
