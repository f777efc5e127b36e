"""Local (sliding-window) attention: the CUDA kernels against the fp64 oracle
with the same window, forward and backward, on seeded inputs; plus the
plain causal entry point against its window form."""

import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_37_b200 import _lib, attn_bwd, attn_fwd, device_status
from exact_tiled_attention_37_b200._lib import AttnTensor
from exact_tiled_attention_37_b200.inputs import make_random

from ._util import TOL_LSE, TOL_REL, abs_err, rel_err, to_np

pytestmark = pytest.mark.gpu

WINDOWS = [(111, 0), (0, 0), (200, 200), (64, 300), (1000, 0), (300, -1), (-1, 50), (5, 7)]


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("window", WINDOWS)
@pytest.mark.parametrize("N", [300, 1000])
def test_forward_window(D, window, N):
    q, k, v = make_random(1, 4, 2, N, D, "bf16", seed=N + D + window[0], with_do=False)
    o, lse = attn_fwd(q.cuda(), k.cuda(), v.cuda(), window=window)
    assert device_status()[0] == 0
    o_ref, l_ref = oracle.attention_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                        False, 1 / math.sqrt(D), window=window)
    assert rel_err(to_np(o), o_ref) <= TOL_REL
    assert abs_err(to_np(lse), l_ref) <= TOL_LSE


@pytest.mark.parametrize("window", [(111, 0), (5, 7), (-1, 20)])
def test_forward_window_fp32(window):
    q, k, v = make_random(1, 2, 1, 256, 64, "fp32", seed=5, with_do=False)
    o, lse = attn_fwd(q.cuda(), k.cuda(), v.cuda(), window=window)
    o_ref, l_ref = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), False, 0.125,
                                        window=window)
    assert rel_err(to_np(o), o_ref) <= 1e-4
    assert abs_err(to_np(lse), l_ref) <= 1e-4


@pytest.mark.parametrize("D,store_ds", [(64, True), (128, True), (128, False), (256, True)])
@pytest.mark.parametrize("window", [(111, 0), (0, 0), (200, 200), (64, 300), (-1, 50)])
def test_backward_window(D, window, store_ds):
    N = 700
    q, k, v, do = make_random(1, 4, 2, N, D, "bf16", seed=D + window[1])
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = attn_fwd(qd, kd, vd, window=window)
    dq, dk, dv = attn_bwd(qd, kd, vd, o, lse, dod, window=window, store_ds=store_ds)
    assert device_status()[0] == 0
    ref = oracle.attention_bwd(*(t.float().numpy() for t in (q, k, v, do)), False,
                               1 / math.sqrt(D), window=window)
    for got, r in zip((dq, dk, dv), ref):
        g = to_np(got)
        e = rel_err(g, r) if np.max(np.abs(r)) > 1e-6 else float(np.max(np.abs(g)))
        assert e <= TOL_REL


def test_causal_entry_point_equals_window_form():
    B, H, N, D = 1, 2, 513, 128
    q, k, v = (t.cuda() for t in make_random(B, H, H, N, D, "bf16", seed=9, with_do=False))
    o_w, l_w = attn_fwd(q, k, v, window=(-1, 0))
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device="cuda", dtype=torch.float32)

    def desc(t):
        sb, sh, sn, _ = t.stride()
        return AttnTensor(ctypes.c_void_p(t.data_ptr()), sb, sh, sn)

    code = _lib.lib().attn_fwd(desc(q), desc(k), desc(v), desc(o), ctypes.c_void_p(lse.data_ptr()),
                               B, H, H, N, D, 0, 1, 1 / math.sqrt(D),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0
    torch.cuda.synchronize()
    assert torch.equal(o, o_w) and torch.equal(lse, l_w)
