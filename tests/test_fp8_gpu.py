"""FP8 (e4m3) forward: the CUDA kernel (through the C ABI) against the fp64
oracle run on the dequantised inputs (the e4m3 values times their per-tensor
scales), on seeded inputs."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_37_b200 import attn_fwd_fp8, device_status
from exact_tiled_attention_37_b200.inputs import make_random

from ._util import TOL_LSE, TOL_REL, abs_err, rel_err, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def quantise(x: torch.Tensor):
    """x -> (e4m3 tensor, scale) with x ~ e4m3 * scale (per-tensor scale)."""
    s = float(x.abs().max()) / 240.0
    return (x / s).to(torch.float8_e4m3fn), s


def deq(x8, s):
    return x8.float().numpy() * s


def run(q, k, v, causal, window=None, scale=None):
    (q8, qs), (k8, ks), (v8, vs) = (quantise(t) for t in (q, k, v))
    D = q.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o, lse = attn_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), qs, ks, vs, causal=causal,
                          scale=scale, window=window)
    torch.cuda.synchronize()
    code, where = device_status()
    assert code == 0, f"device status {code} at wait site {where}"
    assert o.dtype == torch.bfloat16
    return o, lse, (deq(q8, qs), deq(k8, ks), deq(v8, vs)), scale


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 200, 256, 700, 2048])
def test_small_shapes(causal, N):
    q, k, v = make_random(1, 4, 2, N, 128, "fp32", seed=N + causal, with_do=False)
    o, lse, (qd, kd, vd), scale = run(q, k, v, causal)
    o_ref, l_ref = oracle.attention_fwd(qd, kd, vd, causal, scale)
    assert rel_err(to_np(o), o_ref) <= TOL_REL
    assert abs_err(to_np(lse), l_ref) <= TOL_LSE


@pytest.mark.parametrize("window", [(111, 0), (200, 200)])
def test_windows(window):
    q, k, v = make_random(2, 2, 2, 900, 128, "fp32", seed=7 + window[0], with_do=False)
    o, lse, (qd, kd, vd), scale = run(q, k, v, False, window=window)
    o_ref, l_ref = oracle.attention_fwd(qd, kd, vd, False, scale, window=window)
    assert rel_err(to_np(o), o_ref) <= TOL_REL
    assert abs_err(to_np(lse), l_ref) <= TOL_LSE


def test_sharp_scores_and_scales():
    # large scores (running maximum grows, P spans many octaves) and scales far from 1
    q, k, v = make_random(1, 2, 1, 1000, 128, "fp32", seed=11, with_do=False)
    q, k, v = q * 40.0, k * 0.05, v * 1e-3
    o, lse, (qd, kd, vd), scale = run(q, k, v, True, scale=0.3)
    o_ref, l_ref = oracle.attention_fwd(qd, kd, vd, True, scale)
    assert rel_err(to_np(o), o_ref) <= TOL_REL
    assert abs_err(to_np(lse), l_ref) <= TOL_LSE


def test_workload_shape_sampled_rows():
    # the 4096-token causal MHA shape, sampled heads and rows
    B, H, N, D = 2, 16, 4096, 128
    q, k, v = make_random(B, H, H, N, D, "fp32", seed=21, with_do=False)
    o, lse, (qd, kd, vd), scale = run(q, k, v, True)
    rows = np.array([0, 1, 127, 128, 2047, 4095])
    for b, h in ((0, 0), (1, 9)):
        o_r, l_r = oracle.attention_fwd_rows(qd, kd, vd, True, scale, b, h, rows)
        assert rel_err(to_np(o[b, h, torch.as_tensor(rows, device=DEV)]), o_r) <= TOL_REL
        assert abs_err(to_np(lse[b, h, torch.as_tensor(rows, device=DEV)]), l_r) <= TOL_LSE
    assert torch.isfinite(o).all()
