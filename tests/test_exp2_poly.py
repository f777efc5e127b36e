"""The FMA-pipe exponential of the softmax kernels: its constants meet the
stated error bound (CPU, emulating the device arithmetic in fp32), and the
device implementation agrees with CUDA's exp2 (GPU, through the C ABI)."""

import ctypes
import os
import re

import numpy as np
import pytest

from exact_tiled_attention_37_b200 import build

PTX = os.path.join(build.CSRC, "ptx.cuh")


def constants():
    text = open(PTX).read()
    return [np.float32(float(re.search(rf"kExp2P{k} = ([0-9.eE+-]+)f;", text).group(1)))
            for k in range(4)]


def poly_exp2_fp32(x):
    """The device algorithm step by step in fp32: round-to-nearest split with
    the 1.5*2^23 constant, degree-3 Horner, exponent-field addition."""
    c0, c1, c2, c3 = constants()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (f * c3 + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_polynomial_error_bound_on_reduced_range():
    f = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    rel = np.abs(poly_exp2_fp32(f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    assert rel.max() < 1e-4


def test_full_range_including_reduction():
    x = np.concatenate([np.linspace(-125.9, 8.0, 200001, dtype=np.float32),
                        np.float32([-1e-7, 0.0, -0.5, 0.5, -1.5, -20.25])])
    rel = np.abs(poly_exp2_fp32(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4
    # below the clamp the result is at most 2^-126 (negligible against a row sum >= 1)
    tiny = poly_exp2_fp32(np.float32([-200.0, -np.inf]))
    assert np.all(tiny >= 0) and np.all(tiny <= 2.0 ** -125)


@pytest.mark.gpu
@pytest.mark.parametrize("mode,tol", [(0, 2e-6), (1, 1e-4)])
def test_device_exp2_matches_cuda(mode, tol):
    import torch

    from exact_tiled_attention_37_b200 import _lib
    x = torch.linspace(-120.0, 8.0, 1 << 20, device="cuda", dtype=torch.float32)
    y = torch.empty_like(x)
    L = _lib.lib()
    code = L.attn_debug_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                             x.numel(), mode,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < tol, rel
