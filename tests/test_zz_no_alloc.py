"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (it uses the library's fixed 64 MiB scratch array instead of a
caller-provided workspace).  Its gradients must match the workspace entry
point attn_bwd on the same inputs, on two calls in a row (the second call
reuses the scratch the first one left behind).  This file is collected last
so that a run stopping at the first failure has run every other test."""

import ctypes
import math

import pytest
import torch

from exact_tiled_attention_37_b200 import _lib, attn_bwd, attn_fwd, device_status
from exact_tiled_attention_37_b200._lib import AttnTensor
from exact_tiled_attention_37_b200.inputs import make_random

from ._util import TOL_REL, rel_err, to_np

pytestmark = pytest.mark.gpu


def _desc(t):
    sb, sh, sn, _ = t.stride()
    return AttnTensor(ctypes.c_void_p(t.data_ptr()), sb, sh, sn)


def _noalloc():
    L = _lib.lib()
    f = L.attn_bwd_noalloc
    T, i, vp = AttnTensor, ctypes.c_int, ctypes.c_void_p
    f.restype = i
    f.argtypes = [T, T, T, T, vp, T, T, T, T, i, i, i, i, i, i, i, ctypes.c_float, vp]
    return f


@pytest.mark.parametrize("D,causal,hq,hkv", [(128, True, 4, 2), (256, False, 2, 2)])
def test_noalloc_backward_matches_workspace_backward(D, causal, hq, hkv):
    B, N = 2, 333
    scale = 1.0 / math.sqrt(D)
    q, k, v, do = (t.cuda() for t in make_random(B, hq, hkv, N, D, "bf16", seed=D + hq))
    o, lse = attn_fwd(q, k, v, causal=causal, scale=scale)
    ref = attn_bwd(q, k, v, o, lse, do, causal=causal, scale=scale)
    torch.cuda.synchronize()
    f = _noalloc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        code = f(_desc(q), _desc(k), _desc(v), _desc(o), ctypes.c_void_p(lse.data_ptr()),
                 _desc(do), _desc(dq), _desc(dk), _desc(dv), B, hq, hkv, N, D, 0,
                 1 if causal else 0, scale, stream)
        assert code == 0
        torch.cuda.synchronize()
        assert device_status()[0] == 0
        for got, want in zip((dq, dk, dv), ref):
            assert rel_err(to_np(got), to_np(want)) <= TOL_REL


def test_noalloc_rejects_sizes_beyond_the_scratch():
    f = _noalloc()
    # head dimension 256 accumulates dQ in an fp32 scratch: ~537 MB here, more than 64 MiB
    B, H, N, D = 4, 32, 4096, 256
    x = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    t = AttnTensor(ctypes.c_void_p(x.data_ptr()), H * N * D, N * D, D)
    code = f(t, t, t, t, ctypes.c_void_p(x.data_ptr()), t, t, t, t, B, H, H, N, D, 0, 1,
             0.1, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 4  # ATTN_ERR_WORKSPACE, nothing launched
