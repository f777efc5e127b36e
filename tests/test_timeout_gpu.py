"""Bounded waits: a kernel whose wait can never be satisfied (the producer is
told to drop one tile load) gives up after the configured limit, reports
ATTN_ERR_DEVICE_TIMEOUT through the device status word, and leaves the
context usable -- nothing hangs or faults."""

import math

import pytest
import torch

import oracle
from exact_tiled_attention_37_b200 import (attn_bwd, attn_fwd, device_status, set_debug_flags,
                                           set_wait_limit_ns)
from exact_tiled_attention_37_b200.inputs import make_random

from ._util import TOL_REL, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [128, 256])
def test_dropped_load_times_out_and_recovers(D):
    q, k, v = (t.to("cuda") for t in make_random(1, 2, 2, 384, D, "bf16", seed=4, with_do=False))
    assert device_status()[0] == 0
    set_wait_limit_ns(50_000_000)  # 50 ms
    set_debug_flags(1)
    try:
        attn_fwd(q, k, v, causal=False)
        code, where = device_status()
    finally:
        set_debug_flags(0)
        set_wait_limit_ns(0)
    assert code == 6, (code, where)
    assert where != 0
    # the context is still usable and the next call is correct
    o, lse = attn_fwd(q, k, v, causal=False)
    assert device_status()[0] == 0
    o_ref, _ = oracle.attention_fwd(to_np(q), to_np(k), to_np(v), False, 1 / math.sqrt(D))
    assert rel_err(to_np(o), o_ref) <= TOL_REL


@pytest.mark.parametrize("D", [64, 128, 256])
def test_dropped_bwd_load_times_out_and_recovers(D):
    """The dK/dV kernel's producer drops its second Q tile load: the MMA
    warp's wait for it runs out, every role leaves its loop, the kernel
    drains what it started and returns; the next backward is correct."""
    q, k, v, do = (t.to("cuda") for t in make_random(1, 2, 2, 384, D, "bf16", seed=6))
    o, lse = attn_fwd(q, k, v, causal=False)
    assert device_status()[0] == 0
    set_wait_limit_ns(50_000_000)  # 50 ms
    set_debug_flags(2)
    try:
        attn_bwd(q, k, v, o, lse, do, causal=False)
        code, where = device_status()
    finally:
        set_debug_flags(0)
        set_wait_limit_ns(0)
    assert code == 6, (code, where)
    assert where != 0
    dq, dk, dv = attn_bwd(q, k, v, o, lse, do, causal=False)
    assert device_status()[0] == 0
    ref = oracle.attention_bwd(*(to_np(t) for t in (q, k, v, do)), False, 1 / math.sqrt(D))
    for got, r in zip((dq, dk, dv), ref):
        assert rel_err(to_np(got), r) <= TOL_REL


@pytest.mark.parametrize("which", ["fwd", "bwd"])
def test_check_option_raises_on_timeout(which):
    """check=True turns a device-side timeout into an AttnError at the call
    (the same dropped loads as above); a normal call with check=True returns."""
    from exact_tiled_attention_37_b200 import AttnError
    q, k, v, do = (t.to("cuda") for t in make_random(1, 2, 2, 384, 128, "bf16", seed=8))
    o, lse = attn_fwd(q, k, v, causal=True, check=True)
    set_wait_limit_ns(50_000_000)  # 50 ms
    set_debug_flags(1 if which == "fwd" else 2)
    try:
        with pytest.raises(AttnError) as ei:
            if which == "fwd":
                attn_fwd(q, k, v, causal=True, check=True)
            else:
                attn_bwd(q, k, v, o, lse, do, causal=True, check=True)
    finally:
        set_debug_flags(0)
        set_wait_limit_ns(0)
    assert ei.value.code == 6
    assert device_status()[0] == 0  # the failed call's status was read and cleared
    attn_bwd(q, k, v, o, lse, do, causal=True, check=True)
