"""CPU checks of the C ABI: the library builds, loads and exports every
function ``include/attn.h`` declares; host-side validation rejects bad
arguments with the documented status codes before touching the GPU."""

import ctypes
import os
import re

import pytest

from exact_tiled_attention_37_b200 import _lib, build

HEADER = os.path.join(build.ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    names = set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_bytes", "attn_device_status",
              "attn_status_string", "attn_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), f"{n} declared in attn.h but not exported"


def test_abi_version_and_status_strings(L):
    assert L.attn_abi_version() == 1
    for code in range(7):
        assert L.attn_status_string(code)


def test_workspace_size(L):
    B, H, N = 2, 16, 4096
    # D <= 128: per-row Delta and log2-scaled lse only (dQ is written directly)
    for D in (64, 128):
        got = L.attn_bwd_workspace_bytes(B, H, N, D)
        assert 2 * B * H * N * 4 <= got <= 2 * B * H * N * 4 + 1024
    # D = 256: plus the fp32 dQ scratch the fused kernel accumulates into
    got = L.attn_bwd_workspace_bytes(B, H, N, 256)
    assert got >= B * H * N * 256 * 4 + 2 * B * H * N * 4
    assert L.attn_bwd_workspace_bytes(0, H, N, 128) == 0


def test_stored_ds_workspace_size(L):
    """Stored dS tiles: 32 KB per visible 128 x 128 tile after the row
    statistics (rounded up to 64 KB); D = 128 only, at most 4 GiB of tiles."""
    f = L.attn_bwd_workspace_bytes_ds
    B, H, N = 2, 16, 4096
    nt = N // 128
    base = L.attn_bwd_workspace_bytes(B, H, N, 128)
    off = -(-base // 65536) * 65536
    assert f(B, H, N, 128, -1, 0) == off + B * H * (nt * (nt + 1) // 2) * 32768   # causal
    assert f(B, H, N, 128, -1, -1) == off + B * H * nt * nt * 32768               # no mask
    # a window of 1023 keys to the left: each query tile sees at most 9 key tiles
    assert f(B, H, N, 128, 1023, 0) == off + B * H * nt * 9 * 32768
    # sides >= N are unbounded
    assert f(B, H, N, 128, N, 0) == f(B, H, N, 128, -1, 0)
    # other head dimensions, or more than 4 GiB of tiles: the smallest workspace
    assert f(B, H, N, 64, -1, 0) == L.attn_bwd_workspace_bytes(B, H, N, 64)
    assert f(B, H, N, 256, -1, 0) == L.attn_bwd_workspace_bytes(B, H, N, 256)
    assert f(1, 32, 32768, 128, -1, 0) == L.attn_bwd_workspace_bytes(1, 32, 32768, 128)
    assert f(0, H, N, 128, -1, 0) == 0
    assert f(B, H, N, 128, -2, 0) == 0


def _visible_key_tiles(N, wl, wr, i):
    """Key tiles (128 rows) holding a key that some query of query tile i may
    see under the window (wl, wr), counted one query and key at a time."""
    qs = range(128 * i, min(N, 128 * i + 128))
    tiles = set()
    for q in qs:
        lo = 0 if wl < 0 else max(0, q - wl)
        hi = N - 1 if wr < 0 else min(N - 1, q + wr)
        tiles.update(range(lo // 128, hi // 128 + 1))
    return tiles


@pytest.mark.parametrize("N", [1, 127, 128, 129, 300, 640, 1000])
@pytest.mark.parametrize("window", [(-1, 0), (-1, -1), (0, 0), (111, 0), (200, 200), (64, 300),
                                    (-1, 50), (1023, 0)])
def test_stored_ds_slots_cover_every_visible_tile(L, N, window):
    """The stored-dS workspace holds, per (batch, head), one slot per query
    tile and key tile it must (causal: the triangle; other windows: a band as
    wide as the widest query tile's run of visible key tiles), checked against
    tiles counted by brute force."""
    wl, wr = window
    wl_n = -1 if wl >= N else wl
    wr_n = -1 if wr >= N else wr
    B, H, D = 1, 2, 128
    nt = -(-N // 128)
    rows = [_visible_key_tiles(N, wl_n, wr_n, i) for i in range(nt)]
    for r in rows:  # each query tile sees one contiguous run of key tiles
        assert not r or max(r) - min(r) + 1 == len(r)
    if wl_n < 0 and wr_n == 0:
        slots = nt * (nt + 1) // 2
        assert [len(r) for r in rows] == [i + 1 for i in range(nt)]
    else:
        slots = nt * max(len(r) for r in rows)
    got = L.attn_bwd_workspace_bytes_ds(B, H, N, D, wl, wr)
    base = L.attn_bwd_workspace_bytes(B, H, N, D)
    off = -(-base // 65536) * 65536
    assert got == off + B * H * slots * 32768


def _t(ptr, sb, sh, sn):
    return _lib.AttnTensor(ctypes.c_void_p(ptr), sb, sh, sn)


def _fwd(L, B=1, Hq=2, Hkv=1, N=256, D=128, dt=0, ptr=0x10000, lse=0x20000, scale=0.1,
         sn=None, qptr=None):
    sn = D if sn is None else sn
    t = _t(ptr, Hq * N * sn, N * sn, sn)
    q = _t(qptr if qptr is not None else ptr, Hq * N * sn, N * sn, sn)
    kv = _t(ptr, Hkv * N * sn, N * sn, sn)
    return L.attn_fwd(q, kv, kv, t, ctypes.c_void_p(lse), B, Hq, Hkv, N, D, dt, 0, scale, None)


def test_fwd_validation_codes(L):
    assert _fwd(L, Hq=3, Hkv=2) == 1           # Hq % Hkv
    assert _fwd(L, N=0) == 1                   # empty sequence
    assert _fwd(L, B=0) == 1
    assert _fwd(L, ptr=0) == 1                 # null
    assert _fwd(L, lse=0) == 1
    assert _fwd(L, scale=0.0) == 1
    assert _fwd(L, scale=float("nan")) == 1
    assert _fwd(L, D=96) == 2                  # head dim not built
    assert _fwd(L, D=128, dt=1) == 2           # fp32 only at D=64
    assert _fwd(L, qptr=0x10008) == 3          # misaligned base
    assert _fwd(L, sn=132) == 3                # row stride not a multiple of 16 bytes
    assert _fwd(L, lse=0x20004) == 3


def test_block_mask_validation_codes(L):
    # refused before anything is launched (no GPU needed): head dim 256, fp32
    # storage, or more than 512 tiles of 128 rows
    B, Hq, N, D = 1, 2, 256, 128
    lse = ctypes.c_void_p(0x20000)
    bm = ctypes.c_void_p(0x30000)

    def fwd(D=D, dt=0, N=N):
        t = _t(0x10000, Hq * N * D, N * D, D)
        return L.attn_fwd_masked(t, t, t, t, lse, B, Hq, Hq, N, D, dt, -1, -1, bm, 0.1, None)

    assert fwd(D=256) == 2
    assert fwd(D=64, dt=1) == 2
    assert fwd(N=512 * 128 + 1) == 2
    t = _t(0x10000, Hq * N * 256, N * 256, 256)
    ws = L.attn_bwd_workspace_bytes(B, Hq, N, 256)
    assert L.attn_bwd_masked(t, t, t, t, lse, t, t, t, t, B, Hq, Hq, N, 256, 0, -1, 0, bm, 0.1,
                             ctypes.c_void_p(0x40000), ws, None) == 2


def test_window_validation_codes(L):
    B, Hq, N, D = 1, 2, 256, 128
    t = _t(0x10000, Hq * N * D, N * D, D)
    lse = ctypes.c_void_p(0x20000)
    assert L.attn_fwd_window(t, t, t, t, lse, B, Hq, Hq, N, D, 0, -2, 0, 0.1, None) == 1
    assert L.attn_fwd_window(t, t, t, t, lse, B, Hq, Hq, N, D, 0, 3, -5, 0.1, None) == 1
    ws = L.attn_bwd_workspace_bytes(B, Hq, N, D)
    assert L.attn_bwd_window(t, t, t, t, lse, t, t, t, t, B, Hq, Hq, N, D, 0, -3, 0, 0.1,
                             ctypes.c_void_p(0x40000), ws, None) == 1


def test_bwd_validation_codes(L):
    B, Hq, Hkv, N, D = 1, 2, 1, 256, 128
    q = _t(0x10000, Hq * N * D, N * D, D)
    kv = _t(0x10000, Hkv * N * D, N * D, D)
    ws = L.attn_bwd_workspace_bytes(B, Hq, N, D)
    lse = ctypes.c_void_p(0x20000)

    def call(D=D, ws_ptr=0x40000, ws_bytes=ws, dt=0, lse=lse):
        return L.attn_bwd(q, kv, kv, q, lse, q, q, kv, kv, B, Hq, Hkv, N, D, dt, 1, 0.1,
                          ctypes.c_void_p(ws_ptr), ws_bytes, None)

    assert call(ws_ptr=0) == 4
    assert call(ws_bytes=ws - 1) == 4
    assert call(ws_ptr=0x40010) == 3           # workspace must be 256-byte aligned
    assert call(D=96) == 2
    assert call(dt=1) == 2
    assert call(lse=ctypes.c_void_p(0)) == 1


def test_python_api_refuses_cpu_tensors():
    import torch
    from exact_tiled_attention_37_b200 import attn_fwd
    q = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        attn_fwd(q, q, q)


def test_overlapping_outputs_are_rejected(L):
    """An output whose rows (or heads, or batches) overlap would be written by
    several CTAs in an undefined order: refused before anything is launched."""
    B, Hq, N, D = 2, 2, 256, 128
    lse = ctypes.c_void_p(0x20000)
    q = _t(0x10000, Hq * N * D, N * D, D)
    for bad in (_t(0x10000, Hq * N * D, N * D, D // 2),       # rows overlap
                _t(0x10000, Hq * N * D, (N - 1) * D, D),      # heads overlap
                _t(0x10000, N * D, N * D, D),                 # batches overlap heads
                _t(0x10000, Hq * N * D, N * D, 0)):           # every row on one
        assert L.attn_fwd(q, q, q, bad, lse, B, Hq, Hq, N, D, 0, 1, 0.1, None) == 1
        ws = L.attn_bwd_workspace_bytes(B, Hq, N, D)
        for slot in range(3):
            outs = [q, q, q]
            outs[slot] = bad
            assert L.attn_bwd(q, q, q, q, lse, q, *outs, B, Hq, Hq, N, D, 0, 1, 0.1,
                              ctypes.c_void_p(0x40000), ws, None) == 1
