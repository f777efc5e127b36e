"""Python entry points over the C ABI (argument marshalling only).

Every step of the computation runs in the CUDA kernels of ``libattn.so``.
Tensors must already live on a CUDA device; nothing here computes attention,
and there is no CPU path.
"""

from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import ATTN_BF16, ATTN_FP32, AttnError, AttnTensor


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    if t.dtype == torch.float32:
        return ATTN_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or fp32 expected")


def _desc(t: torch.Tensor, name: str) -> AttnTensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dim() != 4:
        raise ValueError(f"{name} must be [B, H, N, D], got shape {tuple(t.shape)}")
    if t.stride(3) != 1:
        raise ValueError(f"{name} must have unit stride on D")
    sb, sh, sn, _ = t.stride()
    return AttnTensor(ctypes.c_void_p(t.data_ptr()), sb, sh, sn)


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(code: int, what: str):
    if code != 0:
        raise AttnError(code, what)


def _check_device(device: torch.device, what: str):
    """Waits for the current stream of `device` and raises AttnError when a
    kernel's bounded wait gave up since the device status was last read.  The
    status word is per device and shared by all streams (see attn.h), so a
    failure of work on another stream of the same device is reported here too."""
    code, where = device_status(device)
    if code != 0:
        raise AttnError(code, f"{what} (device wait site {where})")


def _window(causal: bool, window) -> tuple[int, int]:
    """(window_left, window_right) of the C ABI: -1 = unbounded; causal caps the right side at 0."""
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    if causal:
        wr = 0
    return wl, wr


def _block_mask(block_mask, B, Hq, N, device) -> ctypes.c_void_p:
    """Device pointer of a [B, Hq, T, T] uint8 tile mask (T = ceil(N / 128)), or NULL."""
    if block_mask is None:
        return ctypes.c_void_p(0)
    t = (N + 127) // 128
    if (block_mask.dtype != torch.uint8 or not block_mask.is_cuda
            or block_mask.device != device or tuple(block_mask.shape) != (B, Hq, t, t)
            or not block_mask.is_contiguous()):
        raise ValueError(f"block_mask must be a contiguous uint8 CUDA tensor of shape "
                         f"{(B, Hq, t, t)} on {device}")
    return ctypes.c_void_p(block_mask.data_ptr())


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
             scale: float | None = None, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, window=None, block_mask=None,
             check: bool = False):
    """O, lse = attention(q, k, v): q [B,Hq,N,D], k/v [B,Hkv,N,D] on one CUDA device.

    window=(wl, wr): query i sees keys i - wl .. i + wr (-1 = unbounded side).
    block_mask: [B,Hq,T,T] uint8 (T = ceil(N/128)); 128x128 tile pairs whose
    entry is 0 are skipped (rows that see no key get O = 0, lse = -inf).
    Returns O (dtype of q) and lse [B,Hq,N] fp32 (natural log).
    check=True waits for the call to finish and raises AttnError if a kernel's
    bounded wait timed out (otherwise the outputs of such a call are undefined
    and only device_status() reveals it).
    """
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or lse.shape != (B, Hq, N):
        raise ValueError("lse must be a contiguous fp32 [B, Hq, N] tensor")
    L = _lib.lib()
    wl, wr = _window(causal, window)
    bm = _block_mask(block_mask, B, Hq, N, q.device)
    code = L.attn_fwd_masked(_desc(q, "q"), _desc(k, "k"), _desc(v, "v"), _desc(out, "out"),
                             ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, N, D, _dtype_code(q),
                             wl, wr, bm, float(scale), _stream(q.device))
    _check(code, "attn_fwd")
    if check:
        _check_device(q.device, "attn_fwd")
    return out, lse


def bwd_workspace_bytes(B: int, Hq: int, N: int, D: int) -> int:
    """Smallest workspace attn_bwd accepts (dQ recomputed at D <= 128)."""
    return int(_lib.lib().attn_bwd_workspace_bytes(B, Hq, N, D))


def bwd_workspace_bytes_ds(B: int, Hq: int, N: int, D: int, causal: bool = False,
                           window=None) -> int:
    """Workspace with which attn_bwd stores dS tiles and sums dQ from them
    (D = 128; equal to bwd_workspace_bytes where that form does not apply)."""
    wl, wr = _window(causal, window)
    return int(_lib.lib().attn_bwd_workspace_bytes_ds(B, Hq, N, D, wl, wr))


def attn_bwd(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None,
             dq=None, dk=None, dv=None, workspace: torch.Tensor | None = None, window=None,
             block_mask=None, check: bool = False, store_ds: bool = True):
    """dQ, dK, dV of attention from the forward's O and lse and the gradient dO
    (window, block_mask and check as in attn_fwd).  Without a workspace one is
    allocated: with store_ds, large enough for the stored-dS form (see
    bwd_workspace_bytes_ds), else the smallest one.  A given workspace selects
    the form by its size."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if dq is None:
        dq = torch.empty_like(q, memory_format=torch.contiguous_format)
    if dk is None:
        dk = torch.empty_like(k, memory_format=torch.contiguous_format)
    if dv is None:
        dv = torch.empty_like(v, memory_format=torch.contiguous_format)
    L = _lib.lib()
    wl, wr = _window(causal, window)
    need = int(L.attn_bwd_workspace_bytes(B, Hq, N, D))
    if workspace is None:
        want = int(L.attn_bwd_workspace_bytes_ds(B, Hq, N, D, wl, wr)) if store_ds else need
        workspace = torch.empty(want, device=q.device, dtype=torch.uint8)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace too small: {need} bytes needed")
    if not lse.is_contiguous() or lse.dtype != torch.float32:
        raise ValueError("lse must be contiguous fp32")
    bm = _block_mask(block_mask, B, Hq, N, q.device)
    code = L.attn_bwd_masked(_desc(q, "q"), _desc(k, "k"), _desc(v, "v"), _desc(o, "o"),
                             ctypes.c_void_p(lse.data_ptr()), _desc(do, "do"), _desc(dq, "dq"),
                             _desc(dk, "dk"), _desc(dv, "dv"), B, Hq, Hkv, N, D,
                             _dtype_code(q), wl, wr, bm, float(scale),
                             ctypes.c_void_p(workspace.data_ptr()),
                             ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                             _stream(q.device))
    _check(code, "attn_bwd")
    if check:
        _check_device(q.device, "attn_bwd")
    return dq, dk, dv


def device_status(device=None):
    """(status code, wait-site id): syncs the current stream and reads/clears
    the device status word (0 = no kernel wait timed out)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    where = ctypes.c_int(0)
    code = _lib.lib().attn_device_status(_stream(dev), ctypes.byref(where))
    return int(code), int(where.value)


def set_wait_limit_ns(ns: int):
    _lib.lib().attn_debug_set_wait_limit_ns(int(ns))


def set_debug_flags(flags: int):
    _lib.lib().attn_debug_set_flags(int(flags))


def set_fwd_variant(variant: int):
    """Forward kernel for bf16 D = 128 without a block mask: 0 default, 1 one
    CTA per query tile, 2 CTA pairs with 2-CTA tensor-core products."""
    _lib.lib().attn_debug_set_fwd_variant(int(variant))


def _pool_desc(t: torch.Tensor, name: str) -> AttnTensor:
    """[P, 128, Hkv, D] page pool -> (ptr, page stride, head stride, row stride)."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dim() != 4 or t.shape[1] != 128 or t.stride(3) != 1:
        raise ValueError(f"{name} must be [P, 128, Hkv, D] with unit stride on D")
    sp, sr, sh, _ = t.stride()
    return AttnTensor(ctypes.c_void_p(t.data_ptr()), sp, sh, sr)


def decode_workspace_bytes(B: int, Hq: int, Sq: int, D: int, max_pages: int) -> int:
    return int(_lib.lib().attn_decode_workspace_bytes(B, Hq, Sq, D, max_pages))


def attn_decode(q, k_pool, v_pool, block_table, seqlens, causal: bool = False,
                scale: float | None = None, out=None, lse=None, workspace=None,
                check: bool = False):
    """Decode against a paged cache: q [B,Hq,Sq,D] (newest tokens), k_pool/v_pool
    [P,128,Hkv,D], block_table int32 [B,max_pages], seqlens int32 [B].

    Query token i of sequence b sits at position seqlens[b] - Sq + i.
    Returns O [B,Hq,Sq,D] (bf16) and lse [B,Hq,Sq] fp32 (natural log)."""
    B, Hq, Sq, D = q.shape
    P, _, Hkv, _ = k_pool.shape
    if v_pool.shape != k_pool.shape or k_pool.shape[3] != D:
        raise ValueError(f"pool shapes k{tuple(k_pool.shape)} v{tuple(v_pool.shape)} vs q{tuple(q.shape)}")
    for t, name in ((block_table, "block_table"), (seqlens, "seqlens")):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    if block_table.dim() != 2 or block_table.shape[0] != B or seqlens.shape != (B,):
        raise ValueError("block_table must be [B, max_pages] and seqlens [B]")
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), device=q.device, dtype=torch.float32)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or lse.shape != (B, Hq, Sq):
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Sq] tensor")
    L = _lib.lib()
    need = int(L.attn_decode_workspace_bytes(B, Hq, Sq, D, max_pages))
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    code = L.attn_decode_paged(_desc(q, "q"), _pool_desc(k_pool, "k_pool"),
                               _pool_desc(v_pool, "v_pool"), P,
                               ctypes.c_void_p(block_table.data_ptr()), max_pages,
                               ctypes.c_void_p(seqlens.data_ptr()), _desc(out, "out"),
                               ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, Sq, D,
                               _dtype_code(q), int(bool(causal)), float(scale),
                               ctypes.c_void_p(workspace.data_ptr()),
                               ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                               _stream(q.device))
    _check(code, "attn_decode")
    if check:
        _check_device(q.device, "attn_decode")
    return out, lse


def attn_fwd_fp8(q, k, v, q_scale: float = 1.0, k_scale: float = 1.0, v_scale: float = 1.0,
                 causal: bool = False, scale: float | None = None, out=None, lse=None,
                 window=None, check: bool = False):
    """Forward on e4m3 inputs (torch.float8_e4m3fn, D = 128) holding x / scale with
    per-tensor scales; returns O (bf16) and lse of attention on the dequantised inputs."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        if t.dtype != torch.float8_e4m3fn:
            raise TypeError(f"{name} must be torch.float8_e4m3fn")
    if k.shape != (B, Hkv, N, D) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(q.shape, device=q.device, dtype=torch.bfloat16)
    if lse is None:
        lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    wl, wr = _window(causal, window)
    code = _lib.lib().attn_fwd_fp8(_desc(q, "q"), _desc(k, "k"), _desc(v, "v"), _desc(out, "out"),
                                   ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, N, D,
                                   float(q_scale), float(k_scale), float(v_scale), wl, wr,
                                   float(scale), _stream(q.device))
    _check(code, "attn_fwd_fp8")
    if check:
        _check_device(q.device, "attn_fwd_fp8")
    return out, lse
