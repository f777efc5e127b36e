"""ctypes view of the C ABI in ``include/attn.h`` (argument marshalling only).

Loading fails loudly when ``libattn.so`` has not been built: there is no
fallback implementation of any kind.
"""

from __future__ import annotations

import ctypes
import os

from .build import LIB_PATH

ATTN_BF16 = 0
ATTN_FP32 = 1

STATUS = {
    0: "ATTN_OK",
    1: "ATTN_ERR_INVALID_ARG",
    2: "ATTN_ERR_UNSUPPORTED",
    3: "ATTN_ERR_MISALIGNED",
    4: "ATTN_ERR_WORKSPACE",
    5: "ATTN_ERR_CUDA",
    6: "ATTN_ERR_DEVICE_TIMEOUT",
}


class AttnTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("sb", ctypes.c_int64),
                ("sh", ctypes.c_int64), ("sn", ctypes.c_int64)]


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


_LIB = None


def lib(path: str | None = None) -> ctypes.CDLL:
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"CUDA library not built: {p} is missing (run exact_tiled_attention_37_b200.build.build())")
    L = ctypes.CDLL(p)
    T = AttnTensor
    i, f, vp = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
    L.attn_abi_version.restype = i
    L.attn_abi_version.argtypes = []
    L.attn_status_string.restype = ctypes.c_char_p
    L.attn_status_string.argtypes = [i]
    L.attn_fwd.restype = i
    L.attn_fwd.argtypes = [T, T, T, T, vp, i, i, i, i, i, i, i, f, vp]
    L.attn_fwd_window.restype = i
    L.attn_fwd_window.argtypes = [T, T, T, T, vp, i, i, i, i, i, i, i, i, f, vp]
    L.attn_bwd_window.restype = i
    L.attn_bwd_window.argtypes = [T, T, T, T, vp, T, T, T, T, i, i, i, i, i, i, i, i, f, vp,
                                  ctypes.c_size_t, vp]
    L.attn_fwd_masked.restype = i
    L.attn_fwd_masked.argtypes = [T, T, T, T, vp, i, i, i, i, i, i, i, i, vp, f, vp]
    L.attn_bwd_masked.restype = i
    L.attn_bwd_masked.argtypes = [T, T, T, T, vp, T, T, T, T, i, i, i, i, i, i, i, i, vp, f, vp,
                                  ctypes.c_size_t, vp]
    L.attn_fwd_fp8.restype = i
    L.attn_fwd_fp8.argtypes = [T, T, T, T, vp, i, i, i, i, i, f, f, f, i, i, f, vp]
    L.attn_decode_workspace_bytes.restype = ctypes.c_size_t
    L.attn_decode_workspace_bytes.argtypes = [i, i, i, i, i]
    L.attn_decode_paged.restype = i
    L.attn_decode_paged.argtypes = [T, T, T, i, vp, i, vp, T, vp, i, i, i, i, i, i, i, f, vp,
                                    ctypes.c_size_t, vp]
    L.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    L.attn_bwd_workspace_bytes.argtypes = [i, i, i, i]
    L.attn_bwd_workspace_bytes_ds.restype = ctypes.c_size_t
    L.attn_bwd_workspace_bytes_ds.argtypes = [i, i, i, i, i, i]
    L.attn_bwd.restype = i
    L.attn_bwd.argtypes = [T, T, T, T, vp, T, T, T, T, i, i, i, i, i, i, i, f, vp,
                           ctypes.c_size_t, vp]
    L.attn_device_status.restype = i
    L.attn_device_status.argtypes = [vp, ctypes.POINTER(i)]
    L.attn_debug_set_wait_limit_ns.restype = None
    L.attn_debug_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    L.attn_debug_set_flags.restype = None
    L.attn_debug_set_flags.argtypes = [i]
    L.attn_debug_set_fwd_variant.restype = None
    L.attn_debug_set_fwd_variant.argtypes = [i]
    L.attn_debug_exp2.restype = i
    L.attn_debug_exp2.argtypes = [vp, vp, i, i, vp]
    L.attn_debug_set_bwd_events.restype = None
    L.attn_debug_set_bwd_events.argtypes = [vp, vp]
    L.attn_debug_set_bwd_q_events.restype = None
    L.attn_debug_set_bwd_q_events.argtypes = [vp, vp]
    if path is None:
        _LIB = L
    return L
