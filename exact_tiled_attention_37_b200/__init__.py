"""Exact tiled attention for B200 (sm_100a).

``attn_fwd`` / ``attn_bwd`` call the C ABI of ``libattn.so`` (``include/attn.h``)
on CUDA tensors; PyTorch only allocates device memory and provides the stream.
Importing the package does not load the CUDA library; the first call does.
"""

from ._lib import AttnError
from .api import (attn_bwd, attn_decode, attn_fwd, attn_fwd_fp8, bwd_workspace_bytes,
                  bwd_workspace_bytes_ds, decode_workspace_bytes, device_status, set_debug_flags, set_fwd_variant,
                  set_wait_limit_ns)

__all__ = ["attn_fwd", "attn_fwd_fp8", "attn_bwd", "attn_decode", "bwd_workspace_bytes",
           "bwd_workspace_bytes_ds",
           "decode_workspace_bytes", "device_status", "set_debug_flags", "set_fwd_variant",
           "set_wait_limit_ns",
           "AttnError"]
