"""fp64 CPU oracle for exact attention -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  It shares no code with the CUDA library.
"""

from .attention import (attention_bwd, attention_decode, attention_fwd, attention_fwd_rows,
                        softmax_probs)

__all__ = ["attention_fwd", "attention_bwd", "attention_fwd_rows", "attention_decode",
           "softmax_probs"]
