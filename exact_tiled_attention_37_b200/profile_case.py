"""Runs one forward (+ backward) of a named workload through the C ABI, for
profilers: ``python -m exact_tiled_attention_37_b200.profile_case --workload 2``.

Exits non-zero when a kernel reports a device-side timeout.
"""

from __future__ import annotations

import argparse
import sys

import torch

from . import attn_bwd, attn_fwd, device_status
from .inputs import make_inputs, workload


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--repeat", type=int, default=1)
    ap.add_argument("--fwd-only", action="store_true")
    args = ap.parse_args(argv)
    w = workload(args.workload)
    causal = w.causal[-1]
    q, k, v, *rest = (t.to("cuda") for t in make_inputs(w, with_do=w.backward))
    for _ in range(args.repeat):
        o, lse = attn_fwd(q, k, v, causal=causal)
        if w.backward and not args.fwd_only:
            attn_bwd(q, k, v, o, lse, rest[0], causal=causal)
    torch.cuda.synchronize()
    code, where = device_status()
    print(f"{w.name}: device status {code} (wait site {where})")
    return 0 if code == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
