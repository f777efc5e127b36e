"""Runs one forward (+ backward) of a named workload through the C ABI, for
profilers: ``python -m exact_tiled_attention_37_b200.profile_case --workload 2``
(``--batch B`` keeps only the first B sequences, for smaller captures).
``--decode`` instead runs a paged decode: 8 sequences of 32768 cached keys,
Hq=32, Hkv=8, D=128, one new token, the 2048 pages in a seeded random order.

Exits non-zero when a kernel reports a device-side timeout.
"""

from __future__ import annotations

import argparse
import sys

import torch

from . import attn_bwd, attn_decode, attn_fwd, device_status, set_fwd_variant
from .inputs import make_inputs, workload


def decode_case(repeat: int) -> int:
    B, Hq, Hkv, D, L = 8, 32, 8, 128, 32768
    pages = L // 128
    g = torch.Generator(device="cuda").manual_seed(3)
    kp = torch.randn(B * pages, 128, Hkv, D, device="cuda", dtype=torch.bfloat16, generator=g)
    vp = torch.randn(B * pages, 128, Hkv, D, device="cuda", dtype=torch.bfloat16, generator=g)
    q = torch.randn(B, Hq, 1, D, device="cuda", dtype=torch.bfloat16, generator=g)
    table = torch.randperm(B * pages, device="cuda", generator=g).to(torch.int32)
    seqlens = torch.full((B,), L, device="cuda", dtype=torch.int32)
    for _ in range(repeat):
        attn_decode(q, kp, vp, table.reshape(B, pages), seqlens, causal=True)
    torch.cuda.synchronize()
    code, where = device_status()
    print(f"paged decode B={B} Hq={Hq} Hkv={Hkv} L={L}: device status {code} (wait site {where})")
    return 0 if code == 0 else 1


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--repeat", type=int, default=1)
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--decode", action="store_true")
    ap.add_argument("--fwd-variant", type=int, default=0,
                    help="forward kernel for bf16 D=128: 0 default, 1 one CTA per query tile, "
                         "2 CTA pairs with 2-CTA products")
    ap.add_argument("--batch", type=int, default=0,
                    help="run only the first BATCH sequences of the workload (smaller captures)")
    ap.add_argument("--recompute-dq", action="store_true",
                    help="backward with the smallest workspace: the seven-product form, whose "
                         "dQ kernel recomputes S and dP (default: stored dS tiles at D = 128)")
    args = ap.parse_args(argv)
    if args.decode:
        return decode_case(args.repeat)
    if args.fwd_variant:
        set_fwd_variant(args.fwd_variant)
    w = workload(args.workload)
    causal = w.causal[-1]
    ins = make_inputs(w, with_do=w.backward)
    if args.batch > 0:
        ins = tuple(t[: args.batch] for t in ins)
    q, k, v, *rest = (t.to("cuda") for t in ins)
    for _ in range(args.repeat):
        o, lse = attn_fwd(q, k, v, causal=causal)
        if w.backward and not args.fwd_only:
            attn_bwd(q, k, v, o, lse, rest[0], causal=causal, store_ds=not args.recompute_dq)
    torch.cuda.synchronize()
    code, where = device_status()
    name = w.name + (f" (first {args.batch} sequences)" if args.batch > 0 else "")
    print(f"{name}: device status {code} (wait site {where})")
    return 0 if code == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
