"""Benchmark of the exact tiled attention hot path on B200.

One step = one forward (O, lse) and one backward (dQ, dK, dV) of the MHA
workload B=2, H=16, N=4096, D=128, causal, bf16 -- the configuration the
throughput target is quoted at (N >= 4096, D = 128), with both passes of
the method.  Inputs are seeded synthetic N(0,1) tensors resident in HBM.
Throughput counts 4*B*H*N^2*D FLOPs for the forward (halved for causal) and
2.5x that for the backward.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch with torchrun: every rank runs an independent replica of the
workload (the path needs no exchange between GPUs; weak scaling).

Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD_INDEX = 2  # MHA fwd+bwd B=2 H=16 N=4096 D=128 causal

# The dominant kernel of the step: the backward's dK/dV kernel.
DOMINANT_KERNEL = "bwd_kv_kernel<128,2,2>"
# DRAM traffic of one launch of it from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), with the hash of the kernel sources it was taken on;
# it is reported as null once the sources change (profiles/ holds the capture).
DOMINANT_TRAFFIC = {"bytes": 227364864, "src_sha": "4b5594ff11e21fc4"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="rough budget of the oracle CPU-baseline sample")
    return ap.parse_args()


def dist_info():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("ptx.cuh", "bwd.cuh", "bwd_split.cuh"):
        with open(os.path.join(ROOT, "exact_tiled_attention_37_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            pk = json.load(fh)
        return {"bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "hbm_gbs": float(pk["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
                "source": "fallback"}


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


def max_over_ranks(values, device):
    """Element-wise maximum over all ranks (the slowest rank sets the time);
    identity when no process group is initialised."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(flops_per_step_per_rank: float, world: int, ms_per_step: float) -> float:
    """Units all ranks processed per second (every rank runs a full replica)."""
    return world * flops_per_step_per_rank / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------- CPU baseline (oracle)


def cpu_baseline(w, budget_s: float):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: the
    forward and backward of one (batch, head) pair at a time, repeated until
    the time budget is spent.  Returns TFLOPS on the counted FLOPs."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle
    from exact_tiled_attention_37_b200.inputs import make_inputs

    cores = len(os.sched_getaffinity(0))
    q, k, v, do = (t.float().numpy() for t in make_inputs(w))
    causal = w.causal[0]
    per_head = (w.fwd_flops(causal) + w.bwd_flops(causal)) / (w.B * w.Hq)
    done, t0 = 0, time.perf_counter()
    with threadpool_limits(limits=cores):
        while True:
            b, h = divmod(done % (w.B * w.Hq), w.Hq)
            sl = (slice(b, b + 1), slice(h, h + 1))
            oracle.attention_fwd(q[sl], k[sl], v[sl], causal, w.scale)
            oracle.attention_bwd(q[sl], k[sl], v[sl], do[sl], causal, w.scale)
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
    dt = time.perf_counter() - t0
    return {"value": done * per_head / dt / 1e12, "unit": "TFLOPS", "cores": cores,
            "kind": "oracle",
            "sample": f"fwd+bwd of {done} (batch, head) pair(s) of {w.name} (of {w.B * w.Hq}), "
                      f"fp64 NumPy/OpenBLAS, {dt:.1f} s"}


# ---------------------------------------------------------------- native arm


def run_native(args):
    import torch
    import torch.distributed as dist

    from exact_tiled_attention_37_b200 import _lib, attn_bwd, attn_fwd, bwd_workspace_bytes, \
        device_status
    from exact_tiled_attention_37_b200.inputs import make_inputs, workload

    rank, world, local = dist_info()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = workload(WORKLOAD_INDEX)
    causal = w.causal[0]
    host = [t.pin_memory() for t in make_inputs(w)]
    q, k, v, do = (t.to(dev) for t in host)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(bwd_workspace_bytes(w.B, w.Hq, w.N, w.D), device=dev, dtype=torch.uint8)
    flush = torch.empty(256 * 1024 * 1024, device=dev, dtype=torch.uint8)  # > 126 MB L2
    L = _lib.lib()
    stream = torch.cuda.current_stream(dev)

    def step():
        attn_fwd(q, k, v, causal=causal, out=o, lse=lse)
        attn_bwd(q, k, v, o, lse, do, causal=causal, dq=dq, dk=dk, dv=dv, workspace=ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    K, W = args.steps, args.warmup
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    for e in ev:  # create the driver events before the timed region
        for x in e:
            x.record(stream)
    for _ in range(W):
        flush.zero_()
        step()
    barrier()
    code, where = device_status(dev)
    if code != 0:
        raise RuntimeError(f"device status {code} at wait site {where} during warm-up")

    with ClockSampler(local) as clocks:
        barrier()
        for i in range(K):
            flush.zero_()
            s0, s1, m0, m1 = ev[i]
            s0.record(stream)
            L.attn_debug_set_bwd_events(m0.cuda_event, m1.cuda_event)
            step()
            s1.record(stream)
        barrier()
        time.sleep(0.25)
    code, where = device_status(dev)
    if code != 0:
        raise RuntimeError(f"device status {code} at wait site {where} during timing")
    step_ms = [a.elapsed_time(b) for a, b, _, _ in ev]
    main_ms = [c.elapsed_time(d) for _, _, c, d in ev]
    total_ms = sum(step_ms)

    # forward and backward separately (same region shape, fewer steps)
    def timed(fn, n):
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for a, b in es:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return statistics.median(a.elapsed_time(b) for a, b in es)

    fwd_ms = timed(lambda: attn_fwd(q, k, v, causal=causal, out=o, lse=lse), min(K, 50))
    bwd_ms = timed(lambda: attn_bwd(q, k, v, o, lse, do, causal=causal, dq=dq, dk=dk, dv=dv,
                                    workspace=ws), min(K, 50))

    # end to end through the public API with host buffers: every step uploads
    # its inputs (pinned Q, K, V, dO), runs forward + backward and downloads its
    # gradients (dQ, dK, dV).  Uploads run on one stream, compute on another,
    # downloads on a third, double-buffered, so step i+1's upload and step
    # i-1's download overlap step i's compute (as a user pipeline would).
    n_e2e = max(3, min(K, 20))
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    dbuf = [[torch.empty_like(t, device=dev) for t in host] for _ in range(2)]
    gbuf = [[torch.empty_like(t) for t in (dq, dk, dv)] for _ in range(2)]
    hout = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (dq, dk, dv)]
            for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = sum(t.numel() * t.element_size() for t in hout[0])

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_comp + ev_out:
            e.record(stream)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_in.wait_stream(stream)
        s_comp.wait_stream(stream)
        s_out.wait_stream(stream)
        start.record(s_in)
        for i in range(n + 2):
            if i < n:
                with torch.cuda.stream(s_in):
                    s_in.wait_event(ev_comp[i % 2])
                    for d_, h_ in zip(dbuf[i % 2], host):
                        d_.copy_(h_, non_blocking=True)
                    ev_in[i % 2].record(s_in)
            if 1 <= i <= n:
                j = i - 1
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(ev_in[j % 2])
                    s_comp.wait_event(ev_out[j % 2])
                    qq, kk, vv, dd = dbuf[j % 2]
                    oo, ll = attn_fwd(qq, kk, vv, causal=causal)
                    g0, g1, g2 = gbuf[j % 2]
                    attn_bwd(qq, kk, vv, oo, ll, dd, causal=causal, dq=g0, dk=g1, dv=g2,
                             workspace=ws)
                    ev_comp[j % 2].record(s_comp)
            if i >= 2:
                j = i - 2
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[j % 2])
                    for h_, d_ in zip(hout[j % 2], gbuf[j % 2]):
                        h_.copy_(d_, non_blocking=True)
                    ev_out[j % 2].record(s_out)
        stop.record(s_out)
        stop.synchronize()
        return start.elapsed_time(stop) / n

    e2e_run(2)
    barrier()
    e2e_ms = e2e_run(n_e2e)
    barrier()

    flops_step = w.fwd_flops(causal) + w.bwd_flops(causal)
    ms_per_step, e2e_ms = max_over_ranks([total_ms / K, e2e_ms], dev)
    value = whole_job_tflops(flops_step, world, ms_per_step)
    e2e_value = whole_job_tflops(flops_step, world, e2e_ms)

    peaks = load_peaks()
    dom_ms = statistics.mean(main_ms)
    # algorithmic FLOPs of one dK/dV-kernel launch: four products (S^T, dP^T,
    # dV, dK) over the visible tile pairs, each as costly as one of the
    # forward's two products
    dom_flops = 4 * w.fwd_flops(causal) / 2
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    traffic = DOMINANT_TRAFFIC["bytes"] if DOMINANT_TRAFFIC["src_sha"] == kernel_source_sha() else None
    peak = peaks["bf16_tflops_sustained"]
    clk = clocks.summary()

    result = {
        "metric": "attention fwd+bwd TFLOPS (bf16, 1xB200) and % of dense tensor-core peak",
        "value": round(value, 2),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.Hq, "Hkv": w.Hkv, "N": w.N, "D": w.D,
                   "causal": causal, "passes": "fwd+bwd", "l2": "flushed (256 MB write) between steps",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "fwd": {"ms": round(fwd_ms, 4), "tflops": round(w.fwd_flops(causal) / fwd_ms / 1e9, 1),
                "frac_of_peak": round(w.fwd_flops(causal) / fwd_ms / 1e9 / peaks["bf16_tflops"], 4)},
        "bwd": {"ms": round(bwd_ms, 4), "tflops": round(w.bwd_flops(causal) / bwd_ms / 1e9, 1),
                "frac_of_peak": round(w.bwd_flops(causal) / bwd_ms / 1e9 / peaks["bf16_tflops"], 4)},
        "roofline": {"kernel": DOMINANT_KERNEL, "bound": "tensor",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": f"{peaks['source']} bf16 sustained",
                     "launch_ms": round(dom_ms, 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "pipeline": "upload / compute / download on three streams, double-buffered"},
        "clocks": clk,
        "gpu_launches": 4 * K,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ---------------------------------------------------------------- reference arm


def run_reference(args):
    """The oracle (plain fp64 CPU implementation) as the reference arm, on the
    same workload and metric, each step a bounded sample of the workload."""
    rank, world, _ = dist_info()
    if rank != 0:
        return
    from exact_tiled_attention_37_b200.inputs import workload
    w = workload(WORKLOAD_INDEX)
    budget = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, budget)
    vals = [cpu_baseline(w, budget) for _ in range(args.steps)]
    v = statistics.median(x["value"] for x in vals)
    causal = w.causal[0]
    flops_step = w.fwd_flops(causal) + w.bwd_flops(causal)
    result = {
        "impl": "reference",
        "metric": "attention fwd+bwd TFLOPS (bf16, 1xB200) and % of dense tensor-core peak",
        "value": v,
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": flops_step / (v * 1e12) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.Hq, "Hkv": w.Hkv, "N": w.N, "D": w.D,
                   "causal": causal, "passes": "fwd+bwd"},
        "cpu_baseline": {"value": v, "unit": "TFLOPS", "cores": vals[0]["cores"],
                         "kind": "oracle", "sample": vals[0]["sample"]},
        "e2e": {"value": v, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
