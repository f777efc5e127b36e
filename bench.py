"""Benchmark of the exact tiled attention hot path on B200.

One step = one forward (O, lse) and one backward (dQ, dK, dV) of the MHA
workload B=2, H=16, N=4096, D=128, causal, bf16 -- the configuration the
throughput target is quoted at (N >= 4096, D = 128), with both passes of
the method.  Inputs are seeded synthetic N(0,1) tensors resident in HBM.
Throughput counts 4*B*H*N^2*D FLOPs for the forward (halved for causal) and
2.5x that for the backward.

After the timed steps the same process times, with the same clock sampler,
every other workload of the method (both masks of the B=4 H=16 N=2048
forward, the 32K-token grouped-query forward, the D=256 forward and
backward) and the mask and precision variants (sliding windows, block-sparse
tiles, e4m3 forward), each as the median of CUDA-event timings with L2
flushed before every call; these go under "configs" and do not enter the
headline value.

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
METRIC = "attention fwd+bwd TFLOPS (bf16, 1xB200) and % of dense tensor-core peak"

# The dominant kernel of the step: the backward's dK/dV kernel (which also
# stores the dS tiles the dQ kernel sums from).
DOMINANT_KERNEL = "bwd_kv3_kernel<128,3,2,2,true>"
DQ_KERNEL = "bwd_dqs_kernel<3>"
# DRAM traffic of one launch of the dK/dV and dQ kernels from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), with the hash of the kernel
# sources it was taken on; reported as null once the sources change (profiles/
# holds the capture).
DOMINANT_TRAFFIC = {"bytes": 843696640, "src_sha": "71708753997cd66f"}
DQ_TRAFFIC = {"bytes": 589824512, "src_sha": "71708753997cd66f"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration timings after the timed steps")
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
    for f in ("ptx.cuh", "bwd.cuh", "bwd_split.cuh", "bwd_kv3.cuh", "bwd_dqs.cuh"):
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


def choose_peak(peaks, clocks, region_ms):
    """The burst figure describes a kernel timed alone at full clock, the
    sustained one a kernel inside seconds of back-to-back work under the power
    cap: burst when the sampled SM clock stayed within 5 % of its maximum and
    the timed region is short (< 1 s per step), else sustained."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    burst = mhz is not None and mx and mhz >= 0.95 * mx and region_ms < 1000.0
    kind = "burst" if burst else "sustained"
    return (peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]), kind


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi (every 50 ms) while
    it is open; mark() labels time windows so that each timed region's samples
    can be summarised separately."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.samples = []   # (time, sm_mhz, max_mhz, power_w, reasons)
        self.windows = {}

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 7:
                continue
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            try:
                pw = float(parts[2])
            except ValueError:
                pw = None
            reasons = {n for n, v in zip(self.NAMES, parts[3:7]) if v.lower().startswith("active")}
            self.samples.append((time.monotonic(), sm, mx, pw, reasons))

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def mark(self, name, t0, t1):
        self.windows[name] = (t0, t1)

    def summary(self, name=None):
        t0, t1 = self.windows.get(name, (float("-inf"), float("inf"))) if name else \
            (float("-inf"), float("inf"))
        sel = [s for s in self.samples if t0 <= s[0] <= t1]
        sm = [s[1] for s in sel]
        reasons = sorted(set().union(*[s[4] for s in sel])) if sel else []
        pw = [s[3] for s in sel if s[3] is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": sel[-1][2] if sel else None, "samples": len(sm),
                "power_w_median": statistics.median(pw) if pw else None, "reasons": reasons}


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


def visible_pairs(N: int, wl: int = -1, wr: int = -1, tile_mask=None, tile: int = 128) -> int:
    """Number of (query, key) pairs one head computes under a window (wl, wr)
    (-1 = unbounded side) and an optional [T, T] tile mask: the FLOP count of
    masked variants is 4 * D per visible pair (backward 2.5x)."""
    import numpy as np
    i = np.arange(N)
    lo = np.zeros(N, dtype=np.int64) if wl < 0 else np.maximum(0, i - wl)
    hi = np.full(N, N - 1, dtype=np.int64) if wr < 0 else np.minimum(N - 1, i + wr)
    if tile_mask is None:
        return int(np.sum(hi - lo + 1))
    total = 0
    T = tile_mask.shape[0]
    for qt in range(T):
        rows = i[qt * tile:(qt + 1) * tile]
        for kt in range(T):
            if not tile_mask[qt, kt]:
                continue
            k0, k1 = kt * tile, min(N, (kt + 1) * tile) - 1
            a = np.maximum(lo[rows], k0)
            b = np.minimum(hi[rows], k1)
            total += int(np.sum(np.maximum(0, b - a + 1)))
    return total


# ---------------------------------------------------------------- CPU baseline (oracle)


def cpu_baseline(w, budget_s: float, pairs: int | None = None):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: the
    forward and backward of one (batch, head) pair at a time, repeated until
    the time budget is spent (or `pairs` pairs are done).  Returns TFLOPS on
    the counted FLOPs of the pairs it ran."""
    import numpy as np  # noqa: F401
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
            if (pairs is not None and done >= pairs) or \
                    (pairs is None and time.perf_counter() - t0 > budget_s):
                break
    dt = time.perf_counter() - t0
    return {"value": done * per_head / dt / 1e12, "unit": "TFLOPS", "cores": cores,
            "kind": "oracle", "seconds": dt, "pairs": done,
            "sample": f"fwd+bwd of {done} (batch, head) pair(s) of {w.name} (of {w.B * w.Hq}), "
                      f"fp64 NumPy/OpenBLAS, {dt:.1f} s; TFLOPS = counted FLOPs of those pairs / time"}


# ---------------------------------------------------------------- per-configuration timings


def time_calls(fn, flush, stream, n, warm=2):
    """Median device time (ms) of fn() over n calls, L2 flushed before each;
    events on the launching stream."""
    import torch
    for _ in range(warm):
        fn()
    es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for a, b in es:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    stream.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in es)


def run_configs(dev, flush, stream, peak_burst, clocks):
    """Forward/backward timings of the other workloads and of the mask and
    precision variants.  Returns a list of result dicts."""
    import numpy as np
    import torch

    from exact_tiled_attention_37_b200 import (attn_bwd, attn_fwd, attn_fwd_fp8,
                                               bwd_workspace_bytes_ds, device_status)
    from exact_tiled_attention_37_b200.inputs import make_inputs, make_random, workload

    out = []

    def entry(name, kind, ms, flops, extra=None):
        tf = flops / (ms * 1e-3) / 1e12
        e = {"config": name, "pass": kind, "ms": round(ms, 4), "tflops": round(tf, 1),
             "frac_of_burst_peak": round(tf / peak_burst, 4)}
        if extra:
            e.update(extra)
        out.append(e)

    def reps(ms_guess):
        return 30 if ms_guess < 1 else (15 if ms_guess < 10 else 7)

    # the workloads of the method (bf16; the fp32 single-head one is latency-bound)
    for idx, passes in ((1, ("fwd",)), (2, ("fwd", "bwd")), (3, ("fwd",)), (4, ("fwd", "bwd"))):
        w = workload(idx)
        ins = [t.to(dev) for t in make_inputs(w, with_do="bwd" in passes)]
        q, k, v = ins[:3]
        for causal in w.causal:
            o = torch.empty_like(q)
            lse = torch.empty((w.B, w.Hq, w.N), device=dev, dtype=torch.float32)
            t0 = time.monotonic()
            ms = time_calls(lambda: attn_fwd(q, k, v, causal=causal, out=o, lse=lse), flush, stream,
                            reps(w.fwd_flops(causal) / 1e12))
            entry(f"{w.name}{', causal' if causal else ''}", "fwd", ms, w.fwd_flops(causal))
            if "bwd" in passes:
                do = ins[3]
                dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
                ws = torch.empty(bwd_workspace_bytes_ds(w.B, w.Hq, w.N, w.D, causal=causal),
                                 device=dev, dtype=torch.uint8)
                ms = time_calls(lambda: attn_bwd(q, k, v, o, lse, do, causal=causal, dq=dq, dk=dk,
                                                 dv=dv, workspace=ws), flush, stream,
                                reps(2.5 * w.fwd_flops(causal) / 1e12))
                entry(f"{w.name}{', causal' if causal else ''}", "bwd", ms, w.bwd_flops(causal))
                del dq, dk, dv, ws
            clocks.mark(f"cfg{idx}{causal}", t0, time.monotonic())
        del ins, q, k, v
        torch.cuda.empty_cache()

    # sliding windows on the B=2 H=16 N=4096 D=128 shapes (FLOPs over visible pairs)
    w = workload(2)
    q, k, v, do = (t.to(dev) for t in make_inputs(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for win in ((1023, 0), (111, 0)):
        ws = torch.empty(bwd_workspace_bytes_ds(w.B, w.Hq, w.N, w.D, window=win), device=dev,
                         dtype=torch.uint8)
        f = 4.0 * w.D * w.B * w.Hq * visible_pairs(w.N, *win)
        ms = time_calls(lambda: attn_fwd(q, k, v, window=win, out=o, lse=lse), flush, stream, 30)
        entry(f"{w.name}, local window {win}", "fwd", ms, f, {"flops": "visible pairs"})
        ms = time_calls(lambda: attn_bwd(q, k, v, o, lse, do, window=win, dq=dq, dk=dk, dv=dv,
                                         workspace=ws), flush, stream, 30)
        entry(f"{w.name}, local window {win}", "bwd", ms, 2.5 * f, {"flops": "visible pairs"})

    # e4m3 forward on the same inputs (per-tensor scales = max|x| / 448)
    f8 = []
    for t in (q, k, v):
        s = float(t.float().abs().max()) / 448.0
        f8.append(((t.float() / s).to(torch.float8_e4m3fn), s))
    ms = time_calls(lambda: attn_fwd_fp8(f8[0][0], f8[1][0], f8[2][0], f8[0][1], f8[1][1],
                                         f8[2][1], causal=True, out=o, lse=lse),
                    flush, stream, 30)
    entry(f"{w.name}, e4m3 inputs", "fwd", ms, w.fwd_flops(True), {"dtype": "e4m3"})
    del q, k, v, do, o, dq, dk, dv, ws, f8
    torch.cuda.empty_cache()

    # block-sparse tiles: B=2 H=16 N=8192 D=128, a band of +-2 tiles plus every 8th key tile
    B, H, N, D = 2, 16, 8192, 128
    T = N // 128
    qt, kt = np.meshgrid(np.arange(T), np.arange(T), indexing="ij")
    tm = (np.abs(qt - kt) <= 2) | (kt % 8 == 0)
    q, k, v, do = (t.to(dev) for t in make_random(B, H, H, N, D, "bf16", seed=77))
    bm = torch.from_numpy(np.broadcast_to(tm, (B, H, T, T)).astype(np.uint8).copy()).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    # (the stored-dS workspace of the unmasked problem covers every mask)
    ws = torch.empty(bwd_workspace_bytes_ds(B, H, N, D), device=dev, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for causal in (False, True):
        pairs = visible_pairs(N, -1, 0 if causal else -1, tm)
        f = 4.0 * D * B * H * pairs
        frac_vis = pairs / (N * N)
        ms = time_calls(lambda: attn_fwd(q, k, v, causal=causal, block_mask=bm, out=o, lse=lse),
                        flush, stream, 30)
        entry(f"block-sparse B=2 H=16 N=8192 D=128, band +-2 tiles + every 8th key tile"
              f"{', causal' if causal else ''}", "fwd", ms, f,
              {"flops": "visible pairs", "visible": round(frac_vis, 4)})
        ms = time_calls(lambda: attn_bwd(q, k, v, o, lse, do, causal=causal, block_mask=bm, dq=dq,
                                         dk=dk, dv=dv, workspace=ws), flush, stream, 30)
        entry(f"block-sparse B=2 H=16 N=8192 D=128, band +-2 tiles + every 8th key tile"
              f"{', causal' if causal else ''}", "bwd", ms, 2.5 * f,
              {"flops": "visible pairs", "visible": round(frac_vis, 4)})
    del q, k, v, do, o, dq, dk, dv, ws, bm
    torch.cuda.empty_cache()
    code, where = device_status(dev)
    if code != 0:
        raise RuntimeError(f"device status {code} at wait site {where} during the config timings")
    return out


# ---------------------------------------------------------------- native arm


def run_native(args):
    import torch
    import torch.distributed as dist

    from exact_tiled_attention_37_b200 import _lib, attn_bwd, attn_fwd, bwd_workspace_bytes_ds, \
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
    # the workspace that selects the stored-dS backward (dS tiles of the mask)
    ws = torch.empty(bwd_workspace_bytes_ds(w.B, w.Hq, w.N, w.D, causal=causal), device=dev,
                     dtype=torch.uint8)
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
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    # per step: start/stop
    ev = [(mk(), mk()) for _ in range(K)]
    # per-kernel diagnostics (a separate pass: an event recorded between the
    # dK/dV and dQ kernels would keep the dQ kernel from starting on the SMs
    # the dK/dV kernel leaves): dK/dV start/stop, dQ start/stop
    n_diag = max(10, min(K, 50))
    ev_k = [tuple(mk() for _ in range(4)) for _ in range(n_diag)]
    for e in ev + ev_k:  # create the driver events before the timed region
        for x in e:
            x.record(stream)
    for _ in range(W):
        flush.zero_()
        step()
    barrier()
    code, where = device_status(dev)
    if code != 0:
        raise RuntimeError(f"device status {code} at wait site {where} during warm-up")

    peaks = load_peaks()
    with ClockSampler(local) as clocks:
        # let nvidia-smi finish starting up (its first queries run while it
        # initialises its monitoring library) before the timed region
        time.sleep(1.5)
        barrier()
        t_main0 = time.monotonic()
        for i in range(K):
            flush.zero_()
            s0, s1 = ev[i]
            s0.record(stream)
            step()
            s1.record(stream)
        barrier()
        t_main1 = time.monotonic()
        clocks.mark("main", t_main0, t_main1)
        code, where = device_status(dev)
        if code != 0:
            raise RuntimeError(f"device status {code} at wait site {where} during timing")
        # per-kernel times of the dominant backward kernels (same step, hooks on)
        t0 = time.monotonic()
        for m0, m1, d0, d1 in ev_k:
            flush.zero_()
            L.attn_debug_set_bwd_events(m0.cuda_event, m1.cuda_event)
            L.attn_debug_set_bwd_q_events(d0.cuda_event, d1.cuda_event)
            step()
        torch.cuda.synchronize(dev)
        clocks.mark("kernels", t0, time.monotonic())

        # forward and backward separately (same region shape, fewer steps)
        t0 = time.monotonic()
        fwd_ms = time_calls(lambda: attn_fwd(q, k, v, causal=causal, out=o, lse=lse), flush,
                            stream, max(10, min(K, 50)), warm=3)
        bwd_ms = time_calls(lambda: attn_bwd(q, k, v, o, lse, do, causal=causal, dq=dq, dk=dk,
                                             dv=dv, workspace=ws), flush, stream,
                            max(10, min(K, 50)), warm=3)
        clocks.mark("split", t0, time.monotonic())
        configs = None
        if rank == 0 and not args.no_configs:
            t0 = time.monotonic()
            configs = run_configs(dev, flush, stream, peaks["bf16_tflops"], clocks)
            clocks.mark("configs", t0, time.monotonic())
        time.sleep(0.1)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    kv_ms = [e[0].elapsed_time(e[1]) for e in ev_k]
    dq_ms = [e[2].elapsed_time(e[3]) for e in ev_k]
    total_ms = sum(step_ms)

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

    clk_main = clocks.summary("main")
    clk_all = clocks.summary()
    # the main region can be shorter than the sampling interval allows many
    # samples for; the whole timing window (main + fwd/bwd + configs, the same
    # kernels back to back) gives the clock a sample count worth reading
    clk_ref = clk_main if clk_main["samples"] >= 5 else clk_all
    peak, peak_kind = choose_peak(peaks, clk_ref, ms_per_step)

    # dominant kernel: the dK/dV kernel does four of the method's products
    # (S^T, dP^T, dV, dK) over the visible tile pairs, each as costly as one of
    # the forward's two products
    dom_ms = statistics.mean(kv_ms)
    dom_flops = 4 * w.fwd_flops(causal) / 2
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    sha = kernel_source_sha()
    traffic = DOMINANT_TRAFFIC["bytes"] if DOMINANT_TRAFFIC["src_sha"] == sha else None
    # stored dS tiles (bf16 128 x 128) of the visible tile pairs: written by
    # the dK/dV kernel, read by the dQ kernel
    nt = (w.N + 127) // 128
    ds_bytes = w.B * w.Hq * (nt * (nt + 1) // 2 if causal else nt * nt) * 128 * 128 * 2
    # dQ kernel: one product per tile pair (dQ += dS K_j), bound by reading
    # the dS tiles: dS and K in, dQ out
    dq_mean = statistics.mean(dq_ms)
    dq_method = (w.fwd_flops(causal) / 2) / (dq_mean * 1e-3) / 1e12
    dq_alg_bytes = ds_bytes + w.B * w.Hkv * w.N * w.D * 2 + w.B * w.Hq * w.N * w.D * 2
    dq_gbs = dq_alg_bytes / (dq_mean * 1e-3) / 1e9
    dq_traffic = DQ_TRAFFIC["bytes"] if DQ_TRAFFIC["src_sha"] == sha else None

    result = {
        "metric": METRIC,
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
                     "peak_source": f"{peaks['source']} bf16 {peak_kind}",
                     "frac_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "launch_ms": round(dom_ms, 4),
                     "flops_per_launch": dom_flops,
                     # Q, K, V, dO in; dK, dV and the dS tiles out
                     "algorithmic_bytes": (4 * w.B * w.Hq * w.N * w.D * 2 +
                                           2 * w.B * w.Hkv * w.N * w.D * 2 + ds_bytes)},
        "kernels": {
            DQ_KERNEL: {
                "bound": "hbm",
                "launch_ms": round(dq_mean, 4),
                "achieved_gbs": round(dq_gbs, 1), "peak_gbs": peaks["hbm_gbs"],
                "frac": round(dq_gbs / peaks["hbm_gbs"], 4),
                "method_tflops": round(dq_method, 1),
                "note": "one product per tile pair (dQ += dS K_j) from the stored dS tiles",
                "traffic": dq_traffic, "algorithmic_bytes": dq_alg_bytes,
                "traffic_ratio": round(dq_traffic / dq_alg_bytes, 3) if dq_traffic else None},
        },
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "kind": "pipelined throughput through the public API: per step H2D of Q, K, V, dO "
                        "and D2H of the gradients dQ, dK, dV (O and lse stay on the device); "
                        "upload / compute / download on three streams, double-buffered"},
        "clocks": {**clk_ref, "window": "main timed region" if clk_ref is clk_main else
                   "main + fwd/bwd + config timings (main region alone had "
                   f"{clk_main['samples']} samples)",
                   "main_region": clk_main,
                   "ms_x_mhz": round(ms_per_step * clk_ref["sm_mhz"], 1) if clk_ref["sm_mhz"] else None},
        "gpu_launches": 4 * K,  # forward; backward preprocess, dK/dV, dQ
    }
    if configs is not None:
        result["configs"] = configs
        result["configs_clocks"] = clocks.summary("configs")
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
    same workload and metric.  Each step runs a fixed sample of the workload --
    the forward and backward of one of its (batch, head) pairs -- and is timed
    as it runs, so steps x ms_per_step is the time actually spent; the value is
    the sample's counted FLOPs over its time (a whole workload step would take
    about B x H times as long)."""
    rank, world, _ = dist_info()
    if rank != 0:
        return
    from exact_tiled_attention_37_b200.inputs import workload
    w = workload(WORKLOAD_INDEX)
    for _ in range(args.warmup):
        cpu_baseline(w, 0.0, pairs=1)
    t0 = time.perf_counter()
    vals = [cpu_baseline(w, 0.0, pairs=1) for _ in range(args.steps)]
    timed_s = time.perf_counter() - t0
    secs = [x["seconds"] for x in vals]
    causal = w.causal[0]
    sample_flops = (w.fwd_flops(causal) + w.bwd_flops(causal)) / (w.B * w.Hq)
    ms_step = statistics.median(secs) * 1e3
    v = sample_flops / (ms_step * 1e-3) / 1e12
    result = {
        "impl": "reference",
        "metric": METRIC,
        "value": v,
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.Hq, "Hkv": w.Hkv, "N": w.N, "D": w.D,
                   "causal": causal, "passes": "fwd+bwd",
                   "sample": f"each step: fwd+bwd of 1 of the {w.B * w.Hq} (batch, head) pairs; "
                             "value = that sample's counted FLOPs / its time, extrapolated to "
                             "the whole workload only through the TFLOPS unit"},
        "timed_seconds": round(timed_s, 2),
        "cpu_baseline": {"value": v, "unit": "TFLOPS", "cores": vals[0]["cores"],
                         "kind": "oracle",
                         "sample": f"{args.steps} steps of 1 (batch, head) pair each of {w.name}, "
                                   f"fp64 NumPy/OpenBLAS, {timed_s:.1f} s timed"},
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
