#!/usr/bin/env python
"""Benchmark of the multi-tenant LoRA hot path on B200.

Default workload (N=1): the BGMV decode batch -- 36 tokens, 32 of them each
with its own adapter (32 adapters, rank 16) and 4 with id -1, h_in = h_out =
4096 (Llama-2-7B q_proj). One step is one pass of the hot path over one batch:
the segment build (lora_build_segments) and the fused shrink+expand
(lora_apply). Steps rotate over enough copies of the inputs and adapter pools
that the working set exceeds the 126 MB L2, and run as CUDA-graph replays.

Printed (rank 0): one JSON line with the metric (GB/s of algorithmic bytes),
the roofline of the dominant kernel against the measured HBM peak, the
end-to-end number through the public API with host buffers, the fp64 CPU
oracle timed on the host, SM clocks sampled during the timed region, and the
fused FP8 GEMM + LoRA epilogue at M = 16/64/256 (K 8192, N 28672): TFLOP/s,
us per call and the overhead over the same GEMM without LoRA.

Multi-GPU: one process per GPU (torchrun); each rank runs an independent
replica of the workload (no collective on the data path), value = all ranks'
bytes / the slowest rank's time ("scaling": "weak").

--impl reference runs the fp64 CPU oracle (the only reference this method
has) on the host cores for the same metric and workload.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "multi-LoRA apply GB/s & % HBM roofline; fused FP8 GEMM+LoRA TFLOP/s, µs/call"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM = 6650.0
FALLBACK_BF16 = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64000)
    ap.add_argument("--warmup", type=int, default=320)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="bgmv_decode",
                    choices=["bgmv_decode", "sgmv_tiny", "sgmv_prefill", "many_tenants"])
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 GEMM + LoRA section")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--fp8-only", action="store_true",
                    help="run only the FP8 GEMM + LoRA section and print its JSON")
    ap.add_argument("--fp8-m", type=int, nargs="+", default=[16, 64, 256])
    ap.add_argument("--fp8-reps", type=int, default=20, help="graph replays per timing")
    return ap.parse_args()


# ------------------------------------------------------------------ workloads and byte counts

def make_problem(name):
    from adapter_gemm_builder_b200 import workloads as wl
    return {"bgmv_decode": wl.bgmv_decode, "sgmv_tiny": wl.sgmv_tiny,
            "sgmv_prefill": wl.sgmv_prefill, "many_tenants": wl.many_tenants}[name]()


def apply_bytes(p, rows=None, col_frac=1.0):
    """Algorithmic bytes of one lora_apply: x rows and y read+write of tokens
    with an adapter, A_a and B_a (rank r_a, never the padding) of every adapter
    present, per slice. col_frac scales the output-column share (B, y)."""
    import numpy as np
    ids = p.ids if rows is None else p.ids[rows]
    valid = ids[ids >= 0]
    act = np.unique(valid)
    r = p.ranks[act].astype(np.int64)
    per_slice = (len(valid) * p.h_in * 2 + int(r.sum()) * p.h_in * 2
                 + col_frac * (int(r.sum()) * p.h_out * 2 + len(valid) * p.h_out * 4))
    return int(per_slice * p.n_slices)


def workload_config(p, name):
    import numpy as np
    return {"workload": name, "tokens": int(p.T), "adapters": int(p.n_adapters),
            "active_adapters": int(len(np.unique(p.ids[p.ids >= 0]))), "h_in": int(p.h_in),
            "h_out": int(p.h_out), "r_max": int(p.r_max), "slices": int(p.n_slices),
            "scale": float(p.scales[0])}


# ------------------------------------------------------------------ helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained",
                                                                          d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM, FALLBACK_BF16, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) while the timed region runs."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "-i", str(self.index),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((ts, f))
        inside = [f for ts, f in rows if t0 - 0.05 <= ts <= t1 + 0.05]
        use = inside or [f for _, f in rows]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(f[2]) for f in use if f[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for f in use:
            for n, v in zip(names, f[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(use[0][3]) if use[0][3].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(use),
                "samples_in_timed_region": len(inside)}


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "adapter_gemm_builder_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_file, workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, if the kernel source has not changed since (else None)."""
    path = os.path.join(ROOT, "profiles", f"{os.path.splitext(kernel_file)[0]}_{workload}.md")
    if not os.path.exists(path):
        return None
    want = source_hash(kernel_file)
    traffic, src = None, None
    for line in open(path):
        if line.startswith("traffic_bytes_per_launch:"):
            traffic = float(line.split(":", 1)[1])
        if line.startswith("source_sha256_16:"):
            src = line.split(":", 1)[1].strip()
    return traffic if src == want else None


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def dist_max(val, world):
    """Max of a per-rank value over all ranks (NCCL on the GPU, gloo on the host)."""
    if world == 1:
        return val
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([val], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)

def cpu_oracle_throughput(p, seconds):
    """The fp64 oracle as it stands on this host's cores, on the whole batch,
    repeated for about `seconds`: returns (GB/s, cores, repetitions)."""
    import oracle
    n = 0
    t0 = time.perf_counter()
    while True:
        for s in range(p.n_slices):
            oracle.lora_apply(p.x[s], p.A[s], p.B[s], p.ranks, p.scales, p.ids, p.y_in[s])
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    return apply_bytes(p) * n / dt / 1e9, oracle.num_threads(), n


def run_reference(args):
    """--impl reference: the fp64 CPU oracle on the host cores, K steps, each a
    bounded sample of the workload: one token with an adapter (cycling through
    the batch) over a window of 512 output columns, all slices."""
    import numpy as np

    import oracle
    rank, world, _ = dist_setup(args)
    if rank != 0:
        dist_barrier(world)
        return
    p = make_problem(args.workload)
    oracle.set_num_threads(1)
    rows = np.nonzero(p.ids >= 0)[0]
    width = min(512, p.h_out)
    nwin = max(1, p.h_out // width)
    B_win = [[np.ascontiguousarray(p.B[s][:, :, w * width:(w + 1) * width]) for w in range(nwin)]
             for s in range(p.n_slices)]
    y_win = [[np.ascontiguousarray(p.y_in[s][:, w * width:(w + 1) * width]) for w in range(nwin)]
             for s in range(p.n_slices)]

    def step(k):
        t = rows[k % len(rows)]
        w = (k // len(rows)) % nwin
        for s in range(p.n_slices):
            oracle.lora_apply(p.x[s][t:t + 1], p.A[s], B_win[s][w], p.ranks, p.scales,
                              p.ids[t:t + 1], y_win[s][w][t:t + 1])

    for k in range(args.warmup):
        step(k)
    bytes_step = np.mean([apply_bytes(p, rows=[t], col_frac=width / p.h_out) for t in rows[:64]])
    t0 = time.perf_counter()
    for k in range(args.steps):
        step(k)
    dt = time.perf_counter() - t0
    value = bytes_step * args.steps / dt / 1e9
    sample = (f"one token x {width} output columns per step, cycling over the batch's "
              f"{len(rows)} tokens with an adapter")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**workload_config(p, args.workload), "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    dist_barrier(world)


# ------------------------------------------------------------------ GPU arm

class _Events:
    """cudaEventRecordWithFlags(..., External) so that event nodes captured in a
    CUDA graph are recorded on every replay."""

    def __init__(self):
        self.rt = None
        for name in ("libcudart.so.12", "libcudart.so"):
            try:
                self.rt = ctypes.CDLL(name)
                break
            except OSError:
                continue
        if self.rt is not None:
            self.rt.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p,
                                                         ctypes.c_uint]
            self.rt.cudaEventRecordWithFlags.restype = ctypes.c_int

    def record_external(self, ev, stream):
        if self.rt is None:
            return False
        return self.rt.cudaEventRecordWithFlags(ctypes.c_void_p(ev.cuda_event),
                                                ctypes.c_void_p(stream.cuda_stream), 1) == 0


def run_ours(args):
    import numpy as np
    import torch

    from adapter_gemm_builder_b200 import lora as L

    rank, world, local = dist_setup(args)
    torch.cuda.set_device(local)
    L.load()
    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, bf16_sust, peak_src = measured_peaks()

    p = make_problem(args.workload)
    set_bytes = (p.A.nbytes + p.B.nbytes) // max(1, p.n_adapters) * max(1, len(np.unique(p.ids[p.ids >= 0]))) \
        + p.x.nbytes + p.y_in.nbytes
    R = int(min(64, max(1, math.ceil(2.5 * L2_BYTES / max(set_bytes, 1)))))
    bytes_step = apply_bytes(p)

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    base = dict(x=to_dev(p.x), A=to_dev(p.A), B=to_dev(p.B), y=to_dev(p.y_in),
                ids=torch.from_numpy(p.ids).to(dev), ranks=torch.from_numpy(p.ranks).to(dev),
                scales=torch.from_numpy(p.scales).to(dev))
    sets = []
    for k in range(R):
        d = {key: (v.clone() if k else v) for key, v in base.items()}
        d["pool"] = L.Pool(d["A"], d["B"], d["ranks"], d["scales"])
        d["seg"] = L.Segments(p.T, p.n_adapters, device=dev)
        sets.append(d)

    stream = torch.cuda.Stream(device=dev)
    ext = _Events()

    def step(d):
        L.lora_build_segments(d["ids"], p.n_adapters, d["seg"])
        L.lora_apply(d["x"], d["pool"], d["seg"], d["y"])

    K, W = args.steps, max(3, args.warmup)
    nfull, rem = divmod(K, R)
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(R)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(R)]
    with torch.cuda.stream(stream):
        for ev in ev_a + ev_b:  # create the CUDA events before capture
            ev.record(stream)
        for d in sets:          # eager pass: sets kernel attributes before capture
            step(d)
        torch.cuda.synchronize()
        # the timed steps replay a graph without events (the segment builder and the apply
        # overlap through programmatic dependent launch); a copy with an event pair around
        # every apply is replayed once, as the last full replay of the timed region
        g_full = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_full, stream=stream):
            for d in sets:
                step(d)
        g_inst = torch.cuda.CUDAGraph()
        inner_ok = True
        with torch.cuda.graph(g_inst, stream=stream):
            cs = torch.cuda.current_stream()
            for k, d in enumerate(sets):
                L.lora_build_segments(d["ids"], p.n_adapters, d["seg"])
                inner_ok &= ext.record_external(ev_a[k], cs)
                L.lora_apply(d["x"], d["pool"], d["seg"], d["y"])
                inner_ok &= ext.record_external(ev_b[k], cs)
        g_rem = None
        if rem:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem, stream=stream):
                for d in sets[:rem]:
                    step(d)
        # warm-up (untimed): W steps
        for _ in range(math.ceil(W / R)):
            g_full.replay()
        g_inst.replay()
        stream.synchronize()

    try:
        clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    except Exception:
        clocks = ClockSampler(str(local))
    clocks.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    torch.cuda.synchronize()
    t_host0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(nfull):
            (g_inst if (i == nfull - 1 and inner_ok) else g_full).replay()
        if g_rem is not None:
            g_rem.replay()
        end.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    dist_barrier(world)
    clk = clocks.stop(t_host0, t_host1)
    ms = start.elapsed_time(end)
    ms_max = dist_max(ms, world)

    # dominant kernel: lora_apply, events around each launch inside the timed region
    kernel_ms = None
    timing_src = "events around each lora_apply launch in the last graph replay of the timed region"
    if inner_ok and nfull > 0:
        kernel_ms = statistics.mean(ev_a[k].elapsed_time(ev_b[k]) for k in range(R))
    else:
        timing_src = "events around a graph of back-to-back lora_apply launches after the timed region"
        g_k = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g_k, stream=stream):
                for d in sets:
                    L.lora_apply(d["x"], d["pool"], d["seg"], d["y"])
            for _ in range(3):
                g_k.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(20):
                g_k.replay()
            b.record(stream)
        torch.cuda.synchronize()
        kernel_ms = a.elapsed_time(b) / (20 * R)

    value = bytes_step * K * world / (ms_max / 1e3) / 1e9
    achieved = bytes_step / (kernel_ms / 1e3) / 1e9
    traffic = profiled_traffic("sgmv.cu", args.workload)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "kernel": "sgmv_kernel<APPLY> (lora_apply)", "kernel_us": kernel_ms * 1e3,
                "algorithmic_bytes_per_launch": bytes_step,
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
                "timing": timing_src}

    # end to end through the public API with host buffers
    e2e = run_e2e(args, p, sets[0], stream, bytes_step)

    fp8 = None if args.no_fp8 else run_fp8(args, dev, stream, hbm_peak, bf16_peak, bf16_sust, peak_src)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, n = cpu_oracle_throughput(p, args.cpu_seconds)
        cpu = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"the whole batch ({p.T} tokens, {p.n_slices} slice(s)) x {n} repetitions"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(p, args.workload),
                       "l2": f"rotating {R} input sets ({R * set_bytes / 2**20:.0f} MiB > 126 MB L2)",
                       "launch": f"CUDA graph of {R} steps", "parallelism": f"replicas x{world}"},
            "roofline": roofline, "e2e": e2e, "gpu_launches": 2 * K, "clocks": clk,
            "cpu_baseline": cpu, "fp8_gemm_lora": fp8,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(args, p, d, stream, bytes_step):
    """Same metric through the public API: every step copies the batch's x, ids and
    base output y from pinned host memory, builds segments, applies, and reads y back.
    The steps are captured in a CUDA graph of G steps and replayed, as a serving loop
    would drive them, so that Python's per-call launch cost does not set the rate."""
    import torch

    from adapter_gemm_builder_b200 import lora as L
    # the step's inputs travel as one pinned host block (x | ids | y, 256-byte aligned
    # sections) into one device block that the calls take views of: one copy each way.
    # Two device blocks alternate, so that step k+1's upload (its own stream) overlaps
    # step k's kernels and step k-1's download (a third stream).
    def align(n):
        return (n + 255) // 256 * 256
    nx, ni, ny = d["x"].numel() * 2, d["ids"].numel() * 4, d["y"].numel() * 2
    ox, oi, oy = 0, align(nx), align(nx) + align(ni)
    total = oy + align(ny)
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    host[ox:ox + nx].copy_(d["x"].cpu().contiguous().view(-1).view(torch.uint8))
    host[oi:oi + ni].copy_(d["ids"].cpu().contiguous().view(-1).view(torch.uint8))
    host[oy:oy + ny].copy_(d["y"].cpu().contiguous().view(-1).view(torch.uint8))
    blocks = [torch.empty(total, dtype=torch.uint8, device=d["x"].device) for _ in range(2)]
    views = [(bk[ox:ox + nx].view(torch.bfloat16).view(d["x"].shape),
              bk[oi:oi + ni].view(torch.int32).view(d["ids"].shape),
              bk[oy:oy + ny].view(torch.bfloat16).view(d["y"].shape)) for bk in blocks]
    yo = torch.empty(ny, dtype=torch.uint8).pin_memory()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    E = max(10, args.e2e_steps)
    G = 20

    def steps(n):
        ev_up = [torch.cuda.Event() for _ in range(n)]
        ev_run = [torch.cuda.Event() for _ in range(n)]
        ev_down = [torch.cuda.Event() for _ in range(n)]
        up.wait_stream(stream)
        down.wait_stream(stream)
        for k in range(n):
            bk = k % 2
            xv, iv, yv = views[bk]
            with torch.cuda.stream(up):  # block bk is free once step k-2 was read back
                if k >= 2:
                    up.wait_event(ev_down[k - 2])
                blocks[bk].copy_(host, non_blocking=True)
                ev_up[k].record(up)
            stream.wait_event(ev_up[k])
            L.lora_build_segments(iv, p.n_adapters, d["seg"])
            L.lora_apply(xv, d["pool"], d["seg"], yv)
            ev_run[k].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_run[k])
                yo.copy_(blocks[bk][oy:oy + ny], non_blocking=True)
                ev_down[k].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)

    with torch.cuda.stream(stream):
        steps(4)
        stream.synchronize()
        reps = max(1, E // G)
        E = reps * G
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            steps(G)
        for _ in range(2):
            g.replay()
        stream.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    return {"value": bytes_step * E / (ms / 1e3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": int(total), "d2h_bytes_per_step": int(ny),
            "ms_per_step": ms / E, "steps": E,
            "launch": f"CUDA graph of {G} steps, replayed; uploads, kernels and downloads on three streams, two device blocks"}


def run_fp8(args, dev, stream, hbm_peak, bf16_peak, bf16_sust, peak_src):
    """Fused FP8 GEMM + LoRA epilogue, K 8192, N 28672, 16 adapters of rank 16,
    Zipf(1.1) ids, at M = 16, 64, 256, against the same call without LoRA."""
    import numpy as np
    import torch

    from adapter_gemm_builder_b200 import lora as L
    from adapter_gemm_builder_b200 import workloads as wl
    K, N, n_ad, r = 8192, 28672, 16, 16
    gen = torch.Generator(device=dev).manual_seed(3)
    W = (torch.randn((N, K), generator=gen, device=dev) * (1.0 / math.sqrt(K))).to(torch.bfloat16)
    Wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
    sw = torch.empty(N, dtype=torch.float32, device=dev)
    L.fp8_quantize_rows(W, Wq, sw)
    del W
    fp8_peak = 2.0 * bf16_peak  # dense FP8 = 2x dense bf16 (nominal ratio)
    out = {"shape": {"K": K, "N": N, "adapters": n_ad, "r": r, "ids": "zipf(1.1)"},
           "peak_tflops_fp8": fp8_peak, "peak_hbm_gbs": hbm_peak,
           "peak_source": f"{peak_src}: FP8 = 2 x bf16_tflops (nominal dense ratio)", "M": {}}
    for M in args.fp8_m:
        q = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=r, seed=3, W=np.zeros((1, 1), np.uint16))
        tb = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        x = tb(q.x)
        pool = L.Pool(tb(q.A), tb(q.B), torch.from_numpy(q.ranks).to(dev),
                      torch.from_numpy(q.scales).to(dev))
        seg = L.Segments(M, n_ad, device=dev)
        ids = torch.from_numpy(q.ids).to(dev)
        L.lora_build_segments(ids, n_ad, seg)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = L.workspace(L.LORA_OP_FP8_GEMM, M, K, pool, device=dev)
        ws0 = L.workspace(L.LORA_OP_FP8_GEMM, M, K, None, device=dev)
        res = {}
        for tag, pl, sg, w in (("lora", pool, seg, ws), ("base", None, None, ws0)):
            with torch.cuda.stream(stream):
                L.fp8_gemm_lora_epilogue(x, Wq, sw, pl, sg, y, w)
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                reps = 10
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(reps):
                        L.fp8_gemm_lora_epilogue(x, Wq, sw, pl, sg, y, w)
                for _ in range(min(3, args.fp8_reps)):
                    g.replay()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                n_rep = args.fp8_reps
                for _ in range(n_rep):
                    g.replay()
                b.record(stream)
            torch.cuda.synchronize()
            st, detail = L.lora_workspace_status(w)
            res[tag] = a.elapsed_time(b) / (n_rep * reps) * 1e3  # us per call
            res[tag + "_status"] = st
        act = np.unique(q.ids)
        lora_bytes = int(len(act)) * r * (K + N) * 2 + M * r * 4
        bytes_call = N * K + N * 4 + M * K * 2 + M * N * 2 + lora_bytes
        flops = 2.0 * M * N * K
        t = res["lora"] * 1e-6
        out["M"][str(M)] = {
            "us_per_call": res["lora"], "us_per_call_no_lora": res["base"],
            "overhead_vs_no_lora": res["lora"] / res["base"] - 1.0,
            "tflops": flops / t / 1e12, "tensor_frac": flops / t / 1e12 / fp8_peak,
            "hbm_gbs": bytes_call / t / 1e9, "hbm_frac": bytes_call / t / 1e9 / hbm_peak,
            "attainable_frac": (flops / t) / min(fp8_peak * 1e12, flops / bytes_call * hbm_peak * 1e9),
            "distinct_adapters": int(len(act)), "status_ok": res["lora_status"] == 0,
        }
    return out


def main():
    args = parse_args()
    if args.fp8_only:
        import torch
        from adapter_gemm_builder_b200 import lora as L
        L.load()
        dev = torch.device("cuda", 0)
        hbm, bf16, sust, src = measured_peaks()
        print(json.dumps(run_fp8(args, dev, torch.cuda.Stream(device=dev), hbm, bf16, sust, src)))
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
