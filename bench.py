#!/usr/bin/env python
"""Benchmark of the multi-tenant LoRA hot path on B200.

Headline workload (N=1): many tenants -- 512 decode tokens over 256 adapters of
ranks {8, 16, 32, 64} (pool padded to 64), Zipf(1.1) ids with 5% at -1,
h_in = h_out = 5120 (Llama-2-13B o_proj shape), the q/k/v/o projections applied
in one call. One step is one pass of the hot path over one batch: the segment
build (lora_build_segments) and the fused shrink+expand (lora_apply). Steps
rotate over enough copies of the inputs and adapter pools that the working set
exceeds the 126 MB L2 (the label says so, or says "L2-resident" when it cannot),
and run as CUDA-graph replays.

Printed (rank 0): one JSON line with the metric (GB/s of algorithmic bytes),
the roofline of the dominant kernel against the measured HBM peak, the
end-to-end number through the public API with host buffers, the fp64 CPU
oracle timed on the host (all cores and one core, with the CPU model), SM
clocks sampled during the timed region, the other workloads of the method
(BGMV decode, SGMV prefill, SGMV tiny, and Punica's Identical and Uniform
popularity settings) each with its own roofline, and the fused FP8 GEMM +
LoRA epilogue at M = 16/64/256 (K 8192, N 28672): TFLOP/s, us per call and the
overhead over the same GEMM without LoRA.

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
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="many_tenants", choices=list(WORKLOADS))
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 GEMM + LoRA section")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--fp8-only", action="store_true",
                    help="run only the FP8 GEMM + LoRA section and print its JSON")
    ap.add_argument("--no-backward", action="store_true", help="skip the FP8 backward section")
    ap.add_argument("--section", choices=["fp8", "bf16", "w8a16", "mxfp4", "merge", "backward"],
                    help="run only this GEMM / merge section and print its JSON (profiling aid)")
    ap.add_argument("--fp8-m", type=int, nargs="+", default=[16, 64, 256])
    ap.add_argument("--fp8-reps", type=int, default=20, help="graph replays per timing")
    ap.add_argument("--no-bf16", action="store_true", help="skip the bf16 GEMM + LoRA section")
    ap.add_argument("--no-merge", action="store_true", help="skip the adapter-merge section")
    ap.add_argument("--no-mxfp4", action="store_true", help="skip the MX FP4 and W8A16 GEMM + LoRA sections")
    return ap.parse_args()


# ------------------------------------------------------------------ workloads and byte counts

WORKLOADS = {
    # name: (generator, keyword arguments)
    "many_tenants": ("many_tenants", {}),
    "bgmv_decode": ("bgmv_decode", {}),
    "sgmv_prefill": ("sgmv_prefill", {}),
    "sgmv_tiny": ("sgmv_tiny", {}),
    # Punica's popularity settings on the same shapes: Identical (every token on one
    # adapter, BGMV decode shapes) and Uniform (ids uniform over the adapters, many-tenant shapes)
    "identical": ("bgmv_decode", {"ids_kind": "identical"}),
    "uniform": ("many_tenants", {"ids_kind": "uniform"}),
}


def make_problem(name):
    from adapter_gemm_builder_b200 import workloads as wl
    gen, kw = WORKLOADS[name]
    p = getattr(wl, gen)(**kw)
    p.name = name
    return p


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
    """DRAM bytes per lora_apply call (its one launch, or both launches of the
    tensor-core pair) from the committed ncu summary of this kernel source and
    workload, if the source has not changed since (else None)."""
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


def apply_launches(p, sm_count=None):
    """Kernels of this library one lora_apply (with its workspace) launches: for a batch
    of long segments the shrink and the tensor-core expand; otherwise the cluster
    kernel, preceded by the tile-ordering kernel when the batch is not decode-like and
    its clusters need more than one wave of two CTAs per SM (the library's rules)."""
    from adapter_gemm_builder_b200 import lora as L
    if p.T <= 64 and p.T <= 2 * p.n_adapters:
        return 1
    if tc_path(p):
        return 2
    if sm_count is None:
        import torch
        sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    rows = L.max_tiles(p.T, p.n_adapters) * p.n_slices
    slots = 2 * sm_count
    c = min(8, max(1, (p.h_in + 511) // 512))
    if rows * c > slots:
        c = max(slots // rows, min(c, 2)) if rows <= slots else (1 if rows * min(c, 2) > 8 * slots else min(c, 2))
    return 2 if rows * c > slots else 1


def time_apply(p, dev, steps, warmup, stream, ext, world=1, clocks=None):
    """Time `steps` steps (segment build + lora_apply) of workload p on device dev.
    Inputs rotate over R copies whose total exceeds 2.5x the L2 when that takes at
    most 64 copies (else the label says the working set is L2-resident). Returns
    a dict with the step time (max over ranks), the apply's own time from events
    around each launch in the last replay, and the labels."""
    import numpy as np
    import torch

    from adapter_gemm_builder_b200 import lora as L
    act = np.unique(p.ids[p.ids >= 0])
    set_bytes = (p.A.nbytes + p.B.nbytes) // max(1, p.n_adapters) * max(1, len(act)) \
        + p.x.nbytes + p.y_in.nbytes
    want_r = math.ceil(2.5 * L2_BYTES / max(set_bytes, 1))
    R = int(min(64, max(1, want_r)))
    l2_label = (f"rotating {R} input sets ({R * set_bytes / 2**20:.0f} MiB > 2.5 x 126 MB L2)"
                if R == want_r else
                f"L2-resident: {R} rotating input sets of {set_bytes / 2**20:.2f} MiB "
                f"({R * set_bytes / 2**20:.0f} MiB < 126 MB L2)")

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
        d["ws"] = L.workspace(L.LORA_OP_APPLY, p.T, 0, d["pool"], device=dev)
        sets.append(d)

    def step(d):
        L.lora_build_segments(d["ids"], p.n_adapters, d["seg"])
        L.lora_apply(d["x"], d["pool"], d["seg"], d["y"], ws=d["ws"])

    K, W = steps, max(3, warmup)
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
                L.lora_apply(d["x"], d["pool"], d["seg"], d["y"], ws=d["ws"])
                inner_ok &= ext.record_external(ev_b[k], cs)
        g_rem = None
        if rem:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem, stream=stream):
                for d in sets[:rem]:
                    step(d)
        for _ in range(math.ceil(W / R)):  # warm-up (untimed): >= W steps
            g_full.replay()
        g_inst.replay()
        stream.synchronize()

    if clocks is not None:
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
    clk = clocks.stop(t_host0, t_host1) if clocks is not None else None
    ms = start.elapsed_time(end)
    ms_max = dist_max(ms, world)
    statuses = [L.lora_segments_status(d["seg"])[0] for d in sets]

    timing_src = "events around each lora_apply launch in the last graph replay of the timed region"
    if inner_ok and nfull > 0:
        kernel_ms = statistics.mean(ev_a[k].elapsed_time(ev_b[k]) for k in range(R))
    else:
        timing_src = "events around a graph of back-to-back lora_apply launches after the timed region"
        g_k = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g_k, stream=stream):
                for d in sets:
                    L.lora_apply(d["x"], d["pool"], d["seg"], d["y"], ws=d["ws"])
            for _ in range(3):
                g_k.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(20):
                g_k.replay()
            b.record(stream)
        torch.cuda.synchronize()
        kernel_ms = a.elapsed_time(b) / (20 * R)
    return dict(ms_max=ms_max, kernel_ms=kernel_ms, R=R, l2=l2_label, timing=timing_src,
                clocks=clk, sets=sets, status_ok=all(st == L.LORA_OK for st in statuses),
                launch=f"CUDA graph of {R} steps")


def tc_path(p):
    """lora_apply (with its workspace) takes the tensor-core shrink and expand: a batch of
    long segments (not decode-like, T >= 32 n_adapters, h_out >= 128; the library's rule)."""
    return not (p.T <= 64 and p.T <= 2 * p.n_adapters) and p.T >= 32 * p.n_adapters and p.h_out >= 128


def roofline_apply(p, t, hbm_peak, peak_src, workload):
    bytes_step = apply_bytes(p)
    achieved = bytes_step / (t["kernel_ms"] / 1e3) / 1e9
    tc = tc_path(p)
    return {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak,
            "traffic": profiled_traffic("sgmv_tc.cu" if tc else "sgmv.cu", workload),
            "kernel": "lora_apply (tensor-core shrink + expand)" if tc else "lora_apply (sgmv kernels)",
            "kernel_us": t["kernel_ms"] * 1e3,
            "launches_per_call": apply_launches(p),
            "algorithmic_bytes_per_call": bytes_step,  # every launch of one lora_apply together
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
            "timing": t["timing"]}


def run_ours(args):
    import torch

    from adapter_gemm_builder_b200 import lora as L

    rank, world, local = dist_setup(args)
    torch.cuda.set_device(local)
    L.load()
    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, bf16_sust, peak_src = measured_peaks()
    stream = torch.cuda.Stream(device=dev)
    ext = _Events()

    p = make_problem(args.workload)
    bytes_step = apply_bytes(p)
    try:
        clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    except Exception:
        clocks = ClockSampler(str(local))
    t = time_apply(p, dev, args.steps, args.warmup, stream, ext, world, clocks)
    K, W = args.steps, max(3, args.warmup)
    value = bytes_step * K * world / (t["ms_max"] / 1e3) / 1e9
    roofline = roofline_apply(p, t, hbm_peak, peak_src, args.workload)

    # end to end through the public API with host buffers
    e2e = run_e2e(args, p, t["sets"][0], stream, bytes_step)
    del t["sets"]

    # the other workloads of the method, each with its own roofline (not the headline)
    extras = {}
    if not args.no_extras:
        for name in WORKLOADS:
            if name == args.workload:
                continue
            q = make_problem(name)
            tq = time_apply(q, dev, 200, 10, stream, ext, world, None)
            del tq["sets"]
            extras[name] = {
                "config": workload_config(q, name), "l2": tq["l2"],
                "gb_per_s_step": apply_bytes(q) * 200 / (tq["ms_max"] / 1e3) / 1e9,
                "us_per_step": tq["ms_max"] * 1e3 / 200,
                "roofline": roofline_apply(q, tq, hbm_peak, peak_src, name),
                "status_ok": tq["status_ok"]}

    fp8 = None if args.no_fp8 else run_fp8(args, dev, stream, hbm_peak, bf16_peak, bf16_sust, peak_src)
    bf16 = None if args.no_bf16 else run_bf16(args, dev, stream, hbm_peak, bf16_peak, peak_src)
    merge = None if args.no_merge else run_merge(args, dev, stream, hbm_peak, peak_src)
    mxfp4 = None if args.no_mxfp4 else run_mxfp4(args, dev, stream, hbm_peak, bf16_peak, peak_src)
    w8a16 = None if args.no_mxfp4 else run_mxfp4(args, dev, stream, hbm_peak, bf16_peak, peak_src, "w8a16")
    backward = None if args.no_backward else run_backward(args, dev, stream, hbm_peak, bf16_peak, peak_src)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(p, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": t["ms_max"] / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(p, args.workload), "l2": t["l2"], "launch": t["launch"],
                       "parallelism": f"replicas x{world}"},
            "roofline": roofline, "e2e": e2e, "gpu_launches": (1 + apply_launches(p)) * K,
            "clocks": t["clocks"], "status_ok": t["status_ok"],
            "cpu_baseline": cpu, "workloads": extras, "fp8_gemm_lora": fp8, "bf16_gemm_lora": bf16,
            "switch_merge": merge, "mxfp4_gemm_lora": mxfp4, "w8a16_gemm_lora": w8a16,
            "fp8_lora_backward": backward,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(p, seconds):
    """The fp64 oracle as it stands, on this host: all cores on the whole batch for
    about `seconds`, and one core on a bounded sample (a few tokens, all slices)."""
    import numpy as np

    import oracle
    all_cores = oracle.num_threads()
    v_all, _, n = cpu_oracle_throughput(p, seconds)
    oracle.set_num_threads(1)
    try:
        rows = np.nonzero(p.ids >= 0)[0][:8]
        t0 = time.perf_counter()
        reps = 0
        while True:
            for s in range(p.n_slices):
                oracle.lora_apply(p.x[s][rows], p.A[s], p.B[s], p.ranks, p.scales, p.ids[rows],
                                  p.y_in[s][rows])
            reps += 1
            if time.perf_counter() - t0 >= seconds / 2:
                break
        dt = time.perf_counter() - t0
        v_one = apply_bytes(p, rows=rows) * reps / dt / 1e9
    finally:
        oracle.set_num_threads(all_cores)
    return {"value": v_all, "unit": "GB/s", "cores": all_cores, "kind": "oracle",
            "sample": f"the whole batch ({p.T} tokens, {p.n_slices} slice(s)) x {n} repetitions",
            "cpu_model": cpu_model(),
            "one_core": {"value": v_one, "unit": "GB/s", "cores": 1,
                         "sample": f"{len(rows)} tokens with an adapter, all slices, x {reps} repetitions"}}


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
            L.lora_apply(xv, d["pool"], d["seg"], yv, ws=d["ws"])
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
        act = np.unique(q.ids)
        lora_bytes = int(len(act)) * r * (K + N) * 2 + M * r * 4
        # the token activations, the adapters and y rotate over enough copies to pass
        # the L2 (W, 235 MB, is read once per call anyway)
        set_bytes = q.x.nbytes + q.A.nbytes + q.B.nbytes + M * N * 2
        R = int(min(32, max(2, math.ceil(2.5 * L2_BYTES / set_bytes))))
        base = dict(x=tb(q.x), A=tb(q.A), B=tb(q.B), ids=torch.from_numpy(q.ids).to(dev),
                    ranks=torch.from_numpy(q.ranks).to(dev), scales=torch.from_numpy(q.scales).to(dev))
        sets = []
        for k in range(R):
            d = {key: (v.clone() if k else v) for key, v in base.items()}
            d["pool"] = L.Pool(d["A"], d["B"], d["ranks"], d["scales"])
            d["seg"] = L.Segments(M, n_ad, device=dev)
            L.lora_build_segments(d["ids"], n_ad, d["seg"])
            d["y"] = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            d["ws"] = L.workspace(L.LORA_OP_FP8_GEMM, M, K, d["pool"], device=dev)
            d["ws0"] = L.workspace(L.LORA_OP_FP8_GEMM, M, K, None, device=dev)
            sets.append(d)
        res = {}
        for tag in ("lora", "base"):
            def call(d):
                if tag == "lora":
                    L.fp8_gemm_lora_epilogue(d["x"], Wq, sw, d["pool"], d["seg"], d["y"], d["ws"])
                else:
                    L.fp8_gemm_lora_epilogue(d["x"], Wq, sw, None, None, d["y"], d["ws0"])
            with torch.cuda.stream(stream):
                for d in sets:
                    call(d)
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for d in sets:
                        call(d)
                for _ in range(min(3, args.fp8_reps)):
                    g.replay()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                n_rep = args.fp8_reps
                for _ in range(n_rep):
                    g.replay()
                b.record(stream)
            torch.cuda.synchronize()
            res[tag] = a.elapsed_time(b) / (n_rep * R) * 1e3  # us per call
            res[tag + "_status"] = max(L.lora_workspace_status(d["ws" if tag == "lora" else "ws0"])[0]
                                       for d in sets)
        bytes_call = N * K + N * 4 + M * K * 2 + M * N * 2 + lora_bytes
        flops = 2.0 * M * N * K
        t = res["lora"] * 1e-6
        lib_ref = library_fp8_gemm(dev, stream, sets[0]["x"], Wq, sw, args.fp8_reps)
        out["M"][str(M)] = {
            "us_per_call": res["lora"], "us_per_call_no_lora": res["base"],
            "overhead_vs_no_lora": res["lora"] / res["base"] - 1.0,
            "tflops": flops / t / 1e12, "tensor_frac": flops / t / 1e12 / fp8_peak,
            "hbm_gbs": bytes_call / t / 1e9, "hbm_frac": bytes_call / t / 1e9 / hbm_peak,
            "attainable_frac": (flops / t) / min(fp8_peak * 1e12, flops / bytes_call * hbm_peak * 1e9),
            "distinct_adapters": int(len(act)), "status_ok": res["lora_status"] == 0 and res["base_status"] == 0,
            "l2": f"x, adapters and y rotate over {R} copies ({R * set_bytes / 2**20:.0f} MiB); W read once per call",
            "library_base": lib_ref,
        }
        del sets
    return out


def library_fp8_gemm(dev, stream, x, Wq, sw, reps):
    """The base GEMM alone through a library kernel on the same box, as a side
    comparison for the call without LoRA: torch._scaled_mm on the same E4M3 operands
    (x quantised per token by this library's quantiser) with per-row and per-channel
    scales, bf16 out. A library GEMM; nothing of it is on this library's path."""
    import torch

    from adapter_gemm_builder_b200 import lora as L
    M, K = x.shape
    N = Wq.shape[0]
    xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
    sx = torch.empty(M, dtype=torch.float32, device=dev)
    L.fp8_quantize_rows(x, xq, sx)
    a = xq.view(torch.float8_e4m3fn)
    b = Wq.view(torch.float8_e4m3fn).t()
    try:
        def f():
            return torch._scaled_mm(a, b, scale_a=sx.view(M, 1), scale_b=sw.view(1, N), out_dtype=torch.bfloat16)
        with torch.cuda.stream(stream):
            for _ in range(3):
                f()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n = max(5, reps)
            e0.record(stream)
            for _ in range(n):
                f()
            e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / n * 1e3
        return {"kernel": "torch._scaled_mm, row-wise scales (library GEMM)", "us_per_call": us,
                "tflops": 2.0 * M * N * K / (us * 1e-6) / 1e12,
                "note": "same weights back to back: W (235 MB) exceeds L2, x and y stay L2-warm"}
    except Exception as exc:  # a library without this path on this machine: say so
        return {"kernel": "torch._scaled_mm", "unavailable": str(exc).splitlines()[0][:200]}


BF16_CASES = [
    # name, M, K, N, adapters, rank choices, r_max, ids kind, fraction of tokens at -1
    ("llama70b_up_M16", 16, 8192, 28672, 16, (16,), 16, "zipf", 0.0),
    ("llama70b_up_M64", 64, 8192, 28672, 16, (16,), 16, "zipf", 0.0),
    ("llama70b_up_M256", 256, 8192, 28672, 16, (16,), 16, "zipf", 0.0),
    ("bgmv_decode", 36, 4096, 4096, 32, (16,), 16, "distinct36", 0.0),
    ("many_tenants_one_slice", 512, 5120, 5120, 256, (8, 16, 32, 64), 64, "zipf", 0.05),
    ("sgmv_prefill", 2704, 4096, 11008, 8, (64,), 64, "prefill", 0.0),
]


def run_bf16(args, dev, stream, hbm_peak, bf16_peak, peak_src):
    """The 16-bit base GEMM with the fused LoRA term (one call per projection) on the
    decode shapes of the FP8 section and on the bf16 workloads' shapes, each against the
    same call without LoRA. Inputs are drawn on the device from a seeded generator with
    the workloads' distributions; W, x, the adapters and y rotate over enough copies to
    pass the L2."""
    import numpy as np
    import torch

    from adapter_gemm_builder_b200 import lora as L
    from adapter_gemm_builder_b200 import workloads as wl
    out = {"peak_tflops_bf16": bf16_peak, "peak_hbm_gbs": hbm_peak,
           "peak_source": f"{peak_src} (MEASURED_PEAKS.json bf16_tflops, burst cuBLAS)", "cases": {}}
    gen = torch.Generator(device=dev).manual_seed(11)

    def randn(shape, std):
        return (torch.randn(shape, generator=gen, device=dev) * std).to(torch.bfloat16)

    for name, M, K, N, n_ad, rchoice, r_max, kind, none_frac in BF16_CASES:
        rng = np.random.default_rng(M + N)
        if kind == "distinct36":
            ids = rng.permutation(np.concatenate([np.arange(32), np.full(4, -1)])).astype(np.int32)
        elif kind == "prefill":
            ids = np.repeat(np.arange(8, dtype=np.int32), wl.sgmv_prefill_lengths())
            M = int(ids.shape[0])
        else:
            ids = wl.make_ids(kind, rng, M, n_ad, none_frac)
        ranks = rng.choice(np.asarray(rchoice, np.int32), size=n_ad).astype(np.int32)
        act = np.unique(ids[ids >= 0])
        lora_bytes = int(ranks[act].sum()) * (K + N) * 2 + M * r_max * 4
        base_bytes = N * K * 2 + M * K * 2 + M * N * 2
        set_bytes = base_bytes + int(ranks[act].sum()) * (K + N) * 2
        R = int(min(16, max(1, math.ceil(2.5 * L2_BYTES / set_bytes))))
        sets = []
        for k in range(R):
            d = dict(x=randn((M, K), 1.0), W=randn((N, K), 1.0 / math.sqrt(K)),
                     A=randn((n_ad, K, r_max), 1.0 / math.sqrt(K)),
                     B=randn((n_ad, r_max, N), 1.0 / math.sqrt(max(1, r_max))),
                     y=torch.empty((M, N), dtype=torch.bfloat16, device=dev))
            d["pool"] = L.Pool(d["A"], d["B"], torch.from_numpy(ranks).to(dev),
                               torch.full((n_ad,), 2.0, dtype=torch.float32, device=dev))
            d["seg"] = L.Segments(M, n_ad, device=dev)
            L.lora_build_segments(torch.from_numpy(ids).to(dev), n_ad, d["seg"])
            d["ws"] = L.workspace(L.LORA_OP_BF16_GEMM, M, K, d["pool"], device=dev)
            d["ws0"] = L.workspace(L.LORA_OP_BF16_GEMM, M, K, None, device=dev)
            sets.append(d)
        res = {}
        for tag in ("lora", "base"):
            def call(d):
                if tag == "lora":
                    L.bf16_gemm_lora_epilogue(d["x"], d["W"], d["pool"], d["seg"], d["y"], d["ws"])
                else:
                    L.bf16_gemm_lora_epilogue(d["x"], d["W"], None, None, d["y"], d["ws0"])
            with torch.cuda.stream(stream):
                for d in sets:
                    call(d)
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for d in sets:
                        call(d)
                for _ in range(3):
                    g.replay()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                reps = max(2, 40 // R)
                a.record(stream)
                for _ in range(reps):
                    g.replay()
                b.record(stream)
            torch.cuda.synchronize()
            res[tag] = a.elapsed_time(b) / (reps * R) * 1e3
            res[tag + "_status"] = max(L.lora_workspace_status(d["ws" if tag == "lora" else "ws0"])[0]
                                       for d in sets)
        t = res["lora"] * 1e-6
        flops = 2.0 * M * N * K
        bytes_call = base_bytes + lora_bytes
        out["cases"][name] = {
            "M": M, "K": K, "N": N, "adapters": n_ad, "active_adapters": int(len(act)),
            "us_per_call": res["lora"], "us_per_call_no_lora": res["base"],
            "overhead_vs_no_lora": res["lora"] / res["base"] - 1.0,
            "tflops": flops / t / 1e12, "tensor_frac": flops / t / 1e12 / bf16_peak,
            "hbm_gbs": bytes_call / t / 1e9, "hbm_frac": bytes_call / t / 1e9 / hbm_peak,
            "attainable_frac": (flops / t) / min(bf16_peak * 1e12, flops / bytes_call * hbm_peak * 1e9),
            "status_ok": res["lora_status"] == 0 and res["base_status"] == 0,
            "l2": f"W, x, the adapters and y rotate over {R} copies ({R * set_bytes / 2**20:.0f} MiB)",
        }
        del sets
    return out


def run_mxfp4(args, dev, stream, hbm_peak, bf16_peak, peak_src, fmt="mxfp4"):
    """A low-bit weight base with bf16 activations and the fused LoRA term at the FP8
    section's decode shapes (K 8192, N 28672, 16 adapters of rank 16, Zipf ids), against
    the same call without LoRA: us per call, TFLOP/s against the bf16 peak (its MMAs are
    kind::f16) and the HBM fraction of its algorithmic bytes (weight codes and scales, x,
    y and the adapters present). fmt "mxfp4": OCP MX FP4 weights; "w8a16": E4M3 weights
    with one fp32 scale per output channel."""
    import numpy as np
    import torch

    from adapter_gemm_builder_b200 import lora as L
    from adapter_gemm_builder_b200 import workloads as wl
    K, N, n_ad, r = 8192, 28672, 16, 16
    gen = torch.Generator(device=dev).manual_seed(5)
    W = (torch.randn((N, K), generator=gen, device=dev) * (1.0 / math.sqrt(K))).to(torch.bfloat16)
    if fmt == "mxfp4":
        Wp = torch.zeros(L.mxfp4_code_bytes(N, K), dtype=torch.uint8, device=dev)
        Wsc = torch.zeros(L.mxfp4_scale_bytes(N, K), dtype=torch.uint8, device=dev)
        L.mxfp4_quantize_rows(W, Wp, Wsc)
        w_bytes = N * K // 2 + L.mxfp4_scale_bytes(N, K)
        op = L.LORA_OP_MXFP4_GEMM
    else:
        Wp = torch.empty((N, K), dtype=torch.uint8, device=dev)
        Wsc = torch.empty((N,), dtype=torch.float32, device=dev)
        L.fp8_quantize_rows(W, Wp, Wsc)
        w_bytes = N * K + N * 4
        op = L.LORA_OP_W8A16_GEMM
    del W
    out = {"shape": {"K": K, "N": N, "adapters": n_ad, "r": r, "ids": "zipf(1.1)"},
           "peak_tflops_bf16": bf16_peak, "peak_hbm_gbs": hbm_peak,
           "peak_source": f"{peak_src} (MEASURED_PEAKS.json)", "M": {}}
    for M in args.fp8_m:
        q = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=r, seed=3, W=np.zeros((1, 1), np.uint16))
        tb = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        act = np.unique(q.ids)
        set_bytes = q.x.nbytes + q.A.nbytes + q.B.nbytes + M * N * 2
        R = int(min(32, max(2, math.ceil(2.5 * L2_BYTES / set_bytes))))
        base = dict(x=tb(q.x), A=tb(q.A), B=tb(q.B), ids=torch.from_numpy(q.ids).to(dev),
                    ranks=torch.from_numpy(q.ranks).to(dev), scales=torch.from_numpy(q.scales).to(dev))
        sets = []
        for k in range(R):
            d = {key: (v.clone() if k else v) for key, v in base.items()}
            d["pool"] = L.Pool(d["A"], d["B"], d["ranks"], d["scales"])
            d["seg"] = L.Segments(M, n_ad, device=dev)
            L.lora_build_segments(d["ids"], n_ad, d["seg"])
            d["y"] = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            d["ws"] = L.workspace(op, M, K, d["pool"], device=dev)
            d["ws0"] = L.workspace(op, M, K, None, device=dev)
            sets.append(d)
        res = {}
        for tag in ("lora", "base"):
            fn = L.mxfp4_gemm_lora_epilogue if fmt == "mxfp4" else L.w8a16_gemm_lora_epilogue

            def call(d):
                if tag == "lora":
                    fn(d["x"], Wp, Wsc, d["pool"], d["seg"], d["y"], d["ws"])
                else:
                    fn(d["x"], Wp, Wsc, None, None, d["y"], d["ws0"])
            with torch.cuda.stream(stream):
                for d in sets:
                    call(d)
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for d in sets:
                        call(d)
                for _ in range(3):
                    g.replay()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(args.fp8_reps):
                    g.replay()
                b.record(stream)
            torch.cuda.synchronize()
            res[tag] = a.elapsed_time(b) / (args.fp8_reps * R) * 1e3
            res[tag + "_status"] = max(L.lora_workspace_status(d["ws" if tag == "lora" else "ws0"])[0]
                                       for d in sets)
        lora_bytes = int(len(act)) * r * (K + N) * 2 + M * r * 4
        bytes_call = w_bytes + M * K * 2 + M * N * 2 + lora_bytes
        flops = 2.0 * M * N * K
        t = res["lora"] * 1e-6
        out["M"][str(M)] = {
            "us_per_call": res["lora"], "us_per_call_no_lora": res["base"],
            "overhead_vs_no_lora": res["lora"] / res["base"] - 1.0,
            "tflops": flops / t / 1e12, "tensor_frac": flops / t / 1e12 / bf16_peak,
            "hbm_gbs": bytes_call / t / 1e9, "hbm_frac": bytes_call / t / 1e9 / hbm_peak,
            "status_ok": res["lora_status"] == 0 and res["base_status"] == 0,
            "l2": f"x, adapters and y rotate over {R} copies; the weight codes are read once per call",
        }
        del sets
    return out


MERGE_CASES = [
    # name, N, K, adapters in the pool, rank, selected (top-k of the router)
    ("llama7b_q_proj_top2_of_8", 4096, 4096, 8, 16, 2),
    ("llama70b_up_proj_top2_of_16", 28672, 8192, 16, 16, 2),
]


def run_backward(args, dev, stream, hbm_peak, bf16_peak, peak_src):
    """The adapters' backward on the frozen 8-bit base (fp8_lora_backward: dX, dA, dB) at
    the FP8 section's shapes (K 8192, N 28672, 16 adapters of rank 16, Zipf ids): us per
    call, TFLOP/s of dX's 8-bit GEMM against the FP8 peak, and the HBM fraction of its
    algorithmic bytes (WqT and swT, x, dY and dX, the adapters read and transposed, dA
    and dB written in full)."""
    import numpy as np
    import torch

    from adapter_gemm_builder_b200 import lora as L
    from adapter_gemm_builder_b200 import workloads as wl
    K, N, n_ad, r = 8192, 28672, 16, 16
    gen = torch.Generator(device=dev).manual_seed(9)
    Wt = (torch.randn((K, N), generator=gen, device=dev) * (1.0 / math.sqrt(K))).to(torch.bfloat16)
    WqT = torch.empty((K, N), dtype=torch.uint8, device=dev)
    swT = torch.empty(K, dtype=torch.float32, device=dev)
    L.fp8_quantize_rows(Wt, WqT, swT)  # W^T quantised per input channel, once
    del Wt
    fp8_peak = 2.0 * bf16_peak
    out = {"shape": {"K": K, "N": N, "adapters": n_ad, "r": r, "ids": "zipf(1.1)"},
           "peak_tflops_fp8": fp8_peak, "peak_hbm_gbs": hbm_peak,
           "peak_source": f"{peak_src}: FP8 = 2 x bf16_tflops (nominal dense ratio)", "M": {}}
    for M in args.fp8_m:
        q = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=r, seed=4, W=np.zeros((1, 1), np.uint16))
        tb = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        pool = L.Pool(tb(q.A), tb(q.B), torch.from_numpy(q.ranks).to(dev), torch.from_numpy(q.scales).to(dev))
        seg = L.Segments(M, n_ad, device=dev)
        L.lora_build_segments(torch.from_numpy(q.ids).to(dev), n_ad, seg)
        sets = []
        for k in range(2):
            g = torch.Generator(device=dev).manual_seed(100 + k)
            sets.append(dict(
                x=tb(q.x), dY=torch.randn((M, N), generator=g, device=dev).to(torch.bfloat16),
                dX=torch.empty((M, K), dtype=torch.bfloat16, device=dev),
                dA=torch.empty((n_ad, K, r), device=dev), dB=torch.empty((n_ad, r, N), device=dev),
                ws=L.workspace(L.LORA_OP_FP8_BACKWARD, M, K, pool, device=dev)))

        def call(d):
            L.fp8_lora_backward(d["x"], d["dY"], WqT, swT, pool, seg, d["dX"], d["dA"], d["dB"], d["ws"])
        with torch.cuda.stream(stream):
            for d in sets:
                call(d)
            stream.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for d in sets:
                    call(d)
            for _ in range(3):
                gr.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(args.fp8_reps):
                gr.replay()
            b.record(stream)
        torch.cuda.synchronize()
        us = a.elapsed_time(b) / (args.fp8_reps * len(sets)) * 1e3
        status = max(L.lora_workspace_status(d["ws"])[0] for d in sets)
        act = int(len(np.unique(q.ids)))
        bytes_call = (K * N + K * 4 + M * N * 2 + M * K * 2 * 2 + act * r * (K + N) * 2 * 3
                      + n_ad * r * (K + N) * 4)
        flops = 2.0 * M * N * K
        t = us * 1e-6
        out["M"][str(M)] = {"us_per_call": us, "tflops": flops / t / 1e12,
                            "tensor_frac": flops / t / 1e12 / fp8_peak,
                            "hbm_gbs": bytes_call / t / 1e9, "hbm_frac": bytes_call / t / 1e9 / hbm_peak,
                            "status_ok": status == 0,
                            "l2": "two input sets; WqT (235 MB) read once per call"}
        del sets
    return out


def run_merge(args, dev, stream, hbm_peak, peak_src):
    """Token-wise merge of the router-selected adapters into the backbone
    (lora_switch_merge): GB/s of algorithmic bytes (W read, W_out written, the
    selected adapters' A and B read) and the fraction of the HBM peak. W and W_out
    rotate over enough copies to pass the L2."""
    import numpy as np
    import torch

    from adapter_gemm_builder_b200 import lora as L
    gen = torch.Generator(device=dev).manual_seed(13)
    out = {"peak_hbm_gbs": hbm_peak, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
           "cases": {}}
    for name, N, K, n_ad, r, k_sel in MERGE_CASES:
        A = (torch.randn((n_ad, K, r), generator=gen, device=dev) / math.sqrt(K)).to(torch.bfloat16)
        B = (torch.randn((n_ad, r, N), generator=gen, device=dev) / math.sqrt(r)).to(torch.bfloat16)
        pool = L.Pool(A, B, torch.full((n_ad,), r, dtype=torch.int32, device=dev),
                      torch.full((n_ad,), 2.0, dtype=torch.float32, device=dev))
        rng = np.random.default_rng(N)
        sel = torch.from_numpy(rng.choice(n_ad, k_sel, replace=False).astype(np.int32)).to(dev)
        g = rng.random(k_sel).astype(np.float32)
        gates = torch.from_numpy(g / g.sum()).to(dev)
        set_bytes = 2 * N * K * 2
        R = int(min(16, max(1, math.ceil(2.5 * L2_BYTES / set_bytes))))
        Ws = [(torch.randn((N, K), generator=gen, device=dev) / math.sqrt(K)).to(torch.bfloat16)
              for _ in range(R)]
        Wo = [torch.empty_like(w) for w in Ws]
        with torch.cuda.stream(stream):
            for w, o in zip(Ws, Wo):
                L.lora_switch_merge(w, pool, sel, gates, o)
            stream.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for w, o in zip(Ws, Wo):
                    L.lora_switch_merge(w, pool, sel, gates, o)
            for _ in range(3):
                graph.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = max(3, 60 // R)
            a.record(stream)
            for _ in range(reps):
                graph.replay()
            b.record(stream)
        torch.cuda.synchronize()
        us = a.elapsed_time(b) / (reps * R) * 1e3
        nbytes = 2 * N * K * 2 + k_sel * r * (K + N) * 2
        out["cases"][name] = {"N": N, "K": K, "adapters": n_ad, "rank": r, "selected": k_sel,
                              "us_per_call": us, "algorithmic_bytes": nbytes,
                              "gbs": nbytes / (us * 1e-6) / 1e9,
                              "hbm_frac": nbytes / (us * 1e-6) / 1e9 / hbm_peak,
                              "l2": f"W and W_out rotate over {R} pairs ({R * set_bytes / 2**20:.0f} MiB)"}
        del Ws, Wo, A, B
    return out


def main():
    args = parse_args()
    if args.section:
        import torch
        from adapter_gemm_builder_b200 import lora as L
        L.load()
        dev = torch.device("cuda", 0)
        hbm, bf16, sust, src = measured_peaks()
        st = torch.cuda.Stream(device=dev)
        run = {"fp8": lambda: run_fp8(args, dev, st, hbm, bf16, sust, src),
               "bf16": lambda: run_bf16(args, dev, st, hbm, bf16, src),
               "mxfp4": lambda: run_mxfp4(args, dev, st, hbm, bf16, src),
               "w8a16": lambda: run_mxfp4(args, dev, st, hbm, bf16, src, "w8a16"),
               "merge": lambda: run_merge(args, dev, st, hbm, src),
               "backward": lambda: run_backward(args, dev, st, hbm, bf16, src)}[args.section]
        print(json.dumps(run()))
        return
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
