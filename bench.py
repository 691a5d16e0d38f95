"""Benchmark of the weight-only-quantized decode linear on B200.

Workload (default): the Llama-2-7B linear set at M = 1 - qkv (4096 -> 12288),
o (4096 -> 4096), gate_up (4096 -> 22016), down (11008 -> 4096) - in int4 with
group size 32 and with group size 128 (bf16 scale + zero per group).  One step
is one pass over those 8 layers (every layer once per group size), on seeded
synthetic weights of that shape (0.02 randn with 0.1 % x10 outliers) and
activations (randn -> bf16).

Metric: effective weight GB/s = algorithmic bytes (packed W + scales + zeros +
x + y) / device time, and us per layer.  The 8 layers hold 234 MB, more than the
126 MB L2, so every layer is re-read from HBM on the next step.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl wq|reference]
                  [--workload NAME] [--no-pdl] [--no-graph]
Under torchrun (N > 1) every rank runs the same workload on its own GPU
(replicas: the layer does not shard), value = bytes of all ranks / max time.
"""

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

FMT_ID = {"int8": 0, "int4": 1, "fp6": 2, "bf16": 3}


# ------------------------------------------------------------------ workloads
def workload_layers(name):
    """List of layers (label, fmt, groupsize, K, N, M)."""
    if name == "llama2-7b-int4-m1":
        out = []
        for g in (32, 128):
            for lab, (K, N) in workloads.LLAMA2_7B.items():
                out.append((f"{lab}-g{g}", "int4", g, K, N, 1))
        return out
    if name == "int8-4096-m1":
        return [("4096x4096", "int8", 0, 4096, 4096, 1)]
    if name.startswith("llama-70b-fp6-m"):
        M = int(name.rsplit("m", 1)[1])
        return [(lab, "fp6", 0, K, N, M) for lab, (K, N) in workloads.LLAMA_70B.items()]
    if name.startswith("opt-30b-"):  # opt-30b-<fmt>[-g<g>]-m<M>
        parts = name.split("-")
        fmt = parts[2]
        g = int(parts[3][1:]) if parts[3].startswith("g") else 0
        M = int(parts[-1][1:])
        return [(lab, fmt, g, K, N, M) for lab, (K, N) in workloads.OPT_30B.items()]
    if name == "llama2-7b-stack-int4-g32-m1":
        out = []
        for layer in range(32):
            for lab, (K, N) in workloads.LLAMA2_7B.items():
                out.append((f"L{layer}-{lab}", "int4", 32, K, N, 1))
        return out
    raise SystemExit(f"unknown workload {name}")


def algo_bytes(fmt, g, K, N, M):
    """Packed weight + scales (+ zeros) + x + y bytes of one call."""
    if fmt == "int8":
        w = N * K + 2 * N
    elif fmt == "int4":
        w = N * K // 2 + 2 * 2 * N * (K // g)
    elif fmt == "fp6":
        w = 3 * N * K // 4 + 2 * N
    else:
        w = 2 * N * K
    return w + 2 * M * K + 2 * M * N


def layer_seed(idx):
    return 1000 + idx


# ------------------------------------------------------------------ clocks
# clock event reason bits (NVML): the ones that reject a measurement, and the
# power cap (kept and noted)
_REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}


class ClockSampler:
    """Polls the GPU's SM clock, max clock, clock event reasons and power through
    NVML every 2 ms while the timed region runs (a background thread that only
    reads)."""

    def __init__(self, torch_index):
        self.samples = []
        self.handle = None
        self.max_mhz = None
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it instead of clocks
            self.err = f"nvml unavailable: {type(e).__name__}"
        self.stop = None

    def _run(self):
        nv, h = self.nv, self.handle
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((sm, rs, pw))
            except Exception:
                pass
            self.stop.wait(0.002)

    def __enter__(self):
        if self.handle is not None:
            import threading
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.stop is not None:
            self.stop.set()
            self.thread.join(timeout=5)

    def summary(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        reasons = sorted({name for (_, rs, _) in self.samples for bit, name in _REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "power_w_max": max(s[2] for s in self.samples)}


# ------------------------------------------------------------------ measured DRAM traffic
KERNEL_SOURCES = ("gemm_wq_linear_b200/csrc/wq_gemv.cu", "gemm_wq_linear_b200/csrc/decode.cuh",
                  "gemm_wq_linear_b200/csrc/ptx.cuh", "gemm_wq_linear_b200/csrc/wq_kernels.cuh")


def kernel_source_hash():
    """Hash of the GEMV sources with // comments and whitespace removed, so that
    a comment edit does not invalidate a traffic capture of the same code."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            code = re.sub(r"//[^\n]*", "", f.read())
        h.update(re.sub(r"\s+", " ", code).strip().encode())
    return h.hexdigest()[:16]


def measured_traffic(workload):
    """DRAM bytes (read + write) per launch of the GEMV kernel for `workload`, from
    the committed ncu summary, or None when there is none or the kernel sources
    changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"gemv_{workload}_traffic.md")
    try:
        with open(path) as f:
            kv = dict(ln.split(":", 1) for ln in f if ln.startswith(("traffic_bytes_per_launch:", "kernel_source_hash:")))
    except OSError:
        return None
    if kv.get("kernel_source_hash", "").strip() != kernel_source_hash():
        return None
    return float(kv["traffic_bytes_per_launch"])


# ------------------------------------------------------------------ peaks
def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


# ------------------------------------------------------------------ distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(v, world):
    if world == 1:
        return v
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------ oracle (CPU baseline)
def oracle_sample_run(layers, budget_s):
    """Times the oracle (dequant + fp64 product) on a bounded row sample of each layer.

    Returns (GB/s of algorithmic bytes per unit time, description).  Quantization
    of the sample is done by the oracle beforehand and not timed.
    """
    from oracle import formats, linear
    prepared = []
    for idx, (lab, fmt, g, K, N, M) in enumerate(layers[:8]):
        rows = min(N, 256)
        W = workloads.weights(N, K, layer_seed(idx), rows=slice(0, rows)).numpy()
        x = workloads.activations(M, K, layer_seed(idx) + 500)
        xb = x.view(torch.int16).numpy().view(np.uint16)
        if fmt == "int4":
            q, s, z = formats.quantize_int4(W, g)
            prepared.append((lambda q=q, s=s, z=z, g=g: linear.deq_weights("int4", q, s, z, g), xb, fmt, g, K, rows, M))
        elif fmt == "int8":
            q, s = formats.quantize_int8(W)
            prepared.append((lambda q=q, s=s: linear.deq_weights("int8", q, s), xb, fmt, g, K, rows, M))
        elif fmt == "fp6":
            c, s = formats.quantize_fp6(W)
            prepared.append((lambda c=c, s=s: linear.deq_weights("fp6", c, s), xb, fmt, g, K, rows, M))
        else:
            from oracle import rounding
            b = rounding.bf16_bits(rounding.bf16_rne(W.astype(np.float64)))
            prepared.append((lambda b=b: linear.deq_weights("bf16", b), xb, fmt, g, K, rows, M))
    t0 = time.perf_counter()
    nbytes = 0
    reps = 0
    while True:
        for deq, xb, fmt, g, K, rows, M in prepared:
            y = linear.linear_ref(xb, deq())
            linear.to_bf16(y)
            nbytes += algo_bytes(fmt, g, K, rows, M)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = len(os.sched_getaffinity(0))
    desc = (f"oracle (numpy fp64 dequant + x @ deq(W).T) on the first {prepared[0][5]} output rows of each of "
            f"{len(prepared)} layers, {reps} passes, {dt:.1f} s")
    return nbytes / dt / 1e9, cores, desc


def cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def cpu_baseline(layers, budget_s):
    """The oracle timed on the host: with every thread NumPy's BLAS uses on the
    cores this process may run on, then with one thread (half the budget)."""
    v, cores, desc = oracle_sample_run(layers, budget_s)
    out = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc, "cpu_model": cpu_model(),
           "affinity_cores": len(os.sched_getaffinity(0))}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            v1, _, desc1 = oracle_sample_run(layers, budget_s / 2)
        out["single_thread"] = {"value": v1, "unit": "GB/s", "cores": 1, "sample": desc1}
    except ImportError:
        pass
    return out


def derived_rates(layers, ms, world):
    """Rates derived from the device time of one step: the bf16-equivalent
    weight rate (2 N K bytes a layer, as if the weights were unquantized bf16)."""
    bf16_bytes = sum(2 * N * K for (_, _, _, K, N, _) in layers)
    return {"bf16_equivalent_gbps": world * bf16_bytes / (ms * 1e-3) / 1e9,
            "note": "2*N*K bytes per layer / device time: the rate an unquantized bf16 layer would need"}


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="wq", choices=["wq", "reference"])
    ap.add_argument("--workload", default="llama2-7b-int4-m1")
    ap.add_argument("--no-pdl", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle CPU baseline")
    ap.add_argument("--layers-detail", action="store_true", help="also time each layer alone")
    ap.add_argument("--layer", default=None, help="run only the layer with this label (for profiling one kernel)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world, rank, local = dist_setup(args)
    layers = workload_layers(args.workload)
    if args.layer:
        layers = [ly for ly in layers if ly[0] == args.layer]
        if not layers:
            raise SystemExit(f"no layer {args.layer} in {args.workload}")
    total_bytes = sum(algo_bytes(f, g, K, N, M) for (_, f, g, K, N, M) in layers)
    metric = "effective weight GB/s (algorithmic bytes / device time), M=1..32 decode linear"

    if args.impl == "reference":
        if rank != 0:
            return
        per_step = []
        for _ in range(args.warmup):
            oracle_sample_run(layers, 0.0)
        for _ in range(args.steps):
            v, cores, desc = oracle_sample_run(layers, max(args.cpu_budget / max(args.steps, 1), 0.5))
            per_step.append(v)
        v = statistics.median(per_step)
        line = {"impl": "reference", "metric": metric, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": args.workload, "sample": "first 256 output rows per layer"},
                "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
                "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import gemm_wq_linear_b200 as wq

    dev = torch.device("cuda", torch.cuda.current_device())
    flags = 0 if args.no_pdl else wq.WQ_LAUNCH_PDL
    # -------- build the resident layers (product quantizer + packer, uploaded once)
    bufs = []
    cache = {}
    for idx, (lab, fmt, g, K, N, M) in enumerate(layers):
        key = (fmt, g, K, N, idx % 8 if args.workload.endswith("stack-int4-g32-m1") else idx)
        if key not in cache:
            W = workloads.weights(N, K, layer_seed(idx % 8 if "stack" in args.workload else idx))
            cache[key] = wq.PackedWeight.quantize(W, fmt, g, device=dev)
            del W
        pw = cache[key]
        if "stack" in args.workload and idx >= 8:
            # distinct HBM copies for every layer of the stack (same random values)
            src = cache[key]
            pw = wq.PackedWeight(src.fmt, src.N, src.K, src.packed.clone(),
                                 None if src.scales is None else src.scales.clone(),
                                 None if src.zeros is None else src.zeros.clone(), src.groupsize)
        x = workloads.activations(M, K, layer_seed(idx) + 500)
        bufs.append(dict(lab=lab, fmt=fmt, g=g, K=K, N=N, M=M, pw=pw, xc=x))
    # every layer's x and y live in one device buffer each (16-byte aligned
    # views), mirrored by one pinned host buffer each: the end-to-end leg moves
    # a step's inputs and results with one copy each way
    def offsets(sizes):
        offs, o = [], 0
        for n in sizes:
            offs.append(o)
            o += (n + 63) // 64 * 64
        return offs, o
    xo, xn = offsets([b["M"] * b["K"] for b in bufs])
    yo, yn = offsets([b["M"] * b["N"] for b in bufs])
    x_all = torch.zeros(xn, dtype=torch.bfloat16, device=dev)
    y_all = torch.zeros(yn, dtype=torch.bfloat16, device=dev)
    xh_all = torch.zeros(xn, dtype=torch.bfloat16).pin_memory()
    yh_all = torch.zeros(yn, dtype=torch.bfloat16).pin_memory()
    for b, ox, oy in zip(bufs, xo, yo):
        b["x"] = x_all[ox:ox + b["M"] * b["K"]].view(b["M"], b["K"])
        b["y"] = y_all[oy:oy + b["M"] * b["N"]].view(b["M"], b["N"])
        xh_all[ox:ox + b["M"] * b["K"]].copy_(b.pop("xc").reshape(-1))
    x_all.copy_(xh_all)
    stream = torch.cuda.Stream(device=dev)

    def step():
        for b in bufs:
            wq.linear(b["x"], b["pw"], out=b["y"], stream=stream, flags=flags)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()

    def run_steps(k):
        for _ in range(k):
            if graph is not None:
                graph.replay()
            else:
                step()

    # -------- timed region (device time, CUDA events on the launching stream)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            run_steps(args.steps)
            ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1) / args.steps
    ms = max_over_ranks(ms, world)
    value = world * total_bytes / (ms * 1e-3) / 1e9
    launches_per_step = len(bufs) * 1  # one kernel per layer (M <= 4)

    # -------- end to end through the public API with host buffers: every step
    # copies all layers' x from pinned host memory, runs the layers and copies
    # all y back (captured with the step in a CUDA graph, as the device loop)
    h2d = xh_all.numel() * 2
    d2h = yh_all.numel() * 2

    def e2e_step():
        x_all.copy_(xh_all, non_blocking=True)
        step()
        yh_all.copy_(y_all, non_blocking=True)

    e2e_graph = None
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            e2e_step()
    torch.cuda.synchronize()
    if not args.no_graph:
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e2e_graph, stream=stream):
            e2e_step()
        for _ in range(args.warmup):
            e2e_graph.replay()
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            if e2e_graph is not None:
                e2e_graph.replay()
            else:
                e2e_step()
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    e2e_value = world * total_bytes / (e2e_ms * 1e-3) / 1e9
    if e2e_graph is not None:
        del e2e_graph

    # -------- per-layer detail (outside the timed region)
    layer_us = {}
    if True:
        for b in bufs[:8]:
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 20
            with torch.cuda.stream(stream):
                wq.linear(b["x"], b["pw"], out=b["y"], stream=stream, flags=0)
                a0.record(stream)
                for _ in range(reps):
                    wq.linear(b["x"], b["pw"], out=b["y"], stream=stream, flags=0)
                a1.record(stream)
            a1.synchronize()
            us = a0.elapsed_time(a1) * 1e3 / reps
            layer_us[b["lab"]] = round(us, 3)

    peak, peak_kind = hbm_peak()
    achieved = total_bytes / (ms * 1e-3) / 1e9  # one GPU, per launch averaged over the step
    line = {
        "metric": metric,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "us_per_layer": ms * 1e3 / len(bufs),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4xbf16->fp32" if all(b["fmt"] == "int4" for b in bufs) else "mixed",
        "data": "synthetic",
        "config": {"workload": args.workload, "layers": [b["lab"] for b in bufs][:8] + (["..."] if len(bufs) > 8 else []),
                   "M": bufs[0]["M"], "bytes_per_step": total_bytes,
                   "l2": "inputs larger than L2 (%.0f MB per step vs 126 MB)" % (total_bytes / 1e6),
                   "launch": ("cuda graph" if graph is not None else "stream") + (" + PDL" if flags else ""),
                   "parallelism": f"replicas x{world}"},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind, "frac_of_datasheet_8000": achieved / 8000.0,
                     "traffic": None if args.layer else measured_traffic(args.workload),
                     "algorithmic_bytes_per_launch": total_bytes / len(bufs)},
        "layer_us_alone": layer_us,
        "derived": derived_rates(layers, ms, world),
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "how": "per step one copy of every layer's x from pinned host memory, the layers, one copy of every y "
                       "back; " + ("captured in a CUDA graph" if not args.no_graph else "stream launches")},
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and args.cpu_budget > 0:
        line["cpu_baseline"] = cpu_baseline(layers, args.cpu_budget)
    if graph is not None:
        del graph
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
