"""Benchmark of the quantized matmul hot path on B200.

Workload (one step): the decode sweep of a 16-layer Llama-3.2-1B-shaped stack
of distinct bf16 weights quantized 4-bit, group 64 (q/o 2048x2048, k/v
512x2048, gate/up 8192x2048, down 2048x8192; 547 MB of packed weights,
scales and biases, more than 4x the 126 MB L2, so no L2 flush is needed and
every step streams the weights from HBM).  For each M in (1, 2, 4, 8, 16) the
step runs y = x . dequant(W)^T for every projection of every layer through
aq_qmv.  The step is captured once in a CUDA graph and replayed.

Metric: qmv weight-stream GB/s = (packed weights + scales + biases + x + y
bytes of all calls) / device time of the step, whole job (all ranks).

--impl reference times the CPU oracle on a bounded sample of the same
workload (one layer at M = 1 per step) on the host cores.

Multi-GPU: each rank runs the same workload on its own GPU (independent
replicas, weak scaling, no collective on the data path); the step time is the
max over ranks.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

LAYERS = 16
QMV_M = (1, 2, 4, 8, 16)
BITS, GS = 4, 64
METRIC = "qmv weight-stream GB/s (M<=16), % of B200 HBM roofline"
WORKLOAD = ("decode sweep: 16-layer Llama-3.2-1B-shaped stack (q/o 2048x2048, k/v 512x2048, "
            "gate/up 8192x2048, down 2048x8192), bf16, 4-bit affine g64, M in 1,2,4,8,16")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def layer_bytes(M):
    """Algorithmic bytes of one layer at M rows: packed weights, scales,
    biases, x and y (bf16)."""
    from group_wise_affine_quant_b200.inputs import LLAMA_1B_PROJ
    tot = 0
    for _, n, k in LLAMA_1B_PROJ:
        tot += n * k * BITS // 8 + 2 * 2 * n * (k // GS) + 2 * M * k + 2 * M * n
    return tot


class ClockSampler:
    """Samples nvidia-smi during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                      "--format=csv,noheader,nounits"], capture_output=True,
                                     text=True, timeout=5).stdout.strip()
                if out:
                    self.samples.append([v.strip() for v in out.split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4)
                          if len(s) > 4 + i and s[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def traffic_for(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, if the kernel's
    source has not changed since (profiles/traffic.json)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        src = os.path.join(ROOT, rec["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if h != rec["source_sha256_16"] or rec["workload"] != workload:
            return None
        return rec["dram_bytes_per_launch"]
    except Exception:
        return None


def cpu_baseline(seconds_hint=10.0):
    """The oracle as it stands, on the host cores, over a bounded sample: one
    layer of the stack at M = 1, 2, 4, 8, 16 (the same inputs recipe)."""
    import numpy as np
    import oracle
    from group_wise_affine_quant_b200 import inputs
    ws = inputs.decode_layer(seed=0)
    q = {name: oracle.quantize(inputs.as_u16(w), BITS, GS, 1) for name, w in ws.items()}
    tot_bytes, tot_t = 0, 0.0
    for M in QMV_M:
        for name, n, k in inputs.LLAMA_1B_PROJ:
            x = inputs.as_u16(inputs.decode_x(M, k))
            wq, s, b = q[name]
            t0 = time.perf_counter()
            oracle.qmm(x, wq, s, b, n, BITS, GS, 0, 1)
            tot_t += time.perf_counter() - t0
        tot_bytes += layer_bytes(M)
    return {"value": tot_bytes / tot_t / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "one layer of the stack (7 projections) at M = 1,2,4,8,16, %.1f s" % tot_t}


def run_reference(args):
    world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    import oracle
    from group_wise_affine_quant_b200 import inputs
    ws = inputs.decode_layer(seed=0)
    q = {name: oracle.quantize(inputs.as_u16(w), BITS, GS, 1) for name, w in ws.items()}
    xs = {k: inputs.as_u16(inputs.decode_x(1, k)) for k in (2048, 8192)}

    def step():
        for name, n, k in inputs.LLAMA_1B_PROJ:
            wq, s, b = q[name]
            oracle.qmm(xs[k], wq, s, b, n, BITS, GS, 0, 1)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    val = layer_bytes(1) / dt / 1e9
    line = {"metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "one layer at M=1 per step"},
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": "one layer (7 projections) at M=1 per step"},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    from group_wise_affine_quant_b200 import api, inputs

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm, tf, peak_kind = peaks()

    # Quantize the stack once (on the device, through the library).
    layers = []
    for li in range(LAYERS):
        ws = inputs.decode_layer(seed=100 + li)
        q = {}
        for name, w in ws.items():
            q[name] = api.aq_quantize(w.to(dev), BITS, GS)
        layers.append(q)
        del ws
    torch.cuda.synchronize()
    projs = inputs.LLAMA_1B_PROJ
    xs = {(M, k): inputs.decode_x(M, k, seed=M).to(dev) for M in QMV_M for k in (2048, 8192)}
    ys = {(M, name): torch.empty((M, n), dtype=torch.bfloat16, device=dev)
          for M in QMV_M for name, n, _ in projs}
    wsp = api.Workspace()
    for M in QMV_M:                       # size the workspace before capture
        for _, n, k in projs:
            wsp.get(dev, api.aq_workspace_size(0, M, n, k, BITS, GS))
    launches_per_step = len(QMV_M) * LAYERS * len(projs)

    def step():
        for M in QMV_M:
            for q in layers:
                for name, n, k in projs:
                    wq, s, b = q[name]
                    api.aq_qmv(xs[(M, k)], wq, s, b, BITS, GS, out=ys[(M, name)], workspace=wsp)

    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        step()                            # eager pass (loads the library, sets attributes)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as clk:
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms, world)
    step_bytes = LAYERS * sum(layer_bytes(M) for M in QMV_M)
    value = world * step_bytes / (ms * 1e-3) / 1e9

    # Per-M view (each M's calls captured separately).
    per_m = {}
    with torch.cuda.stream(stream):
        for M in QMV_M:
            gm = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gm, stream=stream):
                for q in layers:
                    for name, n, k in projs:
                        wq, s, b = q[name]
                        api.aq_qmv(xs[(M, k)], wq, s, b, BITS, GS, out=ys[(M, name)], workspace=wsp)
            for _ in range(3):
                gm.replay()
            a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(10):
                gm.replay()
            c.record(stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(c) / 10
            per_m[str(M)] = round(LAYERS * layer_bytes(M) / (t * 1e-3) / 1e9, 1)
            del gm

    # End to end through the public API with host buffers: pinned x in,
    # every y out, around the same graph.
    host_x = {key: v.cpu().pin_memory() for key, v in xs.items()}
    host_y = {key: torch.empty(v.shape, dtype=v.dtype).pin_memory() for key, v in ys.items()}
    h2d = sum(v.numel() * 2 for v in host_x.values())
    d2h = sum(v.numel() * 2 for v in host_y.values())
    with torch.cuda.stream(stream):
        for _ in range(2):
            for key in xs:
                xs[key].copy_(host_x[key], non_blocking=True)
            g.replay()
            for key in ys:
                host_y[key].copy_(ys[key], non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            for key in xs:
                xs[key].copy_(host_x[key], non_blocking=True)
            g.replay()
            for key in ys:
                host_y[key].copy_(ys[key], non_blocking=True)
        c.record(stream)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(c) / args.steps, world)
    e2e = {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    kernel_ms = ms / launches_per_step
    achieved = (step_bytes / launches_per_step) / (kernel_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_kind": peak_kind,
            "kernel": "qmv_kernel (aq_qmv)",
            "traffic": traffic_for("qmv_kernel", "decode-stack")}
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "layers": LAYERS, "M": list(QMV_M), "bits": BITS,
                       "group_size": GS, "parallelism": "replicas" if world > 1 else "single",
                       "l2": "weights 547 MB > 4x L2 per step; no flush needed",
                       "timing": "CUDA graph replay, CUDA events on the launching stream"},
            "per_m_gbs": per_m, "roofline": roof, "clocks": clk.summary(), "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
