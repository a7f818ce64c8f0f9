"""Benchmark of the quantized matmul hot path on B200.

Headline workload (one step): the decode sweep of a 16-layer
Llama-3.2-1B-shaped stack of distinct bf16 weights quantized 4-bit, group 64
(q/o 2048x2048, k/v 512x2048, gate/up 8192x2048, down 2048x8192; 547 MB of
packed weights, scales and biases, more than 4x the 126 MB L2, so no L2
flush is needed and every step streams the weights from HBM).  For each M in
(1, 2, 4, 8, 16) the step runs y = x . dequant(W)^T for every projection of
every layer through aq_qmv.  The step is captured once in a CUDA graph and
replayed.

Metric: qmv weight-stream GB/s = (packed weights + scales + biases + x + y
bytes of all calls) / device time of the step, whole job (all ranks).
Beside it (not part of the step): the sweep's M = 32, 64 rows through
aq_qmm, and the tensor-core side of the metric in TFLOP/s (2 M N K / time):
the chained fp16 qmm (x[1024,1024] through W1 [4096,1024] and W2
[1024,4096], ten times), FP4 weights at M = 4096, and the conv2d implicit
GEMM.

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
QMM_M = (32, 64)
BITS, GS = 4, 64
METRIC = "qmv weight-stream GB/s (M<=16), % of B200 HBM roofline"
WORKLOAD = ("decode sweep: 16-layer Llama-3.2-1B-shaped stack (q/o 2048x2048, k/v 512x2048, "
            "gate/up 8192x2048, down 2048x8192), bf16, 4-bit affine g64, M in 1,2,4,8,16")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-qmm", action="store_true", help="skip the TFLOP/s side lines")
    ap.add_argument("--only", default="all", choices=["all", "qmm", "qmm-affine", "conv"],
                    help="qmm: run only the TFLOP/s workloads; qmm-affine: only the 4-bit "
                         "affine M = N = K = 4096 product; conv: only the groups-1 4-bit conv "
                         "(the last two for profiling)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def proj_bytes(n, k, M):
    """Algorithmic bytes of one projection call: packed weights, scales,
    biases (bf16), x and y (bf16)."""
    return n * k * BITS // 8 + 2 * 2 * n * (k // GS) + 2 * M * k + 2 * M * n


def layer_bytes(M):
    from group_wise_affine_quant_b200.inputs import LLAMA_1B_PROJ
    return sum(proj_bytes(n, k, M) for _, n, k in LLAMA_1B_PROJ)


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi's own loop
    (-lms 50) while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self._p = None

    def __enter__(self):
        try:
            self._p = subprocess.Popen(["nvidia-smi", "-i", str(self.index),
                                        "--query-gpu=" + self.FIELDS,
                                        "--format=csv,noheader,nounits", "-lms", "50"],
                                       stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)                      # let the first sample land
        except Exception:
            self._p = None
        return self

    def __exit__(self, *a):
        if self._p is None:
            return
        time.sleep(0.1)
        self._p.terminate()
        try:
            out, _ = self._p.communicate(timeout=5)
        except Exception:
            self._p.kill()
            out = ""
        for ln in out.splitlines():
            f = [v.strip() for v in ln.split(",")]
            if len(f) >= 8:
                self.samples.append(f)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        num = lambda v: v.replace(".", "", 1).isdigit()
        sm = [float(s[0]) for s in self.samples if num(s[0])]
        mx = [float(s[1]) for s in self.samples if num(s[1])]
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
        h = hashlib.sha256()
        for src in rec["sources"]:
            h.update(open(os.path.join(ROOT, src), "rb").read())
        if h.hexdigest()[:16] != rec["sources_sha256_16"] or rec["workload"] != workload:
            return None
        return rec["dram_bytes_per_launch"]
    except Exception:
        return None


def graph_time_ms(torch, stream, fn, reps, warm=3):
    """Device time per call of fn, captured `reps` times in one CUDA graph."""
    torch.cuda.synchronize()              # inputs written on other streams are complete
    with torch.cuda.stream(stream):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                fn()
        for _ in range(warm):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / reps


def cpu_baseline():
    """The oracle as it stands, on the host cores, over a bounded sample: one
    layer of the stack at M = 1, 2, 4, 8, 16 (the same inputs recipe)."""
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
    return {"value": round(tot_bytes / tot_t / 1e9, 3), "unit": "GB/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "one layer of the stack (7 projections) at M = 1,2,4,8,16, %.1f s" % tot_t}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
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


def qmm_lines(torch, api, inputs, dev, stream, tf_peak, tf_sust, affine_only=False,
              conv_only=False):
    """TFLOP/s of the tensor-core workloads (not part of the timed step).
    Every weight here is quantized before its timed calls and no timed kernel
    writes one, so the kernels may stream weights before their dependency wait
    (the same setting as the decode step)."""
    out = {}
    api.aq_set_weight_prefetch(True)

    def conv_g1():
        # conv2d, groups 1, 4-bit: batch 2, 64x64, 320 -> 320 channels, 3x3, pad 1
        xc, wcv = inputs.conv(1)
        w2 = inputs.flatten_pad_conv_weight(wcv, 64)
        qc = api.aq_quantize(w2.to(dev), 4, 64)
        xcd = xc.to(dev)
        yc = torch.empty((2, 64, 64, 320), dtype=torch.bfloat16, device=dev)
        t = graph_time_ms(torch, stream, lambda: api.aq_qconv2d_nhwc(
            xcd, *qc, 320, 3, 3, (1, 1), (1, 1), 1, 4, 64, out=yc), 10)
        fl = 2 * 8192 * 320 * 2880
        out["conv2d_g1_4bit"] = {"tflops": round(fl / (t * 1e-3) / 1e12, 1), "ms": round(t, 4)}

    if conv_only:
        conv_g1()
        return out, None
    if affine_only:
        xf = inputs.fp4_x(4096, 4096).to(dev)
        yf = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
        wa = api.aq_quantize(inputs.normal((4096, 4096), 0.02, 1, inputs.gen(8)).to(dev), 4, 64)
        t = graph_time_ms(torch, stream, lambda: api.aq_qmm(xf, *wa, 4, 64, out=yf), 10)
        out["affine4_M4096"] = {"tflops": round(2 * 4096 ** 3 / (t * 1e-3) / 1e12, 1), "ms": round(t, 4)}
        return out, None
    # chained fp16 qmm, 4-bit g64: 20 products per chain
    x, w1, w2 = inputs.chained()
    q1 = api.aq_quantize(w1.to(dev), 4, 64)
    q2 = api.aq_quantize(w2.to(dev), 4, 64)
    xd = x.to(dev)
    h = torch.empty((1024, 4096), dtype=torch.float16, device=dev)
    o = torch.empty((1024, 1024), dtype=torch.float16, device=dev)

    def chain():
        cur = xd
        for _ in range(10):
            api.aq_qmm(cur, *q1, 4, 64, out=h)
            api.aq_qmm(h, *q2, 4, 64, out=o)
            cur = o
    t = graph_time_ms(torch, stream, chain, 5)
    fl = 20 * 2 * 1024 * 4096 * 1024
    out["chained_fp16_4bit"] = {"tflops": round(fl / (t * 1e-3) / 1e12, 1), "ms_per_chain": round(t, 4)}
    # FP4, M = 4096, E8M0 (finite) scales, bf16
    codes, scales = inputs.fp4(4096, 4096, 32, seed=7)
    xf = inputs.fp4_x(4096, 4096).to(dev)
    wc, sc = codes.to(dev), scales.to(dev)
    yf = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
    t = graph_time_ms(torch, stream, lambda: api.aq_qmm(xf, wc, sc, None, 4, 32, out=yf), 10)
    fl = 2 * 4096 ** 3
    fp4 = {"tflops": round(fl / (t * 1e-3) / 1e12, 1), "ms": round(t, 4)}
    out["fp4_e8m0_M4096"] = fp4
    # affine 4-bit, M = N = K = 4096, bf16 (same shape as FP4)
    wa = api.aq_quantize(inputs.normal((4096, 4096), 0.02, 1, inputs.gen(8)).to(dev), 4, 64)
    t = graph_time_ms(torch, stream, lambda: api.aq_qmm(xf, *wa, 4, 64, out=yf), 10)
    aff = {"tflops": round(fl / (t * 1e-3) / 1e12, 1), "ms": round(t, 4)}
    out["affine4_M4096"] = aff
    conv_g1()
    roof = {"bound": "tensor", "achieved": aff["tflops"], "peak": tf_peak, "unit": "TFLOP/s",
            "frac": round(aff["tflops"] / tf_peak, 4), "peak_kind": "measured burst bf16",
            "kernel": "qmm_tc_kernel (aq_qmm, 4-bit affine, M=N=K=4096)",
            "traffic": traffic_for("qmm_tc_kernel", "affine4-M4096")}
    return out, roof


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    from group_wise_affine_quant_b200 import api, inputs

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm, tf, tf_sust, peak_kind = peaks()
    if args.only in ("qmm", "qmm-affine", "conv"):
        stream = torch.cuda.Stream(dev)
        qmm, roof_qmm = qmm_lines(torch, api, inputs, dev, stream, tf, tf_sust,
                                  affine_only=args.only == "qmm-affine",
                                  conv_only=args.only == "conv")
        if rank == 0:
            print(json.dumps({"qmm_tflops": qmm, "roofline_qmm": roof_qmm}))
        return

    # Quantize the stack once (on the device, through the library).  The
    # timed calls never follow a kernel that writes their weights, so the
    # library may stream weights before waiting on the previous kernel.
    layers = []
    for li in range(LAYERS):
        ws = inputs.decode_layer(seed=100 + li)
        layers.append({name: api.aq_quantize(w.to(dev), BITS, GS) for name, w in ws.items()})
        del ws
    torch.cuda.synchronize()
    api.aq_set_weight_prefetch(True)
    projs = inputs.LLAMA_1B_PROJ
    all_m = QMV_M + QMM_M
    xs = {(M, k): inputs.decode_x(M, k, seed=M).to(dev) for M in all_m for k in (2048, 8192)}
    ys = {(M, name): torch.empty((M, n), dtype=torch.bfloat16, device=dev)
          for M in all_m for name, n, _ in projs}
    launches_per_step = len(QMV_M) * LAYERS * len(projs)

    def calls(M):
        fn = api.aq_qmv if M <= 16 else api.aq_qmm
        for q in layers:
            for name, n, k in projs:
                wq, s, b = q[name]
                fn(xs[(M, k)], wq, s, b, BITS, GS, out=ys[(M, name)])

    def step():
        for M in QMV_M:
            calls(M)

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

    # The same calls as independent problems: every x is written before the
    # step and every call writes its own y, so the input-prefetch contract
    # holds and each kernel may read its weights and x while the previous one
    # runs (y stays ordered).  Reported beside the value, which keeps every
    # call waiting for its predecessor as a chain of dependent layers would.
    ys_ind = {(M, li, name): torch.empty((M, n), dtype=torch.bfloat16, device=dev)
              for M in QMV_M for li in range(LAYERS) for name, n, _ in projs}

    def step_ind():
        for M in QMV_M:
            for li, q in enumerate(layers):
                for name, n, k in projs:
                    wq, s, b = q[name]
                    api.aq_qmv(xs[(M, k)], wq, s, b, BITS, GS, out=ys_ind[(M, li, name)])

    with torch.cuda.stream(stream):
        api.aq_set_input_prefetch(True)
        try:
            step_ind()
            torch.cuda.synchronize()
            g_ind = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_ind, stream=stream):
                step_ind()
        finally:
            api.aq_set_input_prefetch(False)
        for _ in range(args.warmup):
            g_ind.replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        i0, i1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        i0.record(stream)
        for _ in range(args.steps):
            g_ind.replay()
        i1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
    ms_ind = max_over_ranks(i0.elapsed_time(i1) / args.steps, world)
    independent = {"value": round(world * step_bytes / (ms_ind * 1e-3) / 1e9, 1), "unit": "GB/s",
                   "ms_per_step": round(ms_ind, 4),
                   "frac_of_hbm": round(step_bytes / (ms_ind * 1e-3) / 1e9 / hbm, 4),
                   "calls": "same 560 calls; x written before the step, one y per call, "
                            "weight and input prefetch on"}

    # Per-M view: each M's 112 calls captured alone; per-kernel averages.
    per_m, per_m_us = {}, {}
    for M in all_m:
        t = graph_time_ms(torch, stream, lambda: calls(M), 1)
        per_m[str(M)] = round(LAYERS * layer_bytes(M) / (t * 1e-3) / 1e9, 1)
        per_m_us[str(M)] = round(t * 1e3 / (LAYERS * len(projs)), 2)

    # End to end through the public API with host buffers: pinned x in,
    # every y out, around the same graph.
    host_x = {key: xs[key].cpu().pin_memory() for key in xs if key[0] in QMV_M}
    host_y = {key: torch.empty(ys[key].shape, dtype=ys[key].dtype).pin_memory()
              for key in ys if key[0] in QMV_M}
    h2d = sum(v.numel() * 2 for v in host_x.values())
    d2h = sum(v.numel() * 2 for v in host_y.values())
    with torch.cuda.stream(stream):
        def e2e_step():
            for key in host_x:
                xs[key].copy_(host_x[key], non_blocking=True)
            g.replay()
            for key in host_y:
                host_y[key].copy_(ys[key], non_blocking=True)
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        c.record(stream)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(c) / args.steps, world)
    e2e = {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # Dominant kernel of the step: every call of the sweep (K = 2048 / 8192,
    # group 64: 16-byte packed rows and scale rows) runs the tensor-core
    # decode kernel, so its average launch is the step time over the calls.
    dom = "qmv_tc_kernel (aq_qmv, M = 1..16)"
    dom_us = ms * 1e3 / launches_per_step
    achieved = step_bytes / launches_per_step / (dom_us * 1e-6) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_kind": peak_kind + " copy bandwidth",
            "kernel": dom, "avg_launch_us": round(dom_us, 3),
            "bytes_per_launch": round(step_bytes / launches_per_step),
            "traffic": traffic_for("qmv_tc_kernel", "decode-stack")}
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "layers": LAYERS, "M": list(QMV_M), "bits": BITS,
                       "group_size": GS, "parallelism": "replicas" if world > 1 else "single",
                       "l2": "weights 547 MB > 4x L2 per step; no flush needed",
                       "timing": "CUDA graph replay, CUDA events on the launching stream",
                       "weight_prefetch": "on (weights streamed before each kernel's dependency wait)"},
            "per_m_gbs": per_m, "per_call_us": per_m_us, "roofline": roof,
            "independent_calls": independent,
            "clocks": clk.summary(), "e2e": e2e, "gpu_launches": launches_per_step * args.steps}
    if not args.no_qmm:
        qmm, roof_qmm = qmm_lines(torch, api, inputs, dev, stream, tf, tf_sust)
        line["qmm_tflops"] = qmm
        line["roofline_qmm"] = roof_qmm
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
