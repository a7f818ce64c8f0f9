"""Benchmark of the quantized matmul hot path on B200.

Headline workload (one step): the decode sweep of a 16-layer
Llama-3.2-1B-shaped stack of distinct bf16 weights quantized 4-bit, group 64
(q/o 2048x2048, k/v 512x2048, gate/up 8192x2048, down 2048x8192; 547 MB of
packed weights, scales and biases per step, more than 4x the 126 MB L2, so no
L2 flush is needed and every step streams the weights from HBM).  For each M
in (1, 2, 4, 8, 16) the step computes y = x . dequant(W)^T for all 112
projections of the stack as independent problems through aq_qmv_batched (one
launch per 40 problems).  The step is captured once in a CUDA graph and
replayed.

Metric: qmv weight-stream GB/s = (packed weights + scales + biases + x + y
bytes of all products) / device time of the step, whole job (all ranks).

Beside it (not part of the step):
  * per_call_chain: the same 560 products as 560 aq_qmv calls in order, each
    waiting for its predecessor (the per-call latency view), with the
    per-projection times;
  * per-M views of the batched step; the sweep's M = 32, 64 through aq_qmm;
  * the tiny fp16 config (512x512, M = 1, 8) and the FP4 qmv config
    (4096x4096, M = 1, 16, E8M0 g32 and E4M3 g16 scales);
  * the tensor-core side in TFLOP/s (2 M N K / time): the chained fp16 qmm
    (x[1024,1024] through W1 [4096,1024] and W2 [1024,4096], ten times) at
    bits 2, 3, 4, 6, 8; the conv2d implicit GEMM at groups 1 and 4, 4- and
    8-bit; FP4 weights at M = 256 and 4096 with both scale kinds; the 4-bit
    affine 4096^3 product;
  * the oracle on the host cores (all cores and one thread).

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
            "gate/up 8192x2048, down 2048x8192), bf16, 4-bit affine g64, M in 1,2,4,8,16; "
            "per M the 112 projections as independent problems through aq_qmv_batched")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layers of the stack (default 16; fewer for small profiling runs)")
    ap.add_argument("--no-qmm", action="store_true", help="skip the side configurations")
    ap.add_argument("--only", default="all", choices=["all", "qmm"],
                    help="qmm: run only the side configurations")
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


def max_over_ranks(v, world, device="cuda"):
    """The largest of the ranks' values (a step time: the job is as slow as
    its slowest rank).  `device`: where the collective's tensor lives (the
    process group's backend: cuda for nccl, cpu for gloo)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, bytes_per_rank_step, ms_per_step):
    """Whole-job throughput of `world` replicas, each streaming
    bytes_per_rank_step per step, over the max-over-ranks step time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def traffic_for(kernel, workload):
    """DRAM bytes per algorithmic byte of `kernel` from a committed ncu
    capture (profiles/traffic.json), if the kernel's sources have not changed
    since; None otherwise."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        h = hashlib.sha256()
        for src in rec["sources"]:
            h.update(open(os.path.join(ROOT, src), "rb").read())
        if h.hexdigest()[:16] != rec["sources_sha256_16"] or rec["workload"] != workload:
            return None
        return rec["dram_bytes_per_algorithmic_byte"]
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


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def cpu_baseline():
    """The oracle as it stands, on the host cores, over a bounded sample: one
    layer of the stack at M = 1, 2, 4, 8, 16 (the same inputs recipe), on all
    cores and then on one thread (one layer at M = 1)."""
    import oracle
    from oracle import build_oracle
    from group_wise_affine_quant_b200 import inputs
    ws = inputs.decode_layer(seed=0)
    q = {name: oracle.quantize(inputs.as_u16(w), BITS, GS, 1) for name, w in ws.items()}

    xs = {(M, k): inputs.as_u16(inputs.decode_x(M, k)) for M in QMV_M for k in (2048, 8192)}

    def run(ms, min_s):
        # whole passes over the sample until at least min_s seconds of oracle time
        tot_bytes, tot_t, passes = 0, 0.0, 0
        while tot_t < min_s:
            for M in ms:
                for name, n, k in inputs.LLAMA_1B_PROJ:
                    wq, s, b = q[name]
                    t0 = time.perf_counter()
                    oracle.qmm(xs[(M, k)], wq, s, b, n, BITS, GS, 0, 1)
                    tot_t += time.perf_counter() - t0
                tot_bytes += layer_bytes(M)
            passes += 1
        return tot_bytes, tot_t, passes

    cores = oracle.num_threads()
    b_all, t_all, p_all = run(QMV_M, 10.0)
    oracle.set_num_threads(1)
    try:
        b_one, t_one, p_one = run((1,), 5.0)
    finally:
        oracle.set_num_threads(cores)
    return {"value": round(b_all / t_all / 1e9, 3), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": "%d passes over one layer of the stack (7 projections) at M = 1,2,4,8,16, "
                      "%.1f s" % (p_all, t_all),
            "single_thread": {"value": round(b_one / t_one / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": "%d passes over one layer at M = 1, %.1f s" % (p_one, t_one)},
            "cpu_model": cpu_model(), "build": "g++ " + " ".join(build_oracle.FLAGS)}


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


def stack_problems(layers, xs, ys, M):
    """The 112 projections of the stack at M rows as (x, w_q, s, b, y) lists."""
    from group_wise_affine_quant_b200.inputs import LLAMA_1B_PROJ
    X, W, S, B, Y = [], [], [], [], []
    for li, q in enumerate(layers):
        for name, n, k in LLAMA_1B_PROJ:
            wq, sc, bi = q[name]
            X.append(xs[(M, k)]); W.append(wq); S.append(sc); B.append(bi)
            Y.append(ys[(M, li, name)])
    return X, W, S, B, Y


def side_lines(torch, api, inputs, dev, stream, hbm, tf_peak):
    """The other configurations, each timed alone (not part of the step).
    Every weight here is quantized before its timed calls and no timed kernel
    writes one, so the kernels may stream weights before their dependency wait
    (the same setting as the decode step)."""
    import random
    out, tfl = {}, {}
    api.aq_set_weight_prefetch(True)
    # --- tiny fp16 qmv/qmm (512x512, 4-bit g64), M = 1 and 8: L2-resident, so
    # the time per call (a chain of 100 calls) is the meaningful number
    for M in (1, 8):
        x, w = inputs.tiny(M, seed=0)
        q = api.aq_quantize(w.to(dev), 4, 64)
        xd = x.to(dev)
        y = torch.empty((M, 512), dtype=torch.float16, device=dev)
        t = graph_time_ms(torch, stream, lambda: api.aq_qmv(xd, *q, 4, 64, out=y), 100)
        out["tiny_fp16_qmv_M%d" % M] = {"us_per_call": round(t * 1e3, 2), "l2_resident": True}
    # --- FP4 qmv, 4096x4096, M = 1, 16; 20 distinct weight copies (180 MB > L2)
    for gs, kind in ((32, "e8m0"), (16, "e4m3")):
        copies = [inputs.fp4(4096, 4096, gs, seed=40 + i) for i in range(20)]
        wcs = [(c.to(dev), sc.to(dev)) for c, sc in copies]
        del copies
        for M in (1, 16):
            xf = inputs.fp4_x(M, 4096).to(dev)
            yf = [torch.empty((M, 4096), dtype=torch.bfloat16, device=dev) for _ in wcs]
            byt = 20 * (4096 * 2048 + 4096 * (4096 // gs) + 2 * M * 4096 * 2)

            def chain():
                for (c, sc), yy in zip(wcs, yf):
                    api.aq_qmv(xf, c, sc, None, 4, gs, out=yy)
            t = graph_time_ms(torch, stream, chain, 2)

            def batched():
                api.aq_qmv_batched([xf] * 20, [c for c, _ in wcs], [sc for _, sc in wcs],
                                   None, 4, gs, outs=yf)
            tb = graph_time_ms(torch, stream, batched, 2)
            out["fp4_%s_qmv_M%d" % (kind, M)] = {
                "per_call_gbs": round(byt / (t * 1e-3) / 1e9, 1),
                "us_per_call": round(t * 1e3 / 20, 2),
                "batched_gbs": round(byt / (tb * 1e-3) / 1e9, 1),
                "batched_frac_of_hbm": round(byt / (tb * 1e-3) / 1e9 / hbm, 4)}
        # FP4 qmm at M = 256 and 4096 (tensor-bound), one weight
        wc, sc = wcs[0]
        for M in (256, 4096):
            xf = inputs.fp4_x(M, 4096).to(dev)
            yf = torch.empty((M, 4096), dtype=torch.bfloat16, device=dev)
            t = graph_time_ms(torch, stream, lambda: api.aq_qmm(xf, wc, sc, None, 4, gs, out=yf), 10)
            tfl["fp4_%s_M%d" % (kind, M)] = {"tflops": round(2 * M * 4096 * 4096 / (t * 1e-3) / 1e12, 1),
                                            "ms": round(t, 4)}
        del wcs
    # --- W4A4 (aq_qqmm): x fake-quantized to FP4 E8M0 g32, FP4 weights
    # 4096 x 4096 (20 copies for the decode rows, 180 MB > L2)
    copies = [inputs.fp4(4096, 4096, 32, seed=80 + i) for i in range(20)]
    wcs = [(c.to(dev), sc.to(dev)) for c, sc in copies]
    del copies
    for M in (1, 16):
        xf = inputs.fp4_x(M, 4096).to(dev)
        yf = [torch.empty((M, 4096), dtype=torch.bfloat16, device=dev) for _ in wcs]
        byt = 20 * (4096 * 2048 + 4096 * 128 + 2 * M * 4096 * 2)

        def chain_qq():
            for (c, sc), yy in zip(wcs, yf):
                api.aq_qqmm(xf, c, sc, 32, out=yy)
        t = graph_time_ms(torch, stream, chain_qq, 2)
        out["w4a4_qqmm_M%d" % M] = {"per_call_gbs": round(byt / (t * 1e-3) / 1e9, 1),
                                    "us_per_call": round(t * 1e3 / 20, 2),
                                    "launches_per_call": 2}
    wc, sc = wcs[0]
    for M in (256, 4096):
        xf = inputs.fp4_x(M, 4096).to(dev)
        yf = torch.empty((M, 4096), dtype=torch.bfloat16, device=dev)
        t = graph_time_ms(torch, stream, lambda: api.aq_qqmm(xf, wc, sc, 32, out=yf), 10)
        out["w4a4_qqmm_M%d" % M] = {"tflops": round(2 * M * 4096 * 4096 / (t * 1e-3) / 1e12, 1),
                                    "ms": round(t, 4), "launches_per_call": 2}
    del wcs
    # --- gather (aq_gather_qmm): a mixture-of-experts decode step, 8 experts
    # of 1408 x 2048 (bf16, 4-bit g64), 48 token rows routed to 2 experts each:
    # 96 pairs, grouped by expert (each expert streamed once per call)
    E, NE, KE, TOK = 8, 1408, 2048, 48
    qs = [api.aq_quantize(inputs.normal((NE, KE), 0.02, 1, inputs.gen(90 + e)).to(dev), 4, 64)
          for e in range(E)]
    wq_e, s_e, b_e = (torch.stack([q[j] for q in qs]) for j in range(3))
    del qs
    xg = inputs.normal((TOK, 1, KE), 1.0, 1, inputs.gen(98)).to(dev)
    grng = random.Random(5)
    lhs = [t for t in range(TOK) for _ in range(2)]
    rhs = [e for t in range(TOK) for e in grng.sample(range(E), 2)]
    yg = torch.empty((len(lhs), 1, NE), dtype=torch.bfloat16, device=dev)
    t = graph_time_ms(torch, stream, lambda: api.aq_gather_qmm(xg, wq_e, s_e, b_e, lhs, rhs, 4, 64,
                                                               out=yg), 5)
    pair_bytes = NE * KE // 2 + 4 * NE * (KE // 64) + 2 * KE + 2 * NE
    expert_bytes = E * (NE * KE // 2 + 4 * NE * (KE // 64)) + len(lhs) * 2 * (KE + NE)
    out["gather_moe_decode_96pairs"] = {
        "us_per_call": round(t * 1e3, 2),
        "gbs_expert_bytes": round(expert_bytes / (t * 1e-3) / 1e9, 1),
        "gbs_pair_equivalent": round(len(lhs) * pair_bytes / (t * 1e-3) / 1e9, 1),
        "note": "pairs grouped by expert: 8 problems of up to 16 rows, x rows gathered and "
                "y rows scattered by two copy kernels"}
    del wq_e, s_e, b_e
    # --- non-transposed product (aq_qmm_nt, dy . W): the down projection's
    # weight (2048 x 8192, bf16, 4-bit g64), x [M, 2048] -> y [M, 8192];
    # 16 weight copies (150 MB > L2)
    wts = [api.aq_quantize(inputs.normal((2048, 8192), 0.02, 1, inputs.gen(120 + i)).to(dev), 4, 64)
           for i in range(16)]
    for M in (1, 16):
        xn = inputs.normal((M, 2048), 1.0, 1, inputs.gen(130)).to(dev)
        yn = torch.empty((M, 8192), dtype=torch.bfloat16, device=dev)

        def chain_nt():
            for q in wts:
                api.aq_qmm_nt(xn, *q, 4, 64, out=yn)
        t = graph_time_ms(torch, stream, chain_nt, 2)
        byt = 16 * (2048 * 4096 + 4 * 2048 * 128 + 2 * M * 2048 + 2 * M * 8192)
        out["qmm_nt_down_M%d" % M] = {"gbs": round(byt / (t * 1e-3) / 1e9, 1),
                                      "us_per_call": round(t * 1e3 / 16, 2),
                                      "frac_of_hbm": round(byt / (t * 1e-3) / 1e9 / hbm, 4)}
    del wts
    # --- chained fp16 qmm, 20 products per chain, bits 2, 3, 4, 6, 8
    x, w1, w2 = inputs.chained()
    xd = x.to(dev)
    h = torch.empty((1024, 4096), dtype=torch.float16, device=dev)
    o = torch.empty((1024, 1024), dtype=torch.float16, device=dev)
    for bits in (2, 3, 4, 6, 8):
        q1 = api.aq_quantize(w1.to(dev), bits, 64)
        q2 = api.aq_quantize(w2.to(dev), bits, 64)

        def chain():
            cur = xd
            for _ in range(10):
                api.aq_qmm(cur, *q1, bits, 64, out=h)
                api.aq_qmm(h, *q2, bits, 64, out=o)
                cur = o
        t = graph_time_ms(torch, stream, chain, 3)
        tfl["chained_fp16_%dbit" % bits] = {
            "tflops": round(20 * 2 * 1024 * 4096 * 1024 / (t * 1e-3) / 1e12, 1),
            "ms_per_chain": round(t, 4)}
    # --- conv2d implicit GEMM, bf16, batch 2, 64x64, 320 -> 320, 3x3, pad 1
    for groups in (1, 4):
        xc, wcv = inputs.conv(groups)
        w2d = inputs.flatten_pad_conv_weight(wcv, 64)
        xcd = xc.to(dev)
        yc = torch.empty((2, 64, 64, 320), dtype=torch.bfloat16, device=dev)
        for bits in (4, 8):
            qc = api.aq_quantize(w2d.to(dev), bits, 64)
            t = graph_time_ms(torch, stream, lambda: api.aq_qconv2d_nhwc(
                xcd, *qc, 320, 3, 3, (1, 1), (1, 1), groups, bits, 64, out=yc), 10)
            fl = 2 * 8192 * 320 * 9 * 320 // groups
            tfl["conv2d_g%d_%dbit" % (groups, bits)] = {
                "tflops": round(fl / (t * 1e-3) / 1e12, 1), "ms": round(t, 4)}
    # --- 4-bit affine 4096^3, bf16
    xf = inputs.fp4_x(4096, 4096).to(dev)
    yf = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
    wa = api.aq_quantize(inputs.normal((4096, 4096), 0.02, 1, inputs.gen(8)).to(dev), 4, 64)
    t = graph_time_ms(torch, stream, lambda: api.aq_qmm(xf, *wa, 4, 64, out=yf), 10)
    tfl["affine4_M4096"] = {"tflops": round(2 * 4096 ** 3 / (t * 1e-3) / 1e12, 1), "ms": round(t, 4)}
    # the qmm roofline on the workloads the >= 60 % target is judged on (M >= 1024)
    judged = {"chained_fp16_4bit": "qmm_tc_kernel (chained fp16 qmm, 4-bit, M = 1024)",
              "conv2d_g1_4bit": "qmm_tc_kernel (conv2d implicit GEMM, groups 1, 4-bit, M = 8192)",
              "fp4_e8m0_M4096": "qmm_tc_kernel (FP4 E8M0, M = 4096)"}
    roof = {"bound": "tensor", "peak": tf_peak, "unit": "TFLOP/s", "peak_kind": "measured burst bf16",
            "workloads": {k: {"achieved": tfl[k]["tflops"], "frac": round(tfl[k]["tflops"] / tf_peak, 4),
                              "kernel": v} for k, v in judged.items()}}
    worst = min(roof["workloads"].items(), key=lambda kv: kv[1]["frac"])
    roof.update({"achieved": worst[1]["achieved"], "frac": worst[1]["frac"], "kernel": worst[1]["kernel"],
                 "traffic": None})
    return out, tfl, roof


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
    stream = torch.cuda.Stream(dev)
    if args.only == "qmm":
        side, tfl, roof_qmm = side_lines(torch, api, inputs, dev, stream, hbm, tf)
        if rank == 0:
            print(json.dumps({"side": side, "qmm_tflops": tfl, "roofline_qmm": roof_qmm}))
        return

    # Quantize the stack once (on the device, through the library).  The
    # timed calls never follow a kernel that writes their weights, so the
    # library may stream weights before waiting on the previous kernel.
    n_layers = args.layers
    layers = []
    for li in range(n_layers):
        ws = inputs.decode_layer(seed=100 + li)
        layers.append({name: api.aq_quantize(w.to(dev), BITS, GS) for name, w in ws.items()})
        del ws
    torch.cuda.synchronize()
    api.aq_set_weight_prefetch(True)
    projs = inputs.LLAMA_1B_PROJ
    all_m = QMV_M + QMM_M
    xs = {(M, k): inputs.decode_x(M, k, seed=M).to(dev) for M in all_m for k in (2048, 8192)}
    ys = {(M, li, name): torch.empty((M, n), dtype=torch.bfloat16, device=dev)
          for M in all_m for li in range(n_layers) for name, n, _ in projs}
    probs = {M: stack_problems(layers, xs, ys, M) for M in QMV_M}
    n_problems = n_layers * len(projs)
    launches_per_m = (n_problems + 39) // 40
    launches_per_step = len(QMV_M) * launches_per_m

    def step_m(M):
        X, W, S, B, Y = probs[M]
        api.aq_qmv_batched(X, W, S, B, BITS, GS, outs=Y)

    def step():
        for M in QMV_M:
            step_m(M)

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
    step_bytes = n_layers * sum(layer_bytes(M) for M in QMV_M)
    value = whole_job_gbs(world, step_bytes, ms)

    # Per-M views of the batched step.
    per_m = {}
    for M in QMV_M:
        t = graph_time_ms(torch, stream, lambda: step_m(M), 1)
        per_m[str(M)] = {"gbs": round(n_layers * layer_bytes(M) / (t * 1e-3) / 1e9, 1),
                         "ms": round(t, 4)}

    # The same products as 560 aq_qmv calls in order (each kernel waits for
    # the previous one before reading x and writing y): the per-call view.
    def calls(M, names=None):
        fn = api.aq_qmv if M <= 16 else api.aq_qmm
        for li, q in enumerate(layers):
            for name, n, k in projs:
                if names and name not in names:
                    continue
                wq, sc, bi = q[name]
                fn(xs[(M, k)], wq, sc, bi, BITS, GS, out=ys[(M, li, name)])
    tc = graph_time_ms(torch, stream, lambda: [calls(M) for M in QMV_M], 1)
    chain = {"gbs": round(step_bytes / (tc * 1e-3) / 1e9, 1), "ms_per_step": round(tc, 4),
             "us_per_call": round(tc * 1e3 / (len(QMV_M) * n_problems), 2), "per_projection": {}}
    for name, n, k in projs:
        for M in (1, 16):
            t = graph_time_ms(torch, stream, lambda: calls(M, (name,)), 1)
            chain["per_projection"]["%s_M%d" % (name, M)] = {
                "us_per_call": round(t * 1e3 / n_layers, 2),
                "gbs": round(n_layers * proj_bytes(n, k, M) / (t * 1e-3) / 1e9, 1)}
    # the sweep's M = 32 and 64 rows through aq_qmm (per call, same stack)
    qmm_m = {}
    for M in QMM_M:
        t = graph_time_ms(torch, stream, lambda: calls(M), 1)
        qmm_m[str(M)] = {"gbs": round(n_layers * layer_bytes(M) / (t * 1e-3) / 1e9, 1),
                         "us_per_call": round(t * 1e3 / n_problems, 2)}

    # End to end through the public API with host buffers: pinned x in,
    # every y out, around the same graph.
    host_x = {key: xs[key].cpu().pin_memory() for key in xs if key[0] in QMV_M}
    y_keys = [key for key in ys if key[0] in QMV_M]
    host_y = {key: torch.empty(ys[key].shape, dtype=ys[key].dtype).pin_memory() for key in y_keys}
    h2d = sum(v.numel() * 2 for v in host_x.values())
    d2h = sum(v.numel() * 2 for v in host_y.values())
    with torch.cuda.stream(stream):
        def e2e_step():
            for key in host_x:
                xs[key].copy_(host_x[key], non_blocking=True)
            g.replay()
            for key in y_keys:
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
    e2e = {"value": round(whole_job_gbs(world, step_bytes, e2e_ms), 1), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # Dominant kernel: every launch of the step is qmv_mma_kernel (4-bit
    # affine, K a multiple of the 512-column sub-slice), so its average launch
    # is the step time over the launches.
    dom = "qmv_mma_kernel (aq_qmv_batched, M = 1..16)"
    dom_us = ms * 1e3 / launches_per_step
    bpl = step_bytes / launches_per_step
    achieved = bpl / (dom_us * 1e-6) / 1e9
    ratio = traffic_for("qmv_mma_kernel", "decode-stack-batched")
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_kind": peak_kind + " copy bandwidth",
            "kernel": dom, "avg_launch_us": round(dom_us, 3), "bytes_per_launch": round(bpl),
            "traffic": None if ratio is None else round(ratio * bpl)}
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "layers": n_layers, "M": list(QMV_M), "bits": BITS,
                       "group_size": GS, "parallelism": "replicas" if world > 1 else "single",
                       "l2": "stack of %.0f MB of weights (> L2) streamed once per M; no flush "
                             "needed" % (n_layers * layer_bytes(0) / 1e6),
                       "timing": "CUDA graph replay, CUDA events on the launching stream",
                       "weight_prefetch": "on (weights streamed before each kernel's dependency wait)"},
            "per_m": per_m, "per_call_chain": chain, "qmm_decode_m": qmm_m, "roofline": roof,
            "clocks": clk.summary(), "e2e": e2e, "gpu_launches": launches_per_step * args.steps}
    if not args.no_qmm:
        side, tfl, roof_qmm = side_lines(torch, api, inputs, dev, stream, hbm, tf)
        line["side"] = side
        line["qmm_tflops"] = tfl
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
