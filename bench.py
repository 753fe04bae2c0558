"""Benchmark of the SVDQuant W4A4 (NVFP4) linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--legs]

One step = one pass of the layer over one batch: the quantize call
(smoothing + NVFP4 activation quantization + low-rank down-projection) and
the W4A4 GEMM call (block-scaled FP4 MMA + low-rank up-projection + bias +
bf16 store), on the attention-projection workload M=4096 tokens, K=N=3072,
r=32.  Prints one JSON line (rank 0).  Multi-GPU runs are independent
replicas (weak scaling: each rank runs its own batch; the layer needs no
exchange); timing is the max over ranks of the device-timed region.

The oracle (``oracle/``, CPU) is used only by the ``cpu_baseline`` leg and
by ``--impl reference``.
"""
import argparse
import hashlib
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

CASE = workloads.HEADLINE
METRIC = "SVDQ NVFP4 linear TFLOP/s & % dense-FP4 peak (M4096 K3072 N3072 r32)"
UNIT = "TFLOP/s"
WORKLOAD = "attn-proj SVDQ W4A4 NVFP4 linear M4096 K3072 N3072 r32 (quantize + GEMM)"
FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PF)
DATASHEET_FP4_TFLOPS = 9000.0


def layer_flops(M, K, N, r):
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def aggregate(total_ms, steps, flops_per_step, world, device=None):
    """Whole-job throughput of ``world`` replicas: every rank processed
    ``steps`` steps; the job time is the max of the ranks' device times.
    Returns (max_ms, TFLOP/s).  All ranks must call it (one collective)."""
    if world > 1:
        t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    return total_ms, flops_per_step * steps * world / (total_ms * 1e-3) / 1e12


def peaks():
    p = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
    except OSError:
        pass
    return p


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 20 ms
    while the timed region runs (the same counters nvidia-smi reports)."""
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, dev):
        self.dev = dev
        self.samples = []
        self.max_mhz = None
        self._stop = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devid = getattr(props, "pci_device_id", 0)
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devid:02x}.0")
            except pynvml.NVMLError:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(torch.device(self.dev).index or 0)

    def __enter__(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            while not self._stop.is_set():
                try:
                    self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                         int(get_reasons(h))))
                except Exception:
                    pass
                self._stop.wait(0.02)
        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)

    def summary(self):
        sm = [c for c, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, b in self.REASONS.items() if r & b})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm)}


# ------------------------------------------------------- device workload --
def make_sets(dev, l2_bytes, case=None):
    """Independent copies of one layer (weights + activations + outputs),
    prepared on the device by the library's own offline prep, enough of them
    that their total exceeds 3x L2: rotating through them keeps every step's
    operands out of L2."""
    import svdquant_w4a4_gemm_b200 as sv
    from svdquant_w4a4_gemm_b200 import prep as dprep
    case = CASE if case is None else case
    d = workloads.draw_svdq(case)
    x0 = torch.from_numpy(d["x"]).to(dev).to(torch.bfloat16)
    W0 = torch.from_numpy(d["W"]).to(dev).to(torch.bfloat16)
    b0 = torch.from_numpy(d["bias"]).to(dev).to(torch.bfloat16)
    xc = torch.from_numpy(d["x_cal"]).to(dev).to(torch.bfloat16)
    w0 = dprep.prepare_svdq(W0, b0, xc, case.r)
    M, K, N, r = case.M, case.K, case.N, case.r
    gs = torch.empty(1, device=dev)
    sv.quantize_act(x0, w0.smooth, w0.L1t, None, out=(
        torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
        torch.empty(sv.scale_bytes(M, K), dtype=torch.uint8, device=dev),
        torch.empty(M, r, device=dev), gs))     # static activation scale from the data
    per = (x0.numel() * 2 + M * K // 2 + sv.scale_bytes(M, K) + M * r * 4 + M * N * 2 +
           w0.q_w.numel() + w0.sf_w.numel() + w0.L1t.numel() * 2 + w0.L2t.numel() * 2)
    nsets = max(2, int(np.ceil(3 * l2_bytes / per)))
    sets = []
    for i in range(nsets):
        # distinct copies (same values) so that no two steps share memory
        w = sv.SvdqWeights(q_w=w0.q_w.clone(), sf_w=w0.sf_w.clone(), gs_w=w0.gs_w.clone(),
                           L1t=w0.L1t.clone(), L2t=w0.L2t.clone(), smooth=w0.smooth.clone(),
                           bias=w0.bias.clone())
        sets.append(dict(
            w=w, x=x0.clone(), gs=gs.clone(),
            q=torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
            sf=torch.empty(sv.scale_bytes(M, K), dtype=torch.uint8, device=dev),
            lora=torch.empty(M, r, device=dev), gso=torch.empty(1, device=dev),
            y=torch.empty(M, N, dtype=torch.bfloat16, device=dev)))
    return sets, per


def run_step(sv, s):
    sv.quantize_act(s["x"], s["w"].smooth, s["w"].L1t, s["gs"], out=(s["q"], s["sf"], s["lora"], s["gso"]))
    sv.w4a4_linear(s["q"], s["sf"], s["gso"], s["lora"], s["w"], y=s["y"])


def kernel_traffic(kernel_file, kernel_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            tab = json.load(f)
        src = open(os.path.join(ROOT, "svdquant_w4a4_gemm_b200", "csrc", kernel_file), "rb").read()
        h = hashlib.sha256(src).hexdigest()[:16]
        ent = tab.get(kernel_name)
        if ent and ent.get("source_sha256_16") == h:
            return ent.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def bench_device(args, rank, world, dev):
    import svdquant_w4a4_gemm_b200 as sv
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    sets, per = make_sets(dev, l2)
    nsets = len(sets)
    stream = torch.cuda.current_stream(dev)
    M, K, N, r = CASE.M, CASE.K, CASE.N, CASE.r

    for i in range(args.warmup):
        run_step(sv, sets[i % nsets])
    sv.check_device_errors()

    # ---- the K timed steps, captured once into a CUDA graph so that the
    # device time is not limited by host launch overhead ----
    gsteps = min(args.steps, 200)                 # steps per captured graph
    replays = max(1, -(-args.steps // gsteps))
    cap = torch.cuda.Stream(dev)

    def capture(body):
        g = torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap):
            for i in range(gsteps):
                body(sets[i % nsets])
        g.replay()                      # untimed: uploads the graph
        torch.cuda.synchronize(dev)
        return g

    def k1(s):
        sv.quantize_act(s["x"], s["w"].smooth, s["w"].L1t, s["gs"], out=(s["q"], s["sf"], s["lora"], s["gso"]))

    def k2(s):
        sv.w4a4_linear(s["q"], s["sf"], s["gso"], s["lora"], s["w"], y=s["y"])

    graph = capture(lambda s: (k1(s), k2(s)))
    sv.check_device_errors()

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        t_start.record(stream)
        for _ in range(replays):
            graph.replay()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    sv.check_device_errors()
    steps_done = gsteps * replays
    total_ms, _ = aggregate(t_start.elapsed_time(t_end), steps_done,
                            layer_flops(CASE.M, CASE.K, CASE.N, CASE.r), world, dev)
    # ---- per-kernel device times: each kernel alone, in a graph of its own
    # over the same rotating sets (events around whole replays, on the stream
    # the kernels run on) ----
    per_kernel = {}
    for name, body in (("k1", k1), ("k2", k2)):
        g = capture(body)
        reps = max(1, min(replays, 10))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        per_kernel[name] = [a.elapsed_time(b) * 1e3 / (reps * gsteps)]
        del g
    k1_us, k2_us = per_kernel["k1"], per_kernel["k2"]

    # ---- e2e: the same call with host buffers, copies inside the timed region ----
    x_host = sets[0]["x"].cpu().pin_memory()
    y_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    s0 = sets[0]
    for _ in range(2):
        s0["x"].copy_(x_host, non_blocking=True)
        run_step(sv, s0)
        y_host.copy_(s0["y"], non_blocking=True)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(e2e_steps):
        s = sets[i % nsets]
        s["x"].copy_(x_host, non_blocking=True)
        run_step(sv, s)
        y_host.copy_(s["y"], non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize(dev)
    # whole-job, like `value`: the slowest rank's time, every rank's steps
    e2e_total_ms, e2e_tflops = aggregate(a.elapsed_time(b), e2e_steps, layer_flops(M, K, N, r), world, dev)
    e2e_ms = e2e_total_ms / e2e_steps

    del graph
    legs = None
    if args.legs and rank == 0:
        legs = bench_awq_legs(sv, dev, l2)
        legs.update(bench_gelu_leg(sv, dev, l2))
        try:
            legs.update(bench_dynamic_scale_leg(sv, dev, sets, gsteps, capture))
        except Exception as e:  # noqa: BLE001 - report it on the line, keep the line
            legs["quantize_dynamic_error"] = str(e)[:200]
    return dict(steps=steps_done, total_ms=total_ms, k1_us=k1_us, k2_us=k2_us, clocks=clk.summary(), nsets=nsets,
                set_mb=per / 2 ** 20, e2e_ms=e2e_ms, e2e_tflops=e2e_tflops, h2d=x_host.numel() * 2,
                d2h=y_host.numel() * 2, legs=legs)


def bench_dynamic_scale_leg(sv, dev, sets, gsteps, capture, reps=5):
    """The headline activation quantized three ways: static gs_a (the
    step's K1), dynamic gs_a by a max pass + K1 + finalize, and dynamic gs_a
    in one cooperative launch.  Device time per call over rotating sets."""
    stream = torch.cuda.current_stream(dev)
    ws = [torch.zeros(sv.QUANTIZE_WORKSPACE_BYTES, dtype=torch.uint8, device=dev) for _ in sets]
    for s_ in sets:
        s_["gdyn"] = torch.empty(1, device=dev)
    bodies = {
        "static": lambda s_: sv.quantize_act(s_["x"], s_["w"].smooth, s_["w"].L1t, s_["gs"],
                                             out=(s_["q"], s_["sf"], s_["lora"], s_["gso"])),
        "dynamic_max_pass": lambda s_: sv.quantize_act(s_["x"], s_["w"].smooth, s_["w"].L1t, None,
                                                       out=(s_["q"], s_["sf"], s_["lora"], s_["gdyn"])),
    }
    idx = {id(s_): i for i, s_ in enumerate(sets)}
    bodies["dynamic_single_pass"] = lambda s_: sv.quantize_act_dynamic(
        s_["x"], s_["w"].smooth, s_["w"].L1t, out=(s_["q"], s_["sf"], s_["lora"], s_["gdyn"]),
        workspace=ws[idx[id(s_)]])
    out = {}
    for name, body in bodies.items():
        for i in range(3):
            body(sets[i % len(sets)])
        try:
            g = capture(body)
            how = "graph"
        except Exception:            # a launch kind the stream capture refuses: time it eagerly
            torch.cuda.synchronize(dev)
            g, how = None, "eager"
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            if g is not None:
                g.replay()
            else:
                for i in range(gsteps):
                    body(sets[i % len(sets)])
        b.record(stream)
        torch.cuda.synchronize(dev)
        out[f"quantize_{name}"] = {"us": round(a.elapsed_time(b) * 1e3 / (reps * gsteps), 3), "timed": how}
        del g
    sv.check_device_errors()
    return out


def bench_gelu_leg(sv, dev, l2, steps=200, reps=5):
    """The MLP up-projection GEMM (M4096 K3072 N12288 r32) with the plain
    epilogue and with GELU(tanh) fused into it: device time per launch,
    graphs over rotating sets > 3x L2."""
    case = workloads.MLP_UP
    sets, _ = make_sets(dev, l2, case)
    for s in sets:
        sv.quantize_act(s["x"], s["w"].smooth, s["w"].L1t, s["gs"], out=(s["q"], s["sf"], s["lora"], s["gso"]))
    stream = torch.cuda.current_stream(dev)
    cap = torch.cuda.Stream(dev)
    out = {}
    for act in (None, "gelu"):
        g = torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap):
            for i in range(steps):
                s = sets[i % len(sets)]
                sv.w4a4_linear(s["q"], s["sf"], s["gso"], s["lora"], s["w"], y=s["y"], act=act)
        g.replay()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        us = a.elapsed_time(b) * 1e3 / (reps * steps)
        fl = layer_flops(case.M, case.K, case.N, case.r)
        out[f"mlp_up_gemm_{act or 'plain'}"] = {"us": round(us, 3), "TFLOP/s": round(fl / us / 1e6, 1)}
        del g
    sv.check_device_errors()
    return out


def bench_awq_legs(sv, dev, l2):
    """The AWQ W4A16 modulation layer (M = 1, 2, 8; K = 3072, N = 18432),
    HBM-bound: GB/s of algorithmic bytes, rotating weight copies > 3x L2."""
    from svdquant_w4a4_gemm_b200 import prep as dprep
    out = {}
    for Mw, case in workloads.AWQ.items():
        d = workloads.draw_awq(case)
        W = torch.from_numpy(d["W"]).to(dev).to(torch.bfloat16)
        xc = torch.from_numpy(d["x_cal"]).to(dev).to(torch.bfloat16)
        ainv, qw, sc, z = dprep.prepare_awq(W, xc)
        wbytes = qw.numel() * 4 + sc.numel() * 2 + z.numel() * 2
        n = max(2, int(np.ceil(3 * l2 / wbytes)))
        copies = [(qw.clone(), sc.clone(), z.clone()) for _ in range(n)]
        x = torch.from_numpy(d["x"]).to(dev).to(torch.bfloat16)
        b = torch.from_numpy(d["bias"]).to(dev).to(torch.bfloat16)
        y = torch.empty(Mw, case.N, dtype=torch.bfloat16, device=dev)
        for i in range(5):
            c = copies[i % n]
            sv.awq_w4a16_linear(x, ainv, c[0], c[1], c[2], b, y=y)
        iters = 60
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for i in range(iters):
            c = copies[i % n]
            sv.awq_w4a16_linear(x, ainv, c[0], c[1], c[2], b, y=y)
        e1.record()
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) / iters * 1e3
        algo = wbytes + x.numel() * 2 + ainv.numel() * 4 + b.numel() * 2 + y.numel() * 2
        out[f"awq_M{Mw}"] = {"us": round(us, 3), "GB/s": round(algo / us / 1e3, 1),
                             "algorithmic_bytes": int(algo)}
    return out


# ----------------------------------------------------------------- oracle --
def oracle_sample(rows, seed_rows=0):
    """Prepare the oracle's layer once and return a closure that runs the
    oracle's whole layer on ``rows`` rows of the workload."""
    from oracle import prep as oprep, svdq as osv
    d = workloads.draw_svdq(CASE)
    L = oprep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], CASE.r)
    gs = osv.act_tensor_scale(d["x"], L["s"])
    xs = d["x"][seed_rows:seed_rows + rows]

    def run():
        return osv.svdq_forward(xs, L, gs)["y"]
    return run


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(rows=1024, reps=3):
    run = oracle_sample(rows)
    run()  # warm
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    dt = (time.perf_counter() - t0) / reps
    fl = layer_flops(rows, CASE.K, CASE.N, CASE.r)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} of {CASE.M} rows of the layer (numpy fp64 oracle: quantize, "
                      f"down-projection, dequantized GEMM + low-rank + bias), {reps} reps, "
                      f"{dt:.2f} s per rep"}


def run_reference(args, rank, world, budget_s=90.0):
    """The reference arm: the oracle, as it stands, on the host cores.  Each
    step runs the oracle's whole layer on a 32-row sample of the workload;
    the number of timed steps is capped so the run ends within ~budget_s
    (the line reports the steps actually timed and the ones requested)."""
    if rank != 0:
        return
    rows = 32
    run = oracle_sample(rows)
    t0 = time.perf_counter()
    for _ in range(args.warmup):
        run()
    per = (time.perf_counter() - t0) / max(1, args.warmup)
    steps = max(1, min(args.steps, int(budget_s / max(per, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(steps):
        run()
    dt = (time.perf_counter() - t0) / steps
    fl = layer_flops(rows, CASE.K, CASE.N, CASE.r)
    v = fl / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": CASE.M, "K": CASE.K, "N": CASE.N, "r": CASE.r,
                       "parallelism": "replicas" if world > 1 else "single"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{rows} of {CASE.M} rows per step (numpy fp64 oracle: "
                                       f"quantize, down-projection, dequantized GEMM + low-rank + bias)"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- main --
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--legs", action="store_true", help="also time the AWQ W4A16 modulation layer")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    # the CPU baseline runs before any CUDA work (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    dev = f"cuda:{local}"
    if world > 1:
        import datetime
        torch.cuda.set_device(dev)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device(dev))
    res = bench_device(args, rank, world, dev)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    M, K, N, r = CASE.M, CASE.K, CASE.N, CASE.r
    fl = layer_flops(M, K, N, r)
    steps = res["steps"]
    ms = res["total_ms"] / steps
    value = fl * steps * world / (res["total_ms"] * 1e-3) / 1e12
    pk = peaks()
    sustained = pk.get("bf16_tflops_sustained")
    burst = pk.get("bf16_tflops")
    if sustained:
        peak, peak_src = sustained * FP4_PER_BF16, "of measured (sustained bf16 x nominal fp4/bf16 = 4)"
    else:
        peak, peak_src = 1590.0 * FP4_PER_BF16, "of fallback (1.59 PF bf16 x 4)"
    k2 = statistics.mean(res["k2_us"])
    k1 = statistics.mean(res["k1_us"])
    achieved = fl / (k2 * 1e-6) / 1e12
    k1_bytes = M * K * 2 + K * 4 + r * K * 2 + M * K // 2 + (M * K // 16) + M * r * 4
    hbm = pk.get("hbm_gbs", 6650.0)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N, "r": r, "group": 16,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": f"rotating {res['nsets']} distinct input+weight sets of "
                         f"{res['set_mb']:.0f} MB (> 3x L2), no flush"},
        "pct_dense_fp4_peak": {"of_measured": round(value / world / peak, 4),
                               "of_datasheet_9PF": round(value / world / DATASHEET_FP4_TFLOPS, 4)},
        "roofline": {"bound": "tensor", "kernel": "w4a4_gemm_kernel", "achieved": round(achieved, 1),
                     "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": peak_src,
                     "traffic": kernel_traffic("gemm.cu", "w4a4_gemm_kernel"),
                     "algorithmic_flops_per_launch": fl, "avg_launch_us": round(k2, 3)},
        "kernels": {"quantize_act_kernel": {"avg_launch_us": round(k1, 3),
                                            "GB/s": round(k1_bytes / k1 / 1e3, 1),
                                            "frac_hbm": round(k1_bytes / k1 / 1e3 / hbm, 4),
                                            "algorithmic_bytes": k1_bytes,
                                            "traffic": kernel_traffic("quantize.cu", "quantize_act_kernel")},
                    "w4a4_gemm_kernel": {"avg_launch_us": round(k2, 3)}},
        "clocks": res["clocks"],
        "timed_region_ms": round(res["total_ms"], 3),
        "e2e": {"value": res["e2e_tflops"], "unit": UNIT,
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": 2 * steps,
        "cpu_baseline": cpu,
    }
    if res["legs"]:
        line["legs"] = res["legs"]
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
