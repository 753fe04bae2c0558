"""Benchmark of the SVDQuant W4A4 (NVFP4) linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-legs]

One step = one pass of the layer over one batch: the quantize call
(smoothing + NVFP4 activation quantization + low-rank down-projection) and
the W4A4 GEMM call (block-scaled FP4 MMA + low-rank up-projection + bias +
bf16 store), on the attention-projection workload M=4096 tokens, K=N=3072,
r=32.  Prints one JSON line (rank 0).  Multi-GPU runs are independent
replicas (weak scaling: each rank runs its own batch; the layer needs no
exchange); timing is the max over ranks of the device-timed region.

Besides the K timed steps, a single-GPU run times (outside that region, on
the same device, each over >= 10 separately timed graph replays, median and
range):
* each kernel of the step alone (``kernels``, ``roofline``);
* ``legs``: the other workloads (the tiny layer; the MLP pair: up-projection
  with the plain and the GELU epilogue, down-projection, the whole pair; the
  fused QKV projection at r = 0, 16, 32, 64, 128 with the low-rank overhead
  against r = 0; the AWQ W4A16 modulation layer at M = 1, 2, 8; the three ways
  of taking the activation tensor scale; cuBLASLt's plain NVFP4 GEMM at the
  headline shape and at 8192^3 for context; the on-device weight prep).

The oracle (``oracle/``, CPU) is used only by the ``cpu_baseline`` leg and
by ``--impl reference``.
"""
import os

# BLAS threads of the CPU baseline, set before numpy loads (threadpoolctl
# narrows them to one thread for the one-core time)
_CORES = len(os.sched_getaffinity(0))
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_v, str(_CORES))

import argparse  # noqa: E402
import hashlib  # noqa: E402
import json  # noqa: E402
import statistics  # noqa: E402
import sys  # noqa: E402
import time  # noqa: E402

import numpy as np  # noqa: E402
import torch  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

CASE = workloads.HEADLINE
METRIC = "SVDQ NVFP4 linear TFLOP/s & % dense-FP4 peak (M4096 K3072 N3072 r32)"
UNIT = "TFLOP/s"
WORKLOAD = "attn-proj SVDQ W4A4 NVFP4 linear M4096 K3072 N3072 r32 (quantize + GEMM)"
FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PF)
DATASHEET_FP4_TFLOPS = 9000.0
REPLAYS = 10                # separately timed graph replays per kernel or leg
LAUNCHES = 40               # launches per captured graph


def layer_flops(M, K, N, r):
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def quantize_bytes(M, K, r):
    """Algorithmic HBM bytes of one quantize call: read x, s, L1ᵀ; write
    codes, scales, xl."""
    return M * K * 2 + K * 4 + r * K * 2 + M * K // 2 + M * K // 16 + M * r * 4


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


def fp4_peak(pk):
    """Dense FP4 peak for a kernel timed in isolation: the measured burst
    bf16 GEMM rate (taken at the maximum SM clock) times the nominal FP4/BF16
    ratio 4; the sustained figure (taken under the power cap at a lower
    clock) is reported beside it."""
    burst, sus = pk.get("bf16_tflops"), pk.get("bf16_tflops_sustained")
    if burst:
        return (burst * FP4_PER_BF16, "of measured: burst bf16 GEMM x nominal fp4/bf16 ratio 4",
                pk.get("sm_max_mhz"), None if not sus else sus * FP4_PER_BF16)
    return 1590.0 * FP4_PER_BF16, "of fallback: 1.59 PF bf16 x nominal 4", None, None


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 5 ms
    while it is open (the same counters nvidia-smi reports)."""
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, dev, period=0.005):
        self.dev = dev
        self.period = period
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
                    self.samples.append((time.perf_counter(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                         int(get_reasons(h))))
                except Exception:
                    pass
                self._stop.wait(self.period)
        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)

    def summary(self, t0=None, t1=None):
        sel = [(c, r) for t, c, r in self.samples if (t0 is None or t >= t0) and (t1 is None or t <= t1)]
        sm = [c for c, _ in sel]
        reasons = sorted({n for _, r in sel for n, b in self.REASONS.items() if r & b})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm)}


# ------------------------------------------------------------- timing ----
def gpu_busy_before_start(dev, us=2000):
    """Queue a short spin kernel (torch's, outside the timed region) so that
    the GPU reaches the start event only after the host has queued the timed
    work: a host-side hiccup (this process's clock-sampler thread, the GIL)
    between recording the start event and launching the replay then adds no
    idle GPU time to the measurement."""
    sleep = getattr(torch.cuda, "_sleep", None)
    if sleep is not None:
        with torch.cuda.device(dev):
            sleep(int(us * 2000))  # ~2 GHz SM clock: cycles for `us` microseconds


class GraphTimer:
    """Captures ``n`` launches of a body over rotating operand sets into one
    CUDA graph and times ``replays`` replays separately with events on the
    stream the kernels run on; reports per-launch microseconds."""

    def __init__(self, dev):
        self.dev = dev
        self.stream = torch.cuda.current_stream(dev)
        self.cap = torch.cuda.Stream(dev)

    def capture(self, body, sets, n):
        g = torch.cuda.CUDAGraph()
        self.cap.wait_stream(self.stream)
        with torch.cuda.graph(g, stream=self.cap):
            for i in range(n):
                body(sets[i % len(sets)])
        g.replay()                      # untimed: uploads the graph
        torch.cuda.synchronize(self.dev)
        return g

    def time(self, body, sets, n=LAUNCHES, replays=REPLAYS):
        g = self.capture(body, sets, n)
        us = []
        for _ in range(replays):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            gpu_busy_before_start(self.dev)
            a.record(self.stream)
            g.replay()
            b.record(self.stream)
            b.synchronize()
            us.append(a.elapsed_time(b) * 1e3 / n)
        del g
        return stats(us)


def stats(us):
    return {"us": round(statistics.median(us), 3), "min_us": round(min(us), 3),
            "max_us": round(max(us), 3), "replays": len(us)}


# ------------------------------------------------------- device workload --
def alloc_set(sv, dev, w, x, M, K, N, r, gs):
    return dict(w=w, x=x, gs=gs,
                q=torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
                sf=torch.empty(sv.scale_bytes(M, K), dtype=torch.uint8, device=dev),
                lora=torch.empty(M, r, device=dev) if r else None, gso=torch.empty(1, device=dev),
                y=torch.empty(M, N, dtype=torch.bfloat16, device=dev))


def clone_weights(sv, w):
    return sv.SvdqWeights(q_w=w.q_w.clone(), sf_w=w.sf_w.clone(), gs_w=w.gs_w.clone(),
                          L1t=w.L1t.clone(), L2t=w.L2t.clone(),
                          smooth=None if w.smooth is None else w.smooth.clone(),
                          bias=None if w.bias is None else w.bias.clone())


def set_bytes(sv, M, K, N, r, w):
    return (M * K * 2 + M * K // 2 + sv.scale_bytes(M, K) + M * r * 4 + M * N * 2 +
            w.q_w.numel() + w.sf_w.numel() + w.L1t.numel() * 2 + w.L2t.numel() * 2)


def static_scale(sv, x, w):
    """The activation tensor scale from the data itself (a calibrated static scale)."""
    M, K = x.shape
    gs = torch.empty(1, device=x.device)
    sv.quantize_act(x, w.smooth, w.L1t if w.rank else None, None, out=(
        torch.empty(M, K // 2, dtype=torch.uint8, device=x.device),
        torch.empty(sv.scale_bytes(M, K), dtype=torch.uint8, device=x.device),
        torch.empty(M, w.rank, device=x.device) if w.rank else None, gs))
    return gs


def make_sets(dev, l2_bytes, case=None, w0=None, x0=None, min_sets=2):
    """Independent copies of one layer (weights + activations + outputs),
    prepared on the device by the library's own offline prep, enough of them
    that their total exceeds 3x L2: rotating through them keeps every step's
    operands out of L2."""
    import svdquant_w4a4_gemm_b200 as sv
    from svdquant_w4a4_gemm_b200 import prep as dprep
    case = CASE if case is None else case
    M, K, N, r = case.M, case.K, case.N, case.r
    if w0 is None or x0 is None:
        d = workloads.draw_svdq(case)
        x0 = torch.from_numpy(d["x"]).to(dev).to(torch.bfloat16)
        W0 = torch.from_numpy(d["W"]).to(dev).to(torch.bfloat16)
        b0 = torch.from_numpy(d["bias"]).to(dev).to(torch.bfloat16)
        xc = torch.from_numpy(d["x_cal"]).to(dev).to(torch.bfloat16)
        w0 = dprep.prepare_svdq(W0, b0, xc, r)
    gs = static_scale(sv, x0, w0)
    per = set_bytes(sv, M, K, N, r, w0)
    nsets = max(min_sets, int(np.ceil(3 * l2_bytes / per)))
    sets = [alloc_set(sv, dev, clone_weights(sv, w0), x0.clone(), M, K, N, r, gs.clone())
            for _ in range(nsets)]
    return sets, per


def k1(sv, s):
    w = s["w"]
    sv.quantize_act(s["x"], w.smooth, w.L1t if w.rank else None, s["gs"],
                    out=(s["q"], s["sf"], s["lora"], s["gso"]))


def k2(sv, s, act=None):
    sv.w4a4_linear(s["q"], s["sf"], s["gso"], s["lora"], s["w"], y=s["y"], act=act)


def run_step(sv, s):
    k1(sv, s)
    k2(sv, s)


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
    timer = GraphTimer(dev)
    M, K, N, r = CASE.M, CASE.K, CASE.N, CASE.r

    for i in range(args.warmup):
        run_step(sv, sets[i % nsets])
    sv.check_device_errors()

    # ---- the K timed steps: graphs of up to 200 steps (the device time is
    # then not limited by host launch overhead), exactly K steps in all ----
    chunk = min(args.steps, 200)
    full, rest = divmod(args.steps, chunk)
    step = lambda s: run_step(sv, s)  # noqa: E731
    graph = timer.capture(step, sets, chunk)
    graph_rest = timer.capture(step, sets, rest) if rest else None
    sv.check_device_errors()

    with ClockSampler(dev) as clk:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        w0 = time.perf_counter()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        gpu_busy_before_start(dev)
        t_start.record(stream)
        for _ in range(full):
            graph.replay()
        if graph_rest is not None:
            graph_rest.replay()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        w1 = time.perf_counter()
        if world > 1:
            torch.distributed.barrier()
        sv.check_device_errors()
        total_ms, _ = aggregate(t_start.elapsed_time(t_end), args.steps, layer_flops(M, K, N, r), world, dev)
        del graph, graph_rest

        # ---- each kernel of the step alone, same rotating sets ----
        kern = {"quantize_act_kernel": timer.time(lambda s: k1(sv, s), sets),
                "w4a4_gemm_kernel": timer.time(lambda s: k2(sv, s), sets)}
        sv.check_device_errors()

        # ---- e2e: the same calls with host buffers, copies inside the timed region ----
        # A pipeline, as a serving loop runs it: step i's input goes host ->
        # device on one stream, the layer runs on the compute stream once it
        # has landed, and step i's output goes device -> host on a third
        # stream (two pinned output buffers, alternating), so the copies of
        # neighbouring steps overlap each other and the compute.
        x_host = sets[0]["x"].cpu().pin_memory()
        y_hosts = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        e2e_steps = max(3, min(args.steps, 20))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(nsteps, a=None, b=None):
            if a is not None:
                a.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            done_comp, done_out = [], []
            for i in range(nsteps):
                s = sets[i % nsets]
                with torch.cuda.stream(s_in):
                    if i >= nsets:  # the set's previous step has read its x
                        s_in.wait_event(done_comp[i - nsets])
                    s["x"].copy_(x_host, non_blocking=True)
                stream.wait_stream(s_in)
                if i >= nsets:      # ... and its y has been copied out
                    stream.wait_event(done_out[i - nsets])
                run_step(sv, s)
                done_comp.append(torch.cuda.Event())
                done_comp[-1].record(stream)
                s_out.wait_stream(stream)
                with torch.cuda.stream(s_out):
                    y_hosts[i % 2].copy_(s["y"], non_blocking=True)
                    done_out.append(torch.cuda.Event())
                    done_out[-1].record(s_out)
            stream.wait_stream(s_out)
            if b is not None:
                b.record(stream)

        e2e_run(2)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(e2e_steps, a, b)
        torch.cuda.synchronize(dev)
        # whole-job, like `value`: the slowest rank's time, every rank's steps
        e2e_total_ms, e2e_tflops = aggregate(a.elapsed_time(b), e2e_steps, layer_flops(M, K, N, r), world, dev)

        legs = None
        if world == 1 and not args.no_legs:
            legs = bench_legs(sv, dev, l2, timer, sets, args.only_legs)
        w2 = time.perf_counter()
    clocks = clk.summary()
    clocks["span"] = "whole measurement (timed steps, per-kernel timings, e2e, legs)"
    clocks["timed_region"] = clk.summary(w0, w1)
    clocks["span_s"] = round(w2 - w0, 2)
    return dict(total_ms=total_ms, kernels=kern, clocks=clocks, nsets=nsets, set_mb=per / 2 ** 20,
                e2e_tflops=e2e_tflops, e2e_total_ms=e2e_total_ms, h2d=x_host.numel() * 2,
                d2h=y_hosts[0].numel() * 2, legs=legs)


# ------------------------------------------------------------------- legs --
def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _tf(flops, t):
    return round(flops / t["us"] / 1e6, 1)


def bench_legs(sv, dev, l2, timer, head_sets, only=None):
    """The other workloads; `only`: a comma-separated subset of their names."""
    legs = {}
    pick = set(only.split(",")) if only else None
    hbm = peaks().get("hbm_gbs", 6650.0)
    peak = fp4_peak(peaks())[0]
    for name, fn in (("tiny_layer", lambda: leg_tiny(sv, dev, l2, timer)),
                     ("quantize_scale_variants", lambda: leg_quantize_variants(sv, dev, timer, head_sets, hbm)),
                     ("mlp", lambda: leg_mlp(sv, dev, l2, timer, peak, hbm)),
                     ("qkv_rank_sweep", lambda: leg_qkv(sv, dev, l2, timer, peak)),
                     ("awq_w4a16", lambda: leg_awq(sv, dev, l2, timer, hbm)),
                     ("cublaslt_nvfp4", lambda: leg_cublaslt(sv, dev, timer, head_sets, peak)),
                     ("device_prep", lambda: leg_prep(dev))):
        if pick is not None and name not in pick:
            continue
        try:
            legs[name] = fn()
        except Exception as e:  # noqa: BLE001 - report it on the line, keep the line
            legs[name] = {"error": f"{type(e).__name__}: {str(e)[:300]}"}
        _free()
        sv.check_device_errors()
    return legs


def leg_tiny(sv, dev, l2, timer):
    """Configuration 0 (M256 K512 N512 r32): the whole layer is ~1.3 MB and
    lives in L2, as it would in a model run."""
    c = workloads.TINY
    sets, _ = make_sets(dev, 0, c, min_sets=4)
    t = timer.time(lambda s: run_step(sv, s), sets)
    t["TFLOP/s"] = _tf(layer_flops(c.M, c.K, c.N, c.r), t)
    t["l2"] = "resident (4 sets of 1.3 MB)"
    return t


def leg_quantize_variants(sv, dev, timer, sets, hbm):
    """The headline activation quantized three ways: static gs_a (the step's
    K1), dynamic gs_a by a max pass + K1 + finalize, and dynamic gs_a in one
    cooperative launch."""
    c = CASE
    ws = [torch.zeros(sv.QUANTIZE_WORKSPACE_BYTES, dtype=torch.uint8, device=dev) for _ in sets]
    for i, s in enumerate(sets):
        s["gdyn"] = torch.empty(1, device=dev)
        s["ws"] = ws[i]
    out = {}
    out["static"] = timer.time(lambda s: k1(sv, s), sets)
    out["dynamic_max_pass"] = timer.time(
        lambda s: sv.quantize_act(s["x"], s["w"].smooth, s["w"].L1t, None,
                                  out=(s["q"], s["sf"], s["lora"], s["gdyn"])), sets)
    out["dynamic_single_pass"] = timer.time(
        lambda s: sv.quantize_act_dynamic(s["x"], s["w"].smooth, s["w"].L1t,
                                          out=(s["q"], s["sf"], s["lora"], s["gdyn"]), workspace=s["ws"]), sets)
    nb = quantize_bytes(c.M, c.K, c.r)
    for v in out.values():
        v["GB/s"] = round(nb / v["us"] / 1e3, 1)
        v["frac_hbm"] = round(nb / v["us"] / 1e3 / hbm, 4)
    out["algorithmic_bytes"] = nb
    for s in sets:
        s.pop("gdyn", None)
        s.pop("ws", None)
    return out


def leg_mlp(sv, dev, l2, timer, peak, hbm):
    """Configuration 2: the MLP pair of a DiT block.  Up-projection M4096
    K3072 N12288 (plain and with the fused GELU(tanh) epilogue), then the
    down-projection M4096 K12288 N3072 on the up-projection's GELU output;
    each layer = quantize + GEMM; the pair = both layers back to back."""
    from svdquant_w4a4_gemm_b200 import prep as dprep
    up, dn = workloads.MLP_UP, workloads.MLP_DOWN
    sets, _ = make_sets(dev, l2, up)
    du = workloads.draw_svdq(up)
    # the down-projection's calibration rows: GELU of the up-projection of
    # the up-projection's calibration rows (fp32, on the device)
    xc = torch.from_numpy(du["x_cal"]).to(dev)
    Wu = torch.from_numpy(du["W"]).to(dev)
    bu = torch.from_numpy(du["bias"]).to(dev)
    xcd = torch.nn.functional.gelu(xc @ Wu.T + bu, approximate="tanh").to(torch.bfloat16)
    dd = workloads.draw_svdq(dn, M=1)
    wd = dprep.prepare_svdq(torch.from_numpy(dd["W"]).to(dev).to(torch.bfloat16),
                            torch.from_numpy(dd["bias"]).to(dev).to(torch.bfloat16), xcd, dn.r)
    del xc, Wu, bu
    for s in sets:                     # the up output feeds the down layer
        k1(sv, s)
        k2(sv, s, act="gelu")
    gsd = static_scale(sv, sets[0]["y"], wd)
    dsets = []
    for s in sets:
        ds = alloc_set(sv, dev, clone_weights(sv, wd), s["y"], dn.M, dn.K, dn.N, dn.r, gsd.clone())
        dsets.append(ds)
    fu, fd = layer_flops(up.M, up.K, up.N, up.r), layer_flops(dn.M, dn.K, dn.N, dn.r)
    out = {"up_quantize": timer.time(lambda s: k1(sv, s), sets),
           "up_gemm_plain": timer.time(lambda s: k2(sv, s), sets),
           "up_gemm_gelu": timer.time(lambda s: k2(sv, s, act="gelu"), sets),
           "down_quantize": timer.time(lambda s: k1(sv, s), dsets),
           "down_gemm": timer.time(lambda s: k2(sv, s), dsets)}
    pairs = [(sets[i], dsets[i]) for i in range(len(sets))]

    def pair(p):
        k1(sv, p[0])
        k2(sv, p[0], act="gelu")
        k1(sv, p[1])
        k2(sv, p[1])
    out["pair"] = timer.time(pair, pairs, n=LAUNCHES // 4)
    for k in ("up_gemm_plain", "up_gemm_gelu"):
        out[k]["TFLOP/s"] = _tf(fu, out[k])
        out[k]["frac_fp4_peak"] = round(out[k]["TFLOP/s"] / peak, 4)
    out["down_gemm"]["TFLOP/s"] = _tf(fd, out["down_gemm"])
    out["down_gemm"]["frac_fp4_peak"] = round(out["down_gemm"]["TFLOP/s"] / peak, 4)
    for k, c in (("up_quantize", up), ("down_quantize", dn)):
        nb = quantize_bytes(c.M, c.K, c.r)
        out[k]["GB/s"] = round(nb / out[k]["us"] / 1e3, 1)
        out[k]["frac_hbm"] = round(nb / out[k]["us"] / 1e3 / hbm, 4)
    out["pair"]["TFLOP/s"] = _tf(fu + fd, out["pair"])
    out["pair"]["note"] = "up quantize + up GEMM with GELU + down quantize + down GEMM, per pair"
    out["layers_summed_us"] = round(out["up_quantize"]["us"] + out["up_gemm_gelu"]["us"] +
                                    out["down_quantize"]["us"] + out["down_gemm"]["us"], 3)
    return out


def leg_qkv(sv, dev, l2, timer, peak):
    """Configuration 3: the fused QKV projection M4608 K3072 N9216 (quantize
    + GEMM with Q, K, V stored apart) at r = 0, 16, 32, 64, 128; the
    low-rank overhead is the time over the r = 0 layer of the same shape."""
    from svdquant_w4a4_gemm_b200 import prep as dprep
    base = workloads.QKV[32]
    d = workloads.draw_svdq(base)
    x0 = torch.from_numpy(d["x"]).to(dev).to(torch.bfloat16)
    W0 = torch.from_numpy(d["W"]).to(dev).to(torch.bfloat16)
    b0 = torch.from_numpy(d["bias"]).to(dev).to(torch.bfloat16)
    xc = torch.from_numpy(d["x_cal"]).to(dev).to(torch.bfloat16)
    M, K, N = base.M, base.K, base.N
    out = {}
    for r in (0, 16, 32, 64, 128):
        w = dprep.prepare_svdq(W0, b0, xc, r)
        c = workloads.SvdqCase(f"qkv r{r}", M, K, N, r)
        sets, _ = make_sets(dev, l2, c, w0=w, x0=x0)
        for s in sets:
            s["ys"] = [torch.empty(M, N // 3, dtype=torch.bfloat16, device=dev) for _ in range(3)]

        def split(s):
            sv.w4a4_linear_split(s["q"], s["sf"], s["gso"], s["lora"], s["w"], parts=3, ys=s["ys"])

        def layer(s):
            k1(sv, s)
            split(s)
        e = {"layer": timer.time(layer, sets), "gemm": timer.time(split, sets)}
        fl = layer_flops(M, K, N, r)
        e["layer"]["TFLOP/s"] = _tf(fl, e["layer"])
        e["gemm"]["TFLOP/s"] = _tf(fl, e["gemm"])
        e["gemm"]["frac_fp4_peak"] = round(e["gemm"]["TFLOP/s"] / peak, 4)
        out[f"r{r}"] = e
        del sets, w
        _free()
    t0 = out["r0"]["layer"]["us"]
    out["lowrank_overhead_vs_r0"] = {f"r{r}": round(out[f"r{r}"]["layer"]["us"] / t0 - 1, 4)
                                     for r in (16, 32, 64, 128)}
    return out


def leg_awq(sv, dev, l2, timer, hbm):
    """Configuration 4: the AWQ W4A16 modulation layer (M = 1, 2, 8; K =
    3072, N = 18432), HBM-bound: GB/s of algorithmic bytes, rotating weight
    copies > 3x L2."""
    from svdquant_w4a4_gemm_b200 import prep as dprep
    out = {}
    for Mw, case in workloads.AWQ.items():
        d = workloads.draw_awq(case)
        W = torch.from_numpy(d["W"]).to(dev).to(torch.bfloat16)
        xc = torch.from_numpy(d["x_cal"]).to(dev).to(torch.bfloat16)
        ainv, qw, sc, z = dprep.prepare_awq(W, xc)
        wbytes = qw.numel() * 4 + sc.numel() * 2 + z.numel() * 2
        n = max(2, int(np.ceil(3 * l2 / wbytes)))
        x = torch.from_numpy(d["x"]).to(dev).to(torch.bfloat16)
        b = torch.from_numpy(d["bias"]).to(dev).to(torch.bfloat16)
        copies = [dict(qw=qw.clone(), sc=sc.clone(), z=z.clone(),
                       y=torch.empty(Mw, case.N, dtype=torch.bfloat16, device=dev)) for _ in range(n)]
        t = timer.time(lambda c: sv.awq_w4a16_linear(x, ainv, c["qw"], c["sc"], c["z"], b, y=c["y"]),
                       copies, n=4 * LAUNCHES)
        algo = wbytes + x.numel() * 2 + ainv.numel() * 4 + b.numel() * 2 + Mw * case.N * 2
        t["GB/s"] = round(algo / t["us"] / 1e3, 1)
        t["frac_hbm"] = round(algo / t["us"] / 1e3 / hbm, 4)
        t["algorithmic_bytes"] = int(algo)
        out[f"M{Mw}"] = t
        del copies
        _free()
    return out


def leg_cublaslt(sv, dev, timer, sets, peak):
    """Context, not a target: cuBLASLt's plain NVFP4 GEMM (block scales only;
    no smoothing, low-rank branch or bias) through torch's scaled_mm, on
    the headline operands (same rotating sets as the library's GEMM) and at
    8192^3."""
    F = torch.nn.functional

    def mm(a, sa, b, sb):
        return F.scaled_mm(a.view(torch.float4_e2m1fn_x2), b.view(torch.float4_e2m1fn_x2).t(), sa,
                           F.ScalingType.BlockWise1x16, sb, F.ScalingType.BlockWise1x16,
                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                           output_dtype=torch.bfloat16)

    def sview(buf, rows, K):
        return buf.view(torch.float8_e4m3fn).reshape(-(-rows // 128) * 128, -(-(K // 16) // 4) * 4)

    c = CASE
    for s in sets:
        s["sfa8"] = sview(s["sf"], c.M, c.K)
        s["sfw8"] = sview(s["w"].sf_w, c.N, c.K)
    out = {}
    mm(sets[0]["q"], sets[0]["sfa8"], sets[0]["w"].q_w, sets[0]["sfw8"])   # eager first: a refusal
    torch.cuda.synchronize(dev)                                           # surfaces outside a capture
    t = timer.time(lambda s: mm(s["q"], s["sfa8"], s["w"].q_w, s["sfw8"]), sets)
    t["TFLOP/s"] = _tf(2.0 * c.M * c.N * c.K, t)
    t["frac_fp4_peak"] = round(t["TFLOP/s"] / peak, 4)
    out["M4096_K3072_N3072"] = t
    for s in sets:
        s.pop("sfa8")
        s.pop("sfw8")
    n = 8192
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev, generator=g)
    b = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev, generator=g)
    sa = torch.full((n * n // 16,), 0x38, dtype=torch.uint8, device=dev)   # E4M3 1.0
    big = [dict(a=a, b=b, sa=sview(sa, n, n), sb=sview(sa.clone(), n, n))]
    mm(a, big[0]["sa"], b, big[0]["sb"])
    torch.cuda.synchronize(dev)
    t = timer.time(lambda s: mm(s["a"], s["sa"], s["b"], s["sb"]), big, n=10, replays=5)
    t["TFLOP/s"] = _tf(2.0 * n ** 3, t)
    t["frac_fp4_peak"] = round(t["TFLOP/s"] / peak, 4)
    out["M8192_K8192_N8192"] = t
    return out


def leg_prep(dev):
    """The on-device weight preparation (smoothing, randomized SVD, residual
    NVFP4) of the headline layer, wall time with the device synchronized
    (offline work, not on the hot path)."""
    from svdquant_w4a4_gemm_b200 import prep as dprep
    d = workloads.draw_svdq(CASE)
    W = torch.from_numpy(d["W"]).to(dev).to(torch.bfloat16)
    b = torch.from_numpy(d["bias"]).to(dev).to(torch.bfloat16)
    xc = torch.from_numpy(d["x_cal"]).to(dev).to(torch.bfloat16)
    dprep.prepare_svdq(W, b, xc, CASE.r)
    ms = []
    for _ in range(3):
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        dprep.prepare_svdq(W, b, xc, CASE.r)
        torch.cuda.synchronize(dev)
        ms.append((time.perf_counter() - t0) * 1e3)
    return {"ms": round(statistics.median(ms), 2), "runs": len(ms),
            "what": "prepare_svdq M4096-calibrated K3072 N3072 r32 (smoothing, randomized SVD, residual NVFP4)"}


# ----------------------------------------------------------------- oracle --
_ORACLE_LAYER = {}


def oracle_sample(rows, seed_rows=0):
    """Prepare the oracle's layer (once per process) and return a closure that
    runs the oracle's whole layer on ``rows`` rows of the workload."""
    from oracle import prep as oprep, svdq as osv
    if not _ORACLE_LAYER:
        d = workloads.draw_svdq(CASE)
        L = oprep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], CASE.r)
        _ORACLE_LAYER.update(d=d, L=L, gs=osv.act_tensor_scale(d["x"], L["s"]))
    d, L, gs = _ORACLE_LAYER["d"], _ORACLE_LAYER["L"], _ORACLE_LAYER["gs"]
    xs = d["x"][seed_rows:seed_rows + rows]

    def run():
        return osv.svdq_forward(xs, L, gs)["y"]
    return run


def _time_oracle(run, reps):
    run()  # warm
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    return (time.perf_counter() - t0) / reps


def cpu_baseline(rows=1024, reps=3, rows_1t=128):
    """The oracle as it stands, on the host cores: all cores (BLAS threads =
    the cores this process may use) and one thread."""
    from threadpoolctl import threadpool_limits
    run = oracle_sample(rows)
    with threadpool_limits(limits=_CORES):
        dt = _time_oracle(run, reps)
    run1 = oracle_sample(rows_1t)
    with threadpool_limits(limits=1):
        dt1 = _time_oracle(run1, 1)
    fl = layer_flops(rows, CASE.K, CASE.N, CASE.r)
    fl1 = layer_flops(rows_1t, CASE.K, CASE.N, CASE.r)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": _CORES, "kind": "oracle",
            "blas_threads": _CORES, "one_thread_value": fl1 / dt1 / 1e12,
            "sample": f"{rows} of {CASE.M} rows of the layer (numpy fp64 oracle: quantize, "
                      f"down-projection, dequantized GEMM + low-rank + bias), {reps} reps, "
                      f"{dt:.2f} s per rep on {_CORES} BLAS threads; one thread: {rows_1t} rows, "
                      f"{dt1:.2f} s"}


def run_reference(args, rank, world, budget_s=90.0):
    """The reference arm: the oracle, as it stands, on the host cores (BLAS
    threads = the cores this process may use).  Each step runs the oracle's
    whole layer on a 32-row sample of the workload; the number of timed steps
    is capped so the run ends within ~budget_s (the line reports the steps
    actually timed and the ones requested)."""
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits
    rows = 32
    run = oracle_sample(rows)
    with threadpool_limits(limits=_CORES):
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
                       "group": 16, "parallelism": "replicas" if world > 1 else "single"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": _CORES, "blas_threads": _CORES,
                             "kind": "oracle",
                             "sample": f"{rows} of {CASE.M} rows per step (numpy fp64 oracle: "
                                       f"quantize, down-projection, dequantized GEMM + low-rank + bias), "
                                       f"BLAS threads = {_CORES} host cores"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- main --
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-legs", action="store_true", help="skip the other workloads")
    ap.add_argument("--legs", action="store_true", help=argparse.SUPPRESS)  # legs are the default
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only-legs", default=None,
                    help="comma-separated subset of the other workloads (tiny_layer, quantize_scale_variants, "
                         "mlp, qkv_rank_sweep, awq_w4a16, cublaslt_nvfp4, device_prep)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    args.steps = max(1, args.steps)

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
    steps = args.steps
    ms = res["total_ms"] / steps
    value = fl * steps * world / (res["total_ms"] * 1e-3) / 1e12
    pk = peaks()
    peak, peak_src, peak_mhz, peak_sus = fp4_peak(pk)
    kg, kq = res["kernels"]["w4a4_gemm_kernel"], res["kernels"]["quantize_act_kernel"]
    achieved = fl / (kg["us"] * 1e-6) / 1e12
    kq_bytes = quantize_bytes(M, K, r)
    hbm = pk.get("hbm_gbs", 6650.0)
    kq.update({"GB/s": round(kq_bytes / kq["us"] / 1e3, 1), "frac_hbm": round(kq_bytes / kq["us"] / 1e3 / hbm, 4),
               "hbm_peak_gbs": hbm, "algorithmic_bytes": kq_bytes,
               "traffic": kernel_traffic("quantize.cu", "quantize_act_kernel")})
    kg.update({"TFLOP/s": round(achieved, 1), "frac_fp4_peak": round(achieved / peak, 4)})
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
                     "peak_source": peak_src, "peak_sm_mhz": peak_mhz,
                     "frac_of_sustained_peak": None if not peak_sus else round(achieved / peak_sus, 4),
                     "frac_of_datasheet_9PF": round(achieved / DATASHEET_FP4_TFLOPS, 4),
                     "traffic": kernel_traffic("gemm.cu", "w4a4_gemm_kernel"),
                     "algorithmic_flops_per_launch": fl, "avg_launch_us": kg["us"],
                     "launch_us_range": [kg["min_us"], kg["max_us"]], "replays": kg["replays"]},
        "kernels": res["kernels"],
        "clocks": res["clocks"],
        "timed_region_ms": round(res["total_ms"], 3),
        "e2e": {"value": res["e2e_tflops"], "unit": UNIT,
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
        # per step: the xl clear kernel (r > 0), the quantize kernel, the GEMM
        "gpu_launches": (3 if CASE.r > 0 else 2) * steps,
        "cpu_baseline": cpu,
    }
    if res["legs"]:
        line["legs"] = res["legs"]
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
