"""Benchmark of the W8A8 activation-quantized linear on B200.

Headline: W8A8 per-channel linear, M=4096 tokens, N=10240, K=2560 (the
Cider pages' single-op table shape), fp16 in / fp16 out.  One step = one full
call of ``cider_w8a8_linear_pc`` (per-token quantize + tcgen05 GEMM + fused
dequant).  Reported as TOPS = 2*M*N*K / time.  Inputs: seeded synthetic
activations (N(0,1), 1% of input channels x50) and N(0, 0.02) weights
quantized per output channel on the GPU; enough input sets rotate between
steps that their total exceeds 3x the L2 cache.

The K timed steps are captured once into a CUDA graph and replayed inside
the timed region, so the device time is not inflated by Python launch
overhead; the W warm-up steps run eagerly before capture.  `e2e` times the
same call through the public API, called eagerly from Python, with pinned
host buffers: each step copies x host->device, runs the linear and copies y
device->host.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cider|reference] [--no-rows]

N>1 runs under torch.distributed.run: every rank runs an independent replica
of the same per-GPU workload (the linear has no cross-GPU exchange); the
time is the max over ranks.  --impl reference times the CPU oracle (plain C)
on this host's cores on a bounded sample of the same workload (rank 0 only).
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

import numpy as np  # noqa: E402,F401
import torch  # noqa: E402

METRIC = "W8A8 linear TOPS & % INT8 tensor peak (M=4096,N=10240,K=2560); ms/op"
UNIT = "TOPS"
M0, N0, K0 = 4096, 10240, 2560
SEED0 = 1000 + M0
L2_BYTES = 126 * 1024 * 1024
# dense INT8 tensor peak = a measured bf16 GEMM peak x the nominal int8/bf16 ratio (4.5 / 2.25)
INT8_PER_BF16 = 2.0


def gemm_traffic():
    """DRAM bytes per launch of the headline GEMM from the committed ncu capture,
    or None when the kernel's sources changed since that capture."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
            rec = json.load(f)
        m = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                m.update(f.read())
        return rec["traffic_bytes_per_launch"] if m.hexdigest() == rec["source_sha256"] else None
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons while the timed region runs
    (NVML; nvidia-smi polling if NVML is unavailable).  Reads only."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index, period_s=0.002):
        self.dev = device_index
        self.period = period_s
        self.samples = []  # (sm_mhz, reasons_mask): background samples
        self.polled = []   # samples taken by poll_until, while the timed work runs
        self.max_mhz = None
        self._stop = threading.Event()
        self._nvml = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        try:
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
        return pynvml, h

    def _loop_nvml(self, pynvml, h):
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        while not self._stop.is_set():
            clk = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            try:
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            except AttributeError:
                rs = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
            self.samples.append((float(clk), int(rs)))
            time.sleep(self.period)

    def _loop_smi(self):
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        bits = [0x8, 0x40, 0x20, 0x4]
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={q}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip().split(",")
                mask = sum(b for b, v in zip(bits, out[2:6]) if v.strip().lower().startswith("active"))
                self.samples.append((float(out[0]), mask))
                self.max_mhz = float(out[1])
            except Exception:
                pass
            time.sleep(0.05)

    def __enter__(self):
        try:
            pynvml, h = self._handle()
            self._nvml = (pynvml, h)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self._t = threading.Thread(target=self._loop_nvml, args=(pynvml, h), daemon=True)
        except Exception:
            self._t = threading.Thread(target=self._loop_smi, daemon=True)
        self._t.start()
        time.sleep(0.01)
        return self

    def _sample_nvml(self):
        pynvml, h = self._nvml
        clk = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        try:
            rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        except AttributeError:
            rs = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        self.polled.append((float(clk), int(rs)))

    def poll_until(self, event):
        """Samples from this thread while queued GPU work runs, until `event`
        completes: a timed region shorter than the background period still
        gets samples taken under load (at least one, before the first check)."""
        if self._nvml is None:
            return
        while True:
            self._sample_nvml()
            if event.query():
                return

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        # samples taken while the timed work ran, when there are any
        samples = self.polled or self.samples
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mask = 0
        for _, m in samples:
            mask |= m
        return {"sm_mhz": statistics.median(c for c, _ in samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for n, b in self.REASONS.items() if mask & b),
                "samples": len(samples)}


# ----------------------------------------------------------------------------- timing

def _dist():
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(v, ws, device):
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def capture(fn, steps, warmup):
    """Run `warmup` eager calls, then capture `steps` calls into a CUDA graph.
    fn(i) must enqueue on torch's current stream."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for i in range(warmup):
            fn(i)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            fn(i)
    torch.cuda.synchronize()
    return g


def replay_ms(g, steps, reps=1):
    """Device time per step of a captured graph of `steps` calls (CUDA events)."""
    g.replay()  # untimed warm replay
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(reps):
        g.replay()
    b.record(st)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / (steps * reps)


def graph_time(fn, steps, warmup):
    g = capture(fn, steps, warmup)
    ms = replay_ms(g, steps)
    del g
    return ms


def rotating(n_bytes_per_set):
    return max(2, -(-3 * L2_BYTES // max(1, n_bytes_per_set)))


# ----------------------------------------------------------------------------- CPU oracle

def cpu_baseline(M, N, K, seed, min_s=10.0):
    """The oracle (plain C, OpenMP over token rows) on the full headline workload,
    repeated until about `min_s` seconds of CPU work."""
    import oracle
    from w8a8_activation_quantized_b200 import synth
    x = synth.activations(M, K, seed)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed))
    runs, total = 0, 0.0
    while total < min_s and runs < 50:
        t0 = time.perf_counter()
        oracle.linear_pc(x, qw, sw)
        total += time.perf_counter() - t0
        runs += 1
    tops = 2.0 * M * N * K * runs / total / 1e12
    return {"value": tops, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"the full M={M} N={N} K={K} per-channel linear, {runs} run(s), {total:.1f} s"}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle
    from w8a8_activation_quantized_b200 import synth
    threads = oracle.num_threads()
    rows = max(16, 2 * threads)  # a bounded sample of token rows per step
    x = synth.activations(M0, K0, SEED0)[:rows]
    qw, sw = oracle.quantize_weight_pc(synth.weights(N0, K0, SEED0))
    for _ in range(args.warmup):
        oracle.linear_pc(x, qw, sw)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear_pc(x, qw, sw)
    dt = (time.perf_counter() - t0) / args.steps
    tops = 2.0 * rows * N0 * K0 / dt / 1e12
    print(json.dumps({
        "metric": METRIC, "value": tops, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"w8a8_linear_pc M={M0} N={N0} K={K0}, CPU oracle on {rows} sampled token rows per step"},
        "cpu_baseline": {"value": tops, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of the {M0} token rows per step (rows are independent)"},
        "e2e": {"value": tops, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def run_cider(args):
    import w8a8_activation_quantized_b200 as cider
    from w8a8_activation_quantized_b200 import synth
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    if not cider.cider_is_available():
        raise RuntimeError("device is not sm_100-family")
    pk = peaks()
    int8_peak = pk["bf16"] * INT8_PER_BF16
    M, N, K = M0, N0, K0
    ops = 2.0 * M * N * K

    x0 = torch.from_numpy(synth.activations(M, K, SEED0)).to(device)
    w0, sw0 = cider.cider_quantize_weight_pc(torch.from_numpy(synth.weights(N, K, SEED0)).to(device))
    set_bytes = x0.numel() * 2 + w0.numel() + M * N * 2 + M * K
    n_sets = rotating(set_bytes)
    sets = [(x0, w0, sw0)] + [(x0.roll(i, 0).contiguous(), w0.roll(i, 0).contiguous(), sw0.roll(i, 0).contiguous())
                              for i in range(1, n_sets)]
    ys = [torch.empty((M, N), dtype=torch.float16, device=device) for _ in range(n_sets)]
    wsb = cider.cider_workspace_bytes_mnk(M, N, K)
    wss = [torch.empty((wsb,), dtype=torch.uint8, device=device) for _ in range(n_sets)]

    def step(i):
        x, w, sw = sets[i % n_sets]
        cider.cider_w8a8_linear_pc(x, w, sw, y=ys[i % n_sets], workspace=wss[i % n_sets])

    g = capture(step, args.steps, args.warmup)
    g.replay()
    torch.cuda.synchronize()
    _barrier(ws)
    st = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        a.record(st)
        g.replay()
        b.record(st)
        clk.poll_until(b)
        torch.cuda.synchronize()
    _barrier(ws)
    ms = _max_over_ranks(a.elapsed_time(b) / args.steps, ws, device)
    del g
    value = ws * ops / (ms * 1e-3) / 1e12

    # the dominant kernel alone (tcgen05 GEMM on pre-quantized activations), and the quantize kernel
    qs = [cider.cider_quantize_act(s[0]) for s in sets]
    ms_gemm = graph_time(lambda i: cider.cider_w8a8_gemm_pc_q(qs[i % n_sets][0], qs[i % n_sets][1], sets[i % n_sets][1],
                                                               sets[i % n_sets][2], y=ys[i % n_sets]),
                         args.steps, args.warmup)
    ms_quant = graph_time(lambda i: cider.cider_quantize_act(sets[i % n_sets][0], q=qs[i % n_sets][0],
                                                             scale_x=qs[i % n_sets][1]), args.steps, args.warmup)
    achieved = ops / (ms_gemm * 1e-3) / 1e12

    # end to end through the public API, host buffers, copies inside the timed region.
    # A step is pipelined in row chunks over three streams -- copy in, compute
    # (the public linear on the chunk's rows), copy out -- so the two PCIe
    # directions and the kernels overlap; device rows are double-buffered by
    # step parity and per-chunk events order every reuse.
    n_chunks = 8
    mc = M // n_chunks
    xh = x0.cpu().pin_memory()
    yh = torch.empty((M, N), dtype=torch.float16).pin_memory()
    xd = [torch.empty_like(x0) for _ in range(2)]
    yd = [torch.empty((M, N), dtype=torch.float16, device=device) for _ in range(2)]
    wsc = torch.empty((max(1, cider.cider_workspace_bytes_mnk(mc, N, K)),), dtype=torch.uint8, device=device)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [[torch.cuda.Event() for _ in range(n_chunks)] for _ in range(2)] for k in ("in", "comp", "out")}
    for k in ev:  # recorded once, so the first waits on them pass
        for e in ev[k][0] + ev[k][1]:
            e.record(st)

    def e2e(i):
        p = i % 2
        for j in range(n_chunks):
            rows = slice(j * mc, (j + 1) * mc)
            s_in.wait_event(ev["comp"][p][j])  # the compute that last read these input rows
            with torch.cuda.stream(s_in):
                xd[p][rows].copy_(xh[rows], non_blocking=True)
                ev["in"][p][j].record(s_in)
            st.wait_event(ev["in"][p][j])
            st.wait_event(ev["out"][p][j])  # the copy-out that last read these output rows
            cider.cider_w8a8_linear_pc(xd[p][rows], w0, sw0, y=yd[p][rows], workspace=wsc, stream=st)
            ev["comp"][p][j].record(st)
            s_out.wait_event(ev["comp"][p][j])
            with torch.cuda.stream(s_out):
                yh[rows].copy_(yd[p][rows], non_blocking=True)
                ev["out"][p][j].record(s_out)

    # eager calls: the host-side cost of the public API is part of end to end
    e2e_steps = max(5, min(args.steps, 50))
    for i in range(args.warmup):
        e2e(i)
    torch.cuda.synchronize()
    a.record(st)
    for i in range(e2e_steps):
        e2e(i)
    st.wait_stream(s_out)
    b.record(st)
    torch.cuda.synchronize()
    ms_e2e = a.elapsed_time(b) / e2e_steps
    e2e_tops = ws * ops / (ms_e2e * 1e-3) / 1e12

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": f"w8a8_linear_pc M={M} N={N} K={K} fp16 in/out (quantize + tcgen05 GEMM + dequant)",
                   "inputs": "x fp16 N(0,1) with 1% of channels x50; w N(0,0.02) -> int8 per channel",
                   "parallelism": f"{ws} independent replicas" if ws > 1 else "single GPU",
                   "l2": f"inputs larger than L2: {n_sets} rotating sets, {n_sets * set_bytes / 2**20:.0f} MiB",
                   "launch": "K steps in one CUDA graph, replayed once in the timed region"},
        "pct_int8_peak": 100.0 * (value / ws) / int8_peak,
        "breakdown_ms": {"quantize_act": ms_quant, "gemm_pc": ms_gemm},
        "roofline": {"bound": "tensor", "kernel": "k_gemm_pair (tcgen05.mma.cta_group::2 kind::i8)",
                     "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s", "frac": achieved / int8_peak,
                     "traffic": gemm_traffic(), "algorithmic_bytes": M * K + N * K + M * N * 2 + 4 * (M + N),
                     "peak_note": f"INT8 = {INT8_PER_BF16:g} x {pk['src']} bf16 burst {pk['bf16']:.1f} TFLOP/s"},
        "e2e": {"value": e2e_tops, "unit": UNIT, "ms_per_step": ms_e2e,
                "h2d_bytes_per_step": x0.numel() * 2, "d2h_bytes_per_step": M * N * 2,
                "pipeline": f"{n_chunks} row chunks, copy-in / compute / copy-out streams"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    rows = []
    if not args.no_rows:
        try:
            rows = bench_rows(device, pk, steps=min(args.steps, 100), warmup=args.warmup)
        except Exception as e:  # a failing extra row must not cost the headline line
            line["rows_error"] = f"{type(e).__name__}: {e}"
    cider.cider_device_status()
    if rank == 0 and ws == 1:
        line["cpu_baseline"] = None if args.no_cpu_baseline else cpu_baseline(M, N, K, SEED0)
    if rank == 0:
        # every row in full, then a compact summary, then the headline last
        for r in rows:
            print(json.dumps({"bench_row": r}), flush=True)
        if rows:
            print(json.dumps({"rows_summary_us_frac": rows_summary(rows)}), flush=True)
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def row_key(r):
    """Short name of a bench row: kind, parameters and shape."""
    n = r["row"]
    if n == "w8a8_linear_pc":
        return f"pc M{r['M']}"
    if n == "w8a8_linear_pg":
        return f"pg{r['gs']} M{r['M']}"
    if n == "w4a8_linear_pg":
        return f"w4pg{r['gs']} M{r['M']}"
    if n == "w4a8_linear_pc":
        return f"w4pc M{r['M']}"
    if n in ("w8a16_mv_pc", "w8a16_mv_pg"):
        return n.replace("w8a16_", "") + (f"{r['gs']}" if r.get("gs") else "") + f" M{r['M']}"
    if n == "quantize_act":
        return f"quant {r['M']}x{r['K']}"
    if n == "sdpa_decode":
        return f"sdpa {r['H_q']}/{r['H_kv']} N{r['N']}"
    if n == "decoder_linear_stack":
        return "stack8b"
    return n + (f" M{r['M']}" if "M" in r else "")


def rows_summary(rows):
    """{short name: [microseconds per call, fraction of the row's roofline]}."""
    return {row_key(r): [round(r["ms"] * 1e3, 2), round(r["frac"], 3)] for r in rows}


def bench_rows(device, pk, steps, warmup):
    """Every hot-path row at the pages' shapes: device time per call and its roofline."""
    import w8a8_activation_quantized_b200 as cider
    from w8a8_activation_quantized_b200 import synth
    hbm, int8_peak = pk["hbm"], pk["bf16"] * INT8_PER_BF16
    ridge = int8_peak * 1e12 / (hbm * 1e9)  # ops per byte
    out = []

    def record(row, ms, ops, mbytes, **kw):
        tops = ops / (ms * 1e-3) / 1e12 if ops else None
        gbs = mbytes / (ms * 1e-3) / 1e9
        bound = "hbm" if (not ops or ops / mbytes < ridge) else "tensor"
        out.append(dict(row=row, ms=ms, TOPS=tops, **{"GB/s": gbs}, bound=bound,
                        frac=(gbs / hbm) if bound == "hbm" else tops / int8_peak, **kw))

    # per-channel, N=10240 K=2560, the M sweep of the pages' table
    N, K = 10240, 2560
    w8, s8 = cider.cider_quantize_weight_pc(torch.from_numpy(synth.weights(N, K, 1001)).to(device))
    for M in (1, 128, 1024, 4096, 8192):
        x = torch.from_numpy(synth.activations(M, K, 1000 + M)).to(device)
        n = rotating(N * K + M * K * 3 + M * N * 2)
        ws_ = [w8] + [w8.roll(i, 0).contiguous() for i in range(1, n)]
        ys = [torch.empty((M, N), dtype=torch.float16, device=device) for _ in range(n)]
        wsp = torch.empty((max(1, cider.cider_workspace_bytes_mnk(M, N, K)),), dtype=torch.uint8, device=device)
        ms = graph_time(lambda i: cider.cider_w8a8_linear_pc(x, ws_[i % n], s8, y=ys[i % n], workspace=wsp),
                        steps, warmup)
        record("w8a8_linear_pc", ms, 2.0 * M * N * K, N * K + N * 4 + M * K * 2 + M * N * 2, M=M, N=N, K=K,
               path="small-M fused kernel" if cider.cider_workspace_bytes(M, K) == 0 else "quantize + tcgen05 GEMM")
        del ws_, ys
    # W8A16 decode product (no activation quantization), M=1, N=10240 K=2560
    x1 = torch.from_numpy(synth.activations(1, K, 1001)).to(device)
    n = rotating(N * K)
    ws_ = [w8] + [w8.roll(i, 0).contiguous() for i in range(1, n)]
    y1 = torch.empty((1, N), dtype=torch.float16, device=device)
    ms = graph_time(lambda i: cider.cider_w8a16_mv_pc(x1, ws_[i % n], s8, y=y1), steps, warmup)
    record("w8a16_mv_pc", ms, 2.0 * N * K, N * K + N * 4 + K * 2 + N * 2, M=1, N=N, K=K,
           path="W8A16 decode kernel (no activation quantization)")
    del ws_
    del w8
    # per-group, N=2560 K=10240, gs 128 and 64
    N, K = 2560, 10240
    W = torch.from_numpy(synth.weights(N, K, 2001)).to(device)
    for gs in (128, 64):
        wg, sg = cider.cider_quantize_weight_pg(W, gs)
        for M in (1, 128, 1024, 4096, 8192):
            x = torch.from_numpy(synth.activations(M, K, 2000 + M)).to(device)
            n = rotating(N * K + M * K * 3 + M * N * 2)
            wgs = [wg] + [wg.roll(i, 0).contiguous() for i in range(1, n)]
            ys = [torch.empty((M, N), dtype=torch.float16, device=device) for _ in range(n)]
            wsp = torch.empty((max(1, cider.cider_workspace_bytes_mnk(M, N, K)),), dtype=torch.uint8, device=device)
            ms = graph_time(lambda i: cider.cider_w8a8_linear_pg(x, wgs[i % n], sg, gs, y=ys[i % n], workspace=wsp),
                            steps, warmup)
            record("w8a8_linear_pg", ms, 2.0 * M * N * K, N * K + sg.numel() * 4 + M * K * 2 + M * N * 2,
                   gs=gs, M=M, N=N, K=K)
            del wgs, ys
        # W8A16 decode product with per-group scales (no activation quantization), M=1
        x1 = torch.from_numpy(synth.activations(1, K, 2001)).to(device)
        n = rotating(N * K)
        wgs = [wg] + [wg.roll(i, 0).contiguous() for i in range(1, n)]
        y1 = torch.empty((1, N), dtype=torch.float16, device=device)
        ms = graph_time(lambda i: cider.cider_w8a16_mv_pg(x1, wgs[i % n], sg, gs, y=y1), steps, warmup)
        record("w8a16_mv_pg", ms, 2.0 * N * K, N * K + sg.numel() * 4 + K * 2 + N * 2, gs=gs, M=1, N=N, K=K,
               path="W8A16 per-group decode kernel (no activation quantization)")
        del wgs, wg, sg
    del W
    # W4A8, N=12288 K=4096 M=2048 gs=64
    M, N, K, gs = 2048, 12288, 4096, 64
    p4, s4 = cider.cider_pack_weight_int4_pg(torch.from_numpy(synth.weights(N, K, 3001)).to(device), gs)
    x = torch.from_numpy(synth.activations(M, K, 3000 + M)).to(device)
    n = rotating(N * K // 2 + M * K * 3 + M * N * 2)
    p4s = [p4] + [p4.roll(i, 0).contiguous() for i in range(1, n)]
    ys = [torch.empty((M, N), dtype=torch.float16, device=device) for _ in range(n)]
    wsp = torch.empty((cider.cider_workspace_bytes_mnk(M, N, K),), dtype=torch.uint8, device=device)
    ms = graph_time(lambda i: cider.cider_w4a8_linear_pg(x, p4s[i % n], s4, gs, y=ys[i % n], workspace=wsp), steps, warmup)
    record("w4a8_linear_pg", ms, 2.0 * M * N * K, N * K // 2 + s4.numel() * 4 + M * K * 2 + M * N * 2, gs=gs, M=M, N=N, K=K)
    del p4s
    # W4A8 with one scale per output channel, same shape
    p4, s4 = cider.cider_pack_weight_int4_pc(torch.from_numpy(synth.weights(N, K, 3001)).to(device))
    p4s = [p4] + [p4.roll(i, 0).contiguous() for i in range(1, n)]
    ms = graph_time(lambda i: cider.cider_w4a8_linear_pc(x, p4s[i % n], s4, y=ys[i % n], workspace=wsp), steps, warmup)
    record("w4a8_linear_pc", ms, 2.0 * M * N * K, N * K // 2 + N * 4 + M * K * 2 + M * N * 2, M=M, N=N, K=K)
    del p4s, ys
    # memory-bound producers
    for (M, K) in ((4096, 2560), (8192, 10240)):
        n = rotating(M * K * 3)
        xs = [torch.from_numpy(synth.activations(M, K, 7 + i)).to(device) for i in range(min(n, 4))]
        qb = [torch.empty((M, K), dtype=torch.int8, device=device) for _ in range(len(xs))]
        sb = torch.empty((M,), dtype=torch.float32, device=device)
        ms = graph_time(lambda i: cider.cider_quantize_act(xs[i % len(xs)], q=qb[i % len(xs)], scale_x=sb), steps, warmup)
        record("quantize_act", ms, 0, M * K * 3 + M * 4, M=M, K=K)
    M, F = 2048, 12288
    gts = [torch.from_numpy(synth.activations(M, F, 8 + i)).to(device) for i in range(3)]
    uts = [torch.from_numpy(synth.activations(M, F, 18 + i)).to(device) for i in range(3)]
    qb = [torch.empty((M, F), dtype=torch.int8, device=device) for _ in range(3)]
    sb = torch.empty((M,), dtype=torch.float32, device=device)
    ms = graph_time(lambda i: cider.cider_silu_mul_quantize(gts[i % 3], uts[i % 3], q=qb[i % 3], scale_x=sb), steps, warmup)
    record("silu_mul_quantize", ms, 0, M * F * 5 + M * 4, M=M, F=F)
    del gts, uts, qb
    # offline conversion with percentile-clipped scales (clip_percentile = 99.9)
    for (N, K, gs) in ((10240, 2560, 0), (2560, 10240, 64)):
        n = rotating(N * K * 5)
        Ws = [torch.from_numpy(synth.weights(N, K, 4000 + i)).to(device) for i in range(n)]
        if gs == 0:
            ms = graph_time(lambda i: cider.cider_quantize_weight_pc_clip(Ws[i % n], 99.9), steps, warmup)
            record("quantize_weight_pc_clip", ms, 0, N * K * 5 + N * 4, N=N, K=K, clip_percentile=99.9)
        else:
            ms = graph_time(lambda i: cider.cider_quantize_weight_pg_clip(Ws[i % n], gs, 99.9), steps, warmup)
            record("quantize_weight_pg_clip", ms, 0, N * K * 5 + N * (K // gs) * 4, gs=gs, N=N, K=K,
                   clip_percentile=99.9)
        del Ws
    # decode attention, the pages' SDPA table configurations (D = 128, fp16)
    for (H_kv, N) in ((32, 4096), (8, 4096), (4, 4096), (32, 32768), (8, 32768), (4, 32768)):
        H_q, D = 32, 128
        kv_bytes = 2 * H_kv * N * D * 2
        n = rotating(kv_bytes)
        g = torch.Generator(device=device)
        g.manual_seed(5000 + H_kv + N)
        qs = torch.randn((H_q, D), generator=g, device=device).half()
        ks = [torch.randn((H_kv, N, D), generator=g, device=device).half() for _ in range(n)]
        vs = [torch.randn((H_kv, N, D), generator=g, device=device).half() for _ in range(n)]
        os_ = torch.empty((H_q, D), dtype=torch.float16, device=device)
        wsd = torch.empty((max(16, cider.cider_sdpa_decode_workspace_bytes(H_q, H_kv, N, D)),), dtype=torch.uint8,
                          device=device)
        ms = graph_time(lambda i: cider.cider_sdpa_decode(qs, ks[i % n], vs[i % n], out=os_, workspace=wsd),
                        steps, warmup)
        record("sdpa_decode", ms, 0, kv_bytes + 2 * H_q * D * 2, H_q=H_q, H_kv=H_kv, N=N, D=D)
        del ks, vs
    out.append(bench_stack(device, pk, steps=max(3, steps // 20), warmup=warmup))
    return out


def bench_stack(device, pk, steps, warmup, layers=36, M=2048):
    """The linear stack of an 8B-class decoder: `layers` layers x 7 W8A8
    per-channel linears with SiLU(gate)*up fused into down_proj's quantize."""
    from w8a8_activation_quantized_b200 import stack, synth
    int8_peak = pk["bf16"] * INT8_PER_BF16
    stk = stack.DecoderLinearStack(layers, device=device)
    H = torch.from_numpy(synth.activations(M, stack.HIDDEN, seed=4000 + M, outlier_frac=0.005,
                                           outlier_scale=100.0)).to(device)
    ms = graph_time(lambda i: stk.forward(H), steps, warmup)
    ops = layers * stack.ops_per_layer(M)
    wbytes = layers * sum(n * k for _, n, k in stack.LINEARS)
    tops = ops / (ms * 1e-3) / 1e12
    del stk
    return dict(row="decoder_linear_stack", layers=layers, M=M, ms=ms, TOPS=tops,
                **{"GB/s": wbytes / (ms * 1e-3) / 1e9}, bound="tensor", frac=tops / int8_peak,
                launches_per_step=layers * 11, weight_bytes=wbytes)


ROW_CASES = {
    # name: (kind, M, N, K, gs)
    "pc_m1": ("pc", 1, 10240, 2560, 0), "pc_m128": ("pc", 128, 10240, 2560, 0),
    "pc_m512": ("pc", 512, 10240, 2560, 0), "pc_m1024": ("pc", 1024, 10240, 2560, 0),
    "pc_m2048": ("pc", 2048, 10240, 2560, 0), "pc_m4096": ("pc", 4096, 10240, 2560, 0),
    "pc_m8192": ("pc", 8192, 10240, 2560, 0),
    "pg128_m1": ("pg", 1, 2560, 10240, 128), "pg128_m4096": ("pg", 4096, 2560, 10240, 128),
    "mv_m1": ("mv", 1, 10240, 2560, 0), "mvpg64_m1": ("mvpg", 1, 2560, 10240, 64),
    "mvpg128_m1": ("mvpg", 1, 2560, 10240, 128),
    "pg64_m1": ("pg", 1, 2560, 10240, 64), "pg64_m4096": ("pg", 4096, 2560, 10240, 64),
    "pg128_m128": ("pg", 128, 2560, 10240, 128), "pg64_m128": ("pg", 128, 2560, 10240, 64),
    "pg64_m1024": ("pg", 1024, 2560, 10240, 64), 
    "w4a8_m2048": ("w4", 2048, 12288, 4096, 64), "w4a8pc_m2048": ("w4pc", 2048, 12288, 4096, 0),
    "stack_8b": ("stack", 2048, 0, 0, 0),
    "quant_m4096_k2560": ("quant", 4096, 0, 2560, 0), "quant_m8192_k10240": ("quant", 8192, 0, 10240, 0),
    # offline conversion with percentile-clipped scales (p = 99.9): (kind, 0, N, K, gs)
    "clip_pc": ("clip", 0, 10240, 2560, 0), "clip_pg64": ("clip", 0, 2560, 10240, 64),
    # decode attention: (kind, H_kv, N keys, 0, 0) with H_q = 32, D = 128
    "sdpa_mha_n32k": ("sdpa", 32, 32768, 0, 0), "sdpa_gqa4_n32k": ("sdpa", 8, 32768, 0, 0),
    "sdpa_gqa8_n32k": ("sdpa", 4, 32768, 0, 0), "sdpa_gqa8_n4k": ("sdpa", 4, 4096, 0, 0),
}


def run_row(args):
    """One hot-path row alone (for profiling): device time per call, one JSON line."""
    import w8a8_activation_quantized_b200 as cider
    from w8a8_activation_quantized_b200 import synth
    if args.row == "stack_8b":
        torch.cuda.set_device(0)
        print(json.dumps(bench_stack(torch.device("cuda", 0), peaks(), args.steps, args.warmup)), flush=True)
        return 0
    kind, M, N, K, gs = ROW_CASES[args.row]
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    cider.cider_test_set_fused_quantize({"auto": 0, "off": 1, "on": 2}[args.fused])
    if kind == "sdpa":  # decode attention alone, K/V rotated beyond L2
        cider.cider_test_set_sdpa_kernel(args.sdpa_kernel)
        H_q, H_kv, Nk, D = 32, M, N, 128
        kv_bytes = 2 * H_kv * Nk * D * 2
        n = rotating(kv_bytes)
        g = torch.Generator(device=device)
        g.manual_seed(5000 + H_kv + Nk)
        q = torch.randn((H_q, D), generator=g, device=device).half()
        ks = [torch.randn((H_kv, Nk, D), generator=g, device=device).half() for _ in range(n)]
        vs = [torch.randn((H_kv, Nk, D), generator=g, device=device).half() for _ in range(n)]
        out = torch.empty((H_q, D), dtype=torch.float16, device=device)
        wsd = torch.empty((max(16, cider.cider_sdpa_decode_workspace_bytes(H_q, H_kv, Nk, D)),), dtype=torch.uint8,
                          device=device)
        ms = graph_time(lambda i: cider.cider_sdpa_decode(q, ks[i % n], vs[i % n], out=out, workspace=wsd),
                        args.steps, args.warmup)
        cider.cider_device_status()
        print(json.dumps({"row": args.row, "kind": kind, "H_q": H_q, "H_kv": H_kv, "N": Nk, "ms": ms,
                          "GB/s": (kv_bytes + 2 * H_q * D * 2) / (ms * 1e-3) / 1e9}), flush=True)
        return 0
    if kind == "clip":  # percentile-clipped weight quantizer alone, weights rotated beyond L2
        n = rotating(N * K * 5)
        Ws = [torch.from_numpy(synth.weights(N, K, 4000 + i)).to(device) for i in range(n)]
        if gs == 0:
            ms = graph_time(lambda i: cider.cider_quantize_weight_pc_clip(Ws[i % n], 99.9), args.steps, args.warmup)
        else:
            ms = graph_time(lambda i: cider.cider_quantize_weight_pg_clip(Ws[i % n], gs, 99.9), args.steps,
                            args.warmup)
        cider.cider_device_status()
        nbytes = N * K * 5 + N * (K // gs if gs else 1) * 4
        print(json.dumps({"row": args.row, "kind": kind, "N": N, "K": K, "gs": gs, "ms": ms,
                          "GB/s": nbytes / (ms * 1e-3) / 1e9}), flush=True)
        return 0
    if kind == "quant":  # activation quantization alone, inputs rotated beyond L2
        n = rotating(M * K * 3)
        xs = [torch.from_numpy(synth.activations(M, K, 7 + i)).to(device) for i in range(min(n, 4))]
        qb = [torch.empty((M, K), dtype=torch.int8, device=device) for _ in range(len(xs))]
        sb = torch.empty((M,), dtype=torch.float32, device=device)
        ms = graph_time(lambda i: cider.cider_quantize_act(xs[i % len(xs)], q=qb[i % len(xs)], scale_x=sb),
                        args.steps, args.warmup)
        cider.cider_device_status()
        print(json.dumps({"row": args.row, "kind": kind, "M": M, "K": K, "ms": ms,
                          "GB/s": (M * K * 3 + M * 4) / (ms * 1e-3) / 1e9}), flush=True)
        return 0
    cider.cider_test_set_small_m_kernel(args.small_kernel)
    cider.cider_test_set_gemm_variant(args.gemm_variant)
    x = torch.from_numpy(synth.activations(M, K, 1000 + M)).to(device)
    W = torch.from_numpy(synth.weights(N, K, 1001)).to(device)
    if kind == "pc":
        w, s = cider.cider_quantize_weight_pc(W)
        call = lambda w, y, ws_: cider.cider_w8a8_linear_pc(x, w, s, y=y, workspace=ws_)
    elif kind == "mv":
        w, s = cider.cider_quantize_weight_pc(W)
        call = lambda w, y, ws_: cider.cider_w8a16_mv_pc(x, w, s, y=y)
    elif kind == "pg":
        w, s = cider.cider_quantize_weight_pg(W, gs)
        call = lambda w, y, ws_: cider.cider_w8a8_linear_pg(x, w, s, gs, y=y, workspace=ws_)
    elif kind == "mvpg":
        w, s = cider.cider_quantize_weight_pg(W, gs)
        call = lambda w, y, ws_: cider.cider_w8a16_mv_pg(x, w, s, gs, y=y)
    elif kind == "w4pc":
        w, s = cider.cider_pack_weight_int4_pc(W)
        call = lambda w, y, ws_: cider.cider_w4a8_linear_pc(x, w, s, y=y, workspace=ws_)
    else:
        w, s = cider.cider_pack_weight_int4_pg(W, gs)
        call = lambda w, y, ws_: cider.cider_w4a8_linear_pg(x, w, s, gs, y=y, workspace=ws_)
    del W
    # as in the bench rows: weight copies rotate beyond the L2 cache between calls
    n = rotating(w.numel() + M * K * 3 + M * N * 2)
    wr = [w] + [w.roll(i, 0).contiguous() for i in range(1, n)]
    ys = [torch.empty((M, N), dtype=torch.float16, device=device) for _ in range(min(n, 4))]
    wsp = torch.empty((max(1, cider.cider_workspace_bytes_mnk(M, N, K)),), dtype=torch.uint8, device=device)
    ms = graph_time(lambda i: call(wr[i % n], ys[i % len(ys)], wsp), args.steps, args.warmup)
    cider.cider_device_status()
    print(json.dumps({"row": args.row, "kind": kind, "M": M, "N": N, "K": K, "gs": gs, "ms": ms,
                      "TOPS": 2.0 * M * N * K / (ms * 1e-3) / 1e12}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cider", "reference"], default="cider")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--row", choices=sorted(ROW_CASES), help="time one hot-path row alone (for profiling)")
    ap.add_argument("--fused", choices=["auto", "off", "on"], default="auto",
                    help="with --row: where the per-channel linear quantizes (inside the GEMM launch or not)")
    ap.add_argument("--small-kernel", type=int, default=0, choices=[0, 1, 2, 3, 4],
                    help="with --row: decode kernel (0 auto, 1 register ring, 2 bulk, 3 bulk in half of smem, 4 one-shot)")
    ap.add_argument("--gemm-variant", type=int, default=0, choices=[0, 1, 2, 3, 4, 5],
                    help="with --row: per-channel GEMM (0 auto, 1 128x128, 2 128x256, 3 CTA pair 256x256, "
                         "4 128x80, 5 CTA pair 256x192)")
    ap.add_argument("--sdpa-kernel", type=int, default=0, choices=[0, 1, 2],
                    help="with --row: decode attention (0 auto, 1 CUDA cores, 2 tensor cores)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.row:
        return run_row(args)
    return run_cider(args)


if __name__ == "__main__":
    sys.exit(main())
