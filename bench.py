"""Benchmark of the W8A8 activation-quantized linear on B200.

Headline: W8A8 per-channel linear, M=4096 tokens, N=10240, K=2560 (the
Cider pages' single-op table shape), fp16 in / fp16 out, one step = one full
call (per-token quantize + tcgen05 GEMM + dequant epilogue).  Reported as
TOPS (2*M*N*K / time).  Inputs are seeded synthetic activations (N(0,1) with
1% outlier channels x50) and N(0, 0.02) weights quantized per output channel
on the GPU; several input sets larger than L2 in total rotate between steps.

Usage (one process per GPU; N>1 under torch.distributed.run):
    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cider|reference] [--rows]

--impl reference times the CPU oracle (the plain C reference) on this host's
cores on a bounded sample of the same workload; rank 0 only.
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

HEADLINE = dict(workload="w8a8_linear_pc", M=4096, N=10240, K=2560)
METRIC = "W8A8 linear TOPS & % INT8 tensor peak (M=4096,N=10240,K=2560); ms/op"
UNIT = "TOPS"
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


# Dense INT8 tensor peak = measured bf16 cuBLAS peak x the nominal int8/bf16 ratio (4.5 / 2.25).
INT8_PER_BF16 = 2.0


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _max_over_ranks(v, ws, device):
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _inputs(M, N, K, seed, device):
    from w8a8_activation_quantized_b200 import synth
    import w8a8_activation_quantized_b200 as cider
    x = torch.from_numpy(synth.activations(M, K, seed)).to(device)
    W = torch.from_numpy(synth.weights(N, K, seed)).to(device)
    w, sw = cider.cider_quantize_weight_pc(W)
    del W
    return x, w, sw


def _event_time(fn, steps, warmup, stream):
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        fn(i)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps  # ms per call


def _cpu_baseline(M, N, K, seed, target_s=12.0):
    """The oracle (plain C, OpenMP over rows) on a bounded sample of rows."""
    import oracle
    from w8a8_activation_quantized_b200 import synth
    threads = oracle.num_threads()
    rows = max(16, 2 * threads)
    x = synth.activations(M, K, seed)[:rows]
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed))
    t0 = time.perf_counter()
    oracle.linear_pc(x[:threads], qw, sw)   # calibration pass
    t1 = time.perf_counter()
    per_row = (t1 - t0) / max(1, threads)
    rows = int(min(max(threads, target_s / max(per_row, 1e-6)), rows * 8))
    x = synth.activations(max(rows, 1), K, seed)
    t0 = time.perf_counter()
    oracle.linear_pc(x, qw, sw)
    dt = time.perf_counter() - t0
    tops = 2.0 * rows * N * K / dt / 1e12
    return {"value": tops, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} of {M} token rows of the M={M} N={N} K={K} per-channel linear "
                      f"({dt:.1f} s; rows are independent, so TOPS scale with rows)"}, dt


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    M, N, K = HEADLINE["M"], HEADLINE["N"], HEADLINE["K"]
    base, _ = _cpu_baseline(M, N, K, seed=1000 + M, target_s=4.0)
    # each step is one bounded sample of the workload, like the calibration above
    import oracle
    from w8a8_activation_quantized_b200 import synth
    rows = max(1, oracle.num_threads())
    x = synth.activations(rows, K, 1000 + M)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, 1000 + M))
    for _ in range(args.warmup):
        oracle.linear_pc(x, qw, sw)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear_pc(x, qw, sw)
    dt = (time.perf_counter() - t0) / args.steps
    tops = 2.0 * rows * N * K / dt / 1e12
    line = {"metric": METRIC, "value": tops, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8->int32, fp32 dequant, fp16 out", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "w8a8_linear_pc M=4096 N=10240 K=2560 (CPU oracle, sampled rows)",
                       "rows_per_step": rows},
            "cpu_baseline": {"value": tops, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{rows} token rows per step of the M=4096 N=10240 K=2560 linear"},
            "e2e": {"value": tops, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_cider(args):
    import w8a8_activation_quantized_b200 as cider
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    if not cider.cider_is_available():
        raise RuntimeError("device is not sm_100-family")
    stream = torch.cuda.current_stream(device)
    M, N, K = HEADLINE["M"], HEADLINE["N"], HEADLINE["K"]
    seed = 1000 + M
    peaks = _peaks()
    int8_peak = peaks["bf16"] * INT8_PER_BF16  # burst: each kernel is timed alone, in a short loop

    x0, w0, sw0 = _inputs(M, N, K, seed, device)
    set_bytes = x0.numel() * 2 + w0.numel() + M * N * 2 + M * K
    n_sets = max(2, -(-3 * L2_BYTES // set_bytes))
    sets = [(x0, w0, sw0)] + [(x0.roll(i, 0).contiguous(), w0.roll(i, 0).contiguous(), sw0.roll(i, 0).contiguous())
                              for i in range(1, n_sets)]
    ys = [torch.empty((M, N), dtype=torch.float16, device=device) for _ in range(n_sets)]
    wsb = cider.cider_workspace_bytes(M, K)
    wss = [torch.empty((wsb,), dtype=torch.uint8, device=device) for _ in range(n_sets)]
    ops = 2.0 * M * N * K

    def step(i):
        x, w, sw = sets[i % n_sets]
        cider.cider_w8a8_linear_pc(x, w, sw, y=ys[i % n_sets], workspace=wss[i % n_sets], stream=stream)

    # warm-up, then exactly `steps` timed steps bracketed by barrier + synchronize
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    _barrier(ws)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(args.steps):
            step(i)
        end.record(stream)
        torch.cuda.synchronize()
    _barrier(ws)
    ms = _max_over_ranks(start.elapsed_time(end) / args.steps, ws, device)
    value = ws * ops / (ms * 1e-3) / 1e12

    # dominant kernel alone: the tcgen05 GEMM on pre-quantized activations
    qs = [cider.cider_quantize_act(s[0]) for s in sets]

    def gemm(i):
        q, sx = qs[i % n_sets]
        _, w, sw = sets[i % n_sets]
        cider.cider_w8a8_gemm_pc_q(q, sx, w, sw, y=ys[i % n_sets], stream=stream)

    ms_gemm = _event_time(gemm, args.steps, args.warmup, stream)

    def quant(i):
        cider.cider_quantize_act(sets[i % n_sets][0], q=qs[i % n_sets][0], scale_x=qs[i % n_sets][1], stream=stream)

    ms_quant = _event_time(quant, args.steps, args.warmup, stream)
    achieved = ops / (ms_gemm * 1e-3) / 1e12

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    xh = x0.cpu().pin_memory()
    yh = torch.empty((M, N), dtype=torch.float16).pin_memory()
    xd = torch.empty_like(x0)

    def e2e(i):
        xd.copy_(xh, non_blocking=True)
        cider.cider_w8a8_linear_pc(xd, w0, sw0, y=ys[0], workspace=wss[0], stream=stream)
        yh.copy_(ys[0], non_blocking=True)

    ms_e2e = _event_time(e2e, max(3, args.steps // 2), max(3, args.warmup), stream)
    e2e_tops = ws * ops / (ms_e2e * 1e-3) / 1e12

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8 x int8 -> int32, fp32 dequant, fp16 in/out", "data": "synthetic",
        "config": {"workload": "w8a8_linear_pc", "M": M, "N": N, "K": K, "x": "fp16 N(0,1), 1% channels x50",
                   "w": "N(0,0.02) -> int8 per output channel", "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "l2": f"{n_sets} rotating input sets, {n_sets * set_bytes / 2**20:.0f} MiB > L2"},
        "tops_per_gpu": value / ws, "pct_int8_peak": 100.0 * (value / ws) / int8_peak,
        "breakdown_ms": {"quantize": ms_quant, "gemm": ms_gemm},
        "roofline": {"bound": "tensor", "kernel": "k_gemm_sm100 (per-channel, BN=256)",
                     "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s",
                     "frac": achieved / int8_peak, "traffic": None,
                     "peak_note": f"dense INT8 = {INT8_PER_BF16:g} x {peaks['src']} bf16 cuBLAS burst {peaks['bf16']:.1f}"},
        "e2e": {"value": e2e_tops, "unit": UNIT, "ms_per_step": ms_e2e,
                "h2d_bytes_per_step": x0.numel() * 2, "d2h_bytes_per_step": M * N * 2},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if args.rows:
        line["rows"] = bench_rows(args, device, stream, peaks)
    if rank == 0 and not args.no_cpu_baseline and ws == 1:
        line["cpu_baseline"], _ = _cpu_baseline(M, N, K, seed)
    elif rank == 0 and ws == 1:
        line["cpu_baseline"] = None
    cider.cider_device_status()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def bench_rows(args, device, stream, peaks):
    """One measurement per hot-path row: kernel time (CUDA events) and roofline."""
    import w8a8_activation_quantized_b200 as cider
    from w8a8_activation_quantized_b200 import synth
    hbm = peaks["hbm"]
    int8_peak = peaks["bf16"] * INT8_PER_BF16
    out = []
    steps, warm = max(10, args.steps), max(3, args.warmup)

    def rot(make, nbytes):
        n = max(2, -(-3 * L2_BYTES // max(nbytes, 1)))
        return [make(i) for i in range(n)]

    # per-channel M=1 (decode) and other M of the N=10240, K=2560 sweep
    N, K = 10240, 2560
    W = torch.from_numpy(synth.weights(N, K, 1001)).to(device)
    w8, s8 = cider.cider_quantize_weight_pc(W)
    for M in (1, 128, 1024, 4096, 8192):
        x = torch.from_numpy(synth.activations(M, K, 1000 + M)).to(device)
        nbytes = N * K + M * K * 2 + M * N * 2
        sets = rot(lambda i: (x, w8.roll(i, 0).contiguous() if i else w8, torch.empty((M, N), dtype=torch.float16, device=device)), nbytes)
        wsb = torch.empty((max(1, cider.cider_workspace_bytes(M, K)),), dtype=torch.uint8, device=device)
        ms = _event_time(lambda i: cider.cider_w8a8_linear_pc(sets[i % len(sets)][0], sets[i % len(sets)][1], s8,
                                                              y=sets[i % len(sets)][2], workspace=wsb, stream=stream),
                         steps, warm, stream)
        ops = 2.0 * M * N * K
        mbytes = N * K + N * 4 + M * K * 2 + M * N * 2
        tops = ops / (ms * 1e-3) / 1e12
        gbs = mbytes / (ms * 1e-3) / 1e9
        bound = "hbm" if ops / mbytes < int8_peak * 1e12 / (hbm * 1e9) else "tensor"
        out.append({"row": "w8a8_linear_pc", "M": M, "N": N, "K": K, "ms": ms, "TOPS": tops, "GB/s": gbs,
                    "bound": bound, "frac": (gbs / hbm) if bound == "hbm" else (tops / int8_peak),
                    "path": "small-M kernel" if cider.cider_workspace_bytes(M, K) == 0 else "quantize+tcgen05"})
        del sets
    del W, w8
    # per-group, N=2560, K=10240
    N, K = 2560, 10240
    W = torch.from_numpy(synth.weights(N, K, 2001)).to(device)
    for gs in (128, 64):
        wg, sg = cider.cider_quantize_weight_pg(W, gs)
        for M in (1, 4096):
            x = torch.from_numpy(synth.activations(M, K, 2000 + M)).to(device)
            y = torch.empty((M, N), dtype=torch.float16, device=device)
            wsb = torch.empty((max(1, cider.cider_workspace_bytes(M, K)),), dtype=torch.uint8, device=device)
            wsets = rot(lambda i: wg.roll(i, 0).contiguous() if i else wg, N * K)
            ms = _event_time(lambda i: cider.cider_w8a8_linear_pg(x, wsets[i % len(wsets)], sg, gs, y=y, workspace=wsb,
                                                                  stream=stream), steps, warm, stream)
            ops = 2.0 * M * N * K
            mbytes = N * K + sg.numel() * 4 + M * K * 2 + M * N * 2
            tops, gbs = ops / (ms * 1e-3) / 1e12, mbytes / (ms * 1e-3) / 1e9
            bound = "hbm" if M == 1 else "tensor"
            out.append({"row": "w8a8_linear_pg", "gs": gs, "M": M, "N": N, "K": K, "ms": ms, "TOPS": tops, "GB/s": gbs,
                        "bound": bound, "frac": (gbs / hbm) if bound == "hbm" else (tops / int8_peak)})
        del wg, sg
    del W
    # W4A8, N=12288, K=4096, M=2048, gs=64
    M, N, K, gs = 2048, 12288, 4096, 64
    W = torch.from_numpy(synth.weights(N, K, 3001)).to(device)
    p4, s4 = cider.cider_pack_weight_int4_pg(W, gs)
    del W
    x = torch.from_numpy(synth.activations(M, K, 3000 + M)).to(device)
    y = torch.empty((M, N), dtype=torch.float16, device=device)
    wsb = torch.empty((cider.cider_workspace_bytes(M, K),), dtype=torch.uint8, device=device)
    ms = _event_time(lambda i: cider.cider_w4a8_linear_pg(x, p4, s4, gs, y=y, workspace=wsb, stream=stream),
                     steps, warm, stream)
    ops = 2.0 * M * N * K
    out.append({"row": "w4a8_linear_pg", "gs": gs, "M": M, "N": N, "K": K, "ms": ms,
                "TOPS": ops / (ms * 1e-3) / 1e12, "bound": "tensor", "frac": ops / (ms * 1e-3) / 1e12 / int8_peak})
    # quantize alone and SiLU*up -> quantize (memory-bound)
    for (M, K) in ((4096, 2560), (8192, 10240)):
        x = torch.from_numpy(synth.activations(M, K, 7)).to(device)
        q = torch.empty((M, K), dtype=torch.int8, device=device)
        s = torch.empty((M,), dtype=torch.float32, device=device)
        ms = _event_time(lambda i: cider.cider_quantize_act(x, q=q, scale_x=s, stream=stream), steps, warm, stream)
        b = M * K * 3 + M * 4
        out.append({"row": "quantize_act", "M": M, "K": K, "ms": ms, "GB/s": b / (ms * 1e-3) / 1e9, "bound": "hbm",
                    "frac": b / (ms * 1e-3) / 1e9 / hbm})
    M, F = 2048, 12288
    g = torch.from_numpy(synth.activations(M, F, 8)).to(device)
    u = torch.from_numpy(synth.activations(M, F, 9)).to(device)
    q = torch.empty((M, F), dtype=torch.int8, device=device)
    s = torch.empty((M,), dtype=torch.float32, device=device)
    ms = _event_time(lambda i: cider.cider_silu_mul_quantize(g, u, q=q, scale_x=s, stream=stream), steps, warm, stream)
    b = M * F * 5 + M * 4
    out.append({"row": "silu_mul_quantize", "M": M, "F": F, "ms": ms, "GB/s": b / (ms * 1e-3) / 1e9, "bound": "hbm",
                "frac": b / (ms * 1e-3) / 1e9 / hbm})
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cider", "reference"], default="cider")
    ap.add_argument("--rows", action="store_true", help="also measure every hot-path row")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_cider(args)


if __name__ == "__main__":
    sys.exit(main())
