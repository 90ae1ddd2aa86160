#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear hot path on B200.

Headline (the JSON line's `value`): forward + adapter backward of the
prefill/training layer -- W 11008x4096 NF4 (block 64, double quant), x of
4096 tokens, r = 64, alpha = 16 -- in TFLOP/s of algorithmic work
(4 M N K + 6 M r (N + K) per step), inputs resident in HBM, L2 flushed
before every timed step.  The same line carries the dominant kernel's
roofline, the CPU oracle's time on this host, an end-to-end figure through
the C ABI from pinned host buffers, the SM clocks seen while timing, and the
other rows of the hot path (quantize / dequantize GB/s, decode GEMV GB/s,
the seven-target decoder block).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the same layer on its own 4096 tokens (weak
scaling) and the adapter gradients are all-reduced over NCCL each step; the
secondary rows and the CPU baseline are taken at N = 1 only.
--impl reference times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA NF4 linear fwd+bwd TFLOP/s; NF4 (de)quant & GEMV GB/s vs B200 roofline"
FLUSH_BYTES = 256 << 20          # > 2x the 126 MB L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel from an ncu capture, keyed by
# the hash of the kernel source it was taken on; reported as null once the
# source changes.
NCU_TRAFFIC = {
    # forward 127.4 MB, dx 181.0 MB per launch
    "0afa7f14ba671346": {"fwd": 72_147_712 + 55_230_976, "dx": 162_442_240 + 18_569_984},
}


def linear_flops(m, n, k, r):
    return 4 * m * n * k + 6 * m * r * (n + k)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash():
    h = hashlib.sha256()
    for name in ("qlora_gemm.cu", "tc_common.cuh", "nf4_common.cuh"):
        with open(os.path.join(ROOT, "qlora_linear_layers_nf4_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------------- clocks

_NVML_POLLER = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
uuid, period = sys.argv[1], float(sys.argv[2])
try:
    h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
except pynvml.NVMLError:
    h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[3]))
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
        pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
print("ready", flush=True)
while True:
    t = time.monotonic()
    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
    act = "|".join(n for n, b in zip(names, bits) if rs & b)
    print(f"{t:.6f},{sm},{mx},{pw:.1f},{act}", flush=True)
    time.sleep(period)
"""


class ClockSampler:
    """SM clock, power and throttle reasons sampled while timing.

    A separate process polls NVML every few milliseconds (no GIL shared with
    the launching thread), with CLOCK_MONOTONIC stamps; the summary keeps the
    samples that fall inside [start(), stop()].  The device is found by UUID
    (CUDA and NVML may number GPUs differently).  Without NVML, nvidia-smi is
    sampled at its shortest interval instead.  Raw samples go to
    BENCH_OUT_DIR (default: the temp dir)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device, period_s=0.002):
        self.device = device
        self.period = period_s
        self.proc = None
        self.kind = None
        out_dir = os.environ.get("BENCH_OUT_DIR", tempfile.gettempdir())
        self.path = os.path.join(out_dir, f"nf4_bench_clocks_gpu{getattr(device, 'index', 0) or 0}.csv")

    def launch(self):
        """Start the poller (before warm-up: it takes a moment to come up)."""
        import torch
        os.makedirs(os.path.dirname(self.path) or ".", exist_ok=True)
        self.fh = open(self.path, "w")
        idx = getattr(self.device, "index", 0) or 0
        uuid = str(getattr(torch.cuda.get_device_properties(self.device), "uuid", "") or "")
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _NVML_POLLER, uuid, str(self.period), str(idx)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            if self.proc.stdout.readline().strip() == "ready":
                self.kind = "nvml"
                return self
            self.proc.kill()
        except OSError:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(idx), "-lms", "10"], stdout=self.fh, stderr=subprocess.DEVNULL)
            self.kind = "nvidia-smi"
        except OSError:
            self.proc = None
        return self

    def start(self):
        if self.proc is None and self.kind is None:
            self.launch()
        self.t0 = time.monotonic()

    def stop(self):
        t1 = time.monotonic()
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0,
                    "reasons": ["no clock source (NVML and nvidia-smi unavailable)"]}
        time.sleep(2 * self.period)
        self.proc.terminate()
        samples = []
        if self.kind == "nvml":
            out, _ = self.proc.communicate(timeout=10)
            self.fh.write(out)
            for line in out.splitlines():
                parts = line.split(",")
                if len(parts) != 5:
                    continue
                t = float(parts[0])
                if self.t0 <= t <= t1:
                    samples.append((float(parts[1]), float(parts[2]), float(parts[3]),
                                    {r for r in parts[4].split("|") if r}))
        else:
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        vals = float(parts[1]), float(parts[2]), float(parts[3])
                    except ValueError:
                        continue
                    rs = {n for n, v in zip(self.NAMES, parts[5:9]) if v.lower().startswith("active")}
                    samples.append((*vals, rs))
        if not self.fh.closed:
            self.fh.close()
        self.proc = None
        sm = [x[0] for x in samples]
        reasons, counts = set(), {}
        for x in samples:
            reasons |= x[3]
            for n in x[3]:
                counts[n] = counts.get(n, 0) + 1
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(x[1] for x in samples) if samples else None,
                "sm_min_mhz": min(sm) if sm else None,
                "power_w_max": max(x[2] for x in samples) if samples else None,
                "samples": len(sm), "window_ms": 1e3 * (t1 - self.t0), "source": self.kind,
                "reasons": sorted(reasons), "reason_samples": counts}


def choose_bf16_peak(pk, clk):
    """The bf16 peak that the clocks seen while timing justify.

    The burst figure was measured at full clock and the sustained one under
    the power cap.  The sustained figure applies only when the timed region
    itself ran capped: sw_power_cap seen in at least a tenth of the samples,
    or a median SM clock more than 5 % below the maximum.  Returns
    (peak, which, why)."""
    burst, sustained = pk.get("bf16_tflops"), pk.get("bf16_tflops_sustained")
    n = clk.get("samples") or 0
    med, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    capped = (clk.get("reason_samples") or {}).get("sw_power_cap", 0)
    if not n or med is None or mx is None:
        return burst or sustained, "bf16_tflops", "no clock samples: burst peak (the stricter one)"
    if sustained and (capped >= max(1, n // 10) or med < 0.95 * mx):
        return sustained, "bf16_tflops_sustained", (
            f"power-capped timing: median SM {med:.0f} of {mx:.0f} MHz, sw_power_cap in {capped}/{n} samples")
    return burst or sustained, "bf16_tflops", (
        f"full-clock timing: median SM {med:.0f} of {mx:.0f} MHz, sw_power_cap in {capped}/{n} samples")


# --------------------------------------------------------------------- helpers

def bf16_dev(bits, dev):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def cpu_cores():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    threads = n
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            threads = max(i.get("num_threads", n) for i in info)
    except Exception:
        pass
    return n, threads


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_step_sample(case, m_sample):
    """One bounded oracle step: dequantize W (bf16) and run fwd + bwd on
    m_sample tokens of the workload.  Returns (seconds, flops)."""
    import numpy as np
    from oracle import nf4_oracle as O
    from qlora_linear_layers_nf4_b200 import workloads as WL
    inp = WL.draw_linear(case, m=m_sample)
    ref_q = O.quantize(inp.w, case.block_size, double=case.double_quant)
    f = WL.bf16_bits_to_f32
    x, a, b, dy = (f(v) for v in (inp.x, inp.a, inp.b, inp.dy))

    def step():
        w_hat = O.bf16_to_f32(O.dequantize(ref_q, "bf16"))
        O.qlora_forward(x, w_hat, a, b, case.alpha)
        O.qlora_backward(x, w_hat, a, b, case.alpha, dy)

    return step, linear_flops(m_sample, case.n, case.k, case.r)


# --------------------------------------------------------------------- our arm

class Timer:
    def __init__(self, n):
        import torch
        self.s = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        self.e = [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    def total_ms(self):
        return sum(a.elapsed_time(b) for a, b in zip(self.s, self.e))


def time_steps(fn, steps, warmup, flush=None, barrier=None, on_timed=None):
    """Run warmup + timed steps; each timed step bracketed by events, with an
    L2 flush before it (outside the brackets).  Returns total ms."""
    import torch
    for _ in range(warmup):
        if flush is not None:
            flush()
        fn()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    if on_timed is not None:
        on_timed()
    t = Timer(steps)
    for i in range(steps):
        if flush is not None:
            flush()
        t.s[i].record()
        fn()
        t.e[i].record()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return t.total_ms()


def time_steps_clocked(fn, steps, warmup, device, flush=None, barrier=None):
    """time_steps with the SM clocks sampled over the timed steps."""
    clocks = ClockSampler(device).launch()
    ms = time_steps(fn, steps, warmup, flush=flush, barrier=barrier, on_timed=clocks.start)
    return ms, clocks.stop()


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    from qlora_linear_layers_nf4_b200 import workloads as WL
    from qlora_linear_layers_nf4_b200.dp import AdapterGradBuffer, max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    barrier = (lambda: dist.barrier()) if world > 1 else None
    Q.lib()

    case = WL.PREFILL
    M, N, K, r = case.m, case.n, case.k, case.r
    inp = WL.draw_linear(case)
    q = Q.quantize(torch.from_numpy(inp.w).to(dev), case.block_size, case.double_quant)
    x, A, B, dy = (bf16_dev(v, dev) for v in (inp.x, inp.a, inp.b, inp.dy))
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    T = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    grads = AdapterGradBuffer(r, K, N, dev)
    ws = Q.Workspace(dev)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush = lambda: flush_buf.zero_()

    def step():
        Q.linear_fwd(q, x, A, B, case.alpha, out=y, t_out=T, workspace=ws)
        Q.linear_bwd(q, x, A, B, case.alpha, dy, t=T, dA=grads.dA, dB=grads.dB, dx=dx, workspace=ws)
        if world > 1:
            grads.all_reduce()

    flops = linear_flops(M, N, K, r)
    clocks = ClockSampler(dev).launch()
    for _ in range(max(args.warmup, 0)):
        flush()
        step()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    launches0 = Q.launch_count()
    Q.profile_begin()
    clocks.start()
    t = Timer(args.steps)
    for i in range(args.steps):
        flush()
        t.s[i].record()
        step()
        t.e[i].record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    kernels = Q.profile_end()
    if barrier:
        barrier()
    launches = Q.launch_count() - launches0
    total_ms = max_over_ranks(t.total_ms(), dev)
    ms_per_step = total_ms / args.steps
    value = flops * world * args.steps / (total_ms * 1e-3) / 1e12
    if ws.read_status() != 0:
        raise RuntimeError("device status reported an error during the benchmark")

    pk, pk_kind = peaks()
    # dominant kernel: the fused dequant + tcgen05 GEMM (forward and dx launches)
    fwd_n, fwd_ms = kernels.get("fused_nf4_gemm_fwd", (0, 0.0))
    dx_n, dx_ms = kernels.get("fused_nf4_gemm_dx", (0, 0.0))
    fwd_flops = 2 * M * N * K + 2 * M * r * N
    dx_flops = 2 * M * N * K + 2 * M * r * K
    total_kernel_ms = sum(v[1] for v in kernels.values())
    fused_launches = fwd_n + dx_n
    achieved = ((fwd_n * fwd_flops + dx_n * dx_flops) / ((fwd_ms + dx_ms) * 1e-3) / 1e12
                if fused_launches else None)
    peak, peak_name, peak_why = choose_bf16_peak(pk, clk)
    src = source_hash()
    tr = NCU_TRAFFIC.get(src)
    # bytes per launch, averaged over the step's forward and dx launches
    traffic = (tr["fwd"] + tr["dx"]) / 2 if tr else None
    roofline = {
        "kernel": "fused_nf4_gemm (fwd + dx launches)",
        "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
        "frac": (achieved / peak) if achieved else None, "traffic": traffic,
        "traffic_per_launch": tr,
        "peak_source": f"{pk_kind} {peak_name}: {peak_why}",
        "flops_per_launch": {"fwd": fwd_flops, "dx": dx_flops},
        "share_of_step_kernel_time": (fwd_ms + dx_ms) / total_kernel_ms if total_kernel_ms else None,
        "source_hash": src,
    }
    kern = {k: {"launches": n, "avg_us": 1e3 * ms / n, "share": ms / total_kernel_ms}
            for k, (n, ms) in kernels.items()}

    # ---- end to end through the C ABI from pinned host buffers.  Each step's
    # x and dy are copied host -> device and its dA, dB device -> host inside
    # the timed region.  The copies of step i+1 run on a copy stream into a
    # second buffer set while step i computes, as a data loader would.
    e2e = None
    if not args.no_e2e:
        hx = x.cpu().pin_memory()
        hdy = dy.cpu().pin_memory()
        hdA = torch.empty_like(grads.dA, device="cpu").pin_memory()
        hdB = torch.empty_like(grads.dB, device="cpu").pin_memory()
        xs = [torch.empty_like(x) for _ in range(2)]
        dys = [torch.empty_like(dy) for _ in range(2)]
        main = torch.cuda.current_stream()
        copy = torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()
        e2e_steps = max(3, min(args.steps, 20))

        def e2e_run(n):
            copied = [ev(), ev()]
            consumed = [ev(), ev()]
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(main)
            copy.wait_stream(main)
            with torch.cuda.stream(copy):
                xs[0].copy_(hx, non_blocking=True)
                dys[0].copy_(hdy, non_blocking=True)
                copied[0].record(copy)
            for i in range(n):
                cur, nxt = i % 2, (i + 1) % 2
                if i + 1 < n:
                    with torch.cuda.stream(copy):
                        if i >= 1:
                            copy.wait_event(consumed[nxt])
                        xs[nxt].copy_(hx, non_blocking=True)
                        dys[nxt].copy_(hdy, non_blocking=True)
                        copied[nxt].record(copy)
                main.wait_event(copied[cur])
                flush()
                Q.linear_fwd(q, xs[cur], A, B, case.alpha, out=y, t_out=T, workspace=ws)
                Q.linear_bwd(q, xs[cur], A, B, case.alpha, dys[cur], t=T, dA=grads.dA, dB=grads.dB,
                             dx=dx, workspace=ws)
                if world > 1:
                    grads.all_reduce()
                consumed[cur].record(main)
                hdA.copy_(grads.dA, non_blocking=True)
                hdB.copy_(grads.dB, non_blocking=True)
            t1.record(main)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1)

        e2e_run(2)
        if barrier:
            barrier()
        ms = max_over_ranks(e2e_run(e2e_steps), dev)
        e2e = {"value": flops * world * e2e_steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": hx.numel() * 2 + hdy.numel() * 2,
               "d2h_bytes_per_step": (hdA.numel() + hdB.numel()) * 4,
               "ms_per_step": ms / e2e_steps, "steps": e2e_steps,
               "method": "pinned host x, dy copied on a copy stream into one of two device buffer sets "
                         "while the previous step computes; dA, dB copied back every step; "
                         "L2 flushed before each step's compute"}

    # The secondary rows are single-GPU kernel figures: taken at N = 1 only, so
    # a multi-GPU run holds its GPUs for the data-parallel step alone.
    rows = {}
    if not args.no_rows and world == 1:
        rows = measure_rows(args, dev, flush, pk, pk_kind, barrier)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(case, args.cpu_seconds)

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded normal draws (W ~ N(0, 0.02^2), x, dy ~ N(0, 1), "
                "A ~ N(0, 1/K), B ~ N(0, 0.01^2)), bf16 inputs, NF4 weight quantized on device",
        "config": {
            "workload": "QLoRA linear fwd+bwd, W 11008x4096 NF4 block 64 double-quant, "
                        "M=4096 tokens per GPU, r=64, alpha=16 (dA, dB, dx)",
            "tokens_per_gpu": M, "out_features": N, "in_features": K, "rank": r,
            "flops_per_step_per_gpu": flops, "parallelism": f"dp{world}",
            "l2": "flushed before every timed step (256 MiB memset outside the step events)",
            "grad_allreduce": "NCCL all-reduce of dA+dB (fp32) per step" if world > 1 else "none (1 GPU)",
        },
        "roofline": roofline,
        "kernels": kern,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clk,
        "gpu_launches": launches,
        "gpu_launches_per_step": launches / args.steps,
        "rows": rows,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def graph_time(calls, replays, warmup=2):
    """GPU time per call of `calls` (a list of zero-argument launches), captured
    into one CUDA graph and replayed `replays` times; host overhead is out."""
    import torch
    for _ in range(warmup):
        for c in calls:
            c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(replays):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / (replays * len(calls))
    del g
    return ms


def measure_rows(args, dev, flush, pk, pk_kind, barrier):
    """The other rows of the hot path.  Each is a short kernel, so it is timed
    as CUDA-graph replays of calls on rotating buffers whose footprint exceeds
    the 126 MB L2 (no flush needed, no host launch overhead)."""
    import ctypes
    import numpy as np
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    from qlora_linear_layers_nf4_b200 import workloads as WL

    L = Q.lib()
    hbm = pk.get("hbm_gbs")
    out = {}
    stream = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    def row(name, calls, nbytes, footprint, replays=20):
        # the rotating buffers of one graph replay must be >= 4x the L2, so no
        # call finds its inputs there
        assert footprint >= 4 * l2, f"{name}: rotating footprint {footprint} < 4 x L2"
        ms = graph_time(calls, replays)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"GB/s": gbs, "frac_hbm": gbs / hbm, "us_per_call": 1e3 * ms, "bytes": nbytes,
                     "rotating_bytes": footprint,
                     "method": f"CUDA graph of {len(calls)} calls on rotating buffers "
                               f"({footprint / l2:.1f}x L2), {replays} replays"}

    # ---- quantize / dequantize of 4096x4096: 14 rotating matrices (the fp32
    # inputs alone are 7x the L2), seeded draws of the quantize workload
    R = 14
    ws = [Q.Workspace(dev) for _ in range(R)]
    ws_bytes = Q.workspace_bytes(Q.OP_QUANTIZE, 0, 4096, 4096, 0, 64, True)
    ws_bufs = [w.get(ws_bytes) for w in ws]
    ws_s = [w.numel() for w in ws_bufs]
    base_w = torch.from_numpy(WL.draw_weight(WL.QUANT_SHAPE, WL.QUANT_SEED)).to(dev)
    # the other matrices are row rotations of the seeded one (same values,
    # different addresses and block contents; the kernels' cost does not depend
    # on the values)
    mats = [base_w] + [torch.roll(base_w, 257 * i, dims=0).contiguous() for i in range(1, R)]
    numel, nb = 4096 * 4096, 4096 * 4096 // 64
    codes = [torch.empty(numel // 2, dtype=torch.uint8, device=dev) for _ in range(R)]
    amax = [torch.empty(nb, dtype=torch.float32, device=dev) for _ in range(R)]
    aq = [torch.empty(nb, dtype=torch.uint8, device=dev) for _ in range(R)]
    asc = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(R)]

    def qcall(i, dq):
        def f():
            st = L.nf4_quantize(ptr(mats[i]), 4096, 4096, 64, int(dq), ptr(codes[i]),
                                None if dq else ptr(amax[i]), ptr(aq[i]) if dq else None,
                                ptr(asc[i]) if dq else None, ptr(ws_bufs[i]), ws_s[i], stream())
            assert st == 0, st
        return f

    qfoot = R * (numel * 4 + numel // 2 + nb * 4)
    row("quantize_4096x4096_noDQ", [qcall(i, False) for i in range(R)], numel * 4 + numel // 2 + nb * 4, qfoot)
    row("quantize_4096x4096_DQ", [qcall(i, True) for i in range(R)], numel * 4 + numel // 2 + nb + 4, qfoot)
    # both forms of each weight now exist (codes[i] are identical for both)
    for i in range(R):
        qcall(i, False)()
    torch.cuda.synchronize()
    outs = {"f32": [torch.empty(numel, dtype=torch.float32, device=dev) for _ in range(R)],
            "bf16": [torch.empty(numel, dtype=torch.bfloat16, device=dev) for _ in range(R)]}
    kinds = {"f32": (Q.NF4_F32, 4), "bf16": (Q.NF4_BF16, 2)}

    def dcall(i, dq, kind):
        cw = Q.CWeight(codes=codes[i].data_ptr(), absmax=None if dq else amax[i].data_ptr(),
                       absmax_q=aq[i].data_ptr() if dq else None,
                       absmax_scale=asc[i].data_ptr() if dq else None, rows=4096, cols=4096,
                       block_size=64, double_quant=int(dq))
        def f():
            st = L.nf4_dequantize(ctypes.byref(cw), kinds[kind][0], ptr(outs[kind][i]), stream())
            assert st == 0, st
        return f

    for dq in (False, True):
        if dq:
            for i in range(R):
                qcall(i, True)()
        sb = nb * 4 if not dq else nb + 4
        for kind in ("f32", "bf16"):
            per = numel // 2 + sb + numel * kinds[kind][1]
            row(f"dequantize_{kind}_{'DQ' if dq else 'noDQ'}", [dcall(i, dq, kind) for i in range(R)],
                per, R * per)
    del mats, outs, codes, amax, aq, asc
    torch.cuda.empty_cache()

    # ---- decode forward: 64 rotating 4096x4096 NF4 weights (8.7 MB each, 4.4x
    # the L2), row rotations of one seeded draw quantized on the device
    RD = 64
    base = WL.DECODE[0]
    wd = torch.from_numpy(WL.draw_weight((base.n, base.k), seed=200)).to(dev)
    qws = [Q.quantize(torch.roll(wd, 61 * i, dims=0).contiguous(), 64, True) for i in range(RD)]
    del wd
    for case in WL.DECODE:
        inp = WL.draw_linear(case)
        x, A, B = (bf16_dev(v, dev) for v in (inp.x, inp.a, inp.b))
        y = torch.empty((case.m, case.n), dtype=torch.bfloat16, device=dev)
        wsd = Q.Workspace(dev)
        buf = wsd.get(Q.workspace_bytes(Q.OP_LINEAR_FWD, case.m, case.n, case.k, case.r, 64, True))
        cws = [qq.c_struct() for qq in qws]

        def fcall(cw):
            def f():
                st = L.qlora_linear_fwd(ctypes.byref(cw), ptr(x), case.m, ptr(A), ptr(B), case.r,
                                        float(case.alpha), Q.NF4_BF16, None, ptr(y), None, ptr(buf),
                                        buf.numel(), stream())
                assert st == 0, st
            return f

        nbytes = (case.n * case.k // 2 + case.n * case.k // 64 + 4 + 2 * case.r * case.k
                  + 2 * case.n * case.r + 2 * case.m * (case.k + case.n))
        # 128 calls per graph (each weight twice, 63 others in between)
        row(f"decode_fwd_M{case.m}", [fcall(cw) for cw in cws + cws], nbytes, RD * nbytes, replays=20)
    del qws
    torch.cuda.empty_cache()

    # ---- the headline layer in the F16 compute dtype (same draws rounded to f16)
    case = WL.PREFILL
    inp = WL.draw_linear(case)
    qf = Q.quantize(torch.from_numpy(inp.w).to(dev), 64, True)
    d32 = inp.extra["f32"]
    xf, Af, Bf, dyf = (torch.from_numpy(d32[k]).to(dev).half() for k in ("x", "a", "b", "dy"))
    yf = torch.empty((case.m, case.n), dtype=torch.float16, device=dev)
    Tf = torch.empty((case.m, case.r), dtype=torch.float16, device=dev)
    dxf = torch.empty((case.m, case.k), dtype=torch.float16, device=dev)
    dAf = torch.empty((case.r, case.k), dtype=torch.float32, device=dev)
    dBf = torch.empty((case.n, case.r), dtype=torch.float32, device=dev)
    wsf = Q.Workspace(dev)

    def f16_step():
        Q.linear_fwd(qf, xf, Af, Bf, case.alpha, out=yf, t_out=Tf, workspace=wsf)
        Q.linear_bwd(qf, xf, Af, Bf, case.alpha, dyf, t=Tf, dA=dAf, dB=dBf, dx=dxf, workspace=wsf)

    fsteps = max(3, min(args.steps, 20))
    ms, clk = time_steps_clocked(f16_step, fsteps, 3, dev, flush=flush, barrier=barrier)
    fl = linear_flops(case.m, case.n, case.k, case.r)
    tf = fl * fsteps / (ms * 1e-3) / 1e12
    peak, peak_name, why = choose_bf16_peak(pk, clk)
    out["prefill_11008x4096_M4096_f16_fwd_bwd"] = {
        "TFLOP/s": tf, "ms_per_step": ms / fsteps, "frac_peak": tf / peak,
        "peak": peak, "peak_source": f"{pk_kind} {peak_name} (the f16 dense peak equals the bf16 one): {why}",
        "method": "eager steps, L2 flushed before each"}
    if wsf.read_status() != 0:
        raise RuntimeError("device status reported an error in the f16 row")
    del xf, dyf, yf, dxf
    torch.cuda.empty_cache()

    # ---- the same layer in the F32 compute dtype (fp32 FMAs on the CUDA cores),
    # against the fp32 ALU peak: SMs x 128 FP32 lanes x 2 FLOP x the max SM clock
    xs, As_, Bs_, dys = (torch.from_numpy(np.ascontiguousarray(d32[k])).to(dev) for k in ("x", "a", "b", "dy"))
    ys = torch.empty((case.m, case.n), dtype=torch.float32, device=dev)
    Ts = torch.empty((case.m, case.r), dtype=torch.float32, device=dev)
    dxs = torch.empty((case.m, case.k), dtype=torch.float32, device=dev)

    def f32_step():
        Q.linear_fwd(qf, xs, As_, Bs_, case.alpha, out=ys, t_out=Ts, workspace=wsf)
        Q.linear_bwd(qf, xs, As_, Bs_, case.alpha, dys, t=Ts, dA=dAf, dB=dBf, dx=dxs, workspace=wsf)

    ssteps = 3
    ms = time_steps(f32_step, ssteps, 3, flush=flush, barrier=barrier)
    tf = fl * ssteps / (ms * 1e-3) / 1e12
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    alu_peak = sms * 128 * 2 * 1.965e9 / 1e12
    out["prefill_11008x4096_M4096_f32_fwd_bwd"] = {
        "TFLOP/s": tf, "ms_per_step": ms / ssteps, "bound": "alu",
        "peak_tflops": alu_peak, "frac_fp32_alu": tf / alu_peak,
        "peak_source": f"derived: {sms} SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz (max SM clock)",
        "method": "eager steps, L2 flushed before each"}
    if wsf.read_status() != 0:
        raise RuntimeError("device status reported an error in the f32 row")
    del qf, xs, dys, ys, dxs, Ts
    torch.cuda.empty_cache()

    # ---- dense merge of the 11008x4096 layer with its r = 64 adapter (bf16 out),
    # 6 rotating outputs (541 MB, 4.3x the L2)
    case = WL.PREFILL
    inp = WL.draw_linear(case)
    qm = Q.quantize(torch.from_numpy(inp.w).to(dev), 64, True)
    Am, Bm = bf16_dev(inp.a, dev), bf16_dev(inp.b, dev)
    outs_m = [torch.empty((case.n, case.k), dtype=torch.bfloat16, device=dev) for _ in range(6)]
    wsm = Q.Workspace(dev)
    bufm = wsm.get(Q.workspace_bytes(Q.OP_MERGE, 0, case.n, case.k, case.r, 64, True))
    cwm = qm.c_struct()

    def mcall(o):
        def f():
            st = L.nf4_merge(ctypes.byref(cwm), ptr(Am), ptr(Bm), case.r, float(case.alpha), Q.NF4_BF16,
                             ptr(o), ptr(bufm), bufm.numel(), stream())
            assert st == 0, st
        return f

    mbytes = (case.n * case.k // 2 + case.n * case.k // 64 + 4 + 2 * case.r * (case.n + case.k)
              + 2 * case.n * case.k)
    row("merge_11008x4096_r64_bf16", [mcall(o) for o in outs_m], mbytes,
        len(outs_m) * 2 * case.n * case.k + mbytes - 2 * case.n * case.k)
    del outs_m, qm
    torch.cuda.empty_cache()

    # ---- the seven targets of one decoder block, fwd + bwd each (long kernels: eager).
    # The block's forward runs its targets in layer order and its backward in
    # reverse; q, k, v (which read the same activations) and gate, up are
    # independent of one another, so each group runs on parallel streams, as
    # a training step schedules them.  Every target has its own workspace.
    if not args.no_block:
        ws_q = Q.Workspace(dev)
        layers = {}
        for case in WL.BLOCK:
            inp = WL.draw_linear(case)
            qb = Q.quantize(torch.from_numpy(inp.w).to(dev), 64, True, workspace=ws_q)
            x, A, B, dy = (bf16_dev(v, dev) for v in (inp.x, inp.a, inp.b, inp.dy))
            layers[case.name.split()[1]] = (
                case, qb, x, A, B, dy,
                torch.empty((case.m, case.n), dtype=torch.bfloat16, device=dev),
                torch.empty((case.m, case.r), dtype=torch.bfloat16, device=dev),
                torch.empty((case.m, case.k), dtype=torch.bfloat16, device=dev),
                Q.Workspace(dev))
        groups = [["q_proj", "k_proj", "v_proj"], ["o_proj"], ["gate_proj", "up_proj"], ["down_proj"]]
        assert sorted(n for g in groups for n in g) == sorted(layers)
        side = [torch.cuda.Stream(device=dev) for _ in range(3)]

        def fwd(name):
            case, qb, x, A, B, dy, y, T, dx, wsl = layers[name]
            Q.linear_fwd(qb, x, A, B, case.alpha, out=y, t_out=T, workspace=wsl)

        def bwd(name):
            case, qb, x, A, B, dy, y, T, dx, wsl = layers[name]
            Q.linear_bwd(qb, x, A, B, case.alpha, dy, t=T, dx=dx, workspace=wsl)

        def run_group(fn, group):
            if len(group) == 1:
                fn(group[0])
                return
            main = torch.cuda.current_stream()
            start = torch.cuda.Event()
            start.record(main)
            for st, name in zip(side, group):
                st.wait_event(start)
                with torch.cuda.stream(st):
                    fn(name)
            for st in side[:len(group)]:
                done = torch.cuda.Event()
                done.record(st)
                main.wait_event(done)

        def block_step():
            for g in groups:
                run_group(fwd, g)
            for g in reversed(groups):
                run_group(bwd, g)

        flops = sum(linear_flops(c.m, c.n, c.k, c.r) for c in WL.BLOCK)
        bsteps = max(3, min(args.steps, 10))
        ms, clk = time_steps_clocked(block_step, bsteps, 3, dev, flush=flush, barrier=barrier)
        tf = flops * bsteps / (ms * 1e-3) / 1e12
        peak, peak_name, why = choose_bf16_peak(pk, clk)
        out["decoder_block_7_targets_fwd_bwd"] = {
            "TFLOP/s": tf, "ms_per_block": ms / bsteps, "flops": flops, "frac_peak": tf / peak,
            "peak": peak, "peak_source": f"{pk_kind} {peak_name}: {why}",
            "method": "eager steps, L2 flushed before each; forward in layer order, backward in reverse; "
                      "q/k/v and gate/up on parallel streams"}
    return out


def cpu_baseline(case, seconds):
    """The oracle on this host's cores, on a bounded sample of the workload."""
    n_cores, threads = cpu_cores()
    m_sample = 256
    step, flops = oracle_step_sample(case, m_sample)
    t0 = time.perf_counter()
    step()
    one = time.perf_counter() - t0
    reps = max(1, int(seconds / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        step()
    dt = time.perf_counter() - t0
    return {"value": flops * reps / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{m_sample} of the 4096 tokens of the 11008x4096 r=64 layer: NF4 dequant of "
                      f"the whole weight + fp64 fwd+bwd on those tokens, {reps} reps "
                      f"({dt:.1f} s); NumPy fp64, BLAS threads={threads}, host cores={n_cores}, "
                      f"cpu={cpu_model()}"}


def profile_row(args):
    """Eager launches of one secondary row, for an ncu capture of its kernels:
    `warmup + steps` calls of each variant, no timing, no JSON line."""
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    from qlora_linear_layers_nf4_b200 import workloads as WL

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n = args.warmup + args.steps
    ws = Q.Workspace(dev)
    if args.profile_row in ("quantize", "dequantize"):
        w = torch.from_numpy(WL.draw_weight(WL.QUANT_SHAPE, WL.QUANT_SEED)).to(dev)
        if args.profile_row == "quantize":
            for _ in range(n):
                Q.quantize(w, 64, False, workspace=ws)
                Q.quantize(w, 64, True, workspace=ws)
        else:
            qs = [Q.quantize(w, 64, dq, workspace=ws) for dq in (False, True)]
            for _ in range(n):
                for q in qs:
                    Q.dequantize(q, "f32")
                    Q.dequantize(q, "bf16")
    elif args.profile_row == "merge":
        case = WL.PREFILL
        inp = WL.draw_linear(case)
        q = Q.quantize(torch.from_numpy(inp.w).to(dev), 64, True)
        A, B = bf16_dev(inp.a, dev), bf16_dev(inp.b, dev)
        for _ in range(n):
            Q.merge(q, A, B, case.alpha, "bf16", workspace=ws)
    elif args.profile_row == "f32":
        # the 11008x4096 layer, M = 4096, fwd + bwd in the F32 compute dtype:
        # per step six gemm_f32 launches (T, y, U, dB, dA, dx)
        case = WL.PREFILL
        inp = WL.draw_linear(case)
        q = Q.quantize(torch.from_numpy(inp.w).to(dev), 64, True)
        d32 = inp.extra["f32"]
        x, A, B, dy = (torch.from_numpy(d32[k]).to(dev) for k in ("x", "a", "b", "dy"))
        for _ in range(n):
            y, T = Q.linear_fwd(q, x, A, B, case.alpha, workspace=ws)
            Q.linear_bwd(q, x, A, B, case.alpha, dy, t=T, workspace=ws)
    elif args.profile_row == "decode":
        base = WL.DECODE[0]
        q = Q.quantize(torch.from_numpy(WL.draw_weight((base.n, base.k), seed=200)).to(dev), 64, True)
        for case in WL.DECODE:
            inp = WL.draw_linear(case)
            x, A, B = (bf16_dev(v, dev) for v in (inp.x, inp.a, inp.b))
            for _ in range(n):
                Q.linear_fwd(q, x, A, B, case.alpha, workspace=ws)
    torch.cuda.synchronize()
    if ws.read_status() != 0:
        raise RuntimeError("device status reported an error")
    print(f"profile_row {args.profile_row}: {Q.launch_count()} launches", flush=True)


# --------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from qlora_linear_layers_nf4_b200 import workloads as WL
    case = WL.PREFILL
    n_cores, threads = cpu_cores()
    m_sample = 128
    step, flops = oracle_step_sample(case, m_sample)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = (f"each step: NF4 dequant of the whole 11008x4096 weight + fp64 fwd+bwd on "
              f"{m_sample} of the 4096 tokens; NumPy, BLAS threads={threads}, host cores={n_cores}, "
              f"cpu={cpu_model()}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same recipe as our arm)",
        "config": {"workload": "QLoRA linear fwd+bwd, W 11008x4096 NF4 block 64 double-quant, "
                               "M=4096 tokens per GPU, r=64, alpha=16 (dA, dB, dx)",
                   "reference": "CPU oracle (oracle/nf4_oracle.py) on the host cores, bounded sample"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the secondary rows")
    ap.add_argument("--no-block", action="store_true", help="skip the decoder-block row")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile-row", choices=["quantize", "dequantize", "decode", "merge", "f32"],
                    help="only launch one secondary row eagerly (for ncu); no bench line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile_row:
        profile_row(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
