#!/usr/bin/env python
"""Benchmark: fused GEMM + bias (+ ReLU / GELU, + sign mask) TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one call of gemm_epi_run over one batch of seeded synthetic inputs
already resident in HBM: a single launch of the fused persistent kernel that
loads A and B tiles with TMA, multiplies on the tcgen05 tensor cores into
tensor memory, and finishes each tile (bias, activation, sign mask, rounding)
before its one store.  Throughput counts 2*m*n*k flops per step (epilogue
work is not counted).  Between timed steps the inputs rotate over enough
distinct buffer sets to exceed the 126 MB L2, so every step reads its
operands from HBM.

N > 1 (torchrun, one process per GPU): every rank runs its own independent
replica of the problem (weak scaling, no data-path collective); the timed
region is bracketed by a barrier and the slowest rank's time is used.

Printed on rank 0: one JSON line with the contract's keys plus ``roofline``
(dominant kernel vs. the measured tensor / HBM peak), ``cpu_baseline`` (the
fp64 oracle on the host cores, a bounded sample), ``e2e`` (host buffers,
copies inside the timed region), ``unfused`` (the library's own GEMM-then-
elementwise path), ``clocks`` and ``gpu_launches``.

``--impl reference`` times the CPU oracle itself, as it stands, on the same
workload and metric (bounded samples per step); under torchrun only rank 0
runs it.

``--mlp m,d_model,d_ff,dtype,act,layout`` times the MLP block instead (two
fused GEMMs per step, 4*m*d_model*d_ff flops; for e4m3 the up-projection's
epilogue requantises H, with s_H set from a first run's amax).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused GEMM+bias(+act) TFLOP/s on 1 B200 and % of dense tensor peak"
DEFAULT_WORKLOAD = "relu_aux_bias_bf16_4096x4096x4096"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0        # nominal dense ratio (4.5 / 2.25 PFLOP/s)
FP8_PEAK_NOTE = (", NOMINAL e4m3 peak: the measured bf16 burst x 2 (the dense fp8/bf16 ratio of the "
                 "spec); no e4m3 peak is measured")


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--shape", default=None,
                    help="custom problem m,n,k,dtype,epilogue,bias_axis,b_layout[,km] (overrides --workload; "
                         "operands N(0,1)/64, bias N(0,1), seed 0; km = A stored (k, m))")
    ap.add_argument("--kernel", default="auto", choices=["auto", "tc1", "tc2", "splitk"])
    ap.add_argument("--block-n", type=int, default=0)
    ap.add_argument("--stream-k", default="auto", choices=["auto", "off", "on"])
    ap.add_argument("--split-k", type=int, default=0,
                    help="split-K kernel: CTAs per cluster along k; TC kernels: parts per tail tile "
                         "(0 = the plan's choice)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: target CPU time of the whole warm-up + timed run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-unfused", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps directly instead of replaying them from a CUDA graph")
    ap.add_argument("--mlp", default=None,
                    help="time the MLP block m,d_model,d_ff,dtype,act,layout instead of one GEMM")
    ap.add_argument("--warm-l2", action="store_true",
                    help="one input set reused every step (L2-warm); the default rotates sets beyond L2")
    ap.add_argument("--clock-window", type=float, default=0.5,
                    help="seconds of back-to-back replays of the timed steps, right after the timed "
                         "region, over which the SM clock is sampled (0 = the timed region only)")
    ap.add_argument("--cublas", action="store_true",
                    help="also time cuBLAS's bare GEMM (torch.matmul, no epilogue) at this shape, "
                         "as context only (16-bit workloads)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured (MEASURED_PEAKS.json)"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback (profiling recipe)"


def kernel_source_hash():
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "activation_epilogue_tcgen05_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:12]


def recorded_traffic(workload: str, kernel_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == workload \
                    and parts[1] == kernel_hash:
                return int(parts[2])
    return None


class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) over a window."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 50):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 f"-lms={period_ms}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 10:
                self.samples.append((time.time(), parts))

    def wait_first(self, timeout=10.0):
        t0 = time.time()
        while self.proc and not self.samples and time.time() - t0 < timeout:
            time.sleep(0.05)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        win = [p for (t, p) in self.samples if t0 - 0.1 <= t <= t1 + 0.1]
        if len(win) < 3:                      # short region: nearest samples around it
            near = sorted(self.samples, key=lambda s: abs(s[0] - (t0 + t1) / 2))[:5]
            win = [p for (_, p) in near]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(p[2]) for p in win if num(p[2]) is not None]
        mx = [num(p[3]) for p in win if num(p[3]) is not None]
        power = [num(p[4]) for p in win if num(p[4]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in win for i in range(4) if p[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "power_w_max": max(power) if power else None, "samples": len(win)}


def hold_clock_window(replay, region_s: float, hold_s: float, stream, device):
    """Repeat ``replay`` (the timed region's work) back to back for about ``hold_s`` seconds.

    The timed region of a short workload lasts a few milliseconds, shorter than the clock
    sampler's period, so its clock is read over this longer window of the same launches
    instead.  Returns (replays, device seconds, wall-clock end)."""
    import torch
    reps = max(1, min(100000, math.ceil(hold_s / max(region_s, 1e-6))))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        replay()
    b.record(stream)
    torch.cuda.synchronize(device)
    return reps, a.elapsed_time(b) / 1000.0, time.time()


def clock_record(sampler, wall0, wall1, window, flops_per_region, value):
    """The clock block of the JSON line.

    ``sm_mhz`` etc. summarise the samples over the timed region and the back-to-back window
    after it (``hold_clock_window``).  A timed region of a few milliseconds holds at most one
    sampler period, so ``timed_region`` gives its own samples (often none) and ``window`` the
    window's throughput, its own median clock and their ratio (work per clock cycle at the
    clock the power cap settles to)."""
    if sampler is None:
        return None
    if window is None:
        return sampler.summary(wall0, wall1)
    reps, secs, wall2 = window
    rec = sampler.summary(wall0, wall2)
    inside = [p for (t, p) in sampler.samples if wall0 <= t <= wall1]
    rec["timed_region"] = {"samples": len(inside), "value": value}
    if inside:
        mhz = [float(p[2]) for p in inside if p[2].replace(".", "", 1).isdigit()]
        if mhz:
            rec["timed_region"]["sm_mhz"] = statistics.median(mhz)
    w = {"seconds": secs, "replays_of_timed_region": reps,
         "value": flops_per_region * reps / secs / 1e12, "unit": "TFLOP/s",
         "what": "the timed region's launches replayed back to back right after it"}
    ws = [p for (t, p) in sampler.samples if wall1 <= t <= wall2]
    wm = [float(p[2]) for p in ws if p[2].replace(".", "", 1).isdigit()]
    w["samples"] = len(wm)
    if wm:
        w["sm_mhz"] = statistics.median(wm)
        w["value_per_ghz"] = w["value"] / (w["sm_mhz"] / 1000.0)
    rec["window"] = w
    return rec


def workload_from_args(args):
    from activation_epilogue_tcgen05_b200.workloads import WORKLOADS, Workload
    if not args.shape:
        return WORKLOADS[args.workload]
    parts = args.shape.split(",")
    m, n, k, dt, epi, axis, lay = parts[:7]
    a_lay = parts[7] if len(parts) > 7 else "mk"
    std = 1.0 if dt == "e4m3" else 1.0 / 64
    name = f"custom_{dt}_{epi}_{m}x{n}x{k}_{lay}" + ("_at" if a_lay == "km" else "")
    return Workload(name, int(m), int(n), int(k), dt, epi, axis, lay,
                    ("normal", std), ("normal", std), ("normal", 1.0), a_layout=a_lay)


# ----------------------------------------------------------------------------- CPU oracle legs
def oracle_rows_rate(wl, prob, target_s: float, max_rows=None):
    """Time the oracle (as it stands) on the first R rows of the workload; R sized to ~target_s.

    Returns (TFLOP/s, rows, seconds, threads)."""
    import numpy as np
    import oracle
    from activation_epilogue_tcgen05_b200.workloads import storage

    from activation_epilogue_tcgen05_b200.workloads import make_mask

    Bs = storage(prob.B)
    bias_full = storage(prob.bias)
    bwd = wl.epilogue in ("drelu", "drelu_bgrad")

    # the oracle reads A as (m, k); an A stored (k, m) is handed over row by row of its transpose
    A_mk = prob.A.t() if wl.a_layout == "km" else prob.A

    def run(rows):
        As = storage(A_mk[:rows].contiguous())
        bias = bias_full[:rows] if wl.bias_axis == "row" else bias_full
        t0 = time.perf_counter()
        if bwd:
            oracle.gemm_epi_bwd(As, Bs, make_mask(rows, wl.n, seed=wl.seed), dtype=wl.dtype,
                                epilogue=wl.epilogue, bias_axis=wl.bias_axis, b_layout=wl.b_layout,
                                scale_a=prob.scale_a, scale_b=prob.scale_b)
        else:
            oracle.gemm_epi(As, Bs, bias, dtype=wl.dtype, epilogue=wl.epilogue, bias_axis=wl.bias_axis,
                            b_layout=wl.b_layout, scale_a=prob.scale_a, scale_b=prob.scale_b)
        return time.perf_counter() - t0

    threads = oracle.threads()
    cap = wl.m if max_rows is None else min(wl.m, max_rows)
    rows = min(cap, max(1, threads))
    run(rows)                      # warm-up (thread start-up, first touch), not timed
    dt = run(rows)
    # grow the sample towards target_s (a few rounds: the first timings are the noisiest)
    for _ in range(4):
        if dt >= 0.8 * target_s or rows >= cap:
            break
        rows = int(min(cap, max(rows + 1, rows * target_s / max(dt, 1e-6))))
        dt = run(rows)
    flops = 2.0 * rows * wl.n * wl.k
    return flops / dt / 1e12, rows, dt, threads


def reference_arm(args):
    """--impl reference: the fp64 CPU oracle as it stands, on this workload."""
    from activation_epilogue_tcgen05_b200 import replicas
    rank, world, _ = replicas.env_rank()
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    from activation_epilogue_tcgen05_b200.workloads import make_problem, storage
    wl = workload_from_args(args)
    gen_dev = "cpu"
    if wl.m * wl.k > (1 << 28):              # very large operands: draw only what the samples need
        wl_small = wl.with_(m=min(wl.m, 4096))
        prob = make_problem(wl_small, device=gen_dev)
    else:
        prob = make_problem(wl, device=gen_dev)
    As = storage((prob.A.t() if wl.a_layout == "km" else prob.A).contiguous())      # (m, k) for the oracle
    Bs, bias = storage(prob.B), storage(prob.bias)
    m_avail = As.shape[0]
    rng = np.random.default_rng(0)

    bwd = wl.epilogue in ("drelu", "drelu_bgrad")
    if bwd:
        from activation_epilogue_tcgen05_b200.workloads import make_mask
        mask_full = make_mask(m_avail, wl.n, seed=wl.seed)

    def step(count):
        t0 = time.perf_counter()
        if bwd:     # backward: `count` whole output rows (mask, D row and its dbias share)
            r0 = int(rng.integers(0, max(1, m_avail - count + 1)))
            oracle.gemm_epi_bwd(As[r0:r0 + count], Bs, mask_full[r0:r0 + count], dtype=wl.dtype,
                                epilogue=wl.epilogue, bias_axis=wl.bias_axis, b_layout=wl.b_layout,
                                scale_a=prob.scale_a, scale_b=prob.scale_b)
            return time.perf_counter() - t0
        rows = rng.integers(0, m_avail, count)
        cols = rng.integers(0, wl.n, count)
        oracle.gemm_epi_sampled(As, Bs, bias if wl.bias_axis == "col" else bias[:m_avail], rows, cols,
                                dtype=wl.dtype, epilogue=wl.epilogue, bias_axis=wl.bias_axis,
                                b_layout=wl.b_layout, scale_a=prob.scale_a, scale_b=prob.scale_b)
        return time.perf_counter() - t0

    threads = oracle.threads()
    # size one step so that warmup + steps take about --ref-seconds (a minute) in total
    per_unit = wl.n if bwd else 1          # output positions per counted unit (row or position)
    probe = max(threads, 1) if bwd else max(threads * 4, 64)
    t_probe = step(probe)
    per_pos = t_probe / probe
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    count = int(max(threads if not bwd else 1, min((1 << 20) // per_unit, budget / max(per_pos, 1e-9))))
    count = min(count, m_avail) if bwd else count
    for _ in range(args.warmup):
        step(count)
    total = 0.0
    for _ in range(args.steps):
        total += step(count)
    flops = 2.0 * wl.k * count * per_unit * args.steps
    value = flops / total / 1e12
    sample = (f"{count} consecutive seeded output rows per step (backward oracle, all {wl.n} columns)" if bwd
              else f"{count} seeded output positions per step (one fp64 dot product of length k each)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "m": wl.m, "n": wl.n, "k": wl.k, "dtype": wl.dtype,
                   "epilogue": wl.epilogue, "bias_axis": wl.bias_axis, "b_layout": wl.b_layout},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def mlp_arm(args):
    """The MLP block (gemm_epi_mlp_run): H = act(X.W1 + b1), Y = H.W2 + b2 per step."""
    import torch
    from activation_epilogue_tcgen05_b200 import gemm_epi as g
    from activation_epilogue_tcgen05_b200 import replicas
    from activation_epilogue_tcgen05_b200.workloads import TORCH_DTYPE, Workload, make_problem

    rank, world, local_rank = replicas.env_rank()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback exists)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    have_pg = replicas.init("nccl", timeout_s=120, device_id=dev)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    m, dm, dff, dt, act, lay = args.mlp.split(",")
    m, dm, dff = int(m), int(dm), int(dff)
    std = 1.0 if dt == "e4m3" else 1.0 / 64
    up = Workload("mlp_up", m, dff, dm, dt, act, "col", lay, ("normal", 1.0), ("normal", std), ("normal", 0.1))
    down = Workload("mlp_down", m, dm, dff, dt, "bias", "col", lay, ("normal", 1.0), ("normal", std),
                    ("normal", 0.1), seed=1)
    big = m * dm > (1 << 28)
    pu, pd = make_problem(up, device="cuda" if big else "cpu"), make_problem(down, device="cuda")
    X, W1, b1 = pu.A.to(dev), pu.B.to(dev), pu.bias.to(dev)
    W2, b2 = pd.B.to(dev), pd.bias.to(dev)
    h_t = torch.uint8 if dt == "e4m3" else TORCH_DTYPE[dt]
    H = torch.empty((m, dff), dtype=h_t, device=dev)
    Y = torch.empty((m, dm), dtype=TORCH_DTYPE[up.out_dtype], device=dev)
    mp = g.MlpPlan(m, dm, dff, dt, act, lay)
    stream = torch.cuda.current_stream(dev)
    if dt == "e4m3":
        f32 = lambda v: torch.tensor([v], dtype=torch.float32, device=dev)
        s_x, s_w1, s_w2 = f32(pu.scale_a), f32(pu.scale_b), f32(pd.scale_b)
        s_h, amax = f32(1.0), f32(0.0)
        mp.set_scales(s_x, s_w1, s_h, amax, s_w2)
        mp.run(X, W1, b1, W2, b2, H, Y, stream=stream)        # delayed scaling: s_H from this amax
        torch.cuda.synchronize(dev)
        s_h.copy_(amax / 448.0)
    t0 = time.perf_counter()
    mp.run(X, W1, b1, W2, b2, H, Y, stream=stream)
    torch.cuda.synchronize(dev)
    first_call_ms = 1000 * (time.perf_counter() - t0)
    mp.check(stream)
    for _ in range(args.warmup):
        mp.run(X, W1, b1, W2, b2, H, Y, stream=stream)
    torch.cuda.synchronize(dev)
    mp.check(stream)
    if sampler:
        sampler.wait_first()
    K = args.steps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cs = torch.cuda.current_stream(dev)
        for _ in range(K):
            mp.run(X, W1, b1, W2, b2, H, Y, stream=cs)
    graph.replay()
    torch.cuda.synchronize(dev)
    replicas.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    start.record(stream)
    graph.replay()
    end.record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    region_ms = start.elapsed_time(end)
    window = (hold_clock_window(graph.replay, region_ms / 1000.0, args.clock_window, stream, dev)
              if args.clock_window > 0 else None)
    replicas.barrier()
    mp.check(stream)
    del graph
    elapsed_ms = replicas.max_over_ranks(region_ms, device=dev)
    flops = 4.0 * m * dm * dff
    value = flops * world * K / (elapsed_ms / 1000.0) / 1e12
    clocks = clock_record(sampler, wall0, wall1, window, flops * K, value / world)
    # the library's own unfused sequence: bare GEMM, bias + activation kernel, (e4m3) amax and
    # quantise passes over a bf16 H, bare GEMM, bias kernel
    unfused = None
    if not args.no_unfused:
        Hw = torch.empty((m, dff), dtype=torch.bfloat16, device=dev) if dt == "e4m3" else None
        for _ in range(3):
            mp.run(X, W1, b1, W2, b2, H, Y, stream=stream, fused=False, H_wide=Hw)
        torch.cuda.synchronize(dev)
        Ku = K                      # as many steps as the fused leg: the same clock regime
        ugraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ugraph):
            cs = torch.cuda.current_stream(dev)
            for _ in range(Ku):
                mp.run(X, W1, b1, W2, b2, H, Y, stream=cs, fused=False, H_wide=Hw)
        ugraph.replay()
        torch.cuda.synchronize(dev)
        u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        uw0 = time.time()
        u0.record(stream)
        ugraph.replay()
        u1.record(stream)
        torch.cuda.synchronize(dev)
        uw1 = time.time()
        u_region_ms = u0.elapsed_time(u1)
        uwin = (hold_clock_window(ugraph.replay, u_region_ms / 1000.0, args.clock_window, stream, dev)
                if args.clock_window > 0 else None)
        mp.check(stream)
        del ugraph
        ums = replicas.max_over_ranks(u_region_ms, device=dev) / Ku
        uclk = clock_record(sampler, uw0, uw1, uwin, flops * Ku, flops / (ums / 1000) / 1e12)
        unfused = {"ms_per_step": ums, "value": 4.0 * m * dm * dff * world / (ums / 1000) / 1e12,
                   "unit": "TFLOP/s", "steps": Ku, "launches_per_step": 6 if dt == "e4m3" else 4,
                   "fused_speedup": ums / (elapsed_ms / K), "clocks": uclk}
        f_mhz, u_mhz = (clocks or {}).get("sm_mhz"), (uclk or {}).get("sm_mhz")
        if f_mhz and u_mhz:
            unfused["fused_speedup_equal_clock"] = (ums * u_mhz) / ((elapsed_ms / K) * f_mhz)
    if sampler:
        sampler.stop()
    peaks, peak_src = load_peaks()
    peak = peaks["bf16_tflops"] * (FP8_OVER_BF16 if dt == "e4m3" else 1.0)
    achieved = flops / (elapsed_ms / K / 1000.0) / 1e12
    up_info, down_info = mp.info
    mp.close()
    if rank == 0:
        esz = 1 if dt == "e4m3" else 2
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dt, "data": "synthetic",
            "config": {"workload": f"mlp_{dt}_{act}_{m}x{dm}x{dff}_{lay}", "m": m, "d_model": dm, "d_ff": dff,
                       "dtype": dt, "act": act, "w_layout": lay, "parallelism": f"replicas x{world}",
                       "plans": {"up": up_info, "down": down_info}, "first_call_ms": first_call_ms,
                       "l2": f"one set: X, W1, W2, H, Y = {((m * dm + 2 * dm * dff) * esz + m * dff * esz + m * dm * 2) / 2**20:.0f} MiB",
                       "launch": "CUDA graph of the K steps (two kernel launches each)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": peak_src + (FP8_PEAK_NOTE if dt == "e4m3" else ", bf16 burst"),
                         "note": "per-step time of both GEMM launches"},
            "cpu_baseline": None, "e2e": None, "unfused": unfused, "gpu_launches": 2 * K, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if have_pg:
        replicas.barrier()
        replicas.finalize()
    return 0


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        return reference_arm(args)
    if args.mlp:
        return mlp_arm(args)

    import torch
    from activation_epilogue_tcgen05_b200 import gemm_epi as g
    from activation_epilogue_tcgen05_b200 import replicas
    from activation_epilogue_tcgen05_b200.workloads import (TORCH_DTYPE, WORKLOADS, make_mask, make_problem,
                                                            pack_mask)

    rank, world, local_rank = replicas.env_rank()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback exists)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    have_pg = replicas.init("nccl", timeout_s=120, device_id=dev)
    sampler = ClockSampler(local_rank) if rank == 0 else None

    wl = workload_from_args(args)
    out_t = TORCH_DTYPE[wl.out_dtype]
    big = wl.m * wl.k > (1 << 28)
    prob = make_problem(wl, device="cuda" if big else "cpu")
    A0, B0 = prob.A.to(dev), prob.B.to(dev)
    # Each step's arguments are (A, B, x, D, y): forward x = bias, y = aux mask (written);
    # backward x = the packed forward mask (read), y = dbias (written)
    bwd = wl.epilogue in g.BACKWARD
    if bwd:
        import numpy as np
        x0 = torch.from_numpy(pack_mask(make_mask(wl.m, wl.n, seed=wl.seed)).view(np.int32)).to(dev)
        y_shape, y_dtype = ((wl.m if wl.bias_axis == "row" else wl.n,), out_t) \
            if wl.epilogue == "drelu_bgrad" else (None, None)
    else:
        x0 = prob.bias.to(dev)
        aux_words = wl.m * g.aux_pitch_words(wl.n) if wl.epilogue in g.HAS_AUX else 0
        y_shape, y_dtype = ((aux_words,), torch.int32) if aux_words else (None, None)

    def new_y():
        return torch.empty(y_shape, dtype=y_dtype, device=dev) if y_shape else None

    y_bytes = (math.prod(y_shape) * torch.empty((), dtype=y_dtype).element_size()) if y_shape else 0
    esz = 1 if wl.dtype == "e4m3" else 2
    in_bytes = (wl.m * wl.k + wl.k * wl.n) * esz + x0.numel() * x0.element_size()
    out_bytes = wl.m * wl.n * 2 + y_bytes
    set_bytes = in_bytes + out_bytes
    n_sets = 1 if (set_bytes > 2 * L2_BYTES or args.warm_l2) else max(2, math.ceil(3 * L2_BYTES / set_bytes))
    # launches per step: the GEMM (+ the dbias reduction); unfused: + the elementwise pass (+ the sums)
    launches = 2 if wl.epilogue == "drelu_bgrad" else 1
    launches_unfused = 3 if wl.epilogue == "drelu_bgrad" else 2

    sets = []
    for i in range(n_sets):
        A = A0 if i == 0 else A0.clone()
        B = B0 if i == 0 else B0.clone()
        x = x0 if i == 0 else x0.clone()
        D = torch.empty((wl.m, wl.n), dtype=out_t, device=dev)
        sets.append((A, B, x, D, new_y()))
    plan = g.Plan(wl.m, wl.n, wl.k, wl.dtype, wl.epilogue, wl.bias_axis, wl.b_layout,
                  kernel=args.kernel, block_n=args.block_n, stream_k=args.stream_k, split_k=args.split_k,
                  a_layout=wl.a_layout)
    run = plan.run_bwd if bwd else plan.run
    if wl.dtype == "e4m3":
        plan.set_scales(torch.tensor([prob.scale_a], dtype=torch.float32, device=dev),
                        torch.tensor([prob.scale_b], dtype=torch.float32, device=dev))
    info = plan.info
    stream = torch.cuda.current_stream(dev)
    flops = 2.0 * wl.m * wl.n * wl.k

    # first call (tensor-map encode) timed apart from the steady state
    t0 = time.perf_counter()
    run(*sets[0], stream=stream)
    torch.cuda.synchronize(dev)
    first_call_ms = 1000 * (time.perf_counter() - t0)
    plan.check(stream)

    for i in range(args.warmup):
        run(*sets[i % n_sets], stream=stream)
    torch.cuda.synchronize(dev)
    plan.check(stream)
    if sampler:
        sampler.wait_first()

    K = args.steps
    use_graph = not args.no_graph

    def capture(fused: bool, count: int):
        """The count steps (one launch each) captured into a CUDA graph."""
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cs = torch.cuda.current_stream(dev)
            for i in range(count):
                run(*sets[i % n_sets], stream=cs, fused=fused)
        return graph

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if use_graph:
        graph = capture(True, K)
        graph.replay()                          # upload / first replay, untimed
        torch.cuda.synchronize(dev)
        plan.check(stream)
        replicas.barrier()
        torch.cuda.synchronize(dev)
        wall0 = time.time()
        start.record(stream)
        graph.replay()
        end.record(stream)
        torch.cuda.synchronize(dev)
        wall1 = time.time()
        elapsed_ms = start.elapsed_time(end)
        window = (hold_clock_window(graph.replay, elapsed_ms / 1000.0, args.clock_window, stream, dev)
                  if args.clock_window > 0 else None)
        replicas.barrier()
        plan.check(stream)
        # launches replay back to back: the average launch lasts the region over K
        avg_launch_s = elapsed_ms / K / 1000.0
        del graph
    else:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        replicas.barrier()
        torch.cuda.synchronize(dev)
        wall0 = time.time()
        start.record(stream)
        for i in range(K):
            ev[i][0].record(stream)
            run(*sets[i % n_sets], stream=stream)
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
        wall1 = time.time()
        elapsed_ms = start.elapsed_time(end)

        def direct_steps():
            for i in range(K):
                run(*sets[i % n_sets], stream=stream)
        window = (hold_clock_window(direct_steps, elapsed_ms / 1000.0, args.clock_window, stream, dev)
                  if args.clock_window > 0 else None)
        replicas.barrier()
        plan.check(stream)
        avg_launch_s = statistics.fmean(a.elapsed_time(b) for a, b in ev) / 1000.0
    elapsed_ms_max = replicas.max_over_ranks(elapsed_ms, device=dev)

    value = flops * world * K / (elapsed_ms_max / 1000.0) / 1e12
    ms_per_step = elapsed_ms_max / K
    clocks = clock_record(sampler, wall0, wall1, window, flops * K, value / world)

    # ---- roofline of the dominant (only) kernel: one launch per step
    peaks, peak_src = load_peaks()
    khash = kernel_source_hash()
    traffic = recorded_traffic(wl.name, khash)
    if info["kernel"] == g.KERNEL_SPLITK:
        alg_bytes = in_bytes + out_bytes
        achieved = alg_bytes / avg_launch_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "algorithmic_bytes": alg_bytes, "peak_source": peak_src + ", hbm copy"}
    else:
        peak = peaks["bf16_tflops"] * (FP8_OVER_BF16 if wl.dtype == "e4m3" else 1.0)
        achieved = flops / avg_launch_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "algorithmic_bytes": in_bytes + out_bytes,
                "peak_source": peak_src + (FP8_PEAK_NOTE if wl.dtype == "e4m3" else ", bf16 burst")}
    roof["kernel_source"] = khash
    if launches > 1:
        roof["note"] = "per-step time: the GEMM launch plus the dbias reduction launch"

    # ---- the library's own unfused path (bare GEMM, then the elementwise kernel)
    unfused = None
    if not args.no_unfused and wl.epilogue != "none":
        # long enough for the clock sampler to see it: under the power cap the two sequences
        # run at different clocks (the elementwise pass lowers the average power)
        Ku = min(K, 2000)
        for i in range(3):
            run(*sets[i % n_sets], stream=stream, fused=False)
        torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        def unfused_steps():
            for i in range(Ku):
                run(*sets[i % n_sets], stream=stream, fused=False)
        if use_graph:
            ugraph = capture(False, Ku)
            ugraph.replay()
            torch.cuda.synchronize(dev)
            uw0 = time.time()
            s0.record(stream)
            ugraph.replay()
            s1.record(stream)
        else:
            uw0 = time.time()
            s0.record(stream)
            unfused_steps()
            s1.record(stream)
        torch.cuda.synchronize(dev)
        uw1 = time.time()
        u_region_ms = s0.elapsed_time(s1)
        uwin = (hold_clock_window(ugraph.replay if use_graph else unfused_steps, u_region_ms / 1000.0,
                                  args.clock_window, stream, dev) if args.clock_window > 0 else None)
        if use_graph:
            del ugraph
        plan.check(stream)
        ums = replicas.max_over_ranks(u_region_ms, device=dev) / Ku
        uclk = clock_record(sampler, uw0, uw1, uwin, flops * Ku, flops / (ums / 1000) / 1e12)
        unfused = {"ms_per_step": ums, "value": flops * world / (ums / 1000) / 1e12, "unit": "TFLOP/s",
                   "steps": Ku, "launches_per_step": launches_unfused, "fused_speedup": ums / ms_per_step,
                   "clocks": uclk}
        f_mhz, u_mhz = (clocks or {}).get("sm_mhz"), (uclk or {}).get("sm_mhz")
        if f_mhz and u_mhz:
            # the same comparison at equal SM clocks (time x clock: cycles per step)
            unfused["fused_speedup_equal_clock"] = (ums * u_mhz) / (ms_per_step * f_mhz)

    # ---- end to end through the public API with host buffers: every step copies its inputs
    # from pinned host memory and reads its result back; copies of neighbouring steps overlap
    # the compute (H2D, compute and D2H on three streams, two device buffer sets)
    e2e = None
    if not args.no_e2e:
        Ke = min(K, 50)
        hA = torch.empty(A0.shape, dtype=A0.dtype, pin_memory=True)
        hB = torch.empty(B0.shape, dtype=B0.dtype, pin_memory=True)
        hx = torch.empty(x0.shape, dtype=x0.dtype, pin_memory=True)
        hA.copy_(A0)
        hB.copy_(B0)
        hx.copy_(x0)
        e_sets = [sets[0], sets[1] if n_sets > 1 else (
            torch.empty_like(A0), torch.empty_like(B0), torch.empty_like(x0),
            torch.empty((wl.m, wl.n), dtype=out_t, device=dev), new_y())]
        hD = [torch.empty((wl.m, wl.n), dtype=out_t, pin_memory=True) for _ in range(2)]
        hy = [torch.empty(y_shape, dtype=y_dtype, pin_memory=True) if y_shape else None for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(count, t_start=None, t_end=None):
            used = [False, False]
            for i in range(count):
                j = i % 2
                A, B, x, D, y = e_sets[j]
                with torch.cuda.stream(h2d_s):
                    if i == 0 and t_start is not None:
                        t_start.record(h2d_s)
                    if used[j]:
                        h2d_s.wait_event(ev_comp[j])      # step i-2 has finished reading set j
                    A.copy_(hA, non_blocking=True)
                    B.copy_(hB, non_blocking=True)
                    x.copy_(hx, non_blocking=True)
                    ev_in[j].record(h2d_s)
                stream.wait_event(ev_in[j])
                if used[j]:
                    stream.wait_event(ev_out[j])          # step i-2's result has been read back
                run(A, B, x, D, y, stream=stream)
                ev_comp[j].record(stream)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(ev_comp[j])
                    hD[j].copy_(D, non_blocking=True)
                    if y is not None:
                        hy[j].copy_(y, non_blocking=True)
                    ev_out[j].record(d2h_s)
                used[j] = True
            if t_end is not None:
                t_end.record(d2h_s)

        e2e_steps(2)
        torch.cuda.synchronize(dev)
        replicas.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps(Ke, s0, s1)
        torch.cuda.synchronize(dev)
        plan.check(stream)
        ems = replicas.max_over_ranks(s0.elapsed_time(s1), device=dev) / Ke
        e2e = {"value": flops * world / (ems / 1000) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(in_bytes), "d2h_bytes_per_step": int(out_bytes),
               "ms_per_step": ems, "steps": Ke,
               "api": f"{'gemm_epi_run_bwd' if bwd else 'gemm_epi_run'} (C ABI) with pinned host buffers; "
                      "H2D, compute and D2H of "
                      "neighbouring steps overlap on three streams"}

    # ---- context only: the vendor library's bare GEMM (no bias, no activation) at this shape
    cublas = None
    if args.cublas and wl.dtype in ("f16", "bf16"):
        Bt = B0 if wl.b_layout == "kn" else B0.t()
        outc = torch.empty((wl.m, wl.n), dtype=out_t, device=dev)
        for _ in range(5):
            torch.matmul(A0, Bt, out=outc)
        Kc = min(K, 500)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        c0.record(stream)
        for _ in range(Kc):
            torch.matmul(A0, Bt, out=outc)
        c1.record(stream)
        torch.cuda.synchronize(dev)
        cms = c0.elapsed_time(c1) / Kc
        cublas = {"value": flops / (cms / 1000) / 1e12, "unit": "TFLOP/s", "ms_per_step": cms,
                  "steps": Kc, "what": "torch.matmul (cuBLAS) bare GEMM, same operands, L2-warm"}

    if sampler:
        sampler.stop()

    # ---- CPU oracle baseline: rank 0, N = 1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if big:
            prob_cpu = make_problem(wl.with_(m=min(wl.m, 2048)), device="cpu")
        else:
            prob_cpu = make_problem(wl, device="cpu")
        tf, rows, secs, threads = oracle_rows_rate(wl, prob_cpu, args.cpu_seconds,
                                                   max_rows=prob_cpu.A.shape[0])
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"first {rows} of {wl.m} output rows, all {wl.n} columns ({secs:.1f} s; "
                         f"fp64, OpenMP over rows)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "m": wl.m, "n": wl.n, "k": wl.k, "dtype": wl.dtype,
                       "out_dtype": wl.out_dtype, "epilogue": wl.epilogue, "bias_axis": wl.bias_axis,
                       "b_layout": wl.b_layout, "parallelism": f"replicas x{world}",
                       "l2": (f"inputs rotate over {n_sets} buffer sets ({n_sets * set_bytes / 2**20:.0f} MiB"
                              f" > 126 MB L2)" if n_sets > 1 else
                              (f"warm: one set of {set_bytes / 2**20:.0f} MiB reused every step"
                               if args.warm_l2 and set_bytes <= 2 * L2_BYTES else
                               f"one set of {set_bytes / 2**20:.0f} MiB > 126 MB L2")),
                       "plan": info, "first_call_ms": first_call_ms,
                       "launch": "CUDA graph of the K steps (one kernel launch each)" if use_graph
                       else "direct launches",
                       "pdl": os.environ.get("GEMM_EPI_PDL", "1")[:1] != "0"},
            "pct_of_peak": 100.0 * roof["frac"],
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "unfused": unfused,
            "gpu_launches": K * launches, "clocks": clocks,
        }
        if cublas is not None:
            line["cublas_bare_gemm"] = cublas
        print(json.dumps(line), flush=True)
    plan.close()
    if have_pg:
        replicas.barrier()
        replicas.finalize()
    return 0


if __name__ == "__main__":
    sys.exit(main())
