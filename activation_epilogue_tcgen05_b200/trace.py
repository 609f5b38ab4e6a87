"""Per-stage timelines of the kernels from a tracing build of the library.

    python -m activation_epilogue_tcgen05_b200.trace build
    python -m activation_epilogue_tcgen05_b200.trace run --workload NAME [--launches N] [--graph]

``build`` compiles the library with ``-DGEMM_EPI_TRACE=2`` into ``libgemm_epi_trace.so`` beside
the shipped library (which is untouched: its tracing code compiles to nothing).  In that build every role of the
persistent and small-m kernels records, per ring stage and per tile, a pair of 64-bit words
(%globaltimer, SM clock | event | tile | k-block) into a per-launch slot of a device buffer.
``run`` times a few launches of one workload (``bench.py``'s names) with that build, reads
the buffer back through ``gemm_epi_trace_read`` and prints a summary:

* persistent kernels: for every CTA, the latency from a stage's load issue (producer) to the
  MMA issuer passing its full barrier (same SM clock), the MMA issuer's period between stages,
  and its wait for a free accumulator;
* small-m kernels: per launch, the time from the dependency release (griddepcontrol.wait) to
  the first stage, to the last MMA and to the last CTA's exit, and the release-to-release period.

Tracing perturbs what it measures (two global stores per record); compare traced runs with
traced runs.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
TRACE_DIR = os.path.join(ROOT, "_build", "trace")                  # objects
TRACE_LIB = os.path.join(PKG, "libgemm_epi_trace.so")

# record layout (gemm_tc.cuh: trace_stage)
ROLE_CAP = 256
LAUNCH_RECS = 256 * 4 * ROLE_CAP
TRACE_CAP = 1 << 22
EV = {10: "CTA start", 11: "after the dependency wait", 20: "stage load issued", 22: "stage ready (MMA)",
      23: "last MMA issued", 24: "accumulator wait", 25: "accumulator free", 26: "accumulator ready",
      27: "epilogue piece done", 28: "partials received", 29: "CTA end", 30: "finisher: flags seen",
      31: "finisher: partials added", 32: "publisher: flag raised", 33: "unit's partials added",
      34: "unit's outputs stored"}


def build(force: bool = False) -> str:
    from activation_epilogue_tcgen05_b200 import build as b
    b.BUILD = os.path.join(TRACE_DIR, "obj")
    b.LIB = TRACE_LIB
    b.NVCC_FLAGS = b.NVCC_FLAGS[:-4] + ["-DGEMM_EPI_TRACE=2"] + b.NVCC_FLAGS[-4:]
    return b.build(force=force)


def _launches(t, w):
    import numpy as np
    out = []
    for sl in range(len(t) // LAUNCH_RECS):
        tt = t[sl * LAUNCH_RECS:(sl + 1) * LAUNCH_RECS]
        ww = w[sl * LAUNCH_RECS:(sl + 1) * LAUNCH_RECS]
        nz = np.nonzero(tt)[0]
        if len(nz) == 0:
            continue
        region = nz // ROLE_CAP
        out.append(dict(gt=tt[nz].astype(np.int64), cta=region // 4, role=region % 4,
                        clk=(ww[nz] >> np.uint64(32)).astype(np.int64),
                        ev=((ww[nz] >> np.uint64(24)) & np.uint64(0xFF)).astype(np.int64),
                        tile=((ww[nz] >> np.uint64(16)) & np.uint64(0xFF)).astype(np.int64),
                        kb=(ww[nz] & np.uint64(0xFFFF)).astype(np.int64)))
    return out


def _pct(x, qs=(10, 50, 90)):
    import numpy as np
    x = np.asarray(x, dtype=np.float64)
    if not len(x):
        return "n/a"
    fmt = "{:.0f}" if np.abs(x).max() >= 100 else "{:.2f}"
    return " / ".join(fmt.format(np.percentile(x, q)) for q in qs)


def summarise_persistent(launches, last=3):
    import numpy as np
    lines = []
    for L in launches[-last:]:
        lat, per, accw = [], [], []
        for c in np.unique(L["cta"]):
            sel = lambda **kw: np.logical_and.reduce([L["cta"] == c] + [L[k] == v for k, v in kw.items()])
            p, mm = sel(role=0, ev=20), sel(role=1, ev=22)
            if p.any() and mm.any():
                issued = {(int(a), int(b)): int(t) for a, b, t in zip(L["tile"][p], L["kb"][p], L["clk"][p])}
                for a, b, t in zip(L["tile"][mm], L["kb"][mm], L["clk"][mm]):
                    if (int(a), int(b)) in issued:
                        lat.append((int(t) - issued[(int(a), int(b))]) & 0xFFFFFFFF)
                per.extend(np.diff(np.sort(L["clk"][mm])).tolist())
            w0, w1 = L["clk"][sel(role=1, ev=24)], L["clk"][sel(role=1, ev=25)]
            if len(w0) == len(w1):
                accw.extend((w1 - w0).tolist())
        span = (L["gt"].max() - L["gt"].min()) / 1e3
        lines.append(f"launch span {span:.2f} us")
        # phases against the launch's first record (global timer, ns): first stage ready, last
        # stage ready, last epilogue record, per CTA
        g0 = L["gt"].min()
        first_ready, last_ready, last_epi = [], [], []
        for c in np.unique(L["cta"]):
            mm = (L["cta"] == c) & (L["role"] == 1) & (L["ev"] == 22)
            ep = (L["cta"] == c) & (L["role"] == 2) & (L["ev"] == 27)
            if mm.any():
                first_ready.append((L["gt"][mm].min() - g0) / 1e3)
                last_ready.append((L["gt"][mm].max() - g0) / 1e3)
            if ep.any():
                last_epi.append((L["gt"][ep].max() - g0) / 1e3)
        lines.append(f"  first stage ready (us) p10/p50/p90/max: {_pct(first_ready, (10, 50, 90, 100))}".replace(" / ", "/"))
        lines.append(f"  last stage ready (us) p10/p50/p90/max: {_pct(last_ready, (10, 50, 90, 100))}".replace(" / ", "/"))
        lines.append(f"  last tile's epilogue done (us) p10/p50/p90/max: {_pct(last_epi, (10, 50, 90, 100))}".replace(" / ", "/"))
        lines.append(f"  stage load latency, issue -> MMA full barrier (SM clocks) p10/p50/p90: {_pct(lat)}")
        lines.append(f"  MMA issuer period between stages (SM clocks) p10/p50/p90: {_pct(per)}; "
                     f"mean {np.mean(per):.0f}" if per else "  no stages")
        lines.append(f"  MMA issuer wait for a free accumulator (SM clocks) p10/p50/p90: {_pct(accw)}")
    return lines


def _cluster_phases(L):
    """Per-CTA phase durations of one launch of the cluster form, rank 0 and the rest apart:
    last MMA issued -> accumulator ready -> the partials of its column groups received ->
    epilogue done -> end, and the spread of the last-MMA times inside each cluster (what the
    reduction waits for).  CTAs that finish no column group (ranks >= 4) record no receipt."""
    import numpy as np
    at, ck = {}, {}
    for c, e, t, kb, k in zip(L["cta"].tolist(), L["ev"].tolist(), L["gt"].tolist(), L["kb"].tolist(),
                              L["clk"].tolist()):
        d = at.setdefault(c, {})
        if e in (23, 26, 27, 28, 29, 11) or (e in (33, 34) and e not in d):
            d[e] = t
            ck.setdefault(c, {})[e] = k
        if e in (26, 28, 27, 29):
            d["rank"] = kb
    ctas = [c for c, d in at.items() if all(e in d for e in (11, 23, 26, 27, 28, 29)) and "rank" in d]
    if not ctas:
        return []
    ranks = sorted({at[c]["rank"] for c in ctas})
    size = len(ranks)
    out = [f"  per-CTA phases of that launch (us), p10 / p50 / p90 over CTAs, cluster size {size}:"]
    for name, e0, e1 in (("release -> last MMA issued", 11, 23), ("last MMA -> accumulator ready", 23, 26),
                         ("accumulator ready -> partials received", 26, 28),
                         ("partials received -> epilogue done", 28, 27), ("epilogue done -> CTA end", 27, 29),
                         ("  received -> first unit's sum", 28, 33), ("  first unit: sum -> stored", 33, 34)):
        for who, sel in (("rank 0", lambda c: at[c]["rank"] == 0), ("others", lambda c: at[c]["rank"] != 0)):
            x = [(at[c][e1] - at[c][e0]) / 1e3 for c in ctas if sel(c) and e0 in at[c] and e1 in at[c]]
            # the same phase in SM clocks (both events on the CTA's own SM)
            y = [(ck[c][e1] - ck[c][e0]) & 0xFFFFFFFF for c in ctas if sel(c) and e0 in ck[c] and e1 in ck[c]]
            if x:
                out.append(f"    {name:42s} {who:6s} {_pct(x)}   clocks {_pct(y)}")
    spread = []
    for cl in {c // size for c in ctas}:
        t = [at[c][23] for c in ctas if c // size == cl]
        if len(t) == size:
            spread.append((max(t) - min(t)) / 1e3)
    if spread:
        out.append(f"    {'last-MMA spread inside a cluster':42s} {'':6s} {_pct(spread)}")
    return out


def summarise_small_m(launches):
    import numpy as np
    rows = []
    for L in launches:
        g = L["gt"]
        pick = lambda e: g[L["ev"] == e]
        if not (len(pick(11)) and len(pick(22)) and len(pick(23)) and len(pick(29))):
            continue
        rows.append((pick(11).min(), pick(22).min(), pick(23).max(), pick(29).max(), len(np.unique(L["cta"]))))
    rows.sort()
    lines = []
    # the chain of the last launch's latest events, against its dependency release
    if launches:
        Lz = max(launches, key=lambda L: L["gt"].min())
        rel = Lz["gt"][Lz["ev"] == 11].min() if (Lz["ev"] == 11).any() else Lz["gt"].min()
        for e in sorted(set(Lz["ev"].tolist())):
            x = (Lz["gt"][Lz["ev"] == e] - rel) / 1e3
            lines.append(f"  ev{e:2d} {EV.get(e, ''):28s} min {x.min():7.2f}  p50 {np.median(x):7.2f}  "
                         f"max {x.max():7.2f} us (from the release)")
    if launches and (Lz["ev"] == 28).any():
        lines += _cluster_phases(Lz)
    for i in range(1, len(rows)):
        r0, r1 = rows[i - 1], rows[i]
        lines.append(f"launch {i} ({r1[4]} CTAs): release-to-release {(r1[0] - r0[0]) / 1e3:.2f} us | previous end -> "
                     f"release {(r1[0] - r0[3]) / 1e3:.2f} | release -> first stage {(r1[1] - r1[0]) / 1e3:.2f} | "
                     f"release -> last MMA {(r1[2] - r1[0]) / 1e3:.2f} | release -> last CTA end "
                     f"{(r1[3] - r1[0]) / 1e3:.2f} us")
    return lines


def run(args) -> int:
    import numpy as np
    import torch
    sys.path.insert(0, ROOT)
    from activation_epilogue_tcgen05_b200 import gemm_epi as g
    from activation_epilogue_tcgen05_b200.workloads import TORCH_DTYPE, make_problem
    import bench
    if not os.path.exists(TRACE_LIB):
        raise SystemExit(f"{TRACE_LIB} is missing: run `python -m activation_epilogue_tcgen05_b200.trace build`")
    g.LIB_PATH = TRACE_LIB
    L = g.lib()
    L.gemm_epi_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    wl = bench.workload_from_args(argparse.Namespace(shape=args.shape, workload=args.workload))
    prob = make_problem(wl, device="cpu")
    dev = torch.device("cuda", 0)
    sets = []
    for _ in range(4):           # rotate operands so that each launch reads them from HBM as bench.py does
        D = torch.empty((wl.m, wl.n), dtype=TORCH_DTYPE[wl.out_dtype], device=dev)
        aux = (torch.empty(wl.m * g.aux_pitch_words(wl.n), dtype=torch.int32, device=dev)
               if wl.epilogue in g.HAS_AUX else None)
        sets.append((prob.A.to(dev), prob.B.to(dev), prob.bias.to(dev), D, aux))
    plan = g.Plan(wl.m, wl.n, wl.k, wl.dtype, wl.epilogue, wl.bias_axis, wl.b_layout, kernel=args.kernel,
                  block_n=args.block_n, split_k=args.split_k)
    if wl.dtype == "e4m3":
        plan.set_scales(torch.tensor([prob.scale_a], device=dev), torch.tensor([prob.scale_b], device=dev))
    info = plan.info
    s = torch.cuda.current_stream()
    for i in range(5):
        plan.run(*sets[i % 4], stream=s)
    torch.cuda.synchronize()
    cap = (2 + 2 * TRACE_CAP) * 8
    host = np.zeros(cap // 8, dtype=np.uint64)
    L.gemm_epi_trace_read(host.ctypes.data, cap)          # clears the buffer
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(args.launches):
                plan.run(*sets[i % 4], stream=torch.cuda.current_stream())
        graph.replay()
        torch.cuda.synchronize()
        L.gemm_epi_trace_read(host.ctypes.data, cap)
        graph.replay()
    else:
        for i in range(args.launches):
            plan.run(*sets[i % 4], stream=s)
    torch.cuda.synchronize()
    host[:] = 0
    rc = L.gemm_epi_trace_read(host.ctypes.data, cap)
    plan.check(s)
    plan.close()
    if rc != 0:
        raise SystemExit(f"gemm_epi_trace_read: {rc}")
    recs = host[2:].reshape(-1, 2)
    launches = _launches(recs[:, 0], recs[:, 1])
    print(f"workload {wl.name}; plan {info}; {len(launches)} launches traced "
          f"({'CUDA graph' if args.graph else 'direct launches'})")
    lines = summarise_small_m(launches) if info["kernel"] == g.KERNEL_SPLITK else summarise_persistent(launches)
    print("\n".join(lines))
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    sub = ap.add_subparsers(dest="cmd", required=True)
    b = sub.add_parser("build")
    b.add_argument("--force", action="store_true")
    r = sub.add_parser("run")
    r.add_argument("--workload", default="relu_aux_bias_bf16_4096x4096x4096")
    r.add_argument("--shape", default=None)
    r.add_argument("--launches", type=int, default=6)
    r.add_argument("--graph", action="store_true", help="replay the launches from a CUDA graph")
    r.add_argument("--kernel", default="auto", choices=["auto", "tc1", "tc2", "splitk"])
    r.add_argument("--block-n", type=int, default=0)
    r.add_argument("--split-k", type=int, default=0)
    a = ap.parse_args(argv)
    if a.cmd == "build":
        print(build(a.force))
        return 0
    if a.launches < 1 or a.launches > TRACE_CAP // LAUNCH_RECS - 6:
        raise SystemExit(f"--launches must be 1..{TRACE_CAP // LAUNCH_RECS - 6} (per-launch slots of the buffer)")
    return run(a)


if __name__ == "__main__":
    sys.exit(main())
