"""Benchmark of the weight-only NVFP4 GEMV decode-step sweep on B200.

One step = the decode-step sweep: 4 synthetic layers, each with qkv (10240x5120), o (5120x6144),
the fused gate_up dual (2 x 17408x5120) and down (5120x17408) NVFP4 projections, run back to back
on one stream, for every row count M in {1, 2, 4, 8} -- 64 launches, 3.16 GB of packed weights
and scales streamed per step (0.79 GB per M pass, far above the 126 MB L2, so no flush is needed).

Metric: effective HBM GB/s = (packed weights + scales + bf16 activations + bf16 outputs) bytes
per step / device time per step.  Printed as one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload sweep|attn_pairs|wide_rows]

--workload attn_pairs measures nvfp4_gemv_multi instead: 8 layers x {k + v (2 x 1024x5120),
q + gate (2 x 6144x5120)}, one launch per pair sharing x, M in {1, 8}; the same outputs as
separate nvfp4_gemv launches are timed beside it.  --workload wide_rows times the sweep's first
layer at M = 16, 32, 64 and 128 rows (one kernel pass per 8 rows).

Under torchrun (N > 1) every rank runs an independent replica on its own GPU (the GEMV needs no
collective); value = bytes of all ranks / max over ranks of the device time.
--impl reference times the CPU fp64 oracle (the plain C reference) on a bounded sample of the
same workload on rank 0's host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "sweep"
METRIC = "NVFP4 GEMV effective HBM GB/s and % of B200 peak, rows 1/8"
WORKLOAD_DESC = ("decode-step sweep: 4 layers x {qkv 10240x5120, o 5120x6144, gate_up dual "
                 "2x17408x5120, down 5120x17408} NVFP4, M in {1,2,4,8}, back to back on one stream")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("sweep", "attn_pairs", "wide_rows", "prologue_layers"),
                    default="sweep")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--repeats", type=int, default=5,
                    help="repeats of the K-step timed region; the median is reported")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="run this many eager steps and exit (for ncu launch lists)")
    ap.add_argument("--profile-separate", action="store_true",
                    help="sweep: profile the step as 64 separate launches instead of 4 chains")
    return ap.parse_args()


KERNEL_SOURCE = os.path.join(ROOT, "nvfp4_weight_only_03_b200", "csrc", "nvfp4_gemv.cu")


def kernel_code_sha256(path: str = KERNEL_SOURCE) -> str:
    """SHA-256 of the kernel source without comments and blank lines: edits that leave the code
    unchanged keep a captured traffic figure valid."""
    import re
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).strip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


# DRAM bytes of the chained launches from one ncu capture of a bench step (profiles/
# nvfp4_gemv_chain_launch_list.md): the 4 launches' dram__bytes_read.sum + dram__bytes_write.sum
# over their algorithmic bytes.  Valid only for the kernel code with this SHA-256.
CHAIN_TRAFFIC_SHA256 = "a737f146bbdcdd66257a67e7294f0f76d7354d441c258b78449478504bed6de9"
CHAIN_TRAFFIC_RATIO = 3268259328 / 3170058240  # 1.0310


def measured_chain_traffic():
    try:
        if CHAIN_TRAFFIC_SHA256 is None or kernel_code_sha256() != CHAIN_TRAFFIC_SHA256:
            return None
    except OSError:
        return None
    wl = synth.describe(WORKLOAD)
    bytes_avg = sum(step_bytes(wl).values()) / len(wl.rows)
    return {"bytes_per_launch": round(bytes_avg * CHAIN_TRAFFIC_RATIO),
            "ratio": CHAIN_TRAFFIC_RATIO,
            "how": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one step's 4 chained "
                   "launches over their algorithmic bytes, times the mean algorithmic bytes per "
                   "launch"}


def step_bytes(wl) -> dict:
    """Algorithmic bytes per launch, keyed by (projection, M)."""
    out = {}
    for m in wl.rows:
        for p in wl.projections:
            nw = 2 if p.dual else 1
            out[(p.name, m)] = nw * (p.n * p.k // 2 + p.n * p.k // 16) + m * p.k * 2 + m * p.n * 2
    return out


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ----------------------------------------------------------------------------------------------
# clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [t.strip() for t in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        # samples under load: the top half by clock is not a filter we want; keep them all
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------------------------
# distributed plumbing (replicas only)


def dist_setup(gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:  # host-only runs (the rank logic's tests): gloo
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)


SAMPLE_ROWS = 256


def oracle_slice(oracle, p, m, rng, threads) -> int:
    """The fp64 oracle on SAMPLE_ROWS consecutive output rows of projection p at M = m, at a
    random offset; returns the algorithmic bytes of that slice."""
    rows = np.arange(0, min(p.n, SAMPLE_ROWS)) + int(rng.integers(0, max(1, p.n - SAMPLE_ROWS)))
    if p.dual:
        oracle.gemv_dual(p.w.packed, p.w.scales, p.w.g, p.w_up.packed, p.w_up.scales,
                         p.w_up.g, p.x[:m], rows=rows, threads=threads)
    else:
        oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x[:m], rows=rows, threads=threads)
    nw = 2 if p.dual else 1
    return nw * rows.size * (p.k // 2 + p.k // 16) + m * p.k * 2 + m * rows.size * 2


def cpu_oracle_sample(wl, seconds: float):
    """Time the fp64 oracle on row slices of the workload's projections (rank 0, host cores)."""
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    done_bytes, t_total, n = 0, 0.0, 0
    rng = np.random.default_rng(0)
    order = [(p, m) for m in wl.rows for p in wl.projections]
    while t_total < seconds and n < 100000:
        p, m = order[n % len(order)]
        n += 1
        t0 = time.perf_counter()
        done_bytes += oracle_slice(oracle, p, m, rng, threads)
        t_total += time.perf_counter() - t0
    return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{n} calls of {SAMPLE_ROWS} consecutive output rows each at random "
                      f"offsets, cycling over the sweep's projections and M in {{1,2,4,8}} "
                      f"({t_total:.1f} s)"}


# ----------------------------------------------------------------------------------------------
# our arm


def sweep_chain_ops(nv, wl, dw, m, x_key="x", y_key="y", x_of=None, y_of=None):
    """The sweep's 16 projections at M rows as one chain, in sweep order, each with its own x
    (x_of / y_of map an entry to its x / y tensors when given)."""
    ops = []
    for e in dw:
        p = e["p"]
        x = x_of(e, m) if x_of else e[x_key][:m]
        y = y_of(e, m) if y_of else e[y_key][:m]
        if p.dual:
            ops.append(nv.ChainOp.dual(e["W"], e["S"], e["g"], e["Wu"], e["Su"], e["gu"], x=x, y=y))
        else:
            ops.append(nv.ChainOp.single([(e["W"], e["S"], e["g"])], x=x, ys=[y]))
    return ops


def run_ours(args, world, rank, local):
    import torch
    import nvfp4_weight_only_03_b200 as nv
    L = nv.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.make(WORKLOAD)
    bytes_of = step_bytes(wl)
    total_step_bytes = sum(bytes_of.values())
    pass_bytes = {m: sum(bytes_of[(p.name, m)] for p in wl.projections) for m in wl.rows}

    # resident inputs
    dw = []
    for p in wl.projections:
        ent = {"p": p, "W": torch.from_numpy(p.w.packed).to(dev),
               "S": torch.from_numpy(p.w.scales).to(dev), "g": p.w.g,
               "x": torch.from_numpy(p.x.view(np.int16)).view(torch.bfloat16).to(dev),
               "y": torch.empty((8, p.n), dtype=torch.bfloat16, device=dev)}
        if p.dual:
            ent["Wu"] = torch.from_numpy(p.w_up.packed).to(dev)
            ent["Su"] = torch.from_numpy(p.w_up.scales).to(dev)
            ent["gu"] = p.w_up.g
        dw.append(ent)
    ws = nv.workspace(dev)
    wsp, wsn = ws.data_ptr(), ws.numel()
    flags = nv.FLAG_PREFETCH_WEIGHTS  # decode step: weights are constants

    # the step: one chained launch per M (the 16 projections back to back in one persistent
    # kernel); every projection's result is bitwise that of its own launch
    structs = {m: nv._chain_structs(sweep_chain_ops(nv, wl, dw, m)) for m in wl.rows}
    cbytes = 0
    for m, (arr, mm, _, _) in structs.items():
        b = ctypes.c_size_t()
        st = L.nvfp4_chain_workspace_bytes(arr, len(dw), mm, ctypes.byref(b))
        if st != 0:
            raise RuntimeError(f"chain workspace: {nv.STATUS.get(st, st)}")
        cbytes = max(cbytes, int(b.value))
    cws = torch.zeros(cbytes, dtype=torch.uint8, device=dev)

    def chain_launches(sh):
        return [(f"chain@M{m}", m, L.nvfp4_gemv_chain,
                 (structs[m][0], len(dw), m, cws.data_ptr(), cws.numel(), flags, sh))
                for m in wl.rows]

    def separate_launches(sh):
        """The same step as 64 launches (one per projection and M), for comparison."""
        seq = []
        for m in wl.rows:
            for e in dw:
                p = e["p"]
                xp, yp = e["x"].data_ptr(), e["y"].data_ptr()
                if p.dual:
                    a = (e["W"].data_ptr(), e["S"].data_ptr(), ctypes.c_float(e["g"]),
                         e["Wu"].data_ptr(), e["Su"].data_ptr(), ctypes.c_float(e["gu"]), xp,
                         p.k, yp, p.n, m, p.n, p.k, wsp, wsn, flags, sh)
                    seq.append(("nvfp4_gemv_dual", (p.name, m), L.nvfp4_gemv_dual_ex, a))
                else:
                    a = (e["W"].data_ptr(), e["S"].data_ptr(), ctypes.c_float(e["g"]), xp, p.k,
                         yp, p.n, m, p.n, p.k, wsp, wsn, flags, sh)
                    seq.append(("nvfp4_gemv", (p.name, m), L.nvfp4_gemv_ex, a))
        return seq

    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    def run_seq(seq):
        for item in seq:
            st = item[2](*item[3])
            if st != 0:
                raise RuntimeError(f"launch failed: {nv.STATUS.get(st, st)}")

    if args.profile_steps:
        # eager steps only, for ncu: 4 chain launches a step (64 separate launches with
        # --profile-separate); the first max(W, 3) steps are the warm-up
        make = separate_launches if args.profile_separate else chain_launches
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3) + args.profile_steps):
                run_seq(make(sh))
        stream.synchronize()
        return None

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            run_seq(chain_launches(sh))
            run_seq(separate_launches(sh))
    stream.synchronize()

    def capture(make, with_events):
        """A CUDA graph of one step (optionally with an event pair around every launch: those
        events break the launches' overlap, so their durations are for launches run alone)."""
        graph = torch.cuda.CUDAGraph()
        ev = None
        with torch.cuda.graph(graph, stream=stream):
            cs = torch.cuda.current_stream().cuda_stream
            seq = make(cs)
            if with_events:
                ev = [(torch.cuda.Event(enable_timing=True, external=True),
                       torch.cuda.Event(enable_timing=True, external=True)) for _ in seq]
            for i, item in enumerate(seq):
                if ev is not None:
                    ev[i][0].record()
                st = item[2](*item[3])
                if ev is not None:
                    ev[i][1].record()
                if st != 0:
                    raise RuntimeError(f"capture failed: {nv.STATUS.get(st, st)}")
        return graph, ev, seq

    graph, _, cseq = capture(chain_launches, False)
    graph_ev, ev, _ = capture(chain_launches, True)
    graph_sep, _, sseq = capture(separate_launches, False)
    graph_sep_ev, sev, _ = capture(separate_launches, True)
    for g in (graph, graph_ev, graph_sep, graph_sep_ev):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()

    def timed(g, steps):
        t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            t_begin.record()
            for _ in range(steps):
                g.replay()
            t_end.record()
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(t_begin.elapsed_time(t_end), world)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    # the timed region: K steps, repeated `repeats` times; the median repeat is the number
    repeats = max(1, args.repeats)
    rep_ms = [timed(graph, args.steps) for _ in range(repeats)]
    ms = sorted(rep_ms)[len(rep_ms) // 2]
    sep_steps = max(1, min(args.steps, 50))
    sep_ms = timed(graph_sep, sep_steps) / sep_steps
    # per-launch durations of launches run alone: the instrumented graphs, median of 10 replays
    reps = 10

    def launch_us(g, events, seq):
        samples = [[] for _ in seq]
        for _ in range(reps):
            with torch.cuda.stream(stream):
                g.replay()
            torch.cuda.synchronize()
            for i, (e0, e1) in enumerate(events):
                samples[i].append(e0.elapsed_time(e1) * 1e3)
        return [sorted(v)[len(v) // 2] for v in samples]

    chain_us = launch_us(graph_ev, ev, cseq)
    sep_us = launch_us(graph_sep_ev, sev, sseq)
    clk = clocks.stop()
    ms_per_step = ms / args.steps
    value = world * total_step_bytes * args.steps / (ms * 1e-3) / 1e9

    # the step is 4 launches of one kernel (the chain), back to back: its mean launch duration
    # inside the timed region is the step time over 4
    peak, peak_src = peaks()
    in_step_us = ms_per_step * 1e3 / len(wl.rows)
    bytes_avg = total_step_bytes / len(wl.rows)
    achieved = bytes_avg / (in_step_us * 1e-6) / 1e9
    iso_us = sum(chain_us) / len(chain_us)
    iso = bytes_avg / (iso_us * 1e-6) / 1e9
    tr = measured_chain_traffic()
    roofline = {"bound": "hbm", "kernel": "nvfp4_gemv_chain (nvfp4_gemv_kernel<3>)",
                "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": tr["bytes_per_launch"] if tr else None,
                "peak_source": peak_src, "traffic_detail": tr,
                "bytes_per_launch_avg": round(bytes_avg), "avg_launch_us": round(in_step_us, 3),
                "timing": "CUDA events around the K timed steps on the launching stream (median "
                          f"of {repeats} repeats); a step is 4 chain launches of this kernel",
                "isolated": {"achieved": round(iso, 1), "frac": round(iso / peak, 4),
                             "avg_launch_us": round(iso_us, 3),
                             "timing": f"events around each chain launch, median of {reps} "
                                       "replays"}}
    per_pass = {}
    for (name, m, _, _), us in zip(cseq, chain_us):
        gbps = pass_bytes[m] / (us * 1e-6) / 1e9
        per_pass[name] = {"us": round(us, 2), "GBps": round(gbps, 1), "frac": round(gbps / peak, 4)}
    detail = {}
    for (kind, (name, m), _, _), us in zip(sseq, sep_us):
        b = bytes_of[(name, m)]
        detail[f"{name}@M{m}"] = {"us": round(us, 2), "GBps": round(b / (us * 1e-6) / 1e9, 1),
                                  "frac": round(b / (us * 1e-6) / 1e9 / peak, 4)}

    mlp = mlp_pairs(nv, L, wl, dw, dev, stream, flags, peak)

    # end to end through the public API: pinned host x in, y out, every step
    e2e = run_e2e(args, wl, dw, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(wl, args.cpu_seconds)

    del graph, graph_ev, graph_sep, graph_sep_ev
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4(e2m1+e4m3) x bf16 -> fp32 accumulate, bf16 out",
            "data": "synthetic (seeded N(0,0.02) weights quantised to NVFP4, N(0,1) bf16 x)",
            "config": {"workload": WORKLOAD_DESC, "seed": wl.seed, "rows": list(wl.rows),
                       "bytes_per_step": total_step_bytes,
                       "l2": "inputs 0.79 GB per M pass > 126 MB L2; no flush",
                       "launch": "one CUDA graph per step: one chained launch per M (the 16 "
                                 "projections in one persistent kernel, grid = SMs), "
                                 "programmatic dependent launch between the 4 launches",
                       "repeats": rep_ms and [round(x / args.steps, 5) for x in rep_ms],
                       "parallelism": f"replicas x{world}"},
            "roofline": roofline, "e2e": e2e, "gpu_launches": len(cseq) * args.steps * repeats,
            "clocks": clk, "per_pass": per_pass,
            "separate_launches": {
                "ms_per_step": round(sep_ms, 5),
                "GBps": round(world * total_step_bytes / (sep_ms * 1e-3) / 1e9, 1),
                "what": "the same step as 64 launches (nvfp4_gemv_ex / nvfp4_gemv_dual_ex), one "
                        "CUDA graph with programmatic dependent launch"},
            "per_launch": detail, "mlp_pair": mlp}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def mlp_pairs(nv, L, wl, dw, dev, stream, flags, peak, replays: int = 50):
    """The MLP pair of each layer as one chained launch, gate_up dual -> down with down's x the
    dual's output (x_from, a device-side dependency), at M = 1 and 8: 4 launches (one per
    layer) in one CUDA graph, median of 5 timings of `replays` replays."""
    import torch
    out = {}
    layers = [(dw[i], dw[i + 1]) for i in range(len(dw) - 1) if dw[i]["p"].dual]
    for m in (1, 8):
        acts = [torch.empty((m, gu["p"].n), dtype=torch.bfloat16, device=dev) for gu, _ in layers]
        structs, wsb = [], 0
        for (gu, dn), act in zip(layers, acts):
            ops = [nv.ChainOp.dual(gu["W"], gu["S"], gu["g"], gu["Wu"], gu["Su"], gu["gu"],
                                   x=gu["x"][:m], y=act),
                   nv.ChainOp.single([(dn["W"], dn["S"], dn["g"])], x_from=0, ys=[dn["y"][:m]])]
            st = nv._chain_structs(ops)
            b = ctypes.c_size_t()
            if L.nvfp4_chain_workspace_bytes(st[0], 2, st[1], ctypes.byref(b)) != 0:
                raise RuntimeError("mlp chain workspace")
            wsb = max(wsb, int(b.value))
            structs.append((st, ops))
        ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)

        def launch(sh):
            for (arr, mm, _, _), _ in structs:
                st = L.nvfp4_gemv_chain(arr, 2, mm, ws.data_ptr(), ws.numel(), flags, sh)
                if st != 0:
                    raise RuntimeError(f"mlp chain: {nv.STATUS.get(st, st)}")
        with torch.cuda.stream(stream):
            for _ in range(3):
                launch(stream.cuda_stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            launch(torch.cuda.current_stream().cuda_stream)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record()
                for _ in range(replays):
                    g.replay()
                e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / replays / len(layers) * 1e3)
        us = sorted(times)[len(times) // 2]
        gu, dn = layers[0][0]["p"], layers[0][1]["p"]
        nbytes = (2 * (gu.n * gu.k // 2 + gu.n * gu.k // 16) + m * gu.k * 2 + m * gu.n * 2 +
                  dn.n * dn.k // 2 + dn.n * dn.k // 16 + m * dn.k * 2 + m * dn.n * 2)
        gbps = nbytes / (us * 1e-6) / 1e9
        out[f"M{m}"] = {"us_per_launch": round(us, 2), "GBps": round(gbps, 1),
                        "frac": round(gbps / peak, 4), "bytes_per_launch": nbytes}
        del g
    out["what"] = ("one nvfp4_gemv_chain launch per layer: gate_up dual 2x17408x5120 -> down "
                   "5120x17408 reading the dual's output through x_from (cooperative launch); "
                   "4 layers per CUDA graph, median of 5 x 50 replays")
    return out


def run_e2e(args, wl, dw, world):
    """Same metric through the public Python API (nvfp4_weight_only_03_b200.Chain, one prepared
    chain per M and buffer), as a serving loop runs it.  Every step copies the step's inputs
    (each projection's x, 8 rows) from pinned host memory to the device in one copy, runs the
    4 chains, and reads every projection's y back into pinned host memory in one copy; all of
    it is inside the timed region.  The copies run on their own streams (one for H2D, one for
    D2H) with two buffers, so one step's copies overlap the neighbouring steps' kernels; events
    keep every buffer from being overwritten while a copy or kernel still uses it."""
    import torch
    import nvfp4_weight_only_03_b200 as nv
    dev = dw[0]["x"].device
    # one pinned host buffer of all x; two device buffers of all x and of all y, two pinned
    # host buffers of all y (step i uses buffer i % 2)
    x_off, off = {}, 0
    for e in dw:
        x_off[e["p"].name] = off
        off += e["x"].numel()
    hx = torch.empty(off, dtype=torch.bfloat16).pin_memory()
    for e in dw:
        o = x_off[e["p"].name]
        hx[o:o + e["x"].numel()].copy_(torch.from_numpy(e["p"].x.view(np.int16)).view(torch.bfloat16)
                                       .reshape(-1))
    dx = [torch.empty(off, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    y_off, off = {}, 0
    for m in wl.rows:
        for e in dw:
            y_off[(e["p"].name, m)] = off
            off += m * e["p"].n
    hy = [torch.empty(off, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dy = [torch.empty(off, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    compute = torch.cuda.Stream(device=dev)
    h2d = torch.cuda.Stream(device=dev)
    d2h = torch.cuda.Stream(device=dev)
    chains = [[], []]
    for buf in range(2):
        for m in wl.rows:
            def x_of(e, m, buf=buf):
                p = e["p"]
                xo = x_off[p.name]
                return dx[buf][xo:xo + 8 * p.k].view(8, p.k)[:m]

            def y_of(e, m, buf=buf):
                p = e["p"]
                yo = y_off[(p.name, m)]
                return dy[buf][yo:yo + m * p.n].view(m, p.n)
            chains[buf].append(nv.Chain(sweep_chain_ops(nv, wl, dw, m, x_of=x_of, y_of=y_of),
                                        stream=compute, prefetch_weights=True))
    x_ready = [torch.cuda.Event() for _ in range(2)]    # H2D of buffer b done
    x_free = [torch.cuda.Event() for _ in range(2)]     # kernels reading dx[b] done
    y_ready = [torch.cuda.Event() for _ in range(2)]    # kernels writing dy[b] done
    y_free = [torch.cuda.Event() for _ in range(2)]     # D2H of dy[b] done
    for b in range(2):  # every buffer starts free
        x_free[b].record(compute)
        y_free[b].record(d2h)

    def step(i):
        b = i % 2
        with torch.cuda.stream(h2d):
            h2d.wait_event(x_free[b])
            dx[b].copy_(hx, non_blocking=True)
            x_ready[b].record(h2d)
        with torch.cuda.stream(compute):
            compute.wait_event(x_ready[b])
            compute.wait_event(y_free[b])
            for ch in chains[b]:
                ch(stream=compute)
            x_free[b].record(compute)
            y_ready[b].record(compute)
        with torch.cuda.stream(d2h):
            d2h.wait_event(y_ready[b])
            hy[b].copy_(dy[b], non_blocking=True)
            y_free[b].record(d2h)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(h2d)  # the first H2D follows t0; the other streams wait for it too
    compute.wait_event(t0)
    d2h.wait_event(t0)
    for i in range(args.e2e_steps):
        step(i)
    # the last D2H is the last piece of work; every stream ends before t1
    d2h.wait_stream(compute)
    d2h.wait_stream(h2d)
    t1.record(d2h)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    bytes_step = sum(step_bytes(wl).values())
    return {"value": round(world * bytes_step * args.e2e_steps / (ms * 1e-3) / 1e9, 1),
            "unit": "GB/s", "h2d_bytes_per_step": hx.numel() * 2,
            "d2h_bytes_per_step": hy[0].numel() * 2, "steps": args.e2e_steps,
            "api": "nvfp4_weight_only_03_b200.Chain (one prepared chain per M), one H2D copy of "
                   "the step's x and one D2H copy of its y per step, copies on their own streams "
                   "overlapping the neighbouring steps (two buffers)"}


# ----------------------------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample of the same workload


REF_SLICES_PER_STEP = 48  # 3 random 256-row slices of each of the 16 projections per step


def run_reference(args, world, rank):
    """The oracle as it stands on the host cores, on a bounded sample of the sweep: each step is
    REF_SLICES_PER_STEP slices of 256 consecutive output rows at random offsets (the sampler of
    cpu_baseline), three per projection, at one M (cycling over 1, 2, 4, 8)."""
    if rank != 0:
        return None
    wl = synth.make(WORKLOAD)
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    projs = list(wl.projections)

    def step(i):
        m = wl.rows[i % len(wl.rows)]
        return sum(oracle_slice(oracle, projs[j % len(projs)], m, rng, threads)
                   for j in range(REF_SLICES_PER_STEP))

    for i in range(args.warmup):
        step(i)
    steps = args.steps
    t0 = time.perf_counter()
    b = sum(step(i) for i in range(steps))
    dt = time.perf_counter() - t0
    v = b / dt / 1e9
    sample = (f"each step = {REF_SLICES_PER_STEP} slices of {SAMPLE_ROWS} consecutive output rows "
              f"at random offsets, three per projection, at one M cycling over {{1,2,4,8}} ({steps} "
              f"steps, {dt:.1f} s); the cpu_baseline sampler")
    return {"metric": METRIC, "value": round(v, 3), "unit": "GB/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(dt / steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD_DESC, "seed": wl.seed, "rows": list(wl.rows),
                       "sample": f"{SAMPLE_ROWS}-row slices (a bounded sample of the workload)"},
            "cpu_baseline": {"value": round(v, 3), "unit": "GB/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------------------------
# several outputs sharing x (nvfp4_gemv_multi)

PAIRS_LAYERS = 8
PAIRS_ROWS = (1, 8)
PAIRS_DESC = ("attention projection pairs sharing x: 8 layers x {k + v 2x1024x5120, q + gate "
              "2x6144x5120} NVFP4, M in {1,8}, one nvfp4_gemv_multi launch per pair, back to back "
              "on one stream")


def run_pairs(args, world, rank, local):
    import torch
    import nvfp4_weight_only_03_b200 as nv
    L = nv.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    pairs = [synth.make("attn_kv"), synth.make("attn_qgate")]
    # every layer streams its own copy of the pair weights (distinct device buffers: 330 MB per
    # M pass, far above the 126 MB L2); x of each pair is the first projection's draw
    layers = []
    for _ in range(PAIRS_LAYERS):
        for wl in pairs:
            ws_ = [(torch.from_numpy(p.w.packed).to(dev), torch.from_numpy(p.w.scales).to(dev),
                    p.w.g, p.n) for p in wl.projections]
            x = torch.from_numpy(wl.projections[0].x.view(np.int16)).view(torch.bfloat16).to(dev)
            ys = [torch.empty((8, n), dtype=torch.bfloat16, device=dev) for *_, n in ws_]
            layers.append({"name": wl.name, "w": ws_, "x": x, "y": ys, "k": wl.projections[0].k})
    ws = nv.workspace(dev)
    flags = nv.FLAG_PREFETCH_WEIGHTS

    def pass_bytes(m):
        b = 0
        for e in layers:
            for (_, _, _, n) in e["w"]:
                b += n * e["k"] // 2 + n * e["k"] // 16 + m * n * 2
            b += m * e["k"] * 2
        return b
    step_bytes_ = sum(pass_bytes(m) for m in PAIRS_ROWS)

    def calls(h, fused):
        seq = []
        for m in PAIRS_ROWS:
            for e in layers:
                if fused:
                    outs = (nv.Output * len(e["w"]))()
                    for o, ((W, S, g, n), y) in enumerate(zip(e["w"], e["y"])):
                        outs[o].w, outs[o].s, outs[o].global_scale = W.data_ptr(), S.data_ptr(), g
                        outs[o].y, outs[o].ldy, outs[o].n = y.data_ptr(), n, n
                    seq.append((L.nvfp4_gemv_multi, (outs, len(e["w"]), e["x"].data_ptr(), e["k"],
                                                    m, e["k"], ws.data_ptr(), ws.numel(), flags, h)))
                else:
                    for (W, S, g, n), y in zip(e["w"], e["y"]):
                        seq.append((L.nvfp4_gemv_ex, (W.data_ptr(), S.data_ptr(), ctypes.c_float(g),
                                                      e["x"].data_ptr(), e["k"], y.data_ptr(), n, m,
                                                      n, e["k"], ws.data_ptr(), ws.numel(), flags,
                                                      h)))
        return seq

    stream = torch.cuda.Stream(device=dev)

    def graph_of(fused):
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                for fn, a in calls(stream.cuda_stream, fused):
                    if fn(*a) != 0:
                        raise RuntimeError("launch failed")
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            seq = calls(torch.cuda.current_stream().cuda_stream, fused)
            for fn, a in seq:
                if fn(*a) != 0:
                    raise RuntimeError("capture failed")
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        return g, len(seq)

    def timed(g, steps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            t0.record()
            for _ in range(steps):
                g.replay()
            t1.record()
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(t0.elapsed_time(t1), world)

    g_fused, n_fused = graph_of(True)
    g_sep, n_sep = graph_of(False)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms = timed(g_fused, args.steps)
    clk = clocks.stop()
    ms_sep = timed(g_sep, args.steps)
    value = world * step_bytes_ * args.steps / (ms * 1e-3) / 1e9
    value_sep = world * step_bytes_ * args.steps / (ms_sep * 1e-3) / 1e9
    peak, peak_src = peaks()
    per_launch_us = ms / args.steps * 1e3 / n_fused
    bytes_avg = step_bytes_ / n_fused

    # end to end through the public API: all x in from pinned host memory, all y back, per step
    hx = torch.cat([e["x"].reshape(-1) for e in layers]).cpu().pin_memory()
    dx = torch.empty_like(hx, device=dev)
    xs, off = [], 0
    for e in layers:
        xs.append(dx[off:off + e["x"].numel()].view(8, e["k"]))
        off += e["x"].numel()
    ysz = sum(m * n for m in PAIRS_ROWS for e in layers for *_, n in e["w"])
    hy = torch.empty(ysz, dtype=torch.bfloat16).pin_memory()
    dy = torch.empty(ysz, dtype=torch.bfloat16, device=dev)
    e2e_calls, off = [], 0
    for m in PAIRS_ROWS:
        for e, x in zip(layers, xs):
            ys = []
            for *_, n in e["w"]:
                ys.append(dy[off:off + m * n].view(m, n))
                off += m * n
            e2e_calls.append(([(W, S, g) for W, S, g, _ in e["w"]], x[:m], ys))
    cur = torch.cuda.current_stream()

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        for wts, x, ys in e2e_calls:
            nv.gemv_multi(wts, x, ys=ys, ws=ws, stream=cur, prefetch_weights=True)
        hy.copy_(dy, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(cur)
    for _ in range(args.e2e_steps):
        e2e_step()
    t1.record(cur)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(t0.elapsed_time(t1), world)
    e2e = {"value": round(world * step_bytes_ * args.e2e_steps / (ms_e2e * 1e-3) / 1e9, 1),
           "unit": "GB/s", "h2d_bytes_per_step": hx.numel() * 2, "d2h_bytes_per_step": ysz * 2,
           "steps": args.e2e_steps, "api": "nvfp4_weight_only_03_b200.gemv_multi"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        threads = os.cpu_count() or 1
        order = [(p, m) for m in PAIRS_ROWS for wl in pairs for p in wl.projections]
        t_end = time.perf_counter() + args.cpu_seconds
        b, n_calls, t_start = 0, 0, time.perf_counter()
        while time.perf_counter() < t_end:
            p, m = order[n_calls % len(order)]
            x = pairs[0 if p.n == 1024 else 1].projections[0].x[:m]
            oracle.gemv(p.w.packed, p.w.scales, p.w.g, x, rows=np.arange(256), threads=threads)
            b += 256 * (p.k // 2 + p.k // 16) + m * p.k * 2 + m * 256 * 2
            n_calls += 1
        dt = time.perf_counter() - t_start
        cpu = {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_calls} calls of 256 output rows each, cycling over the four "
                         f"projections and M in {{1,8}} ({dt:.1f} s)"}

    del g_fused, g_sep
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4(e2m1+e4m3) x bf16 -> fp32 accumulate, bf16 out",
            "data": "synthetic (seeded N(0,0.02) weights quantised to NVFP4, N(0,1) bf16 x)",
            "config": {"workload": PAIRS_DESC, "rows": list(PAIRS_ROWS),
                       "bytes_per_step": step_bytes_,
                       "l2": "0.33 GB of weights per M pass > 126 MB L2; no flush",
                       "launch": f"one CUDA graph per step ({n_fused} nvfp4_gemv_multi kernels, "
                                 "programmatic dependent launch), persistent grid = SMs",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "kernel": "nvfp4_gemv_kernel<single, multi>",
                         "achieved": round(bytes_avg / (per_launch_us * 1e-6) / 1e9, 1),
                         "peak": peak, "unit": "GB/s",
                         "frac": round(bytes_avg / (per_launch_us * 1e-6) / 1e9 / peak, 4),
                         "traffic": None, "peak_source": peak_src,
                         "bytes_per_launch_avg": bytes_avg,
                         "avg_launch_us": round(per_launch_us, 3),
                         "timing": "CUDA events around the K timed steps; every launch of the "
                                   "step is this kernel"},
            "separate_launches": {"value": round(value_sep, 1), "unit": "GB/s",
                                  "launches_per_step": n_sep,
                                  "ms_per_step": round(ms_sep / args.steps, 5),
                                  "what": "the same outputs as one nvfp4_gemv launch each"},
            "e2e": e2e, "gpu_launches": n_fused * args.steps, "clocks": clk}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


# ----------------------------------------------------------------------------------------------
# input prologues: the decode layer's neighbours of the GEMV fused into its x staging

PRO_ROWS = (1, 8)
PRO_EPS = 1e-6
PRO_DESC = ("decode-step sweep (4 layers x {qkv 10240x5120, o 5120x6144, gate_up dual 2x17408x5120, "
            "down 5120x17408} NVFP4, M in {1,8}) with the layer's neighbours as input prologues "
            "of the GEMV calls: residual add + RMS norm before qkv and gate_up (h written out), the sigmoid "
            "gate before o; x of each layer is the previous down output. Also timed: the same "
            "GEMVs without the neighbours, and with them as separate torch eager kernels")


def prologue_step_bytes(wl, rows=PRO_ROWS):
    """Algorithmic bytes of one step: every weight and scale once per M pass, x and y of each
    call, and the prologue's operands (residual, gamma and h for the norm, the gate)."""
    b = 0
    for m in rows:
        for p in wl.projections:
            b += (2 if p.dual else 1) * (p.n * p.k // 2 + p.n * p.k // 16)
            b += m * p.k * 2 + m * p.n * 2
            kind = p.name.split(".")[1]
            if kind in ("qkv", "gate_up"):
                b += 2 * m * p.k * 2 + p.k * 2   # residual in, h out, gamma
            elif kind == "o":
                b += m * p.k * 2                 # gate
    return b


def run_prologue(args, world, rank, local):
    import torch
    import nvfp4_weight_only_03_b200 as nv
    L = nv.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.make(WORKLOAD, generate_x=False)
    seed = wl.seed
    k_model = wl.projections[0].k          # 5120, the hidden size
    k_attn = [p for p in wl.projections if p.name.endswith(".o")][0].k  # 6144

    def bf16(bits_):
        return torch.from_numpy(np.ascontiguousarray(bits_).view(np.int16)).view(
            torch.bfloat16).to(dev)

    ents = []
    for p in wl.projections:
        e = {"p": p, "W": torch.from_numpy(p.w.packed).to(dev),
             "S": torch.from_numpy(p.w.scales).to(dev), "g": p.w.g,
             "y": torch.empty((8, p.n), dtype=torch.bfloat16, device=dev)}
        if p.dual:
            e["Wu"] = torch.from_numpy(p.w_up.packed).to(dev)
            e["Su"] = torch.from_numpy(p.w_up.scales).to(dev)
            e["gu"] = p.w_up.g
        ents.append(e)
    # activations: the first layer's input and residual, the attention output and its gate per
    # layer, one gain vector per norm; qkv's norm writes h to hbuf[0], gate_up's reads it and
    # writes hbuf[1], the next layer's residual
    x0 = bf16(synth.activations(seed + 200, 0, 8, k_model))
    r0 = bf16(synth.residual_stream(seed + 200, 2 * 8 * k_model, 8, k_model))
    n_layers = len(ents) // 4
    attn = [bf16(synth.activations(seed + 201 + i, 0, 8, k_attn)) for i in range(n_layers)]
    gates = [bf16(synth.gate_logits(seed + 201 + i, 2 * 8 * k_attn, 8, k_attn))
             for i in range(n_layers)]
    gammas = [bf16(synth.norm_gains(seed + 210 + i, 0, k_model)) for i in range(2 * n_layers)]
    hbuf = [torch.empty((8, k_model), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws = nv.wide_workspace(k_attn, k_attn, 8, dev)  # holds the prologue's x' of 8 rows
    wsp, wsn = ws.data_ptr(), ws.numel()
    flags = nv.FLAG_PREFETCH_WEIGHTS
    step_bytes_ = prologue_step_bytes(wl)

    def plan(h):
        """[(fn, args, keepalive)] for one fused step: per M, per layer qkv, o, gate_up, down."""
        seq = []
        for m in PRO_ROWS:
            x, r = x0, r0
            for li in range(n_layers):
                qkv, o, gu, down = ents[4 * li:4 * li + 4]
                # qkv: x' = rmsnorm(x + r), h -> hbuf[0]
                pq = nv.Prologue(kind=nv.PROLOGUE_ADD_RMSNORM, eps=PRO_EPS, residual=r.data_ptr(),
                                 ld_residual=k_model, gamma=gammas[2 * li].data_ptr(),
                                 residual_out=hbuf[0].data_ptr(), ld_residual_out=k_model)
                seq.append((L.nvfp4_gemv_pro, (ctypes.byref(pq), qkv["W"].data_ptr(),
                            qkv["S"].data_ptr(), ctypes.c_float(qkv["g"]), x.data_ptr(), k_model,
                            qkv["y"].data_ptr(), qkv["p"].n, m, qkv["p"].n, k_model, wsp, wsn,
                            flags, h), pq))
                # o: x' = attention output * sigmoid(gate)
                po = nv.Prologue(kind=nv.PROLOGUE_SIGMOID_GATE, gate=gates[li].data_ptr(),
                                 ld_gate=k_attn)
                seq.append((L.nvfp4_gemv_pro, (ctypes.byref(po), o["W"].data_ptr(),
                            o["S"].data_ptr(), ctypes.c_float(o["g"]), attn[li].data_ptr(),
                            k_attn, o["y"].data_ptr(), o["p"].n, m, o["p"].n, k_attn, wsp, wsn,
                            flags, h), po))
                # gate_up: x' = rmsnorm(o + h), the new h -> hbuf[1]
                pg = nv.Prologue(kind=nv.PROLOGUE_ADD_RMSNORM, eps=PRO_EPS,
                                 residual=hbuf[0].data_ptr(), ld_residual=k_model,
                                 gamma=gammas[2 * li + 1].data_ptr(),
                                 residual_out=hbuf[1].data_ptr(), ld_residual_out=k_model)
                seq.append((L.nvfp4_gemv_dual_pro, (ctypes.byref(pg), gu["W"].data_ptr(),
                            gu["S"].data_ptr(), ctypes.c_float(gu["g"]), gu["Wu"].data_ptr(),
                            gu["Su"].data_ptr(), ctypes.c_float(gu["gu"]), o["y"].data_ptr(),
                            k_model, gu["y"].data_ptr(), gu["p"].n, m, gu["p"].n, k_model, wsp,
                            wsn, flags, h), pg))
                seq.append((L.nvfp4_gemv_ex, (down["W"].data_ptr(), down["S"].data_ptr(),
                            ctypes.c_float(down["g"]), gu["y"].data_ptr(), down["p"].k,
                            down["y"].data_ptr(), down["p"].n, m, down["p"].n, down["p"].k, wsp,
                            wsn, flags, h), None))
                x, r = down["y"], hbuf[1]
        return seq

    def plain(h):
        """The same GEMVs on the same inputs without their neighbours."""
        seq = []
        for m in PRO_ROWS:
            x = x0
            for li in range(n_layers):
                qkv, o, gu, down = ents[4 * li:4 * li + 4]
                seq.append((L.nvfp4_gemv_ex, (qkv["W"].data_ptr(), qkv["S"].data_ptr(),
                            ctypes.c_float(qkv["g"]), x.data_ptr(), k_model, qkv["y"].data_ptr(),
                            qkv["p"].n, m, qkv["p"].n, k_model, wsp, wsn, flags, h), None))
                seq.append((L.nvfp4_gemv_ex, (o["W"].data_ptr(), o["S"].data_ptr(),
                            ctypes.c_float(o["g"]), attn[li].data_ptr(), k_attn,
                            o["y"].data_ptr(), o["p"].n, m, o["p"].n, k_attn, wsp, wsn, flags,
                            h), None))
                seq.append((L.nvfp4_gemv_dual_ex, (gu["W"].data_ptr(), gu["S"].data_ptr(),
                            ctypes.c_float(gu["g"]), gu["Wu"].data_ptr(), gu["Su"].data_ptr(),
                            ctypes.c_float(gu["gu"]), o["y"].data_ptr(), k_model,
                            gu["y"].data_ptr(), gu["p"].n, m, gu["p"].n, k_model, wsp, wsn,
                            flags, h), None))
                seq.append((L.nvfp4_gemv_ex, (down["W"].data_ptr(), down["S"].data_ptr(),
                            ctypes.c_float(down["g"]), gu["y"].data_ptr(), down["p"].k,
                            down["y"].data_ptr(), down["p"].n, m, down["p"].n, down["p"].k, wsp,
                            wsn, flags, h), None))
                x = down["y"]
        return seq

    stream = torch.cuda.Stream(device=dev)
    xn_buf = torch.empty((8, k_model), dtype=torch.bfloat16, device=dev)
    xg_buf = torch.empty((8, k_attn), dtype=torch.bfloat16, device=dev)

    def torch_norm(x, r, gamma, hout, m):
        h = (x[:m].float() + r[:m].float()).to(torch.bfloat16)
        hout[:m].copy_(h)
        hf = h.float()
        xn = hf * torch.rsqrt(hf.pow(2).mean(-1, keepdim=True) + PRO_EPS) * gamma.float()
        xn_buf[:m].copy_(xn.to(torch.bfloat16))

    def run_separate(h):
        """The neighbours as torch eager kernels, the GEMVs plain on their outputs."""
        for m in PRO_ROWS:
            x, r = x0, r0
            for li in range(n_layers):
                qkv, o, gu, down = ents[4 * li:4 * li + 4]
                torch_norm(x, r, gammas[2 * li], hbuf[0], m)
                if L.nvfp4_gemv_ex(qkv["W"].data_ptr(), qkv["S"].data_ptr(),
                                   ctypes.c_float(qkv["g"]), xn_buf.data_ptr(), k_model,
                                   qkv["y"].data_ptr(), qkv["p"].n, m, qkv["p"].n, k_model, wsp,
                                   wsn, flags, h) != 0:
                    raise RuntimeError("launch failed")
                xg_buf[:m].copy_((attn[li][:m].float() * torch.sigmoid(gates[li][:m].float()))
                                 .to(torch.bfloat16))
                if L.nvfp4_gemv_ex(o["W"].data_ptr(), o["S"].data_ptr(), ctypes.c_float(o["g"]),
                                   xg_buf.data_ptr(), k_attn, o["y"].data_ptr(), o["p"].n, m,
                                   o["p"].n, k_attn, wsp, wsn, flags, h) != 0:
                    raise RuntimeError("launch failed")
                torch_norm(o["y"], hbuf[0], gammas[2 * li + 1], hbuf[1], m)
                if L.nvfp4_gemv_dual_ex(gu["W"].data_ptr(), gu["S"].data_ptr(),
                                        ctypes.c_float(gu["g"]), gu["Wu"].data_ptr(),
                                        gu["Su"].data_ptr(), ctypes.c_float(gu["gu"]),
                                        xn_buf.data_ptr(), k_model, gu["y"].data_ptr(), gu["p"].n,
                                        m, gu["p"].n, k_model, wsp, wsn, flags, h) != 0:
                    raise RuntimeError("launch failed")
                if L.nvfp4_gemv_ex(down["W"].data_ptr(), down["S"].data_ptr(),
                                   ctypes.c_float(down["g"]), gu["y"].data_ptr(), down["p"].k,
                                   down["y"].data_ptr(), down["p"].n, m, down["p"].n,
                                   down["p"].k, wsp, wsn, flags, h) != 0:
                    raise RuntimeError("launch failed")
                x, r = down["y"], hbuf[1]

    def graph_of(build):
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                build(stream.cuda_stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            build(torch.cuda.current_stream().cuda_stream)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        return g

    def run_seq(make):
        def build(h):
            for fn, a, _keep in make(h):
                st = fn(*a)
                if st != 0:
                    raise RuntimeError(f"launch failed: {nv.STATUS.get(st, st)}")
        return build

    def timed(g, steps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            t0.record()
            for _ in range(steps):
                g.replay()
            t1.record()
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(t0.elapsed_time(t1), world)

    calls = plan(0)
    n_calls = len(calls)
    n_pro = sum(1 for _, _, keep in calls if keep is not None)
    n_launch = n_calls + n_pro  # each prologue call is a prologue grid and a GEMV
    if args.profile_steps:
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3) + args.profile_steps):
                run_seq(plan)(stream.cuda_stream)
        stream.synchronize()
        return None
    g_fused = graph_of(run_seq(plan))
    g_plain = graph_of(run_seq(plain))
    g_sep = graph_of(run_separate)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms = timed(g_fused, args.steps)
    clk = clocks.stop()
    ms_plain = timed(g_plain, args.steps)
    ms_sep = timed(g_sep, args.steps)
    value = world * step_bytes_ * args.steps / (ms * 1e-3) / 1e9
    peak, peak_src = peaks()
    per_call_us = ms / args.steps * 1e3 / n_calls
    bytes_avg = step_bytes_ / n_calls

    # end to end through the public API: the step's first input, residual, attention outputs and
    # gates in from pinned host memory, the last down output of each M pass back
    srcs = [x0, r0] + attn + gates
    hx = torch.cat([t.reshape(-1) for t in srcs]).cpu().pin_memory()
    dx = torch.empty_like(hx, device=dev)
    views, off = [], 0
    for t in srcs:
        views.append(dx[off:off + t.numel()].view(t.shape))
        off += t.numel()
    ex0, er0 = views[0], views[1]
    eattn, egates = views[2:2 + n_layers], views[2 + n_layers:]
    last = ents[-1]
    hy = torch.empty((len(PRO_ROWS), 8, last["p"].n), dtype=torch.bfloat16).pin_memory()
    cur = torch.cuda.current_stream()

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        for mi, m in enumerate(PRO_ROWS):
            x, r = ex0[:m], er0[:m]
            for li in range(n_layers):
                qkv, o, gu, down = ents[4 * li:4 * li + 4]
                nv.gemv(qkv["W"], qkv["S"], qkv["g"], x, y=qkv["y"][:m], ws=ws, stream=cur,
                        prefetch_weights=True, prologue=nv.AddRmsNorm(
                            r, gammas[2 * li], PRO_EPS, hbuf[0][:m]))
                nv.gemv(o["W"], o["S"], o["g"], eattn[li][:m], y=o["y"][:m], ws=ws, stream=cur,
                        prefetch_weights=True, prologue=nv.SigmoidGate(egates[li][:m]))
                nv.gemv_dual(gu["W"], gu["S"], gu["g"], gu["Wu"], gu["Su"], gu["gu"], o["y"][:m],
                             y=gu["y"][:m], ws=ws, stream=cur, prefetch_weights=True,
                             prologue=nv.AddRmsNorm(hbuf[0][:m], gammas[2 * li + 1], PRO_EPS,
                                                    hbuf[1][:m]))
                nv.gemv(down["W"], down["S"], down["g"], gu["y"][:m], y=down["y"][:m], ws=ws,
                        stream=cur, prefetch_weights=True)
                x, r = down["y"][:m], hbuf[1][:m]
            hy[mi, :m].copy_(last["y"][:m], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(cur)
    for _ in range(args.e2e_steps):
        e2e_step()
    t1.record(cur)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(t0.elapsed_time(t1), world)
    d2h = sum(m * last["p"].n * 2 for m in PRO_ROWS)
    e2e = {"value": round(world * step_bytes_ * args.e2e_steps / (ms_e2e * 1e-3) / 1e9, 1),
           "unit": "GB/s", "h2d_bytes_per_step": hx.numel() * 2, "d2h_bytes_per_step": d2h,
           "steps": args.e2e_steps,
           "api": "nvfp4_weight_only_03_b200.gemv / gemv_dual with AddRmsNorm / SigmoidGate"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        threads = os.cpu_count() or 1
        xb = synth.activations(seed + 200, 0, 8, k_model)
        rb = synth.residual_stream(seed + 200, 2 * 8 * k_model, 8, k_model)
        gb = synth.norm_gains(seed + 210, 0, k_model)
        qkv = wl.projections[0]
        t_end = time.perf_counter() + args.cpu_seconds
        b, n_calls, t_start = 0, 0, time.perf_counter()
        while time.perf_counter() < t_end:
            m = PRO_ROWS[n_calls % len(PRO_ROWS)]
            _, xq, _ = oracle.add_rmsnorm(xb[:m], rb[:m], gb, PRO_EPS)
            oracle.gemv(qkv.w.packed, qkv.w.scales, qkv.w.g, xq, rows=np.arange(256),
                        threads=threads)
            b += 256 * (qkv.k // 2 + qkv.k // 16) + 4 * m * qkv.k * 2 + qkv.k * 2 + m * 256 * 2
            n_calls += 1
        dt = time.perf_counter() - t_start
        cpu = {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_calls} calls of the norm prologue then 256 qkv output rows, M "
                         f"alternating 1 and 8 ({dt:.1f} s)"}

    del g_fused, g_plain, g_sep
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4(e2m1+e4m3) x bf16 -> fp32 accumulate, bf16 out",
            "data": "synthetic (seeded N(0,0.02) weights quantised to NVFP4; N(0,1) x, N(0,16) "
                    "residual, 1+N(0,0.01) gains, N(0,4) gate logits, all bf16)",
            "config": {"workload": PRO_DESC, "rows": list(PRO_ROWS), "eps": PRO_EPS,
                       "bytes_per_step": step_bytes_,
                       "l2": "0.79 GB of weights per M pass > 126 MB L2; no flush",
                       "launch": f"one CUDA graph per step ({n_launch} kernels, programmatic "
                                 "dependent launch), persistent grid = SMs",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm",
                         "kernel": "nvfp4_gemv_kernel (all instances) with nvfp4_prologue_kernel",
                         "achieved": round(bytes_avg / (per_call_us * 1e-6) / 1e9, 1),
                         "peak": peak, "unit": "GB/s",
                         "frac": round(bytes_avg / (per_call_us * 1e-6) / 1e9 / peak, 4),
                         "traffic": None, "peak_source": peak_src,
                         "bytes_per_call_avg": round(bytes_avg),
                         "avg_call_us": round(per_call_us, 3),
                         "timing": f"CUDA events around the K timed steps; a step is {n_calls} "
                                   f"GEMV calls, {n_pro} of them with a prologue grid ahead"},
            "without_neighbours": {"ms_per_step": round(ms_plain / args.steps, 5),
                                   "what": "the same GEMVs with no prologue (the neighbours' work "
                                           "left out): the floor the fusion is measured against"},
            "separate_torch_neighbours": {"ms_per_step": round(ms_sep / args.steps, 5),
                                          "what": "plain GEMVs with the neighbours as torch "
                                                  "eager kernels in the same graph"},
            "e2e": e2e, "gpu_launches": n_launch * args.steps, "clocks": clk}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


# ----------------------------------------------------------------------------------------------
# more than 8 rows (one kernel pass per 8-row block)

WIDE_ROWS = (16, 32, 64, 128)
WIDE_DESC = ("sweep layer 0 {qkv 10240x5120, o 5120x6144, gate_up dual 2x17408x5120, down "
             "5120x17408} NVFP4 at M in {16,32,64,128} rows, back to back on one stream, in two "
             "modes: 8-row kernel passes, and the tensor-core tier (NVFP4_FLAG_WIDE_TENSOR) for "
             "all four; value: the tier at M = 128")


def run_wide(args, world, rank, local):
    import torch
    import nvfp4_weight_only_03_b200 as nv
    L = nv.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.make(WORKLOAD, generate_x=False)
    projs = wl.projections[:4]
    ents = []
    for i, p in enumerate(projs):
        e = {"p": p, "W": torch.from_numpy(p.w.packed).to(dev), "S": torch.from_numpy(p.w.scales).to(dev),
             "x": torch.from_numpy(synth.activations(wl.seed + 100, 2 * i * 128 * p.k, 128, p.k)
                                   .view(np.int16)).view(torch.bfloat16).to(dev),
             "y": torch.empty((128, p.n), dtype=torch.bfloat16, device=dev)}
        if p.dual:
            e["Wu"] = torch.from_numpy(p.w_up.packed).to(dev)
            e["Su"] = torch.from_numpy(p.w_up.scales).to(dev)
        ents.append(e)
    ws = torch.zeros(max(nv.workspace_bytes_wide(e["p"].n, e["p"].k, WIDE_ROWS[-1]) for e in ents),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    if args.profile_steps:
        # eager steps of the tier at the largest row count, for ncu launch lists
        m = WIDE_ROWS[-1]
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3) + args.profile_steps):
                for e in ents:
                    p = e["p"]
                    if p.dual:
                        st = L.nvfp4_gemv_dual_ex(e["W"].data_ptr(), e["S"].data_ptr(),
                                                  ctypes.c_float(p.w.g), e["Wu"].data_ptr(),
                                                  e["Su"].data_ptr(), ctypes.c_float(p.w_up.g),
                                                  e["x"].data_ptr(), p.k, e["y"].data_ptr(), p.n,
                                                  m, p.n, p.k, ws.data_ptr(), ws.numel(),
                                                  nv.FLAG_WIDE_TENSOR, stream.cuda_stream)
                    else:
                        st = L.nvfp4_gemv_ex(e["W"].data_ptr(), e["S"].data_ptr(),
                                             ctypes.c_float(p.w.g), e["x"].data_ptr(), p.k,
                                             e["y"].data_ptr(), p.n, m, p.n, p.k, ws.data_ptr(),
                                             ws.numel(), nv.FLAG_WIDE_TENSOR, stream.cuda_stream)
                    if st != 0:
                        raise RuntimeError(f"launch failed: {nv.STATUS.get(st, st)}")
        stream.synchronize()
        return None
    per_mode = {}
    for mode, flags in (("passes", nv.FLAG_PREFETCH_WEIGHTS), ("tensor_tier", nv.FLAG_WIDE_TENSOR)):
        per_mode[mode] = run_wide_mode(args, world, L, ents, ws, stream, flags,
                                       ClockSampler(local) if mode == "tensor_tier" else None)
    top = per_mode["tensor_tier"][WIDE_ROWS[-1]]
    m = WIDE_ROWS[-1]

    # end to end through the public API at M = 128 on the tier: every projection's x in from
    # pinned host memory, every y back, per step
    hx = torch.cat([e["x"].reshape(-1) for e in ents]).cpu().pin_memory()
    dx = torch.empty_like(hx, device=dev)
    xs, off = [], 0
    for e in ents:
        xs.append(dx[off:off + e["x"].numel()].view(e["x"].shape))
        off += e["x"].numel()
    hy = [torch.empty_like(e["y"], device="cpu").pin_memory() for e in ents]
    cur = torch.cuda.current_stream()

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        for e, x in zip(ents, xs):
            p = e["p"]
            if p.dual:
                nv.gemv_dual(e["W"], e["S"], p.w.g, e["Wu"], e["Su"], p.w_up.g, x, y=e["y"],
                             ws=ws, stream=cur, wide_tensor=True)
            else:
                nv.gemv(e["W"], e["S"], p.w.g, x, y=e["y"], ws=ws, stream=cur, wide_tensor=True)
        for e, h in zip(ents, hy):
            h.copy_(e["y"], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(cur)
    for _ in range(args.e2e_steps):
        e2e_step()
    t1.record(cur)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(t0.elapsed_time(t1), world) / args.e2e_steps
    step_b = top["GBps"] * 1e9 * top["ms_per_step"] * 1e-3 / world
    e2e = {"value": round(world * step_b / (ms_e2e * 1e-3) / 1e9, 1), "unit": "GB/s",
           "h2d_bytes_per_step": hx.numel() * 2,
           "d2h_bytes_per_step": sum(e["y"].numel() * 2 for e in ents), "steps": args.e2e_steps,
           "api": "nvfp4_weight_only_03_b200.gemv / gemv_dual with wide_tensor=True, M = 128"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        threads = os.cpu_count() or 1
        qkv = projs[0]
        xb = synth.activations(wl.seed + 100, 0, m, qkv.k)
        t_end = time.perf_counter() + args.cpu_seconds
        b, n_calls, t_start = 0, 0, time.perf_counter()
        while time.perf_counter() < t_end:
            oracle.gemv(qkv.w.packed, qkv.w.scales, qkv.w.g, xb, rows=np.arange(64),
                        threads=threads)
            b += 64 * (qkv.k // 2 + qkv.k // 16) + m * qkv.k * 2 + m * 64 * 2
            n_calls += 1
        dt = time.perf_counter() - t_start
        cpu = {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_calls} calls of 64 qkv output rows at M = {m} ({dt:.1f} s)"}

    line = {"metric": METRIC, "value": top["GBps"], "unit": "GB/s", "n_gpus": world,
            "steps": top["steps"], "warmup": args.warmup, "ms_per_step": top["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4(e2m1+e4m3) x bf16 -> fp32 accumulate, bf16 out",
            "data": "synthetic (seeded N(0,0.02) weights quantised to NVFP4, N(0,1) bf16 x)",
            "config": {"workload": WIDE_DESC, "rows": list(WIDE_ROWS),
                       "l2": "0.2 GB of weights per pass, no flush"},
            "roofline": {"bound": "tensor", "achieved": top["TFLOPs"], "peak": peaks_bf16()[0],
                         "unit": "TFLOP/s", "frac": round(top["TFLOPs"] / peaks_bf16()[0], 4),
                         "traffic": None, "peak_source": peaks_bf16()[1],
                         "note": "f16 tcgen05 MMAs against the measured bf16 cuBLAS burst peak "
                                 "(the same rate for f16); the dual runs both streams on the tier"},
            "per_rows": per_mode,
            "gpu_launches": (top["kernels_per_step"] * top["steps"]
                             if top.get("kernels_per_step") is not None else None),
            "clocks": top.get("clocks"), "e2e": e2e}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def peaks_bf16():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(path))["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def graph_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (captured with keep_graph=True), or None."""
    try:
        from cuda.bindings import runtime as cr
        graph = g.raw_cuda_graph()
        if isinstance(graph, int):
            graph = cr.cudaGraph_t(init_value=graph)
        err, _, count = cr.cudaGraphGetNodes(graph, 0)
        err, nodes, count = cr.cudaGraphGetNodes(graph, count)
        kernels = 0
        for node in nodes[:count]:
            err, kind = cr.cudaGraphNodeGetType(node)
            if kind == cr.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kernels += 1
        return kernels
    except Exception:
        return None


def run_wide_mode(args, world, L, ents, ws, stream, flags, clocks=None):
    import torch
    import nvfp4_weight_only_03_b200 as nv
    per_m = {}
    for m in WIDE_ROWS:
        def launches(h):
            for e in ents:
                p = e["p"]
                if p.dual:
                    st = L.nvfp4_gemv_dual_ex(e["W"].data_ptr(), e["S"].data_ptr(), ctypes.c_float(p.w.g),
                                              e["Wu"].data_ptr(), e["Su"].data_ptr(), ctypes.c_float(p.w_up.g),
                                              e["x"].data_ptr(), p.k, e["y"].data_ptr(), p.n, m, p.n, p.k,
                                              ws.data_ptr(), ws.numel(), flags, h)
                else:
                    st = L.nvfp4_gemv_ex(e["W"].data_ptr(), e["S"].data_ptr(), ctypes.c_float(p.w.g),
                                         e["x"].data_ptr(), p.k, e["y"].data_ptr(), p.n, m, p.n, p.k,
                                         ws.data_ptr(), ws.numel(), flags, h)
                if st != 0:
                    raise RuntimeError(f"launch failed: {nv.STATUS.get(st, st)}")
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                launches(stream.cuda_stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=stream):
            launches(torch.cuda.current_stream().cuda_stream)
        g.instantiate()
        kernels = graph_kernel_nodes(g)
        g.replay()
        torch.cuda.synchronize()
        steps = max(1, args.steps // m)
        if clocks is not None and m == WIDE_ROWS[-1]:
            clocks.start()
            time.sleep(0.3)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            t0.record()
            for _ in range(steps):
                g.replay()
            t1.record()
        torch.cuda.synchronize()
        barrier(world)
        ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
        clk = clocks.stop() if clocks is not None and m == WIDE_ROWS[-1] else None
        b = sum((2 if e["p"].dual else 1) * (e["p"].n * e["p"].k * 9 // 16) + m * e["p"].k * 2
                + m * e["p"].n * 2 for e in ents)
        fl = sum((2 if e["p"].dual else 1) * 2 * m * e["p"].n * e["p"].k for e in ents)
        per_m[m] = {"ms_per_step": round(ms, 5), "GBps": round(world * b / (ms * 1e-3) / 1e9, 1),
                    "TFLOPs": round(world * fl / (ms * 1e-3) / 1e12, 1), "steps": steps,
                    "kernels_per_step": kernels}
        if clk is not None:
            per_m[m]["clocks"] = clk
        del g
    return per_m


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    run = {"sweep": run_ours, "attn_pairs": run_pairs, "wide_rows": run_wide,
           "prologue_layers": run_prologue}[args.workload]
    line = run(args, world, rank, local)
    if line is not None and rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
