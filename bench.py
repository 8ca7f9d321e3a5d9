"""Benchmark of one complete PageWeaver prefill call (pw_group + pw_attn) on B200.

Default workload: 64K-token prefill, Hq=64 / Hkv=8, head dim 128, 64-token FP8 E4M3 pages,
k=32 community-structured page selections, g=8, W=128 (synthetic stand-in for the pages'
64K-context captures).  One step = one complete call over that batch, inputs resident in HBM.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle instead (bounded
sample of the same workload, on the host cores).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0
PAGE, D = 64, 128
METRIC = "complete-call ms and useful TFLOP/s (grouping incl.) at 1 B200; % of roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--W", type=int, default=128)
    ap.add_argument("--g", type=int, default=8)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave out the per-configuration runs of the measurement plan")
    ap.add_argument("--sweep-steps", type=int, default=10)
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, BF16_FALLBACK_TFLOPS, "fallback"


# ------------------------------------------------------------------------------------------
# work accounting (host, from the inputs and the group lists)
# ------------------------------------------------------------------------------------------

def useful_flops(inp, Hq) -> float:
    """sum over (t, hq) of 4 * 128 * (number of keys the query attends to)."""
    sel, cu = inp["sel_pages"], inp["cu_seqlens"]
    T, Hkv, k = sel.shape
    total = 0
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        pos = np.arange(e - s, dtype=np.int64)
        own = pos // PAGE
        for h in range(Hkv):
            rows = np.sort(sel[s:e, h], axis=1)
            valid = rows >= 0
            dup = np.zeros_like(valid)
            dup[:, 1:] = rows[:, 1:] == rows[:, :-1]
            keep = valid & ~dup
            keys = np.where(rows < own[:, None], PAGE, (pos % PAGE + 1)[:, None])
            total += int((keys * keep).sum())
    G = Hq // Hkv
    return float(total) * G * 4 * D


def group_work(gh: dict, G: int):
    """(algorithmic union bytes, executed FLOPs) of one pw_attn launch."""
    usize = np.diff(gh["union_off"]).astype(np.int64)
    union_bytes = float(usize.sum()) * 2 * PAGE * D          # K + V pages, E4M3
    rows = gh["gsize"].astype(np.int64) * G
    exec_flops = float((usize * rows).sum()) * PAGE * D * 4
    return union_bytes, exec_flops


# Tensor-core work the pipelined kernel (tiles of <= 64 rows) issues per union page of a group,
# whatever the group's row count R:
#   S = Q K^T: two E4M3 parts of Q (K-concatenated), M = 64 rows (the tile, zero-padded), N = 64
#     keys, K = 2 x 128 -> 2 * 64 * 64 * 256 FLOP.  An M = 64 product takes as long as an
#     M = 128 one, so its tensor time is that of 2 * 128 * 64 * 256 FLOP at the E4M3 rate.
#   O += P V: P_hi and P_lo stacked as one M = 128 operand, N = 128 dims, K = 64 keys
#     -> 2 * 128 * 128 * 64 FLOP at the f16 rate.
S_ISSUED_PER_PAGE = 2 * 64 * 64 * 256
S_TIME_EQUIV_PER_PAGE = 2 * 128 * 64 * 256
PV_ISSUED_PER_PAGE = 2 * 128 * 128 * 64
FP8_OVER_BF16 = 2.0   # nominal dense E4M3 : bf16 throughput ratio of the tensor cores


def issued_work(gh: dict):
    """(issued tensor FLOPs, seconds those products need at the peaks, as a function of the
    bf16 peak in TFLOP/s) of one pw_attn launch of the pipelined kernel."""
    pages = float(np.diff(gh["union_off"]).astype(np.int64).sum())
    issued = pages * (S_ISSUED_PER_PAGE + PV_ISSUED_PER_PAGE)

    def seconds_at_peak(bf16_tflops: float) -> float:
        return pages * (S_TIME_EQUIV_PER_PAGE / (FP8_OVER_BF16 * bf16_tflops * 1e12) +
                        PV_ISSUED_PER_PAGE / (bf16_tflops * 1e12))
    return issued, seconds_at_peak


def source_hash(*paths) -> str:
    """Fingerprint of the kernel code: comments and blank lines are left out, so that a change
    of comments alone keeps a traffic record taken on the same code."""
    h = hashlib.sha256()
    for p in paths:
        with open(p, encoding="utf-8") as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("\n".join(l.rstrip() for l in src.splitlines() if l.strip()).encode())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel_src_hash: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it
    was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "union_attn_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("kernel_source_sha") == kernel_src_hash:
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------------------------------
# clocks sampler
# ------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    """nvidia-smi samples every 20 ms, started before the warm-up (its start-up takes longer
    than a short timed region) and reduced to the samples taken inside the timed window."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []          # (host monotonic time, csv line)
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            deadline = time.monotonic() + 5.0
            while not self.lines and time.monotonic() < deadline:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, window=None):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = list(self.lines)
        window = window if window is not None else self.window
        if window is not None:
            inside = [x for x in lines if window[0] <= x[0] <= window[1]]
            lines = inside if inside else lines
        for _, ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ------------------------------------------------------------------------------------------

def oracle_sample(inp, wl, W, g, target_s: float):
    """Time the oracle on a bounded sample: the full grouping plus the attention of the rows
    of random groups, grown until about target_s of CPU time.  Returns (useful TFLOP/s of the
    oracle, threads, description, estimated oracle ms of one complete call (extrapolated from
    the sample), measured wall ms of the sample)."""
    from oracle import oracle
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    gr = oracle.group(inp["sel_pages"], inp["cu_seqlens"], W, g)
    t_group = time.perf_counter() - t0
    G = wl.G
    # rows of groups in order, until the estimated cost reaches the budget
    rows_t, rows_h = [], []
    n_groups = gr["n_groups"]
    order = np.random.default_rng(0).permutation(n_groups)
    probe = 0
    t_attn = 0.0
    flops_done = 0.0
    sample_groups = 0
    sel = inp["sel_pages"]
    while t_attn < target_s and probe < n_groups:
        batch = order[probe: probe + 64]
        probe += len(batch)
        rt, rh = [], []
        for gi in batch:
            h = int(gr["gmeta"][gi, 1])
            for t in gr["qids"][gi, : gr["gsize"][gi]]:
                for j in range(G):
                    rt.append(int(t))
                    rh.append(h * G + j)
        sample_groups += len(batch)
        t1 = time.perf_counter()
        oracle.attn_rows(inp, np.array(rt, np.int64), np.array(rh, np.int32), threads)
        t_attn += time.perf_counter() - t1
        # useful flops of these rows
        cu = inp["cu_seqlens"]
        for t, hq in zip(rt, rh):
            b = int(np.searchsorted(cu, t, side="right") - 1)
            pos = t - int(cu[b])
            pages = {int(p) for p in sel[t, hq // G] if p >= 0}
            flops_done += sum(PAGE if p < pos // PAGE else pos % PAGE + 1 for p in pages) * 4 * D
    frac = sample_groups / max(n_groups, 1)
    t_sample = t_attn + t_group * frac
    rate = flops_done / t_sample / 1e12
    full_ms = (t_group + t_attn / max(frac, 1e-12)) * 1e3
    wall_ms = (t_group + t_attn) * 1e3
    desc = (f"full oracle grouping ({t_group:.2f} s) + oracle attention of all rows of "
            f"{sample_groups} random groups of {n_groups} ({frac * 100:.2f}% of the work, "
            f"{t_attn:.1f} s); grouping time apportioned by that fraction")
    return rate, threads, desc, full_ms, wall_ms


# ------------------------------------------------------------------------------------------
# arms
# ------------------------------------------------------------------------------------------

def rank_max(x: float, dist_mod, device) -> float:
    """The largest x over the ranks of the process group: a job's time is its slowest rank's."""
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput in units of 1e12 per second: every rank processes units_per_rank
    (weak scaling), and the job takes ms."""
    return units_per_rank * world / (ms * 1e-3) / 1e12


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from dynamic_sparse_attention_pw_b200 import synth
    wl = synth.WORKLOADS[args.workload].with_(W=args.W, g=args.g)
    inp = synth.make_inputs(wl)
    uflops = useful_flops(inp, wl.Hq)
    per_step = max(args.cpu_seconds / max(args.steps, 1), 2.0)
    for _ in range(args.warmup):
        oracle_sample(inp, wl, args.W, args.g, 0.5)
    rates, threads, desc, full_ms, wall_ms = [], 0, "", [], []
    for _ in range(args.steps):
        r, threads, desc, fm, wm = oracle_sample(inp, wl, args.W, args.g, per_step)
        rates.append(r)
        full_ms.append(fm)
        wall_ms.append(wm)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s (useful)",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        # a step is one bounded sample of the workload (see cpu_baseline.sample): its measured
        # wall time; the time of one whole call is an extrapolation, reported separately
        "ms_per_step": statistics.median(wall_ms),
        "full_call_ms_estimate": statistics.median(full_ms),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s (useful)", "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s (useful)", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_of(wl, args):
    return {"workload": f"{wl.name}: T={wl.T} tokens, Hq={wl.Hq}/Hkv={wl.Hkv}, d=128, "
                        f"page=64, k={wl.kmax}, FP8 E4M3 KV, g={args.g}, W={args.W}",
            "T": wl.T, "Hq": wl.Hq, "Hkv": wl.Hkv, "kmax": wl.kmax, "g": args.g, "W": args.W,
            "l2": "flushed (256 MiB write) before every timed step, outside the timed events",
            "parallelism": f"independent replicas x{args.gpus} (weak)"}


class Timed:
    """One configuration on the device: its inputs, group buffers and output, and the device
    timing of complete calls (pw_group then pw_attn on the current stream, CUDA events)."""

    def __init__(self, wl, W, g, dev, inp=None):
        import torch
        from dynamic_sparse_attention_pw_b200 import api, synth
        self.api, self.wl, self.W, self.g = api, wl, W, g
        self.inp = inp if inp is not None else synth.make_inputs(wl)
        self.d = api.device_inputs(self.inp, dev)
        self.status = api.new_status(dev)
        self.groups = api.Groups.allocate(wl.T, wl.Hkv, self.inp["cu_seqlens"], wl.kmax, W, g, dev)
        self.O = torch.empty_like(self.d["Q"])
        self.stream = torch.cuda.current_stream()

    def group(self):
        d = self.d
        self.api.pw_group(d["sel_pages"], d["cu_seqlens"], d["cu_seqlens_host"], self.W, self.g,
                          groups=self.groups, status=self.status)

    def attn(self):
        d = self.d
        self.api.pw_attn(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], d["cu_seqlens"],
                         self.groups, d["k_scale"], d["v_scale"], d["sm_scale"], O=self.O,
                         status=self.status)

    def run(self, steps, flush, warmup=3):
        """Warm-up calls, then `steps` timed calls with L2 flushed before each (outside the
        events), then up to 10 calls with L2 left warm.  Returns per-call (group, attn,
        complete) ms lists, the warm-L2 list and the host window of the timed calls."""
        import torch
        for _ in range(warmup):
            flush.fill_(1)
            self.group()
            self.attn()
        torch.cuda.synchronize()
        self.api.check_status(self.status, f"{self.wl.name} warm-up")
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        torch.cuda.synchronize()
        t0 = time.monotonic()
        for i in range(steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(self.stream)
            self.group()
            ev[i][1].record(self.stream)
            self.attn()
            ev[i][2].record(self.stream)
        torch.cuda.synchronize()
        window = (t0, time.monotonic())
        wev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(steps, 10))]
        for e in wev:
            e[0].record(self.stream)
            self.group()
            self.attn()
            e[1].record(self.stream)
        torch.cuda.synchronize()
        self.api.check_status(self.status, f"{self.wl.name} timed calls")
        group_ms = [e[0].elapsed_time(e[1]) for e in ev]
        attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
        step_ms = [e[0].elapsed_time(e[2]) for e in ev]
        warm_ms = [e[0].elapsed_time(e[1]) for e in wev]
        return group_ms, attn_ms, step_ms, warm_ms, window

    def work(self):
        gh = self.groups.to_host()
        union_bytes, exec_flops = group_work(gh, self.wl.G)
        issued, at_peak = issued_work(gh)
        usize = np.diff(gh["union_off"])
        return {"gh": gh, "union_bytes": union_bytes, "exec_flops": exec_flops,
                "issued_flops": issued, "tensor_seconds_at_peak": at_peak,
                "useful_flops": useful_flops(self.inp, self.wl.Hq), "usize": usize}


def breakdown(wk, group_ms, attn_ms, step_ms, warm_ms, hbm, bf16):
    attn_mean = statistics.mean(attn_ms)
    call_mean = statistics.mean(step_ms)
    roof_ms = max(wk["union_bytes"] / (hbm * 1e9), wk["exec_flops"] / (bf16 * 1e12)) * 1e3
    usize = wk["usize"]
    return {
        "group_ms": statistics.mean(group_ms), "attn_ms": attn_mean,
        "group_ms_median": statistics.median(group_ms), "attn_ms_median": statistics.median(attn_ms),
        "complete_call_ms": call_mean,
        "complete_call_ms_median": statistics.median(step_ms),
        "complete_call_ms_warm_l2_median": statistics.median(warm_ms),
        "roofline_ms": roof_ms, "complete_call_frac_of_roofline": roof_ms / call_mean,
        "attn_frac_of_roofline": roof_ms / attn_mean,
        "union_pages_mean": float(usize.mean()) if usize.size else 0.0,
        "union_pages_max": int(usize.max()) if usize.size else 0,
        "n_groups": int(wk["gh"]["n_groups"]),
        "useful_tflop": wk["useful_flops"] / 1e12,
        "executed_tflop_algorithmic": wk["exec_flops"] / 1e12,
        "useful_over_executed": wk["useful_flops"] / wk["exec_flops"] if wk["exec_flops"] else None,
        "issued_tflop": wk["issued_flops"] / 1e12,
        "useful_over_issued": wk["useful_flops"] / wk["issued_flops"] if wk["issued_flops"] else None,
        "tensor_frac_issued_at_peak": wk["tensor_seconds_at_peak"](bf16) / (attn_mean * 1e-3),
        "useful_tflops": wk["useful_flops"] / (call_mean * 1e-3) / 1e12,
    }


# The per-configuration runs of the measurement plan: the 64K workload swept over W, the 32K
# workload grouped four ways (contiguous W = g, regrouped W = 128, one query per group, and
# sixteen queries per group, whose 16 x 4 rows fill the 64-row tile that eight queries fill
# only half of), and the remaining workloads at their own W.
SWEEP = [(4, 32, 8), (4, 64, 8), (4, 256, 8), (3, 8, 8), (3, 128, 8), (3, 128, 1),
         (3, 128, 16), (1, 32, 8), (2, 64, 8), (5, 128, 8)]


def launches_per_call(words, W):
    """Kernels of one complete call: pw_group's bitset, greedy (plus the renumbering greedy for
    windows whose staged rows would exceed 2112 words), offset and page kernels, then pw_attn."""
    return 5 + (1 if words > 8 and words * (W + 1) > 2112 else 0)


def run_overlap(dev, inp, W, steps, warmup=3):
    """Grouping of call n + 1 on a second stream beside the attention of call n (two sets of
    group buffers and status words), against the same calls one after the other.  Returns the
    mean ms per call of each schedule; the 64K workload's inputs exceed L2, so no flush."""
    import torch
    from dynamic_sparse_attention_pw_b200 import api, synth
    wl = synth.WORKLOADS[4].with_(W=W, g=8)
    t = Timed(wl, W, 8, dev, inp=inp)
    d = t.d
    bufs = [(t.groups, t.status),
            (api.Groups.allocate(wl.T, wl.Hkv, inp["cu_seqlens"], wl.kmax, W, 8, dev),
             api.new_status(dev))]
    main, side = torch.cuda.current_stream(), torch.cuda.Stream(dev)

    def group(i, stream):
        g_, st = bufs[i % 2]
        api.pw_group(d["sel_pages"], d["cu_seqlens"], d["cu_seqlens_host"], W, 8, groups=g_,
                     status=st, stream=stream)

    def attn(i, stream):
        g_, st = bufs[i % 2]
        api.pw_attn(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], d["cu_seqlens"], g_,
                    d["k_scale"], d["v_scale"], d["sm_scale"], O=t.O, status=st, stream=stream)

    n = warmup + steps
    ev = lambda: torch.cuda.Event(enable_timing=True)
    # one after the other, on one stream
    seq = [ev() for _ in range(2)]
    for i in range(n):
        if i == warmup:
            seq[0].record(main)
        group(i, main)
        attn(i, main)
    seq[1].record(main)
    torch.cuda.synchronize()
    # overlapped: grouping i + 1 (side) waits only for attention i - 1, which read its buffers
    gdone = [torch.cuda.Event() for _ in range(n + 1)]
    adone = [torch.cuda.Event() for _ in range(n)]
    ovl = [ev() for _ in range(2)]
    side.wait_stream(main)
    group(0, side)
    gdone[0].record(side)
    for i in range(n):
        if i >= 1:
            side.wait_event(adone[i - 1])
        if i + 1 < n:
            group(i + 1, side)
            gdone[i + 1].record(side)
        main.wait_event(gdone[i])
        if i == warmup:
            ovl[0].record(main)
        attn(i, main)
        adone[i].record(main)
    ovl[1].record(main)
    main.wait_stream(side)
    torch.cuda.synchronize()
    for _, st in bufs:
        api.check_status(st, f"{wl.name} overlapped calls")
    return {"workload": wl.name, "W": W, "g": 8, "steps": steps,
            "sequential_ms_per_call": seq[0].elapsed_time(seq[1]) / steps,
            "overlapped_ms_per_call": ovl[0].elapsed_time(ovl[1]) / steps}


def run_sweep(args, dev, flush, clocks, hbm, bf16, head_inp):
    """One entry per SWEEP configuration (the headline configuration is the line itself)."""
    import torch
    from dynamic_sparse_attention_pw_b200 import synth
    out = []
    inputs = {args.workload: head_inp}
    for cfg, W, g in SWEEP:
        if (cfg, W, g) == (args.workload, args.W, args.g):
            continue
        wl = synth.WORKLOADS[cfg].with_(W=W, g=g)
        if cfg not in inputs:
            inputs = {cfg: synth.make_inputs(synth.WORKLOADS[cfg])}
        t = Timed(wl, W, g, dev, inp=inputs[cfg])
        gm, am, sm_, wm, window = t.run(args.sweep_steps, flush)
        wk = t.work()
        bd = breakdown(wk, gm, am, sm_, wm, hbm, bf16)
        achieved = wk["union_bytes"] / (bd["attn_ms"] * 1e-3) / 1e9
        entry = {"workload": wl.name, "T": wl.T, "W": W, "g": g, "steps": args.sweep_steps,
                 "union_pages_mean": bd["union_pages_mean"], "union_pages_max": bd["union_pages_max"],
                 "group_ms": bd["group_ms"], "attn_ms": bd["attn_ms"],
                 "complete_call_ms": bd["complete_call_ms"],
                 "complete_call_ms_warm_l2_median": bd["complete_call_ms_warm_l2_median"],
                 "useful_tflops": bd["useful_tflops"],
                 "attn_frac_of_roofline": bd["attn_frac_of_roofline"],
                 "union_byte_rate_gbs": achieved,
                 "useful_over_issued": bd["useful_over_issued"],
                 "tensor_frac_issued_at_peak": bd["tensor_frac_issued_at_peak"],
                 "clocks": clocks.summary(window)}
        out.append(entry)
        del t
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    from dynamic_sparse_attention_pw_b200 import api, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    wl = synth.WORKLOADS[args.workload].with_(W=args.W, g=args.g)
    head = Timed(wl, args.W, args.g, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(dev.index).__enter__()
    K = args.steps

    # ---- device-timed region (the same calls on every rank, then the slowest rank's time) ----
    if world > 1:
        dist.barrier()
    group_ms, attn_ms, step_ms, warm_ms, window = head.run(K, flush, warmup=max(args.warmup, 3))
    clocks.mark(*window)
    if world > 1:
        dist.barrier()
    total_ms = float(sum(step_ms))
    if world > 1:
        total_ms = rank_max(total_ms, dist, dev)
    ms_per_step = total_ms / K
    wk = head.work()
    value = job_rate(wk["useful_flops"], world, ms_per_step)

    # ---- end to end through the public API, host buffers ----
    e2e = None
    d = head.d
    if not args.no_e2e:
        pin = {k: d[k].cpu().pin_memory() for k in ("Q", "K_pages", "V_pages", "page_table",
                                                     "sel_pages", "cu_seqlens")}
        out_host = torch.empty(head.O.shape, dtype=head.O.dtype).pin_memory()
        h2d = int(sum(v.numel() * v.element_size() for v in pin.values()))
        d2h = int(out_host.numel() * out_host.element_size())
        # Successive calls pipelined the way a serving loop would run them: two sets of device
        # inputs and outputs, step i + 1's inputs copied in on one copy stream while step i
        # computes and its output is copied out on another (host-to-device and device-to-host
        # copies share the link in both directions at once).  Every step still copies its own
        # inputs in and reads its own result back.
        sets = [{k: torch.empty_like(d[k]) for k in pin} for _ in range(2)]
        outs = [torch.empty_like(head.O) for _ in range(2)]
        main = head.stream
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            s_in.wait_stream(main)
            s_out.wait_stream(main)
            for i in range(n):
                j = i % 2
                if i >= 2:
                    s_in.wait_event(comp_done[j])     # step i - 2 has read input set j
                with torch.cuda.stream(s_in):
                    for k_, v in pin.items():
                        sets[j][k_].copy_(v, non_blocking=True)
                in_done[j].record(s_in)
                main.wait_event(in_done[j])
                if i >= 2:
                    main.wait_event(out_done[j])      # step i - 2's output is on the host
                api.prefill(sets[j]["Q"], sets[j]["K_pages"], sets[j]["V_pages"],
                            sets[j]["page_table"], sets[j]["sel_pages"], sets[j]["cu_seqlens"],
                            d["cu_seqlens_host"], args.W, args.g, d["k_scale"], d["v_scale"],
                            d["sm_scale"], groups=head.groups, O=outs[j], status=head.status,
                            stream=main)
                comp_done[j].record(main)
                s_out.wait_event(comp_done[j])
                with torch.cuda.stream(s_out):
                    out_host.copy_(outs[j], non_blocking=True)
                out_done[j].record(s_out)
            main.wait_stream(s_in)
            main.wait_stream(s_out)

        e2e_steps(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ne = max(4, min(K, 8))
        e0.record(main)
        e2e_steps(ne)
        e1.record(main)
        torch.cuda.synchronize()
        api.check_status(head.status, f"{wl.name} end-to-end calls")
        e2e_ms = e0.elapsed_time(e1) / ne
        if world > 1:
            e2e_ms = rank_max(e2e_ms, dist, dev)
        e2e = {"value": job_rate(wk["useful_flops"], world, e2e_ms), "unit": "TFLOP/s (useful)",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "schedule": "successive calls pipelined: inputs of step i + 1 copied in while "
                           "step i computes and its output is copied out"}
        del sets, outs
        torch.cuda.empty_cache()

    if rank != 0:
        clocks.__exit__(None, None, None)
        if world > 1:
            dist.destroy_process_group()
        return 0

    hbm, bf16, src = peaks()
    sweep = overlap = None
    if not args.no_sweep and world == 1:
        sweep = run_sweep(args, dev, flush, clocks, hbm, bf16, head.inp)
        if args.workload == 4:
            overlap = [run_overlap(dev, head.inp, W, args.sweep_steps) for W in (128, 256)]
    clocks.__exit__(None, None, None)

    bd = breakdown(wk, group_ms, attn_ms, step_ms, warm_ms, hbm, bf16)
    attn_mean = bd["attn_ms"]
    achieved = wk["union_bytes"] / (attn_mean * 1e-3) / 1e9
    ksrc = os.path.join(ROOT, "dynamic_sparse_attention_pw_b200", "csrc")
    khash = source_hash(*(os.path.join(ksrc, f) for f in
                          ("pw_attn.cu", "pw_attn_ws.cu", "pw_attn_common.cuh", "pw_sm100.cuh")))
    kname = "k_union_attn_ws" if args.g * wl.G <= 64 else "k_union_attn"
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s (useful)",
        "n_gpus": world,
        "steps": K,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 x e4m3 (S, Q split exactly in two e4m3 parts) and f16 x f16 (PV, P split in f16 hi + lo), fp32 accumulate",
        "data": "synthetic",
        "config": config_of(wl, args),
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": traffic_from_profile(khash),
            "kernel": kname, "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)"
            if src == "measured" else "fallback 6650 GB/s",
            "achieved_is": "union-byte rate: the K and V pages of every group's union counted once "
                           "per group, over the kernel's time; pages shared by nearby groups come "
                           "from L2, so DRAM moves far fewer bytes (traffic)",
            "algorithmic_bytes_per_launch": wk["union_bytes"],
            "kernel_ms": attn_mean,
        },
        "breakdown": bd,
        "clocks": clocks.summary(),
        "gpu_launches": launches_per_call(head.groups.words, args.W) * K,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if sweep is not None:
        line["sweep"] = sweep
    if overlap is not None:
        line["grouping_overlap"] = overlap
    if not args.no_cpu_baseline and world == 1:
        rate, threads, desc, _, _ = oracle_sample(head.inp, wl, args.W, args.g, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s (useful)", "cores": threads,
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
