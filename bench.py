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

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        if self.window is not None:
            inside = [x for x in lines if self.window[0] <= x[0] <= self.window[1]]
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
    of the first groups of every kv head, grown until about target_s of CPU time.  Returns
    (useful TFLOP/s of the oracle, threads, description, oracle ms per complete call)."""
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
    desc = (f"full oracle grouping ({t_group:.2f} s) + oracle attention of all rows of "
            f"{sample_groups} random groups of {n_groups} ({frac * 100:.2f}% of the work, "
            f"{t_attn:.1f} s); grouping time apportioned by that fraction")
    return rate, threads, desc, full_ms


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
    rates, threads, desc, full_ms = [], 0, "", []
    for _ in range(args.steps):
        r, threads, desc, fm = oracle_sample(inp, wl, args.W, args.g, per_step)
        rates.append(r)
        full_ms.append(fm)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s (useful)",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median(full_ms), "higher_is_better": True,
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
    inp = synth.make_inputs(wl)
    d = api.device_inputs(inp, dev)
    status = api.new_status(dev)
    groups = api.Groups.allocate(wl.T, wl.Hkv, inp["cu_seqlens"], wl.kmax, args.W, args.g, dev)
    O = torch.empty_like(d["Q"])
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        api.pw_group(d["sel_pages"], d["cu_seqlens"], d["cu_seqlens_host"], args.W, args.g,
                     groups=groups, status=status)
        api.pw_attn(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], d["cu_seqlens"],
                    groups, d["k_scale"], d["v_scale"], d["sm_scale"], O=O, status=status)

    clocks = ClockSampler(dev.index).__enter__()
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    api.check_status(status, "bench warm-up")
    gh = groups.to_host()
    union_bytes, exec_flops = group_work(gh, wl.G)
    uflops = useful_flops(inp, wl.Hq)
    usize = np.diff(gh["union_off"])

    # ---- device-timed region ----
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = time.monotonic()
    for i in range(K):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        api.pw_group(d["sel_pages"], d["cu_seqlens"], d["cu_seqlens_host"], args.W, args.g,
                     groups=groups, status=status)
        ev[i][1].record(stream)
        api.pw_attn(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], d["cu_seqlens"],
                    groups, d["k_scale"], d["v_scale"], d["sm_scale"], O=O, status=status)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks.mark(t_start, time.monotonic())
    clocks.__exit__(None, None, None)
    # secondary figure: the same calls with L2 left warm (no flush between them)
    wev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(K, 10))]
    for e in wev:
        e[0].record(stream)
        step()
        e[1].record(stream)
    torch.cuda.synchronize()
    warm_ms = [e[0].elapsed_time(e[1]) for e in wev]
    if world > 1:
        dist.barrier()
    api.check_status(status, "bench timed region")
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    group_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = float(sum(step_ms))
    if world > 1:
        total_ms = rank_max(total_ms, dist, dev)
    ms_per_step = total_ms / K
    value = job_rate(uflops, world, ms_per_step)

    # ---- end to end through the public API, host buffers ----
    e2e = None
    if not args.no_e2e:
        pin = {k: d[k].cpu().pin_memory() for k in ("Q", "K_pages", "V_pages", "page_table",
                                                     "sel_pages", "cu_seqlens")}
        out_host = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        dev_bufs = {k: torch.empty_like(d[k]) for k in pin}
        h2d = int(sum(v.numel() * v.element_size() for v in pin.values()))
        d2h = int(out_host.numel() * out_host.element_size())

        def e2e_step():
            for k_, v in pin.items():
                dev_bufs[k_].copy_(v, non_blocking=True)
            api.prefill(dev_bufs["Q"], dev_bufs["K_pages"], dev_bufs["V_pages"],
                        dev_bufs["page_table"], dev_bufs["sel_pages"], dev_bufs["cu_seqlens"],
                        d["cu_seqlens_host"], args.W, args.g, d["k_scale"], d["v_scale"],
                        d["sm_scale"], groups=groups, O=O, status=status)
            out_host.copy_(O, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ne = max(2, min(K, 5))
        e0.record(stream)
        for _ in range(ne):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / ne
        if world > 1:
            e2e_ms = rank_max(e2e_ms, dist, dev)
        e2e = {"value": job_rate(uflops, world, e2e_ms), "unit": "TFLOP/s (useful)",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    hbm, bf16, src = peaks()
    attn_mean = statistics.mean(attn_ms)
    achieved = union_bytes / (attn_mean * 1e-3) / 1e9
    ksrc = os.path.join(ROOT, "dynamic_sparse_attention_pw_b200", "csrc")
    khash = source_hash(*(os.path.join(ksrc, f) for f in
                          ("pw_attn.cu", "pw_attn_ws.cu", "pw_attn_common.cuh", "pw_sm100.cuh")))
    kname = "k_union_attn_ws" if args.g * wl.G <= 64 else "k_union_attn"
    roof_ms = max(union_bytes / (hbm * 1e9), exec_flops / (bf16 * 1e12)) * 1e3
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
            "algorithmic_bytes_per_launch": union_bytes,
            "kernel_ms": attn_mean,
        },
        "breakdown": {
            "group_ms": statistics.mean(group_ms), "attn_ms": attn_mean,
            "group_ms_median": statistics.median(group_ms), "attn_ms_median": statistics.median(attn_ms),
            "complete_call_ms_median": statistics.median(step_ms),
            "complete_call_ms_warm_l2_median": statistics.median(warm_ms),
            "complete_call_ms": ms_per_step,
            "roofline_ms": roof_ms, "complete_call_frac_of_roofline": roof_ms / ms_per_step,
            "attn_frac_of_roofline": roof_ms / attn_mean,
            "union_pages_mean": float(usize.mean()), "union_pages_max": int(usize.max()),
            "n_groups": int(gh["n_groups"]),
            "useful_tflop": uflops / 1e12, "executed_tflop_algorithmic": exec_flops / 1e12,
            "useful_over_executed": uflops / exec_flops,
            "tensor_frac_executed": exec_flops / (attn_mean * 1e-3) / (bf16 * 1e12),
        },
        "clocks": clocks.summary(),
        "gpu_launches": 5 * K,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and world == 1:
        rate, threads, desc, _ = oracle_sample(inp, wl, args.W, args.g, args.cpu_seconds)
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
