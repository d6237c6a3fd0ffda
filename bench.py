#!/usr/bin/env python
"""Throughput of the looped recurrent block on B200 through the librdt C ABI.

One step = one rdt_loop_forward call: T = 8 loops of the GQA block (batch 4 x seq 512,
dim 1024, 16/4 heads of 64, 16 experts top-2, SwiGLU hidden 1024, bf16 storage, fp32
state) on seeded synthetic inputs resident in HBM. The L2 cache is flushed (256 MiB
write) before every timed step; each step is timed with CUDA events on its stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--act]

N > 1 runs under torchrun: every rank runs its own full replica (no data-path
collective; weak scaling); the timed region is bracketed by a barrier and a device
synchronise, and the step time is the maximum over ranks. `--impl reference` times the
fp64 CPU oracle on the host cores instead (rank 0 only). `--act` times the same workload
through rdt_loop_forward_act (ACT halting, threshold 0.99, the seeded halting head) and
reports the halting histogram; its tokens·loops count the T = 8 loops asked for.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "gqa-bf16-b4s512-d1024-h16x4-e16k2"
LOOPS = 8
METRIC = "recurrent-block tokens·loops/sec (bf16 fwd, 1 B200) and % of roofline"
UNIT = "tokens*loops/s"
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a kernel, from one
# ncu capture of this workload, valid only while the kernel's code is the one captured
# (fingerprint: first 16 hex digits of the SHA-256 of the listed files' code, concatenated:
# comments removed, each line stripped, blank lines dropped, so that an edit of a comment
# or of indentation keeps the capture while any change to a code token voids it).
KERNEL_SOURCES = {"gemm_up": ("recurrent_depth_transformer_b200/csrc/gemm_tc.cuh",
                              "recurrent_depth_transformer_b200/csrc/gemm_tc.cu",
                              "recurrent_depth_transformer_b200/csrc/gemm_tc_pair.cu",
                              "recurrent_depth_transformer_b200/csrc/rdt_internal.cuh",
                              "recurrent_depth_transformer_b200/csrc/rdt_api.cu")}
MEASURED_TRAFFIC = {"gemm_up": (79.72864e6 + 2.450688e6, "77aada7e305fe0e8")}


def code_text(src: str) -> str:
    """C/C++/CUDA source without its comments: string and character literals are kept whole
    (a '//' inside one is code), each line is stripped and blank lines are dropped."""
    out = []
    i, n = 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c and src[j] != "\n":
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.strip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def source_fingerprint(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(code_text(fh.read()).encode("utf-8"))
        h.update(b"\0")
    return h.hexdigest()[:16]


def measured_traffic(kernel):
    """The captured traffic of `kernel`, or None once its sources differ from the captured."""
    if kernel not in MEASURED_TRAFFIC or kernel not in KERNEL_SOURCES:
        return None
    value, fp = MEASURED_TRAFFIC[kernel]
    try:
        return value if source_fingerprint(KERNEL_SOURCES[kernel]) == fp else None
    except (OSError, ValueError):          # missing or undecodable source: no claim
        return None


# ----------------------------------------------------------------------------- algorithmic work

def kernel_work(wl, T):
    """Algorithmic FLOPs and DRAM bytes per launch of each kernel class (counts of what the
    block must compute and move, not of what a kernel happens to do: causal attention
    counts the S(S+1)/2 unmasked pairs, the expert GEMMs the N*k routed rows)."""
    N, d = wl.batch * wl.seq, wl.dim
    hq, hkv, dh = wl.n_heads, wl.n_kv_heads, wl.head_dim
    E, k, hid, S = wl.n_experts, wl.top_k, wl.expert_hidden, wl.n_shared
    rows = N * (k + S)
    nqkv = (hq + 2 * hkv) * dh
    b2 = 2
    w = {}
    w["gemm_qkv"] = dict(flops=2.0 * N * d * nqkv, bytes=b2 * (N * d + nqkv * d + N * nqkv), bound="tensor")
    pairs = wl.batch * wl.seq * (wl.seq + 1) / 2
    w["attention"] = dict(flops=4.0 * hq * dh * pairs, bytes=b2 * N * (nqkv + hq * dh), bound="tensor")
    # the O projection completes y = x + a and h_next = A h + B e + a with two fp32 reductions
    w["gemm_o"] = dict(flops=2.0 * N * hq * dh * d, bytes=b2 * (N * hq * dh + d * hq * dh) + 4 * 2 * N * d,
                       bound="tensor")
    w["gemm_up"] = dict(flops=2.0 * rows * d * 2 * hid, bytes=b2 * (rows * d + (E + S) * 2 * hid * d + rows * hid),
                        bound="tensor")
    w["gemm_down"] = dict(flops=2.0 * rows * hid * d, bytes=b2 * (rows * hid + (E + S) * d * hid) + 4 * N * d * 2,
                          bound="tensor")
    # RMSNorm1 reads h, e, B e and writes xn, y = x and h_next = A h + B e
    w["norm1"] = dict(flops=0.0, bytes=N * d * (4 + b2 + 4 + b2 + 4 + 4), bound="hbm")
    # RMSNorm2 fused with the fp32 router and the dispatch (W_r staged in shared memory): y in;
    # per (token, slot) the routing (index, weight, row token, row weight) and the yn copy in
    # the expert's rows; yn itself only when shared experts read it
    w["router_topk"] = dict(flops=2.0 * N * d * E,
                            bytes=N * d * 4 + (N * d * b2 if S else 0) + E * d * b2 + N * k * (d * b2 + 16),
                            bound="hbm")
    w["moe_dispatch"] = dict(flops=0.0, bytes=N * k * (d * b2 * 2 + 16), bound="hbm")
    w["hoist"] = dict(flops=0.0, bytes=N * d * (b2 + b2 + 4 + 4), bound="hbm")
    w["check_finite"] = dict(flops=0.0, bytes=N * d * 4, bound="hbm")
    return w


def step_flops(wl, T):
    w = kernel_work(wl, T)
    per_loop = sum(w[k]["flops"] for k in ("gemm_qkv", "attention", "gemm_o", "gemm_up", "gemm_down"))
    per_loop += 2.0 * wl.batch * wl.seq * wl.dim * wl.n_experts      # router logits
    return per_loop * T


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

CLOCK_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    def __init__(self):
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, window=None):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        return parse_clocks(open(self.path).read(), window)


def _stamp(text):
    """nvidia-smi timestamp ('2026/12/02 19:04:21.123', host local time) -> epoch seconds."""
    import datetime
    for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
        try:
            return datetime.datetime.strptime(text, fmt).timestamp()
        except ValueError:
            pass
    return None


def parse_clocks(text, window=None):
    """Median SM clock and the throttle reasons seen. With window = (t0, t1) (host epoch
    seconds of the timed region) only the samples taken inside it count, unless none was."""
    rows = []
    for line in text.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 10:
            continue
        try:
            rows.append((_stamp(parts[0]), float(parts[2]), float(parts[3]), parts[6:10]))
        except ValueError:
            continue
    if window is not None:
        inside = [r for r in rows if r[0] is not None and window[0] <= r[0] <= window[1]]
        if inside:
            rows = inside
    if not rows:
        return None
    reasons = set()
    for r in rows:
        for name, val in zip(REASONS, r[3]):
            if val.lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max(r[2] for r in rows),
            "reasons": sorted(reasons), "samples": len(rows), "in_timed_region": window is not None and
            any(window[0] <= (r[0] or 0) <= window[1] for r in rows)}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def reduce_max(value: float, device=None) -> float:
    """Maximum of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_ms, tokens_per_step, loops, world):
    """Whole-job throughput: every rank processes its own tokens; the job takes as long as
    the slowest rank."""
    ms = max(per_rank_ms)
    return world * tokens_per_step * loops / (ms / 1e3), ms


# ----------------------------------------------------------------------------- CPU baseline

def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info()), default=0)
        if n:
            return int(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(wl, inputs, seconds=10.0):
    """Time the fp64 oracle on one sequence (512 tokens) through all loops, repeated until
    `seconds` of CPU work; returns (tokens*loops/s, description)."""
    import oracle as O
    sub = dict(inputs)
    sub["e"] = inputs["e"][:1]
    sub["h0"] = sub["e"]
    w1 = wl.replace(batch=1)
    t0 = time.perf_counter()
    runs = 0
    while True:
        O.loop_forward(sub["h0"], sub["e"], LOOPS, sub, w1)
        runs += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return runs * wl.seq * LOOPS / el, f"{runs} x (1 of {wl.batch} sequences, {wl.seq} tokens, {LOOPS} loops), {el:.1f} s"


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from workloads import by_name, generate
    import oracle as O
    wl = by_name(WORKLOAD)
    inputs = generate(wl)
    sub = dict(inputs)
    sub["e"] = inputs["e"][:1]
    sub["h0"] = sub["e"]
    w1 = wl.replace(batch=1)
    for _ in range(args.warmup):
        O.loop_forward(sub["h0"], sub["e"], 1, sub, w1)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.loop_forward(sub["h0"], sub["e"], LOOPS, sub, w1)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = wl.seq * LOOPS / (ms / 1e3)
    sample = f"1 of {wl.batch} sequences ({wl.seq} tokens) through all {LOOPS} loops per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": wl.batch, "seq": wl.seq, "dim": wl.dim, "loops": LOOPS,
                   "parallelism": "host cores (fp64 NumPy oracle)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import recurrent_depth_transformer_b200 as R
    from workloads import by_name, generate

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    wl = by_name(WORKLOAD)
    inputs = generate(wl)
    weights = R.device_weights(inputs, True, device=dev)
    h = R.RDT(R.make_config(wl, max_loops=LOOPS), weights)
    del weights
    e = torch.from_numpy(inputs["e"]).to(torch.bfloat16).to(dev)
    out = torch.empty(e.shape, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    N = wl.batch * wl.seq

    nl = None
    if args.act:
        from workloads import act_head
        head = act_head(wl)
        h.set_act(torch.from_numpy(head["w_halt"]).to(dev), head["b_halt"], head["threshold"])
        nl = torch.empty((wl.batch, wl.seq), dtype=torch.int32, device=dev)

        def step():
            h.loop_forward_act(e, e, LOOPS, out=out, n_loops=nl)
    else:
        def step():
            h.loop_forward(e, e, LOOPS, out=out)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    # ---- timed region (device time, CUDA events on the launch stream)
    sampler = ClockSampler() if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = h.launch_count()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_wall0 = time.time()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    launches = h.launch_count() - launches0
    clocks = sampler.stop((t_wall0, t_wall1)) if sampler else None
    ms_rank = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    ms_all = reduce_max(ms_rank, dev)
    value, ms = aggregate([ms_all], N, LOOPS, world)

    # ---- per-kernel event timing over the same number of steps
    h.profile(True)
    for _ in range(args.steps):
        flush.zero_()
        step()
    stats, _ = h.profile_read()
    h.profile(False)

    # ---- end to end through the host-buffer entry point (pinned memory, copies inside)
    if args.act:
        return act_line(args, h, wl, nl, value, ms, world, rank, stats, launches, clocks)
    e_host = e.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    for _ in range(3):                       # eager, graph capture, first replay
        h.loop_forward_host(e_host, e_host, LOOPS, out_host)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e2e_ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        h.loop_forward_host(e_host, e_host, LOOPS, out_host)
        b.record(stream)
        b.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_rank = statistics.mean(e2e_ms)
    e2e_all = reduce_max(e2e_rank, dev)
    e2e_value, _ = aggregate([e2e_all], N, LOOPS, world)
    ok = bool(np.isfinite(out_host.numpy()).all())
    diag = h.diagnostics()

    peaks, peak_src = load_peaks()
    work = kernel_work(wl, LOOPS)
    top = max(stats.items(), key=lambda kv: kv[1][1]) if stats else None
    roof = None
    kernels = {}
    for name, (n, tot) in stats.items():
        kernels[name] = {"launches_per_step": n / args.steps, "ms_per_step": tot / args.steps,
                         "share": tot / max(sum(v[1] for v in stats.values()), 1e-12)}
    if top is not None and top[0] in work:
        name, (n, tot) = top
        wk = work[name]
        avg_s = tot / n / 1e3
        if wk["bound"] == "tensor":
            achieved = wk["flops"] / avg_s / 1e12
            peak = peaks["bf16_tflops"]
            roof = {"kernel": name, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": measured_traffic(name),
                    "peak_source": f"{peak_src} bf16 dense (burst)", "avg_launch_us": avg_s * 1e6,
                    "algorithmic_per_launch": wk["flops"]}
        else:
            achieved = wk["bytes"] / avg_s / 1e9
            peak = peaks["hbm_gbs"]
            roof = {"kernel": name, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "traffic": measured_traffic(name), "peak_source": f"{peak_src} HBM copy",
                    "avg_launch_us": avg_s * 1e6, "algorithmic_per_launch": wk["bytes"]}
    flops = step_flops(wl, LOOPS)
    path_roof = {"step_flops": flops, "achieved_tflops": flops / (ms / 1e3) / 1e12 / world,
                 "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / world / peaks["bf16_tflops"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample = oracle_sample(wl, inputs, seconds=args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": wl.batch, "seq": wl.seq, "dim": wl.dim, "loops": LOOPS,
                       "tokens_per_step": N, "parallelism": f"replicas x{world} (no data-path collective)",
                       "l2": "flushed before every timed step (256 MiB write)"},
            "roofline": roof,
            "path_roofline": path_roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(e_host.numel() * 2),
                    "d2h_bytes_per_step": int(out_host.numel() * 4), "ms_per_step": e2e_all},
            "gpu_launches": int(launches),
            "clocks": clocks,
            "kernels": kernels,
            "finite": ok and diag["nonfinite"] == 0 and diag["timeout"] == 0,
        }
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def act_line(args, h, wl, nl, value, ms, world, rank, stats, launches, clocks):
    """The line of the ACT leg: device-timed throughput and the halting histogram."""
    import numpy as np
    import torch.distributed as dist
    loops = nl.cpu().numpy().ravel()
    diag = h.diagnostics()
    if rank == 0:
        tot = max(sum(v[1] for v in stats.values()), 1e-12)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ours+act",
            "config": {"workload": WORKLOAD + "+act", "batch": wl.batch, "seq": wl.seq, "dim": wl.dim,
                       "loops": LOOPS, "tokens_per_step": wl.batch * wl.seq,
                       "act": {"threshold": 0.99, "head": "w ~ N(0, 0.25/dim), b = -1"},
                       "l2": "flushed before every timed step (256 MiB write)"},
            "act": {"mean_loops": float(loops.mean()),
                    "hist": np.bincount(loops, minlength=LOOPS + 1)[1:].tolist(),
                    "loops_run_fraction": float(loops.mean() / LOOPS)},
            "e2e": None,
            "gpu_launches": int(launches),
            "clocks": clocks,
            "kernels": {k: {"launches_per_step": n / args.steps, "ms_per_step": t / args.steps,
                            "share": t / tot} for k, (n, t) in stats.items()},
            "finite": diag["nonfinite"] == 0 and diag["timeout"] == 0,
        }
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--act", action="store_true", help="time the ACT halting loop instead")
    ap.add_argument("--workload", default=None, help="workload name (default: the headline one)")
    ap.add_argument("--loops", type=int, default=None, help="loops T per step")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    global WORKLOAD, LOOPS
    if args.workload:
        WORKLOAD = args.workload
    if args.loops:
        LOOPS = args.loops
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
