#!/usr/bin/env python
"""Throughput of the looped recurrent block on B200 through the librdt C ABI.

One step = one rdt_loop_forward call: T loops of the block over one batch of seeded
synthetic inputs resident in HBM. The headline workload is the largest single-GPU
configuration: the long-context GQA block with depth-wise LoRA (batch 1 x seq 8192, dim
2048, 32/8 heads of 64, 64 experts top-8 with SwiGLU hidden 512, LoRA rank 16 on Q and O),
T = 16 loops, bf16 storage and an fp32 state. The L2 cache is flushed (256 MiB write)
before every timed step; each step is timed with CUDA events on its stream and the median
step is reported.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--loops T] [--act] [--all]
                    [--decode] [--kernel attention] [--cp]

--decode times rdt_decode_step (one new token per sequence, T loops, over a prompt of the
workload's length) instead. `--kernel attention` times rdt_attention alone on the workload's
sequence-attention shape (the command the attention kernel's ncu captures run). `--cp`
splits one sequence of the workload over the N GPUs (context parallelism; strong scaling).

--gpus N > 1 runs one process per GPU (re-launched under torch.distributed.run when not
started by it): every rank runs a replica of the workload on inputs of its own (no
data-path collective; weak scaling); the timed region is bracketed by a barrier and a
device synchronise and the step time is the maximum over ranks. `--impl reference` times
the fp64 CPU oracle on the host cores instead (rank 0 only). `--act` times the same
workload through rdt_loop_forward_act (ACT halting, threshold 0.99, the seeded halting
head). `--all` prints one line for every configuration and loop count of the workload
list instead of the headline line.
"""
from __future__ import annotations

import argparse
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

WORKLOAD = "long-bf16-b1s8192-d2048-h32x8-e64k8-lora16"
LOOPS = 16
METRIC = "recurrent-block tokens·loops/sec (bf16 fwd, 1 B200) and % of roofline"
UNIT = "tokens*loops/s"
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# CPU-baseline sample: at most this many seconds of oracle work per timed sample
CPU_SECONDS = 30.0

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a kernel on a
# workload, from one ncu capture, valid only while the kernel's code is the one captured
# (fingerprint: first 16 hex digits of the SHA-256 of the listed files' code, concatenated:
# comments removed, each line stripped, blank lines dropped, so that an edit of a comment
# or of indentation keeps the capture while any change to a code token voids it).
KERNEL_SOURCES = {
    "attention": ("recurrent_depth_transformer_b200/csrc/attention_tc.cu",
                  "recurrent_depth_transformer_b200/csrc/rdt_internal.cuh"),
    "gemm_up": ("recurrent_depth_transformer_b200/csrc/gemm_tc.cuh",
                "recurrent_depth_transformer_b200/csrc/gemm_tc.cu",
                "recurrent_depth_transformer_b200/csrc/gemm_tc_pair.cu",
                "recurrent_depth_transformer_b200/csrc/rdt_internal.cuh",
                "recurrent_depth_transformer_b200/csrc/rdt_api.cu"),
}
# (workload, kernel) -> (bytes per launch, source fingerprint)
MEASURED_TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum (1 pass) on one attention launch
    # of the default command: 50.37 MB read + 2.76 MB written (most of o is still in L2 when
    # the kernel ends)
    ("long-bf16-b1s8192-d2048-h32x8-e64k8-lora16", "attention"): (50371328.0 + 2757376.0, "83c8394ee09325bb"),
}


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


def measured_traffic(workload, kernel):
    """The captured traffic of `kernel` on `workload`, or None once its sources differ."""
    key = (workload, kernel)
    if key not in MEASURED_TRAFFIC or kernel not in KERNEL_SOURCES:
        return None
    value, fp = MEASURED_TRAFFIC[key]
    try:
        return value if source_fingerprint(KERNEL_SOURCES[kernel]) == fp else None
    except (OSError, ValueError):          # missing or undecodable source: no claim
        return None


# ----------------------------------------------------------------------------- algorithmic work

def kernel_work(wl):
    """Algorithmic FLOPs and DRAM bytes per launch of each kernel class: counts of what the
    block must compute and move, not of what a kernel happens to do (causal attention counts
    the S(S+1)/2 unmasked pairs, the expert GEMMs the N*k routed rows plus shared rows, the
    depth-wise LoRA its rank-r products; weights are read once, activations once in and
    once out)."""
    N, d = wl.batch * wl.seq, wl.dim
    E, k, hid, S = wl.n_experts, wl.top_k, wl.expert_hidden, wl.n_shared
    rows = N * (k + S)
    b2 = 2 if wl.dtype == "bf16" else 4
    pairs = wl.batch * wl.seq * (wl.seq + 1) / 2
    w = {}
    # the O projection that forms y = x + a and h_next = A h + B e + a reads h (and e, or the
    # hoisted B e) and stores both once; after depth attention it adds a into them instead
    e_in = b2 if wl.inject_e else 0
    be_in = 4 if (wl.b_kind == "dense" or not wl.inject_e) else 0
    resid = N * d * (4 + e_in + be_in + 4 + 4)
    depth = bool(getattr(wl, "da_heads", 0))
    o_out = 4 * 2 * N * d if depth else resid
    if wl.attn == "gqa":
        hq, hkv, dh = wl.n_heads, wl.n_kv_heads, wl.head_dim
        nq, nqkv = hq * dh, (hq + 2 * hkv) * dh
        r = wl.lora_rank if wl.n_lora else 0
        w["gemm_qkv"] = dict(flops=2.0 * N * d * nqkv + 2.0 * N * r * (d + nq),
                             bytes=b2 * (N * d + nqkv * d + N * nqkv), bound="tensor")
        w["attention"] = dict(flops=4.0 * hq * dh * pairs, bytes=b2 * N * (nqkv + nq), bound="tensor")
        ow = nq
        w["gemm_o"] = dict(flops=2.0 * N * nq * d + 2.0 * N * r * (nq + d),
                           bytes=b2 * (N * nq + d * nq) + o_out, bound="tensor")
    else:
        H, ql, kvl, rp = wl.n_heads, wl.q_lora_rank, wl.kv_lora_rank, wl.qk_rope_dim
        lat = ql + kvl + rp
        w["gemm_latent"] = dict(flops=2.0 * N * d * lat, bytes=b2 * (N * d + lat * d) + 4 * N * lat, bound="tensor")
        w["gemm_q_absorbed"] = dict(flops=2.0 * N * ql * H * (kvl + rp),
                                    bytes=b2 * (N * ql + ql * H * (kvl + rp) + N * H * (kvl + rp)), bound="tensor")
        # absorbed attention: every head over the shared (kvl + rope)-wide key, kvl-wide value
        w["attention"] = dict(flops=2.0 * H * (kvl + rp + kvl) * pairs,
                              bytes=b2 * N * (H * (kvl + rp) + kvl + rp + H * kvl), bound="tensor")
        ow = H * kvl
        w["gemm_o"] = dict(flops=2.0 * N * ow * d, bytes=b2 * (N * ow + d * ow) + o_out, bound="tensor")
        w["mla_latent_norm"] = dict(flops=0.0, bytes=N * (4 * lat + b2 * (ql + kvl + rp)), bound="hbm")
    if getattr(wl, "da_heads", 0):
        # depth attention: projections of every token, each query over its T loops' keys
        # (the mean over loops t = 0 .. T-1 of t + 1 keys is counted per launch by the caller)
        hqd, hkvd, dh = wl.da_heads, wl.da_kv_heads, wl.head_dim
        nqd, nqkvd = hqd * dh, (hqd + 2 * hkvd) * dh
        w["gemm_qkv_depth"] = dict(flops=2.0 * N * d * nqkvd, bytes=b2 * (N * d + nqkvd * d + N * nqkvd), bound="tensor")
        T = max(wl.loops)
        keys = (T + 1) / 2.0
        w["depth_attention"] = dict(flops=4.0 * N * hqd * dh * keys,
                                    bytes=b2 * N * (nqd + 2 * hkvd * dh * keys + nqd), bound="hbm")
        w["gemm_o_depth"] = dict(flops=2.0 * N * nqd * d, bytes=b2 * (N * nqd + d * nqd) + resid,
                                 bound="tensor")
    w["gemm_up"] = dict(flops=2.0 * rows * d * 2 * hid, bytes=b2 * (rows * d + (E + S) * 2 * hid * d + rows * hid),
                        bound="tensor")
    w["gemm_down"] = dict(flops=2.0 * rows * hid * d, bytes=b2 * (rows * hid + (E + S) * d * hid) + 4 * N * d * 2,
                          bound="tensor")
    # RMSNorm1 reads h and e and writes xn (after depth attention: reads y, writes xn)
    w["norm1"] = dict(flops=0.0, bytes=N * d * (4 + e_in + b2), bound="hbm")
    if E * d * b2 <= 65536 or wl.dtype != "bf16":
        # the fused router (W_r in shared memory; fp32: FMA): y in, W_r once, per (token,
        # slot) the routing words and the yn copy in the expert's rows; yn itself where
        # shared experts read it
        w["router_topk"] = dict(flops=2.0 * N * d * E,
                                bytes=N * d * 4 + (N * d * b2 if S else 0) + E * d * b2 + N * k * (d * b2 + 16),
                                bound="hbm")
    else:
        # the tensor-core router: yn and its bf16 residual in, W_r once (both halves), per
        # (token, slot) the routing words (index, weight, claimed row, token of the row)
        w["router_topk"] = dict(flops=2.0 * N * 2 * d * E, bytes=N * d * b2 * 2 + 2 * E * d * b2 + N * k * 16,
                                bound="hbm")
    # RMSNorm2 for the tensor-core router: y in, yn and its bf16 residual out
    w["norm2"] = dict(flops=0.0, bytes=N * d * (4 + 2 * b2), bound="hbm")
    w["moe_dispatch"] = dict(flops=0.0, bytes=N * k * (d * b2 * 2 + 4), bound="hbm")
    w["moe_combine"] = dict(flops=0.0, bytes=N * d * 4 * (2 + k + S), bound="hbm")
    # h <- h0; B e only where the O projection does not form it (dense B: a separate matmul)
    keep_be = wl.b_kind == "diag" and not wl.inject_e
    w["hoist"] = dict(flops=0.0, bytes=N * d * (b2 + 4 + ((b2 + 4) if keep_be else 0)), bound="hbm")
    w["check_finite"] = dict(flops=0.0, bytes=N * d * 4, bound="hbm")
    w["act_halting"] = dict(flops=0.0, bytes=N * d * 12, bound="hbm")
    return w


PATH_KERNELS = ("gemm_qkv", "gemm_latent", "gemm_q_absorbed", "attention", "gemm_o", "gemm_up", "gemm_down",
                "gemm_qkv_depth", "depth_attention", "gemm_o_depth")


def step_flops(wl, T):
    """Algorithmic FLOPs of T loops: the dense contractions plus the router logits."""
    w = kernel_work(wl)
    per_loop = sum(w[k]["flops"] for k in PATH_KERNELS if k in w)
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


def roofline_of(name, n_launches, total_ms, work, peaks, peak_src, workload):
    """The roofline object of one kernel class from its event-timed launches."""
    wk = work[name]
    avg_s = total_ms / n_launches / 1e3
    if wk["bound"] == "tensor":
        achieved = wk["flops"] / avg_s / 1e12
        peak = peaks["bf16_tflops"]
        return {"kernel": name, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": measured_traffic(workload, name),
                "peak_source": f"{peak_src} bf16 dense (burst)", "avg_launch_us": avg_s * 1e6,
                "algorithmic_per_launch": wk["flops"]}
    achieved = wk["bytes"] / avg_s / 1e9
    peak = peaks["hbm_gbs"]
    return {"kernel": name, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": measured_traffic(workload, name),
            "peak_source": f"{peak_src} HBM copy", "avg_launch_us": avg_s * 1e6,
            "algorithmic_per_launch": wk["bytes"]}


# ----------------------------------------------------------------------------- clocks

CLOCK_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index=0):
        self.proc = None
        self.path = None
        self.gpu = gpu_index

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={CLOCK_FIELDS}",
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


# ----------------------------------------------------------------------------- ranks

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


def replica_plan(wl, rank, world):
    """Weak scaling by replicas: the sequences of different ranks never interact, so every
    rank runs the whole configuration on inputs of its own (the configuration's seed plus the
    rank: independent sequences, same weights). Returns the rank's input seed and the tokens
    it processes per step."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    return wl.seed + 1000 * rank, wl.batch * wl.seq


def launch_ranks(argv, n):
    """Re-run this script under torch.distributed.run with one process per GPU."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def init_ranks(device=None, backend="nccl", timeout_s=120):
    """Join the process group of a multi-rank run (nothing for one rank)."""
    import datetime
    import torch.distributed as dist
    rank, local, world = dist_env()
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if device is not None else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return rank, local, world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


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


def oracle_sample_plan(wl, budget_s=CPU_SECONDS):
    """A bounded sample of the workload for the fp64 oracle: one loop over the whole batch
    when that fits the budget (every position at its full context, so the per-token cost is
    the workload's), else one loop over a prefix of every sequence. The estimate scales a
    loop's FLOPs by an fp64 rate of 50 GFLOP/s."""
    per_loop = step_flops(wl, 1)
    if per_loop / 50e9 <= budget_s:
        return wl.seq
    seq = wl.seq
    while seq > 128 and step_flops(wl.replace(seq=seq), 1) / 50e9 > budget_s:
        seq //= 2
    return seq


def oracle_sample(wl, inputs, seconds=10.0):
    """Time the fp64 oracle on the sample of oracle_sample_plan, repeated until `seconds`
    of work; returns (tokens*loops/s, description)."""
    import oracle as O
    seq = oracle_sample_plan(wl)
    sub = dict(inputs)
    sub["e"] = inputs["e"][:, :seq]
    sub["h0"] = sub["e"] if inputs["h0"] is inputs["e"] else inputs["h0"][:, :seq]
    w1 = wl.replace(seq=seq)
    t0 = time.perf_counter()
    runs = 0
    while True:
        O.loop_forward(sub["h0"], sub["e"], 1, sub, w1)
        runs += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    what = "the whole batch" if seq == wl.seq else f"the first {seq} of {wl.seq} positions of every sequence"
    return (runs * wl.batch * seq / el,
            f"{runs} x (1 loop over {what}: {wl.batch * seq} tokens), {el:.1f} s")


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from workloads import by_name, generate
    import oracle as O
    wl = by_name(args.workload)
    inputs = generate(wl)
    # per step: one loop of a prefix short enough that the whole run takes minutes
    seq = oracle_sample_plan(wl, budget_s=4.0)
    sub = dict(inputs)
    sub["e"] = inputs["e"][:, :seq]
    sub["h0"] = sub["e"]
    w1 = wl.replace(seq=seq)
    for _ in range(args.warmup):
        O.loop_forward(sub["h0"], sub["e"], 1, sub, w1.replace(seq=min(seq, 64)))
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.loop_forward(sub["h0"], sub["e"], 1, sub, w1)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.median(times)
    value = wl.batch * seq / (ms / 1e3)
    what = "the whole batch" if seq == wl.seq else f"the first {seq} of {wl.seq} positions"
    sample = f"1 of {args.loops} loops over {what} per step (fp64 NumPy oracle)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "batch": wl.batch, "seq": wl.seq, "dim": wl.dim, "loops": args.loops,
                   "parallelism": "host cores (fp64 NumPy oracle)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_one(args, wl_name, T, dev, rank, world, with_cpu):
    """Time one workload; returns the JSON line (rank 0) or None."""
    import numpy as np
    import torch

    import recurrent_depth_transformer_b200 as R
    from workloads import by_name, generate

    wl = by_name(wl_name)
    seed, tokens = replica_plan(wl, rank, world)
    inputs = generate(wl) if seed == wl.seed else generate(wl.replace(seed=seed))
    weights = R.device_weights(generate(wl) if seed != wl.seed else inputs, wl.dtype == "bf16", device=dev)
    h = R.RDT(R.make_config(wl, max_loops=T), weights)
    del weights
    e = torch.from_numpy(inputs["e"]).to(torch.bfloat16 if wl.dtype == "bf16" else torch.float32).to(dev)
    out = torch.empty(e.shape, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    nl = None
    if args.act:
        from workloads import act_head
        head = act_head(wl)
        h.set_act(torch.from_numpy(head["w_halt"]).to(dev), head["b_halt"], head["threshold"])
        nl = torch.empty((wl.batch, wl.seq), dtype=torch.int32, device=dev)

        def step():
            h.loop_forward_act(e, e, T, out=out, n_loops=nl)
    else:
        def step():
            h.loop_forward(e, e, T, out=out)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    # ---- timed region (device time, CUDA events on the launch stream)
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    barrier()
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
    barrier()
    launches = (h.launch_count() - launches0) / args.steps
    clocks = sampler.stop((t_wall0, t_wall1)) if sampler else None
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms_rank = statistics.median(step_ms)
    ms_all = reduce_max(ms_rank, dev)
    value, ms = aggregate([ms_all], tokens, T, world)

    # ---- per-kernel event timing inside graph replay (events are nodes of the loop's graph)
    h.profile(2)
    for _ in range(2):                    # eager call, then capture with the event nodes
        flush.zero_()
        step()
    torch.cuda.synchronize()
    h.profile(2)                          # restart the statistics, keep the graph
    for _ in range(args.steps):
        flush.zero_()
        step()
        h.profile_read()                  # each replay records the graph's events anew
    stats, _ = h.profile_read()
    h.profile(0)

    diag = h.diagnostics()
    e2e = None
    if not args.act:
        # ---- end to end through the host-buffer entry point (pinned memory, copies inside)
        e_host = e.cpu().pin_memory()
        out_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        for _ in range(3):                   # eager, graph capture, first replay
            h.loop_forward_host(e_host, e_host, T, out_host)
        barrier()
        torch.cuda.synchronize()
        e2e_ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            h.loop_forward_host(e_host, e_host, T, out_host)
            b.record(stream)
            b.synchronize()
            e2e_ms.append(a.elapsed_time(b))
        e2e_all = reduce_max(statistics.median(e2e_ms), dev)
        e2e_value, _ = aggregate([e2e_all], tokens, T, world)
        finite = bool(np.isfinite(out_host.numpy()).all())
        e2e = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(e_host.numel() * e_host.element_size()),
               "d2h_bytes_per_step": int(out_host.numel() * 4), "ms_per_step": e2e_all}
    else:
        finite = bool(torch.isfinite(out).all().item())

    peaks, peak_src = load_peaks()
    work = kernel_work(wl)
    tot = max(sum(v[1] for v in stats.values()), 1e-12)
    kernels = {name: {"launches_per_step": n / args.steps, "ms_per_step": t / args.steps, "share": t / tot}
               for name, (n, t) in stats.items()}
    ranked = sorted(((t, name, n) for name, (n, t) in stats.items() if name in work), reverse=True)
    roof = roofline_of(ranked[0][1], ranked[0][2], ranked[0][0], work, peaks, peak_src, wl_name) if ranked else None
    flops = step_flops(wl, T)
    # per GPU: every rank runs the whole workload in the step time
    path_roof = {"step_flops": flops, "achieved_tflops": flops / (ms / 1e3) / 1e12,
                 "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]}

    cpu = None
    if with_cpu and rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample = oracle_sample(wl, inputs, seconds=args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": sample}

    h.close()
    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl_name, "batch": wl.batch, "seq": wl.seq, "dim": wl.dim, "loops": T,
                   "tokens_per_step": tokens, "parallelism": f"replicas x{world} (no data-path collective)",
                   "l2": "flushed before every timed step (256 MiB write)", "step_time": "median of the timed steps"},
        "roofline": roof,
        "path_roofline": path_roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(round(launches)),
        "clocks": clocks,
        "kernels": kernels,
        "kernel_timing": "CUDA events recorded by nodes of the replayed loop graph",
        "finite": finite and diag["nonfinite"] == 0 and diag["timeout"] == 0,
    }
    if args.act:
        line["impl"] = "ours+act"
        line["config"]["workload"] = wl_name + "+act"
        line["config"]["act"] = {"threshold": 0.99, "head": "w ~ N(0, 0.25/dim), b = -1"}
        line["act"] = act_summary(nl.cpu().numpy(), T)
    return line


def act_summary(n_loops, T):
    """Halting histogram of an ACT run: how many positions ran 1 .. T loops, the mean, and
    the fraction of the T loops asked for that positions ran."""
    import numpy as np
    loops = np.asarray(n_loops).ravel()
    return {"mean_loops": float(loops.mean()), "hist": np.bincount(loops, minlength=T + 1)[1:].tolist(),
            "loops_run_fraction": float(loops.mean() / T)}


ALL_RUNS = (("tiny-f32-b1s64-d128-gqa4x2-e4k2", 4), ("gqa-bf16-b4s512-d1024-h16x4-e16k2", 8),
            ("mla-bf16-b4s512-d1024-h16-lat128-e16k2", 3), ("mla-bf16-b4s512-d1024-h16-lat128-e16k2", 8),
            ("widemoe-bf16-b2s2048-d2048-h32x8-e64k8s1", 1), ("widemoe-bf16-b2s2048-d2048-h32x8-e64k8s1", 4),
            ("widemoe-bf16-b2s2048-d2048-h32x8-e64k8s1", 8), ("widemoe-bf16-b2s2048-d2048-h32x8-e64k8s1", 16),
            ("long-bf16-b1s8192-d2048-h32x8-e64k8-lora16", 16))


def decode_bytes(wl, length, experts_used):
    """Algorithmic bytes of one decode step's loop: every projection and router weight once,
    the weights of the experts the step's tokens chose, the cache read up to the new position
    and the new row written, the state and activation rows."""
    d, b2, B = wl.dim, 2, wl.batch
    if wl.attn == "gqa":
        nq, nkv = wl.n_heads * wl.head_dim, wl.n_kv_heads * wl.head_dim
        proj = (nq + 2 * nkv) * d + d * nq
        cache_row = 2 * nkv
    else:
        H, ql, kvl, rp = wl.n_heads, wl.q_lora_rank, wl.kv_lora_rank, wl.qk_rope_dim
        proj = (ql + kvl + rp) * d + ql * H * (kvl + rp) + d * H * kvl
        cache_row = kvl + rp
    experts = (experts_used + wl.n_shared) * 3 * wl.expert_hidden * d
    return b2 * (proj + wl.n_experts * d + experts + B * (length + 1) * cache_row + B * cache_row) + B * d * 4 * 6


def bench_decode(args, dev, rank, world):
    """Decode steps of one token per sequence after a prompt of the workload's length."""
    import numpy as np
    import torch

    import recurrent_depth_transformer_b200 as R
    from workloads import by_name, generate, round_bf16

    wl = by_name(args.workload)
    T = args.loops
    inputs = generate(wl)
    steps = args.warmup + args.steps
    weights = R.device_weights(inputs, True, device=dev)
    h = R.RDT(R.make_config(wl, max_loops=T, max_decode=steps), weights)
    del weights
    e = torch.from_numpy(inputs["e"]).to(torch.bfloat16).to(dev)
    h.decode_prefill(e, e, T)
    rng = np.random.default_rng(wl.seed + 7)
    new = torch.from_numpy(round_bf16(rng.standard_normal((steps, wl.batch, wl.dim)).astype(np.float32)))
    new = new.to(torch.bfloat16).to(dev)
    out = torch.empty((wl.batch, wl.dim), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    xs = [new[i].contiguous() for i in range(steps)]
    buf = torch.empty_like(xs[0])
    for i in range(args.warmup):             # eager, capture, replays (same pointers every step)
        buf.copy_(xs[i])
        h.decode_step(buf, buf, T, out=out)
    torch.cuda.synchronize()
    barrier()
    launches0 = h.launch_count()
    evs = []
    for i in range(args.warmup, steps):
        buf.copy_(xs[i])
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        h.decode_step(buf, buf, T, out=out)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    launches = (h.launch_count() - launches0) / args.steps
    ms = reduce_max(statistics.median(a.elapsed_time(b) for a, b in evs), dev)
    diag = h.diagnostics()
    used = sum(1 for c in diag["expert_counts"][:wl.n_experts] if c > 0)
    length = wl.seq + steps - 1
    nbytes = decode_bytes(wl, length, used) * T
    peaks, src = load_peaks()
    h.close()
    if rank != 0:
        return None
    gbs = nbytes / (ms / 1e3) / 1e9
    return {
        "impl": "ours-decode", "metric": "decode tokens/s (one token per sequence per step, T loops)",
        "value": world * wl.batch / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": wl.batch, "prompt": wl.seq, "dim": wl.dim, "loops": T,
                   "cache_positions": wl.seq + steps, "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "decode step (whole)", "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{src} HBM copy", "algorithmic_per_step": nbytes,
                     "experts_read_last_step": used},
        "gpu_launches": int(round(launches)),
    }


def bench_attention(args, dev, rank, world):
    """rdt_attention alone on the workload's sequence-attention shape (GQA heads; bf16 q, k, v
    drawn from a seeded normal), event-timed per launch: the kernel-level line that the
    attention ncu captures run."""
    import torch

    import recurrent_depth_transformer_b200 as R
    from workloads import by_name

    wl = by_name(args.workload)
    if wl.attn != "gqa" or wl.dtype != "bf16":
        raise SystemExit("--kernel attention times bf16 GQA workloads")
    B, S, Hq, Hkv, D = wl.batch, wl.seq, wl.n_heads, wl.n_kv_heads, wl.head_dim
    g = torch.Generator(device=dev).manual_seed(wl.seed)
    q = torch.randn(B * S, Hq * D, device=dev, generator=g).to(torch.bfloat16)
    k = torch.randn(B * S, Hkv * D, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(B * S, Hkv * D, device=dev, generator=g).to(torch.bfloat16)
    o = torch.empty(B * S, Hq * D, device=dev, dtype=torch.bfloat16)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        R.attention(q, k, v, B, S, Hq, Hkv, D, D, D ** -0.5, o=o)
    torch.cuda.synchronize()
    barrier()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        R.attention(q, k, v, B, S, Hq, Hkv, D, D, D ** -0.5, o=o)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    ms = reduce_max(statistics.median(a.elapsed_time(b) for a, b in evs), dev)
    if rank != 0:
        return None
    peaks, src = load_peaks()
    flops = 4.0 * B * Hq * D * S * (S + 1) / 2
    tf = flops / (ms / 1e3) / 1e12
    return {
        "impl": "ours-kernel", "metric": "causal attention TFLOP/s (one launch)", "value": world * tf,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": B, "seq": S, "heads": Hq, "kv_heads": Hkv, "head_dim": D,
                   "l2": "flushed between launches", "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "attention", "bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"], "traffic": None,
                     "peak_source": f"{src} cuBLAS bf16 burst"},
        "gpu_launches": 1,
    }


def bench_cp(args, dev, rank, world):
    """Context parallelism: one sequence of the workload split over the ranks (rank r holds
    positions [r S / N, (r + 1) S / N)); the keys of every loop travel over peer memory from
    the QKV projection's epilogue. The whole job's tokens per step are the workload's, so the
    scaling is strong."""
    import torch
    import torch.distributed as dist

    import recurrent_depth_transformer_b200 as R
    from workloads import by_name, generate

    wl = by_name(args.workload)
    T = args.loops
    if wl.seq % world or (wl.seq // world) % 128:
        raise SystemExit(f"--cp: {wl.seq} positions do not split into {world} shares of a multiple of 128")
    S = wl.seq // world
    inputs = generate(wl)
    weights = R.device_weights(inputs, wl.dtype == "bf16", device=dev)
    h = R.RDT(R.make_config(wl, max_loops=T, seq=S, cp_size=world if world > 1 else 0,
                            cp_rank=rank if world > 1 else 0), weights)
    del weights
    opened = []
    if world > 1:
        def all_gather(obj):
            out = [None] * world
            dist.all_gather_object(out, obj)
            return out
        opened = R.cp_connect_ranks(h, rank, world, all_gather)
    barrier()
    e_all = torch.from_numpy(inputs["e"]).to(torch.bfloat16)
    e = e_all[:, rank * S:(rank + 1) * S].contiguous().to(dev)
    out = torch.empty(e.shape, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):          # every rank makes the same calls: their loops wait for one another
        flush.zero_()
        h.loop_forward(e, e, T, out=out)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    launches0 = h.launch_count()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_wall0 = time.time()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        h.loop_forward(e, e, T, out=out)
        b.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    launches = (h.launch_count() - launches0) / args.steps
    clocks = sampler.stop((t_wall0, t_wall1)) if sampler else None
    ms = reduce_max(statistics.median(a.elapsed_time(b) for a, b in evs), dev)
    diag = h.diagnostics()
    finite = bool(torch.isfinite(out).all().item()) and diag["nonfinite"] == 0 and diag["timeout"] == 0
    barrier()                              # nobody touches a peer's buffers any more
    for p_ in opened:
        R.ipc_close_handle(p_)
    barrier()
    h.close()
    if rank != 0:
        return None
    tokens = wl.batch * wl.seq
    peaks, _ = load_peaks()
    flops = step_flops(wl, T)
    return {
        "impl": "ours-cp", "metric": METRIC, "value": tokens * T / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": wl.batch, "seq": wl.seq, "dim": wl.dim, "loops": T,
                   "tokens_per_step": tokens, "positions_per_rank": S, "parallelism": f"context parallel x{world}",
                   "l2": "flushed before every timed step (256 MiB write)", "step_time": "median of the timed steps"},
        "path_roofline": {"step_flops": flops, "achieved_tflops": flops / (ms / 1e3) / 1e12,
                          "frac_of_bf16_peak_all_gpus": flops / (ms / 1e3) / 1e12 / (peaks["bf16_tflops"] * world)},
        "e2e": None, "gpu_launches": int(round(launches)), "clocks": clocks, "finite": finite,
    }


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_ranks(dev)
    if args.decode or args.kernel or args.cp:
        line = (bench_attention if args.kernel else bench_cp if args.cp else bench_decode)(args, dev, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        barrier()
        if world > 1:
            dist.destroy_process_group()
        return 0
    runs = ALL_RUNS if args.all else ((args.workload, args.loops),)
    for name, T in runs:
        line = bench_one(args, name, T, dev, rank, world, with_cpu=not args.all or name == args.workload)
        if line is not None:
            print(json.dumps(line), flush=True)
    barrier()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--act", action="store_true", help="time the ACT halting loop instead")
    ap.add_argument("--workload", default=WORKLOAD, help="workload name (default: the headline one)")
    ap.add_argument("--loops", type=int, default=LOOPS, help="loops T per step")
    ap.add_argument("--all", action="store_true", help="one line per configuration and loop count")
    ap.add_argument("--decode", action="store_true", help="time decode steps with the per-loop KV cache")
    ap.add_argument("--kernel", choices=("attention",), help="time one kernel alone on the workload's shape")
    ap.add_argument("--cp", action="store_true",
                    help="context parallelism: split the workload's sequence over the N GPUs (strong scaling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    _, _, world = dist_env()
    if args.gpus > 1 and world == 1 and "LOCAL_RANK" not in os.environ:
        return launch_ranks(argv, args.gpus)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
