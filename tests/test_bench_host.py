"""Host-side logic of bench.py: algorithmic work, clock parsing, the multi-rank reduction
(two gloo ranks on CPU) and the reference arm's JSON line."""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import WORKLOADS, by_name


def test_algorithmic_flops_of_the_bench_workload():
    wl = by_name(bench.WORKLOAD)
    assert wl is WORKLOADS[4] and bench.LOOPS == 16     # the largest configuration is the headline
    per_loop = bench.step_flops(wl, 1)
    # 2N d (Hq+2Hkv) dh + 2N Hq dh d + LoRA 2N r (d + Hq dh) x 2 + 4 B Hq dh S(S+1)/2
    #   + 2N d E + 6 d hid N k
    N, d, S = 8192, 2048, 8192
    want = (2 * N * d * 3072 + 2 * N * 2048 * d + 2 * 2 * N * 16 * (d + 2048) + 4 * 32 * 64 * S * (S + 1) / 2
            + 2 * N * d * 64 + 6 * d * 512 * N * 8)
    assert per_loop == pytest.approx(want)
    assert per_loop == pytest.approx(863.3e9, rel=0.001)
    # the GQA configuration: 38.7 GFLOP per loop
    assert bench.step_flops(WORKLOADS[1], 1) == pytest.approx(38.7e9, rel=0.01)
    # absorbed MLA: latent 2N d (ql + kvl + r), q~ 2N ql H (kvl + r), attention 2 H (2 kvl + r) pairs,
    # O 2N H kvl d, experts as GQA, router
    m = WORKLOADS[2]
    N, d = 2048, 1024
    pairs = 4 * 512 * 513 / 2
    want = (2 * N * d * 544 + 2 * N * 384 * 16 * 160 + 2 * 16 * 288 * pairs + 2 * N * 2048 * d
            + 6 * d * 1024 * N * 2 + 2 * N * d * 16)
    assert bench.step_flops(m, 1) == pytest.approx(want)


def test_replica_plan_gives_each_rank_its_own_inputs():
    wl = WORKLOADS[4]
    seeds = [bench.replica_plan(wl, r, 4)[0] for r in range(4)]
    assert len(set(seeds)) == 4 and seeds[0] == wl.seed
    assert all(bench.replica_plan(wl, r, 4)[1] == wl.batch * wl.seq for r in range(4))
    with pytest.raises(ValueError):
        bench.replica_plan(wl, 4, 4)


def test_launch_ranks_runs_torchrun_with_one_process_per_gpu(monkeypatch):
    seen = {}
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: seen.setdefault("cmd", cmd) and 0)
    bench.launch_ranks(["--gpus", "4", "--steps", "3"], 4)
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-3:] == ["--gpus", "4", "--steps", "3"][-3:]


def test_oracle_sample_is_bounded():
    # the long configuration: one loop of the whole sequence fits the CPU budget's estimate
    # only for the baseline sample; the reference arm's per-step sample is a prefix
    assert bench.oracle_sample_plan(WORKLOADS[1]) == 512
    assert bench.oracle_sample_plan(WORKLOADS[4], budget_s=4.0) < 8192


def test_parse_clocks():
    txt = ("2026/12/02 19:04:21.000, 0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
           "2026/12/02 19:04:21.050, 0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
           "2026/12/02 19:04:21.100, 0, 1700, 1965, 999.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n")
    c = bench.parse_clocks(txt)
    assert c["sm_mhz"] == 1800 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 3 and not c["in_timed_region"]
    # only the samples inside the timed region count when some fall in it
    t0 = bench._stamp("2026/12/02 19:04:21.040")
    c = bench.parse_clocks(txt, (t0, t0 + 0.02))
    assert c["samples"] == 1 and c["sm_mhz"] == 1800 and c["in_timed_region"]
    c = bench.parse_clocks(txt, (t0 + 10, t0 + 11))       # none inside: all samples, flagged
    assert c["samples"] == 3 and not c["in_timed_region"]
    assert bench.parse_clocks("") is None


def test_aggregate_is_whole_job_over_slowest_rank():
    v, ms = bench.aggregate([2.0, 4.0], 2048, 8, 2)
    assert ms == 4.0 and v == pytest.approx(2 * 2048 * 8 / 0.004)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    assert bench.init_ranks(backend="gloo", timeout_s=60) == (rank, rank, world)
    assert dist.get_world_size() == world
    wl = WORKLOADS[1]
    seed, tokens = bench.replica_plan(wl, rank, world)
    m = bench.reduce_max(1.5 + rank, device="cpu")
    v, ms = bench.aggregate([m], tokens, 4, world)
    q.put((rank, m, v, seed))
    bench.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [2.5, 2.5]                       # the slowest rank's time
    assert res[0][2] == pytest.approx(2 * 2048 * 4 / 0.0025)        # both ranks' tokens
    assert res[0][3] != res[1][3]                                   # each rank its own inputs


def test_reference_arm_prints_one_json_line(capsys):
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference" and line["unit"] == bench.UNIT and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_measured_traffic_only_for_unchanged_sources(monkeypatch):
    files = bench.KERNEL_SOURCES["gemm_up"]
    fp = bench.source_fingerprint(files)
    key = (bench.WORKLOAD, "gemm_up")
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, key, (123.0, fp))
    assert bench.measured_traffic(bench.WORKLOAD, "gemm_up") == 123.0
    assert bench.measured_traffic("other-workload", "gemm_up") is None   # captured on another workload
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, key, (123.0, "0" * 16))
    assert bench.measured_traffic(bench.WORKLOAD, "gemm_up") is None     # sources changed since
    assert bench.measured_traffic(bench.WORKLOAD, "norm1") is None       # never captured


def test_fingerprint_ignores_comments_not_code(tmp_path):
    src = 'int f(int a) {  // doubles a\n    /* note */ return 2 * a;\n}\nconst char* s = "p//q";\n'
    f = tmp_path / "k.cu"

    def fp(text):
        f.write_text(text)
        return bench.source_fingerprint([str(f)])

    base = fp(src)
    assert fp(src.replace("doubles a", "twice a")) == base              # comment edit
    assert fp(src.replace("/* note */", "/* longer\n note */")) == base  # block comment
    assert fp("\n" + src.replace("    ", "\t")) == base                  # indentation, blank line
    assert fp(src.replace("2 * a", "3 * a")) != base                     # code
    assert fp(src.replace("p//q", "p//r")) != base                       # '//' inside a string is code



def test_act_summary_reports_the_halting_histogram():
    nl = [[1, 2, 2, 8], [8, 8, 3, 1]]
    a = bench.act_summary(nl, 8)
    assert a["hist"] == [2, 2, 1, 0, 0, 0, 0, 3]
    assert a["mean_loops"] == pytest.approx(33 / 8)
    assert a["loops_run_fraction"] == pytest.approx(33 / 64)


def test_roofline_of_a_tensor_and_an_hbm_kernel():
    wl = by_name(bench.WORKLOAD)
    work = bench.kernel_work(wl)
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    r = bench.roofline_of("attention", 16, 16 * 0.5, work, peaks, "measured", bench.WORKLOAD)
    assert r["bound"] == "tensor" and r["avg_launch_us"] == pytest.approx(500.0)
    assert r["achieved"] == pytest.approx(274.9e9 / 500e-6 / 1e12, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / 1000.0)
    r = bench.roofline_of("norm1", 2, 0.1, work, peaks, "measured", bench.WORKLOAD)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    # RMSNorm1: h (fp32) and e (bf16) in, xn (bf16) out: 8 bytes per element
    assert r["achieved"] == pytest.approx(8192 * 2048 * 8 / 50e-6 / 1e9)


def test_state_traffic_of_the_o_projection_and_the_hoist():
    """The O projection forms y and h_next from h and e (reads h 4 B and e 2 B, stores 2 x 4 B
    per element); after depth attention it adds into them instead (2 x 4 B of reductions).
    The hoist stores B.e only where the O projection cannot form it (no e in the block
    input); with a dense B the product comes from a separate matmul."""
    from workloads import DEPTH_WORKLOAD
    wl = WORKLOADS[4]                                     # long: diagonal B, e injected
    N, d = wl.batch * wl.seq, wl.dim
    nq = wl.n_heads * wl.head_dim
    w = bench.kernel_work(wl)
    assert w["gemm_o"]["bytes"] == 2 * (N * nq + d * nq) + N * d * (4 + 2 + 4 + 4)
    assert w["norm1"]["bytes"] == N * d * (4 + 2 + 2)
    assert w["hoist"]["bytes"] == N * d * (2 + 4)
    w0 = bench.kernel_work(wl.replace(inject_e=False))   # B.e kept by the hoist, read by O
    assert w0["gemm_o"]["bytes"] == 2 * (N * nq + d * nq) + N * d * (4 + 4 + 4 + 4)
    assert w0["hoist"]["bytes"] == N * d * (2 + 4 + 2 + 4)
    wd = bench.kernel_work(DEPTH_WORKLOAD)
    Nd, dd = DEPTH_WORKLOAD.batch * DEPTH_WORKLOAD.seq, DEPTH_WORKLOAD.dim
    nqd = DEPTH_WORKLOAD.n_heads * DEPTH_WORKLOAD.head_dim
    assert wd["gemm_o"]["bytes"] == 2 * (Nd * nqd + dd * nqd) + 4 * 2 * Nd * dd
    nqd_da = DEPTH_WORKLOAD.da_heads * DEPTH_WORKLOAD.head_dim
    assert wd["gemm_o_depth"]["bytes"] == 2 * (Nd * nqd_da + dd * nqd_da) + Nd * dd * (4 + 2 + 4 + 4)
