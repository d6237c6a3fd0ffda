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
    assert wl is WORKLOADS[1]
    per_loop = bench.step_flops(wl, 1)
    # 2N d (Hq+2Hkv) dh + 2N Hq dh d + 4 B Hq dh S(S+1)/2 + 2N d E + 6 d hid N k
    N, d = 2048, 1024
    want = (2 * N * d * 1536 + 2 * N * 1024 * d + 4 * 4 * 16 * 64 * 512 * 513 / 2
            + 2 * N * d * 16 + 6 * d * 1024 * N * 2)
    assert per_loop == pytest.approx(want)
    assert per_loop == pytest.approx(38.7e9, rel=0.01)


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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    assert bench.dist_env() == (rank, rank, world)
    m = bench.reduce_max(1.5 + rank, device="cpu")
    v, ms = bench.aggregate([m], 1000, 4, world)
    q.put((rank, m, v))
    dist.barrier()
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
    assert [r[1] for r in res] == [2.5, 2.5]
    assert res[0][2] == pytest.approx(2 * 1000 * 4 / 0.0025)


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
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "gemm_up", (123.0, fp))
    assert bench.measured_traffic("gemm_up") == 123.0
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "gemm_up", (123.0, "0" * 16))
    assert bench.measured_traffic("gemm_up") is None          # sources changed since the capture
    assert bench.measured_traffic("attention") is None        # never captured


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



def test_act_line_reports_halting_histogram(capsys):
    """The --act leg's JSON line, from a stand-in handle (no GPU): the workload, the
    halting histogram, the mean loops and the kernel shares."""
    import argparse

    class FakeHandle:
        closed = False

        def diagnostics(self):
            return {"nonfinite": 0, "timeout": 0}

        def close(self):
            self.closed = True

    wl = by_name(bench.WORKLOAD)
    nl = torch.tensor([[1, 2, 2, 8], [8, 8, 3, 1]], dtype=torch.int32)
    args = argparse.Namespace(steps=10, warmup=3)
    stats = {"gemm_up": (80, 3.0), "act_halting": (80, 1.0)}
    h = FakeHandle()
    assert bench.act_line(args, h, wl, nl, 2.0e7, 0.82, 1, 0, stats, 1234, None) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert h.closed
    assert line["impl"] == "ours+act" and line["config"]["workload"].endswith("+act")
    assert line["act"]["hist"] == [2, 2, 1, 0, 0, 0, 0, 3]
    assert line["act"]["mean_loops"] == pytest.approx(33 / 8)
    assert line["act"]["loops_run_fraction"] == pytest.approx(33 / 64)
    assert line["kernels"]["gemm_up"]["share"] == pytest.approx(0.75)
    assert line["gpu_launches"] == 1234 and line["finite"] is True
