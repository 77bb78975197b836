"""bench.py's multi-rank path on the CPU: two gloo ranks started the way torchrun starts
them (RANK / WORLD_SIZE / MASTER_ADDR / MASTER_PORT in the environment)."""

import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
import bench  # noqa: E402

_RANK = """
import datetime, json, os, sys
sys.path.insert(0, sys.argv[1])
import torch.distributed as dist
import bench
rank = int(os.environ["RANK"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
# rank-dependent timings: the job is as slow as its slowest rank, per quantity
mine = [10.0 + 2.0 * rank, 30.0 - rank, 5.0]
got = bench.max_over_ranks(mine, dist, "cpu")
# repeated timed regions: rank 0's regions take 100 ms, rank 1's 400 ms; both must run
# the larger count (10 regions for 1 s), so their collectives stay paired
class Clk:
    marks = []
    def mark(self, m):
        self.marks.append(m)
clk = Clk()
calls = []
def region(mk):
    calls.append(mk)
    if mk[0]:
        clk.mark(mk[0])
    dist.barrier()
    return 100.0 if rank == 0 else 400.0
regions = bench._repeated_regions(region, clk, 1.0, dist, "cpu")
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "got": got, "regions": regions, "calls": calls,
                  "marks": clk.marks}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_max_of_every_timing():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", _RANK, str(ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.returncode == 0, e[-2000:]
        outs.append(json.loads(o.strip().splitlines()[-1]))
    for r in outs:
        assert r["got"] == [12.0, 30.0, 5.0]
        assert len(r["regions"]) == 10
        assert r["calls"][0] == ["begin", None]
        assert all(c == [None, None] for c in r["calls"][1:])
        assert r["marks"] == ["begin", "end"]


def test_one_rank_repeats_regions_until_the_minimum_time():
    class Clk:
        def __init__(self):
            self.marks = []

        def mark(self, m):
            self.marks.append(m)

    clk = Clk()
    times = iter([300.0, 310.0, 290.0, 305.0, 999.0])
    regions = bench._repeated_regions(lambda mk: next(times), clk, 1.0, None, "cpu")
    assert regions == [300.0, 310.0, 290.0, 305.0]     # ceil(1000 / 300) = 4
    assert clk.marks == ["end"]                         # the region marks its own begin
    assert bench._repeated_regions(lambda mk: 5000.0, clk, 1.0, None, "cpu") == [5000.0]
    assert bench._repeated_regions(lambda mk: 1.0, clk, 0.0, None, "cpu") == [1.0]


def test_replica_throughput_counts_every_rank_over_the_slowest_time():
    # 2 ranks x 10 steps x 8192 tokens in 12 ms (the slowest rank)
    assert bench.replica_throughput(8192, 2, 10, 12.0) == pytest.approx(8192 * 20 / 0.012)
    assert bench.max_over_ranks([1.5, 2], None, "cpu") == [1.5, 2.0]


def test_reference_arm_on_a_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_contract_line_on_rank_zero():
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference",
                        "--workload", "tiny_fp32", "--steps", "2", "--warmup", "1"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.strip().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"]
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("tiny_fp32")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_algorithmic_bytes_and_flops_of_the_1024px_layer():
    # the roofline numerators: the minimum each kernel moves with H and Y in bf16 (router
    # x, W_r, scores, scores_t; W1|W3, gathered rows, H; W2, H, Y; Y, out), 1024 px CFG
    from diffusion_transformer_moe_b200 import inputs as I
    w = I.WORKLOADS["1024px_cfg"]
    mb = {k: round(v / 1e6, 1) for k, v in bench.stage_bytes(w).items()}
    assert (mb["router"], mb["gemm1_swiglu"], mb["gemm2_scale"], mb["combine"]) == \
        (38.0, 587.2, 318.8, 67.1)
    gf = {k: round(v / 1e9, 2) for k, v in bench.stage_flops(w).items()}
    assert gf == {"router": 2.15, "gemm1_swiglu": 68.72, "gemm2_scale": 34.36}
    # split intermediates move H as a bf16 hi/lo pair and Y in fp32 on purpose: reported
    # beside the algorithmic bytes, never inside them
    alg, des = bench.stage_bytes(w), bench.stage_design_bytes(w, "split")
    assert des["gemm1_swiglu"] - alg["gemm1_swiglu"] == 2 * w.E * w.Ce * w.F + 4 * w.E * w.Ce
    assert des["gemm2_scale"] - alg["gemm2_scale"] == \
        2 * w.E * w.Ce * w.F + 2 * w.E * w.Ce * w.d + 8 * w.E * w.Ce
    assert des["combine"] - alg["combine"] == 2 * w.E * w.Ce * w.d + 4 * (w.T + 1)
    plain = bench.stage_design_bytes(w, "bf16")
    assert plain["gemm2_scale"] - alg["gemm2_scale"] == 8 * w.E * w.Ce


def test_both_arms_carry_the_same_config():
    from diffusion_transformer_moe_b200 import inputs as I
    w = I.WORKLOADS["1024px_cfg"]
    c = bench._workload_config(w)
    assert set(c) == {"workload", "T", "d", "E", "F", "C", "segments", "l2"}
    assert c == bench._workload_config(w, "write+read")


def test_clock_sampler_reports_only_the_timed_region(monkeypatch):
    # a fake NVML whose clock and reasons change when the timed region begins and ends:
    # the record must hold only the samples taken in between
    import time
    import types
    phase = {"v": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0, nvmlInit=lambda: None, nvmlDeviceGetHandleByIndex=lambda i: i,
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: (600, 1900, 700)[phase["v"]],
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: (0x40, 0x4, 0x8)[phase["v"]])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    cs = bench.ClockSampler(0)
    cs.start()
    time.sleep(0.02)
    phase["v"] = 1
    time.sleep(0.005)  # a sample under way when the phase changed has finished
    cs.mark("begin")
    time.sleep(0.02)
    cs.mark("end")
    phase["v"] = 2
    time.sleep(0.02)
    rec = cs.stop()
    assert rec["samples"] >= 3
    assert rec["sm_mhz"] == 1900 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]
