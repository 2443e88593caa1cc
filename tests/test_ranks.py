"""Replica ranks on the CPU: world-size-2 gloo process groups.

The benchmark runs one independent system per GPU; its only collectives
bracket the timed region.  These tests run the same host logic with gloo:
the reported time is the slowest rank's, the units are summed over ranks,
every rank takes the same collective steps, and the reference arm does its
work on rank 0 alone.
"""
import json
import os
import socket
import subprocess
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from molecular_dynamics_b200.ranks import RankGroup, RankInfo, Timed, host_clock, timed_region  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, sleeps, units, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    info = RankInfo.from_env()
    group = RankGroup.init(info, "gloo", timeout_s=60)
    try:
        res = timed_region(group, lambda: time.sleep(sleeps[rank]) or rank, host_clock, units[rank])
        # a second region, as the benchmark's end-to-end leg does, on every rank
        res2 = timed_region(group, lambda: rank * 10, host_clock, units[rank])
        out.put((rank, res.ms, res.units, res.result, res2.units, res2.result))
    finally:
        group.close()


def _run(world, sleeps, units):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, sleeps, units, q)) for r in range(world)]
    for p in procs:
        p.start()
    rows = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(rows)


def test_two_ranks_max_time_and_summed_units():
    rows = _run(2, sleeps=[0.05, 0.4], units=[1000.0, 3000.0])
    ms = [r[1] for r in rows]
    # both ranks report the same (slowest) time, at least rank 1's own sleep
    assert ms[0] == ms[1]
    assert ms[0] >= 400.0
    for rank, _, u, result, u2, result2 in rows:
        assert u == 4000.0 and u2 == 4000.0
        assert result == rank and result2 == 10 * rank


def test_single_process_group_is_identity():
    g = RankGroup()
    res = timed_region(g, lambda: 7, lambda run: (12.5, run()), 100.0)
    assert res.ms == 12.5 and res.units == 100.0 and res.result == 7
    assert res.throughput == pytest.approx(100.0 / 12.5e-3)


def test_throughput_is_whole_job():
    # replicas: value = units of all ranks / the slowest rank's time
    t = Timed(ms=250.0, units=4 * 1_048_576 * 20, result=None)
    assert t.throughput == pytest.approx(4 * 1_048_576 * 20 / 0.25)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "0", "--gpus", "2"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
    assert time.perf_counter() - t0 < 60


def test_reference_arm_prints_the_contract_line():
    # one process (N = 1): the oracle's JSON line carries the metric of the GPU arm, a CPU
    # baseline describing this run and an end-to-end entry with no host-device traffic
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "ag256",
                        "--steps", "1", "--warmup", "0", "--cpu-seconds", "1"],
                       env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "atom-steps/s" and d["higher_is_better"] is True
    assert d["metric"].startswith("atom-steps/s") and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["dtype"] == "f64" and d["data"] == "synthetic" and d["config"]["workload"].startswith("ag256")


def test_roofline_arithmetic():
    import bench
    # 10 launches of 3 ms each of the edge backward; T = 3, N_phi = 8
    prof = {"edge_bwd": (30.0, 10), "density": (9.0, 9), "active": (1.0, 3)}
    pairs = 1_000_000
    roof = bench.roofline(prof, pairs, 8, 3, 50_000, 148, {"sm_max_mhz": 2000.0}, "measured", {"sm_mhz": 1900.0})
    flop = pairs * (bench.FLOP_EDGE_BWD_PER_PAIR[8][0] + 2 * bench.FLOP_EDGE_BWD_PER_PAIR[8][1]) / 3
    assert roof["kernel"] == "k_edge_bwd" and roof["bound"] == "alu"
    assert roof["flop_per_launch"] == pytest.approx(flop)
    assert roof["achieved"] == pytest.approx(flop / 3e-3 / 1e12)
    assert roof["peak"] == pytest.approx(148 * 128 * 2 * 2000e6 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    # a dominant group with no algorithmic count has no entry
    assert bench.roofline({"mlp_bwd": (5.0, 1)}, pairs, 8, 3, 1, 148, {}, "fallback", {}) is None
    json.dumps(roof)
    # dominant fp32 networks: 2 (108*128 + 128*128 + 128*24) flop per forward, doubled for the VJP launch
    r2 = bench.roofline({"mlp_bwd": (8.0, 2), "edge_bwd": (1.0, 3)}, pairs, 8, 3, 1000, 148, {"sm_max_mhz": 2000.0},
                        "measured", {}, net=(108, 24, (128, 128), "simt"))
    assert r2["bound"] == "alu"
    assert r2["flop_per_launch"] == 1000 * 2 * 2 * (108 * 128 + 128 * 128 + 128 * 24)
    assert r2["achieved"] == pytest.approx(r2["flop_per_launch"] / 4e-3 / 1e12)
    # bf16 tensor-core networks: against the sustained bf16 peak
    r3 = bench.roofline({"mlp_fwd": (8.0, 2)}, pairs, 8, 3, 1000, 148, {"bf16_tflops_sustained": 1382.5}, "measured",
                        {}, net=(24, 24, (128, 128), "bf16"))
    assert r3["bound"] == "tensor" and r3["peak"] == 1382.5
    # three-pass tf32 networks: against the tf32 peak (bf16 x the nominal 1.1 / 2.25), algorithmic flops
    r4 = bench.roofline({"mlp_fwd": (8.0, 2)}, pairs, 8, 3, 1000, 148, {"bf16_tflops_sustained": 1382.5}, "measured",
                        {}, net=(24, 24, (64, 64), "tf32x3"))
    assert r4["bound"] == "tensor" and r4["peak"] == pytest.approx(1382.5 * 1.1 / 2.25)
    assert r4["flop_per_launch"] == 1000 * 2 * (24 * 64 + 64 * 64 + 64 * 24)


def test_per_kernel_roofline_arithmetic():
    import bench
    prof = {"active": (2.0, 4), "density": (6.0, 3), "mlp_fwd": (1.0, 2), "energy_sum": (0.1, 1)}
    pk = {"hbm_gbs": 6500.0, "sm_max_mhz": 2000.0, "bf16_tflops_sustained": 1400.0}
    n, pairs, nnz = 1000, 54_000, 78_000
    a = bench.kernel_roofline("active", prof, pairs, 8, 3, n, 148, pk, "measured", {}, nnz=nnz)
    bytes_ = 4 * nnz + 4 * (n + 1) + 16 * n + 20 * pairs + 4 * n
    assert a["bound"] == "hbm" and a["unit"] == "GB/s"
    assert a["achieved"] == pytest.approx(bytes_ / 0.5e-3 / 1e9)
    assert a["frac"] == pytest.approx(a["achieved"] / 6500.0)
    d = bench.kernel_roofline("density", prof, pairs, 8, 3, n, 148, pk, "measured", {})
    assert d["achieved"] == pytest.approx(pairs * bench.FLOP_DENSITY_PER_PAIR[8] / 2e-3 / 1e12)
    m = bench.kernel_roofline("mlp_fwd", prof, pairs, 8, 3, n, 148, pk, "measured", {}, net=(24, 24, (128, 128), "bf16"))
    assert m["bound"] == "tensor" and m["peak"] == 1400.0
    assert m["achieved"] == pytest.approx(n * bench.network_flop_per_atom("mlp_fwd", 24, 24, (128, 128)) / 0.5e-3 / 1e12)
    # groups without an algorithmic count, or absent, have no entry
    assert bench.kernel_roofline("energy_sum", prof, pairs, 8, 3, n, 148, pk, "measured", {}) is None
    assert bench.kernel_roofline("edge_bwd", prof, pairs, 8, 3, n, 148, pk, "measured", {}) is None
    assert bench.kernel_roofline("active", prof, pairs, 8, 3, n, 148, pk, "measured", {}) is None
