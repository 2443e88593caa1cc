#!/usr/bin/env python
"""Throughput of REANN velocity-Verlet MD (energy + forces, T = 3) on one B200.

One step = one pass of the whole hot path over the workload: half kick and
drift, the skin check (and, when it trips, the cell binning and neighbour-list
rebuild), one energy+force evaluation (active-pair compaction, T density
layers, coefficient networks, energy network, T edge backward passes and
force gather, energy reduction) and the second half kick.

Default workload: Ag FCC 64x64x64 cells (1,048,576 atoms), a = 4.09 A,
sigma = 0.05 A, T = 3, r_c = 6.0 A, 8 radial functions, L = 2, networks
[128, 128], 1 fs steps, Maxwell-Boltzmann 300 K.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (one process per GPU under torchrun) every rank runs its own
replica of the workload (independent systems, no data-path collective):
value = atom-steps of all ranks / the slowest rank's time.
--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from molecular_dynamics_b200 import presets, synth  # noqa: E402
from molecular_dynamics_b200.ranks import RankGroup, RankInfo, cuda_event_clock, timed_region  # noqa: E402

METRIC = "atom-steps/s (MD step = E+F, T=3)"
UNIT = "atom-steps/s"
L2_BYTES = 126 * 1024 * 1024

# algorithmic FP32 operations per active (directed) pair, from the arithmetic
# the two edge passes perform per pair (FMA = 2; exp, sin/cos, sqrt, rcp = 1)
FLOP_DENSITY_PER_PAIR = {8: 240, 10: 298}
FLOP_EDGE_BWD_PER_PAIR = {8: (754, 930), 10: (938, 1158)}   # (layer 0 without dE/dc, layers >= 1)


# DRAM read + write (dram__bytes_read.sum + dram__bytes_write.sum) of one
# k_edge_bwd launch (a layer >= 1 launch: the scalar kernel) from an ncu
# capture on 256,000 Ag atoms of the 1M-atom Ag model, scaled to the atom count
# of the run; other models (other densities, cut-offs, radial counts) report null.  The capture
# belongs to the kernel source whose SHA-256 prefix is recorded beside it (the
# text of the scalar k_edge_bwd kernel in edge.cu): once that text changes, the
# figure no longer describes the kernel and the line reports null.
EDGE_BWD_CAPTURE = {"bytes_per_atom": (448.216192e6 + 23.258240e6) / 256000, "source_sha": "73c818a4f0abbb25",
                    "workload": "ag1m"}
EDGE_BWD_TRAFFIC_NOTE = "bytes per launch: DRAM read+write of a 256,000-atom ncu capture scaled by the atom count"


def edge_source_sha() -> str:
    import hashlib
    with open(os.path.join(ROOT, "molecular_dynamics_b200", "csrc", "edge.cu")) as f:
        src = f.read()
    a = src.index("k_edge_bwd(int n")
    b = src.index("\n// Packed form of the backward", a)
    return hashlib.sha256(src[a:b].encode()).hexdigest()[:16]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 20 ms, started
    before the warm-up so that samples flow when the timed region begins;
    stop() keeps the samples taken between mark_begin() and mark_end() (for a
    region shorter than the sampling interval, the nearest sample on each
    side)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.t0 = self.t1 = None

    def wait_ready(self, timeout: float = 5.0):
        """Block until the sampler has written its first sample (nvidia-smi takes
        a moment to start), so that short timed regions are covered."""
        if self.proc is None:
            return
        t_end = time.time() + timeout
        while time.time() < t_end:
            self.file.flush()
            if os.path.getsize(self.file.name) > 0:
                return
            time.sleep(0.02)

    def mark_begin(self):
        import datetime
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        import datetime
        self.t1 = datetime.datetime.now()

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        import datetime
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        rows = []
        for line in self.file.read().strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(parts[1]), float(parts[2]),
                             {n for n, v in zip(names, parts[5:9]) if v.lower().startswith("active")}))
            except ValueError:
                continue
        os.unlink(self.file.name)
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= self.t1]
        nearest = False
        if not inside and rows and self.t0 is not None:
            before = [r for r in rows if r[0] < self.t0]
            after = [r for r in rows if r[0] > self.t1]
            inside = before[-1:] + after[:1]
            nearest = True
        sm = [r[1] for r in inside]
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": max(r[2] for r in inside) if inside else None,
               "reasons": sorted(set().union(*[r[3] for r in inside])) if inside else [], "samples": len(sm)}
        if nearest:
            out["note"] = "timed region shorter than the 20 ms sampling interval: the nearest sample on each side"
        return out


def cpu_sample_preset(p):
    """The bounded sample of a workload the oracle is timed on: FCC lattices
    cut to at most 12^3 cells (6,912 atoms), the 3,000-atom water box whole,
    the gas mixture in 1/32 of the volume at the same number density and
    composition.  Same model and weights as the workload."""
    if p.kind == "fcc":
        return p.with_(ncell=min(p.ncell, 12))
    if p.kind == "chon":
        f = 32
        return p.with_(n_mol=tuple(max(1, round(k / f)) for k in p.n_mol), box=p.box / f ** (1.0 / 3.0))
    return p


def cpu_sample(p, seconds: float = 12.0, steps: int = 0):
    """The oracle's velocity Verlet on the workload's bounded sample (brute-
    force pairs every step).  steps = 0: one step is timed first and the step
    count is chosen to fill about `seconds` of CPU time (1 to 256 steps)."""
    import oracle
    ps = cpu_sample_preset(p)
    pos, types, box = synth.make_structure(ps)
    v = synth.maxwell_boltzmann(ps, types)
    model = oracle.Model.from_preset(p, synth.weight_blob(p))
    dt_fs = p.dt_fs
    if steps <= 0:
        t0 = time.perf_counter()
        oracle.md_verlet(model, pos.astype(np.float64), v, types, box, ps.masses, dt_fs, 1)
        per_step = (time.perf_counter() - t0) / 2          # the initial evaluation and one step
        steps = int(max(1, min(256, seconds / max(per_step, 1e-6))))
    t0 = time.perf_counter()
    oracle.md_verlet(model, pos.astype(np.float64), v, types, box, ps.masses, dt_fs, steps)
    dt = time.perf_counter() - t0
    n = len(pos)
    return {"value": n * steps / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"fp64 oracle velocity Verlet on a {n}-atom sample of {p.key} (same model), {steps} steps of "
                      f"{dt_fs:g} fs plus the initial force evaluation, brute-force pairs every step; {dt:.1f} s"}, dt


def oracle_breakdown(p):
    """The oracle's parts on the workload's bounded sample: the O(N^2) pair
    search, the cell-list pair search, and one energy+force evaluation given
    the pair list (ms each)."""
    import oracle
    ps = cpu_sample_preset(p)
    pos, types, box = synth.make_structure(ps)
    model = oracle.Model.from_preset(p, synth.weight_blob(p))
    t0 = time.perf_counter()
    pairs = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    t1 = time.perf_counter()
    oracle.pairs_cells(pos, box, p.r_cut, p.skin)
    t2 = time.perf_counter()
    oracle.energy_forces(model, pos, types, box, pairs)
    t3 = time.perf_counter()
    return {"atoms": len(pos), "pairs_brute_ms": 1e3 * (t1 - t0), "pairs_cells_ms": 1e3 * (t2 - t1),
            "energy_forces_given_pairs_ms": 1e3 * (t3 - t2)}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    p = presets.get(args.workload)
    _, dt_w = cpu_sample(p, steps=args.warmup) if args.warmup > 0 else (None, 0.0)
    cb, dt = cpu_sample(p, steps=args.steps)
    parts = oracle_breakdown(p)
    line = {
        "impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{p.key}: {p.description} (oracle timed on a {parts['atoms']}-atom sample of it)",
                   "atoms": p.n_atoms, "T": p.T, "r_cut": p.r_cut, "n_radial": p.n_radial, "l_max": p.l_max,
                   "hidden": list(p.hidden), "dt_fs": p.dt_fs},
        "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
        "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "oracle_breakdown": parts,
    }
    print(json.dumps(line), flush=True)
    return 0


def dd_sweep(args):
    """Monolithic vs domain-decomposed E+F for T = 1..6 on the workload: time,
    ghost bytes per layer and per evaluation, and bit-identity of the results.
    One JSON line per T."""
    import torch
    from molecular_dynamics_b200 import reann

    p = presets.get(args.workload)
    if args.ncell:
        p = presets.scaled(args.workload, ncell=args.ncell)
    pos, types, box = synth.make_structure(p)
    n = len(pos)
    pos_d = torch.from_numpy(pos).cuda()
    types_d = torch.from_numpy(types).cuda()
    grid = tuple(int(x) for x in args.dd_grid.split("x"))
    stream = torch.cuda.current_stream()

    def timed(ctx, F):
        for _ in range(2):
            ctx.reann_energy_forces(pos_d, F)
        times = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            E = ctx.reann_energy_forces(pos_d, F)
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        return E, statistics.median(times)

    for T in range(1, max(p.stats_depth, p.T) + 1):
        w = synth.weight_blob(p, T=T)
        out = {}
        for name, g in (("mono", (0, 0, 0)), ("dd", grid)):
            ctx = reann.Context(reann.ModelSpec.from_preset(p, T=T, dd_grid=g), w)
            ctx.reann_build_neighbors(pos_d, types_d, box)
            F = torch.empty_like(pos_d)
            E, ms = timed(ctx, F)
            out[name] = (E, ms, F.clone(), ctx.reann_get_counters())
            ctx.close()
        c = out["dd"][3]
        print(json.dumps({
            "mode": "dd_sweep", "workload": p.key, "atoms": n, "T": T, "dd_grid": list(grid),
            "ef_ms_monolithic": out["mono"][1], "ef_ms_dd": out["dd"][1],
            "ghost_slots": c.ghost_slots, "ghost_bytes_per_layer_fwd": c.ghost_bytes_fwd,
            "ghost_bytes_per_layer_bwd": c.ghost_bytes_bwd,
            "ghost_bytes_per_evaluation": (T - 1) * c.ghost_bytes_fwd + T * c.ghost_bytes_bwd + 16 * c.ghost_slots,
            "bit_identical": bool(out["mono"][0] == out["dd"][0] and torch.equal(out["mono"][2], out["dd"][2])),
        }), flush=True)
    return 0


def network_flop_per_atom(group, d_in, d_out, hidden):
    """Algorithmic flops of one network launch per atom: a forward pass is
    2 (d_in H1 + H1 H2 + H2 d_out); the energy launch adds its VJP (same
    count with d_out = 1), the coefficient backward recomputes the forward and
    runs the VJP."""
    h1, h2 = hidden
    fwd = lambda o: 2 * (d_in * h1 + h1 * h2 + h2 * o)
    return {"mlp_fwd": fwd(d_out), "mlp_energy": 2 * fwd(1), "mlp_bwd": 2 * fwd(d_out)}[group]


def network_kind(p) -> str:
    """Which network kernels the library runs for this model (include/reann.h,
    mlp_precision): bf16 tensor cores, three-pass tf32 tensor cores, or fp32
    CUDA cores."""
    if p.mlp_precision == 1:
        return "bf16"
    if p.mlp_precision == 0 and tuple(p.hidden) == (64, 64) and p.density_form == 0 and p.n_radial in (8, 10):
        return "tf32x3"
    return "simt"


NETWORK_DESCRIPTION = {"bf16": "bf16 tcgen05 (split bf16 activations), fp32 accumulate",
                       "tf32x3": "fp32-accurate tcgen05: three tf32 passes of hi/lo split operands, fp32 accumulate",
                       "simt": "fp32 CUDA-core"}

KERNEL_NAMES = {"edge_bwd": "k_edge_bwd", "density": "k_density_fwd", "active": "k_active"}
NETWORK_NAMES = {"mlp_fwd": " (coefficient networks)", "mlp_energy": " (energy network + VJP)",
                 "mlp_bwd": " (coefficient-network VJP)"}


def kernel_roofline(group, prof, active_pairs, NP, T, n_atoms, sm_count, pk, pk_kind, clk, net=None, nnz=None):
    """Roofline entry of one kernel group: algorithmic operations (or bytes)
    per launch over its mean CUDA-event launch time.  Edge passes and fp32
    networks: FP32 FMA peak of the SM count at clocks.max.sm; bf16 tensor-core
    networks: the measured sustained bf16 peak; the active-pair compaction:
    the measured HBM copy bandwidth, with the bytes it must move (full-list
    columns and row offsets read, positions read once, active columns and
    geometry and counts written).  `net` = (d_in, d_out, hidden,
    mlp_precision) of the workload's networks; `nnz` the full-list length.
    None for a group without an algorithmic count or launches."""
    if group not in prof or not prof[group][1]:
        return None
    ms, launches = prof[group]
    launch_s = ms / launches * 1e-3
    smax = pk.get("sm_max_mhz", 1965.0)
    clock_mhz = clk.get("sm_mhz") or smax
    fp32_peak = sm_count * 128 * 2 * smax * 1e6 / 1e12
    fp32_note = (f"FP32 FMA peak {sm_count} SMs x 128 lanes x 2 flop x {smax:.0f} MHz "
                 f"(clocks.max.sm, {pk_kind}); median SM clock during the run {clock_mhz} MHz")
    if group == "active":
        if nnz is None:
            return None
        work = 4.0 * nnz + 4.0 * (n_atoms + 1) + 16.0 * n_atoms + 20.0 * active_pairs + 4.0 * n_atoms
        peak = pk.get("hbm_gbs", 6650.0)
        achieved = work / launch_s / 1e9
        return {"kernel": "k_active", "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "bytes_per_launch": work, "launch_ms": launch_s * 1e3,
                "peak_note": f"HBM copy bandwidth ({pk_kind})"}
    tensor = False
    if group == "edge_bwd":
        work = active_pairs * (FLOP_EDGE_BWD_PER_PAIR[NP][0] + (T - 1) * FLOP_EDGE_BWD_PER_PAIR[NP][1]) / T
    elif group == "density":
        work = active_pairs * FLOP_DENSITY_PER_PAIR[NP]
    elif group.startswith("mlp_") and net is not None:
        d_in, d_out, hidden, kind = net
        work = n_atoms * network_flop_per_atom(group, d_in, d_out, hidden)
        tensor = kind != "simt"
    else:
        return None
    achieved = work / launch_s / 1e12
    if tensor and kind == "bf16":
        peak, note = pk.get("bf16_tflops_sustained", 1400.0), f"bf16 dense, sustained ({pk_kind})"
    elif tensor:
        # tf32 dense: the measured sustained bf16 peak x the nominal tf32/bf16 ratio (1.1 / 2.25 PFLOP/s);
        # the three tf32 passes per product are not counted as work
        peak = pk.get("bf16_tflops_sustained", 1400.0) * 1.1 / 2.25
        note = f"tf32 dense = sustained bf16 ({pk_kind}) x 1.1/2.25 nominal; algorithmic flops (each product runs 3 passes)"
    else:
        peak, note = fp32_peak, fp32_note
    kernel = KERNEL_NAMES.get(group) or {"bf16": "k_mlp_tc", "tf32x3": "k_mlp_tc32", "simt": "k_mlp"}.get(
        kind, "k_mlp") + NETWORK_NAMES.get(group, "")
    return {"kernel": kernel, "bound": "tensor" if tensor else "alu", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "flop_per_launch": work, "launch_ms": launch_s * 1e3,
            "peak_note": note}


def roofline(prof, active_pairs, NP, T, n_atoms, sm_count, pk, pk_kind, clk, net=None, workload=None):
    """Roofline entry of the dominant kernel group (largest share of the
    profiled time), with its DRAM traffic per launch where an ncu capture of
    that kernel exists."""
    shares = {k: v_[0] for k, v_ in prof.items()}
    dominant = max(shares, key=shares.get)
    r = kernel_roofline(dominant, prof, active_pairs, NP, T, n_atoms, sm_count, pk, pk_kind, clk, net)
    if r is None:
        return None
    current = (dominant == "edge_bwd" and EDGE_BWD_CAPTURE["source_sha"] == edge_source_sha()
               and workload == EDGE_BWD_CAPTURE["workload"])
    traffic = EDGE_BWD_CAPTURE["bytes_per_atom"] * n_atoms if current else None
    r["traffic"] = traffic
    r["traffic_note"] = EDGE_BWD_TRAFFIC_NOTE if traffic is not None else \
        "no DRAM capture of the current source of this kernel on this model"
    if dominant in ("edge_bwd", "density"):
        # what ncu shows binding the edge passes (the FP32 peak is the arithmetic roofline only)
        r["limiter_note"] = ("ncu: the L1 data pipe at 72-78 % of its wavefront rate and the register "
                             "writeback at 61-67 % (neighbour-row gathers); FP32 pipes about half busy")
    return r


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1, help="GPUs (one process per GPU under torchrun; replicas)")
    ap.add_argument("--steps", type=int, default=100, help="timed MD steps (one call, device-resident)")
    ap.add_argument("--warmup", type=int, default=3, help="untimed MD steps before the timed region")
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"),
                    help="reference: the fp64 oracle on a bounded sample of the workload, host cores")
    ap.add_argument("--workload", default="ag1m", choices=presets.ALL, help="synthetic system and model")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-array end-to-end timing")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle baseline sample")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU time of the oracle baseline sample")
    ap.add_argument("--dd-sweep", action="store_true",
                    help="monolithic vs domain-decomposed E+F for T = 1..6 (one JSON line per T)")
    ap.add_argument("--dd-grid", default="8x8x8", help="subdomain grid of --dd-sweep")
    ap.add_argument("--ncell", type=int, default=0,
                    help="FCC workloads: cells per axis (smaller lattices for profiling captures)")
    ap.add_argument("--ensemble", default="nve", choices=("nve", "nvt"),
                    help="nvt: stochastic velocity rescaling after every step (reann_md_step_nvt)")
    ap.add_argument("--temperature", type=float, default=300.0, help="NVT target temperature, K")
    ap.add_argument("--tau", type=float, default=100.0, help="NVT coupling time, fs")
    ap.add_argument("--mlp-precision", type=int, default=None, choices=(0, 1, 2),
                    help="override the workload's network precision (2: fp32 CUDA-core networks)")
    args = ap.parse_args()

    info = RankInfo.from_env()
    if args.impl == "reference":
        return run_reference(args, info.rank, info.world)
    if args.dd_sweep:
        return dd_sweep(args)

    import torch
    from molecular_dynamics_b200 import reann

    torch.cuda.set_device(info.local)
    group = RankGroup.init(info, "nccl")

    p = presets.get(args.workload)
    if args.ncell:
        p = presets.scaled(args.workload, ncell=args.ncell)
    if args.mlp_precision is not None:
        p = p.with_(mlp_precision=args.mlp_precision)
    pos, types, box = synth.make_structure(p)
    v0 = synth.maxwell_boltzmann(p, types)
    n = len(pos)
    dt_fs = p.dt_fs   # the workload's own step: 1 fs, 0.5 fs for water (ns/day is quoted at 1 fs and at it)
    spec = reann.ModelSpec.from_preset(p)   # the workload's own network precision (bf16 for ag1m)
    ctx = reann.Context(spec, synth.weight_blob(p), device=info.local)
    stream = torch.cuda.current_stream()
    clock = cuda_event_clock(stream)
    x = torch.from_numpy(pos.astype(np.float64)).cuda()
    v = torch.from_numpy(v0.copy()).cuda()
    pos_d = torch.from_numpy(pos).cuda()
    ctx.reann_build_neighbors(pos_d, torch.from_numpy(types).cuda(), box)

    # ---- energy+force evaluations alone (the single-evaluation workloads'
    # unit): reann_energy_forces on the resident start structure
    F_d = torch.empty_like(pos_d)
    for _ in range(args.warmup):
        ctx.reann_energy_forces(pos_d, F_d)
    ef_steps = max(1, min(args.steps, 20))

    def ef_loop():
        for _ in range(ef_steps):
            ctx.reann_energy_forces(pos_d, F_d)

    ef_run = timed_region(group, ef_loop, clock, n * ef_steps)
    del F_d

    # the MD call of the chosen ensemble; NVT draws every step's two random
    # numbers up front on the host (the library takes them as inputs)
    total_steps = args.warmup + args.steps + min(args.steps, 20) + (0 if args.no_e2e else args.steps + 1)
    noise = synth.thermostat_noise(n, total_steps, seed=2024) if args.ensemble == "nvt" else None
    cursor = [0]

    def md(k, xx, vv):
        if noise is None:
            return ctx.reann_md_step(k, dt_fs, xx, vv, p.masses)
        z = noise[cursor[0]:cursor[0] + k]
        cursor[0] += k
        return ctx.reann_md_step_nvt(k, dt_fs, args.temperature, args.tau, z, xx, vv, p.masses)

    # warm-up (the first call also evaluates the entry forces); the clock
    # sampler starts before it so that samples flow through the timed region
    clocks = ClockSampler(info.local)
    clocks.start()
    clocks.wait_ready()
    md(args.warmup, x, v)
    torch.cuda.synchronize()

    # ---- device-resident timed region: K steps in one call (a continuation);
    # each step's energy+forces and half kick replay as one CUDA graph
    launches0 = ctx.reann_get_counters().kernel_launches

    def timed_steps():
        clocks.mark_begin()
        out = md(args.steps, x, v)   # returns after its stream has synchronised
        clocks.mark_end()
        return out

    run = timed_region(group, timed_steps, clock, n * args.steps)
    clk = clocks.stop()
    st = run.result
    t_ms = run.ms
    value = run.throughput
    launches = ctx.reann_get_counters().kernel_launches - launches0

    # ---- kernel breakdown: a separate call with per-launch CUDA events (eager launches)
    prof_steps = min(args.steps, 20)
    ctx.reann_profile(True)
    md(prof_steps, x, v)
    torch.cuda.synchronize()
    prof = ctx.reann_profile_read()
    ctx.reann_profile(False)
    cnt = ctx.reann_get_counters()

    # ---- end to end: one public call per step with pinned host state
    e2e = None
    if not args.no_e2e:
        xh = torch.empty((n, 3), dtype=torch.float64).pin_memory()
        vh = torch.empty((n, 3), dtype=torch.float64).pin_memory()
        xh.copy_(x.cpu())
        vh.copy_(v.cpu())
        md(1, xh.numpy(), vh.numpy())      # warm the host path

        def host_steps():
            for _ in range(args.steps):
                md(1, xh.numpy(), vh.numpy())

        run_e = timed_region(group, host_steps, clock, n * args.steps)
        e2e = {"value": run_e.throughput, "unit": UNIT,
               "h2d_bytes_per_step": 2 * 3 * 8 * n, "d2h_bytes_per_step": 2 * 3 * 8 * n,
               "note": f"{'reann_md_step_nvt' if noise is not None else 'reann_md_step'}(1) per step with pinned "
                       "host x, v: x and v copied in and out every step (the library moves them in and checks "
                       "them against its resident state while the step runs; x goes out during the step's "
                       "force evaluation)"}

    if info.rank != 0:
        group.close()
        return 0
    world = info.world

    # ---- roofline of the dominant kernel group (FP32-ALU bound edge passes)
    pk, pk_kind = peaks()
    sm_count = torch.cuda.get_device_properties(info.local).multi_processor_count
    shares = {k: v_[0] for k, v_ in prof.items()}
    total = sum(shares.values()) or 1.0
    net = (p.DR, p.D, tuple(p.hidden), network_kind(p))
    roof = roofline(prof, cnt.active_pairs, p.n_radial, p.T, n, sm_count, pk, pk_kind, clk, net=net, workload=p.key)
    per_kernel = {}
    for g in ("edge_bwd", "density", "mlp_bwd", "mlp_fwd", "mlp_energy", "active"):
        r = kernel_roofline(g, prof, cnt.active_pairs, p.n_radial, p.T, n, sm_count, pk, pk_kind, clk, net=net,
                            nnz=cnt.nnz)
        if r is not None:
            per_kernel[g] = {k: r[k] for k in ("kernel", "bound", "achieved", "peak", "unit", "frac", "launch_ms")}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (networks bf16, fp32 accumulate)" if p.mlp_precision else "f32",
        "data": "synthetic",
        "config": {"workload": f"{p.key}: {p.description}", "atoms": n, "T": p.T, "r_cut": p.r_cut,
                   "n_radial": p.n_radial, "l_max": p.l_max, "hidden": list(p.hidden), "dt_fs": dt_fs,
                   "networks": NETWORK_DESCRIPTION[network_kind(p)],
                   "launch": "energy+forces and half kick replayed as one CUDA graph per step",
                   "ensemble": "NVE (velocity Verlet)" if noise is None else
                               f"NVT (stochastic velocity rescaling, {args.temperature:g} K, tau {args.tau:g} fs)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"working set > L2 ({n * (p.T * (10 * p.n_radial + 6 * p.n_radial) * 4) / 1e9:.1f} GB of "
                         f"per-layer activations vs 126 MB L2); no flush needed"},
        "ns_per_day": (args.steps / (t_ms * 1e-3)) * 1.0 * 86400 / 1e6,
        "ns_per_day_note": "at the metric's 1 fs per step" + (
            f"; {(args.steps / (t_ms * 1e-3)) * dt_fs * 86400 / 1e6:.4g} ns/day at the workload's own {dt_fs:g} fs"
            if dt_fs != 1.0 else ""),
        "energy_forces": {"value": ef_run.throughput, "unit": "atom-evaluations/s",
                          "ms_per_evaluation": ef_run.ms / ef_steps, "evaluations": ef_steps,
                          "note": "reann_energy_forces alone on the resident start structure (energy read back "
                                  "each call); the unit of the single-evaluation workloads"},
        "rebuilds": st.rebuilds,
        "gpu_launches": launches,
        "clocks": clk,
        "kernel_ms_per_step": {k: v_[0] / prof_steps for k, v_ in prof.items() if v_[1]},
        "kernel_profile_note": (f"per-launch CUDA events over a separate {prof_steps}-step call with eager launches; "
                                f"their sum {total / prof_steps:.4g} ms per step against the timed (graph-replayed) "
                                f"step's {t_ms / args.steps:.4g} ms"),
        "kernel_share": {k: v_ / total for k, v_ in shares.items() if v_},
        "roofline": roof,
        "kernel_roofline": per_kernel,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and world == 1:
        cb, _ = cpu_sample(p, seconds=args.cpu_seconds)
        line["cpu_baseline"] = cb
    print(json.dumps(line), flush=True)
    group.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
