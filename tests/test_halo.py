"""The multi-process decomposition with the per-layer halo exchange
(molecular_dynamics_b200/halo.py; "Efficient Parallelization of Message
Passing Neural Network Potentials for Large-Scale Molecular Dynamics",
section "Parallelization Algorithm", Figs. 3-4), run as gloo ranks on the CPU
with an fp64 numpy stand-in for each process's library share
(tests/halo_engine.py): every rank evaluates its own atoms with ghosts, the
coefficient rows move forward and the gradient and force partials move back
once per layer, and the ranks together reproduce the single-process oracle's
total energy and every force.
"""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from molecular_dynamics_b200.halo import Grid, partition  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, dims, key, out):
    import torch.distributed as dist
    from halo_engine import NumpyHaloEngine
    from helpers import small
    from molecular_dynamics_b200 import synth
    from molecular_dynamics_b200.halo import HaloEvaluator, Transport
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        p, pos, types, box = small(key)
        grid = Grid(box, dims)
        own = partition(grid, pos, rank)
        eng = NumpyHaloEngine(p, synth.weight_blob(p))
        ev = HaloEvaluator(eng, grid, rank, p.r_cut + p.skin, Transport(rank, world, "gloo"))
        pos_own = torch.from_numpy(pos[own])
        ev.setup(pos_own, torch.from_numpy(types[own]))
        F = torch.zeros((len(own), 3), dtype=torch.float64)
        E = ev.energy_forces(pos_own, F)
        out.put((rank, E, own, F.numpy(), ev.plan.n_ghost, ev.plan.send_counts, ev.exchanges))
    finally:
        dist.destroy_process_group()


def _run(world, dims, key):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, dims, key, q)) for r in range(world)]
    for p in procs:
        p.start()
    rows = sorted([q.get(timeout=600) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return rows


@pytest.mark.parametrize("world,dims,key", [(2, (2, 1, 1), "water"), (3, (1, 3, 1), "hea"), (2, (1, 1, 2), "chon")])
def test_ranks_reproduce_the_single_process_result(world, dims, key):
    import oracle
    from helpers import model_for, small
    p, pos, types, box = small(key)
    ref = oracle.energy_forces(model_for(p), pos, types, box)
    rows = _run(world, dims, key)
    owned = np.concatenate([r[2] for r in rows])
    assert np.array_equal(np.sort(owned), np.arange(len(pos)))        # every atom has exactly one owner
    for rank, E, own, F, n_ghost, send_counts, exchanges in rows:
        assert E == pytest.approx(ref.energy, rel=1e-12, abs=1e-12)  # every rank sees the total
        assert np.abs(F - ref.forces[own]).max() <= 1e-10 * max(1.0, np.abs(ref.forces).max())
        assert n_ghost > 0 and sum(send_counts) > 0
        assert exchanges == 2 * (p.T - 1) + 1                           # c^t forward, dE/dc^t back, forces back


def test_grid_geometry():
    g = Grid([10.0, 20.0, 30.0], (2, 1, 3))
    assert g.size == 6
    pts = np.array([[0.5, 1.0, 1.0], [9.9, 19.0, 29.0], [5.0, 0.0, 10.0], [-0.1, 0.0, 0.0]])
    assert list(g.owner(pts)) == [0, 5, 4, 3]
    # periodic distance to region 0 ([0,5) x [0,20) x [0,10)): inside, across the x wrap, beyond z
    d2 = g.distance2(np.array([[1.0, 1.0, 1.0], [9.5, 1.0, 1.0], [1.0, 1.0, 12.0]]), 0)
    assert d2 == pytest.approx([0.0, 0.25, 4.0])
