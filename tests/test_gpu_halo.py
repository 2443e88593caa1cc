"""The library's share of a multi-process decomposition
(reann_halo_plan / reann_energy_forces_halo) driven by
molecular_dynamics_b200/halo.py: ranks as separate processes with gloo
messages staged through host memory (every process uses cuda:0 here; no
kernel waits on another process -- the rows move between calls on the host).
Their total energy and every force meet the oracle tolerances of the
single-process path.
"""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, dims, key, out):
    import torch
    import torch.distributed as dist
    from helpers import small
    from molecular_dynamics_b200 import presets, reann, synth
    from molecular_dynamics_b200.halo import Grid, HaloEvaluator, Transport, partition
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        if key == "hea1372":
            p = presets.scaled("hea108k", ncell=7)
            pos, types, box = synth.make_structure(p)
        else:
            p, pos, types, box = small(key)
        grid = Grid(box, dims)
        own = partition(grid, pos, rank)
        ctx = reann.Context(reann.ModelSpec.from_preset(p), synth.weight_blob(p))
        ev = HaloEvaluator(ctx, grid, rank, p.r_cut + p.skin, Transport(rank, world, "gloo"))
        pos_own = torch.from_numpy(pos[own]).cuda()
        ev.setup(pos_own, torch.from_numpy(types[own]).cuda())
        F = torch.zeros((len(own), 3), dtype=torch.float32, device="cuda")
        E = ev.energy_forces(pos_own, F)
        cnt = ctx.reann_get_counters()
        out.put((rank, E, own, F.cpu().numpy().astype(np.float64), cnt.ghost_slots, cnt.ghost_bytes_fwd,
                 cnt.ghost_bytes_bwd, ev.exchanges))
        ctx.close()
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
        p.join(timeout=120)
        assert p.exitcode == 0
    return rows


@pytest.mark.parametrize("world,dims,key", [(2, (2, 1, 1), "hea1372"), (2, (1, 2, 1), "chon"), (3, (3, 1, 1), "water")])
def test_library_ranks_match_oracle(world, dims, key):
    from gpu_helpers import E_TOL, F_TOL, oracle_eval
    from helpers import small
    from molecular_dynamics_b200 import presets, synth
    if key == "hea1372":
        p = presets.scaled("hea108k", ncell=7)
        pos, types, box = synth.make_structure(p)
    else:
        p, pos, types, box = small(key)
    ref = oracle_eval(p, pos, types, box)
    n = len(pos)
    rows = _run(world, dims, key)
    owned = np.concatenate([r[2] for r in rows])
    assert np.array_equal(np.sort(owned), np.arange(n))
    for rank, E, own, F, ghosts, bfwd, bbwd, exchanges in rows:
        assert abs(E - ref.energy) / n <= E_TOL[0] * max(abs(ref.energy) / n, 1e-2), (E, ref.energy)
        assert np.abs(F - ref.forces[own]).max() <= F_TOL[0], np.abs(F - ref.forces[own]).max()
        assert ghosts > 0 and bfwd > 0 and bbwd == ghosts * p.D * 4
        assert exchanges == 2 * (p.T - 1) + 1
