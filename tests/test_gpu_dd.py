"""Domain-decomposed checking mode (single GPU).

The REANN-MPI paper's scheme ("Parallelization Algorithm", Figs. 3-4): each
subdomain keeps ghost copies of the atoms within the cutoff of its local atoms
and refreshes the ghosts' messages c^t once per message-passing layer.  Here
the subdomains live in one GPU and the refresh is an in-HBM gather.

  * with the refresh, every local atom sees the monolithic run's values in the
    monolithic order: energies and forces are bit-identical;
  * negative control (Fig. 3c): with stale ghost coefficients T = 1 still
    agrees (only c^0 enters) and T >= 2 does not;
  * ghost traffic per layer is fixed by the ghost count, so the bytes moved
    per evaluation grow linearly in T.
"""
import numpy as np
import pytest

from gpu_helpers import torch_cuda
from helpers import small
from molecular_dynamics_b200 import presets, reann, synth

pytestmark = pytest.mark.gpu


def _run(p, pos, types, box, T, dd_grid=(0, 0, 0), stale=0, mlp_precision=0):
    torch = torch_cuda()
    spec = reann.ModelSpec.from_preset(p, T=T, mlp_precision=mlp_precision, dd_grid=dd_grid, dd_stale_ghosts=stale)
    ctx = reann.Context(spec, synth.weight_blob(p, T=T))
    pos_d = torch.from_numpy(pos).cuda()
    ctx.reann_build_neighbors(pos_d, torch.from_numpy(types).cuda(), box)
    F = torch.empty_like(pos_d)
    Ei = torch.empty(len(pos), dtype=torch.float32, device="cuda")
    E = ctx.reann_energy_forces(pos_d, F, Ei)
    return ctx, E, F.cpu().numpy(), Ei.cpu().numpy()


def _ag(ncell):
    p = presets.scaled("ag1m", ncell=ncell)
    return (p, *synth.make_structure(p))


@pytest.mark.parametrize("T", [1, 2, 3, 5])
def test_dd_is_bit_identical_to_monolithic_ag(T):
    p, pos, types, box = _ag(8)
    _, E0, F0, Ei0 = _run(p, pos, types, box, T)
    ctx, E1, F1, Ei1 = _run(p, pos, types, box, T, dd_grid=(2, 2, 2))
    assert E1 == E0
    assert np.array_equal(F1, F0) and np.array_equal(Ei1, Ei0)
    cnt = ctx.reann_get_counters()
    assert cnt.ghost_slots > 0


@pytest.mark.parametrize("key,grid", [("chon", (2, 2, 2)), ("hea", (2, 1, 2)), ("water", (2, 2, 2))])
def test_dd_is_bit_identical_to_monolithic_other_workloads(key, grid):
    p, pos, types, box = small(key)
    _, E0, F0, Ei0 = _run(p, pos, types, box, p.T)
    _, E1, F1, Ei1 = _run(p, pos, types, box, p.T, dd_grid=grid)
    assert E1 == E0 and np.array_equal(F1, F0) and np.array_equal(Ei1, Ei0)


def test_dd_bf16_networks_bit_identical():
    p, pos, types, box = _ag(8)
    _, E0, F0, _ = _run(p, pos, types, box, 3, mlp_precision=1)
    _, E1, F1, _ = _run(p, pos, types, box, 3, dd_grid=(2, 2, 2), mlp_precision=1)
    assert E1 == E0 and np.array_equal(F1, F0)


@pytest.mark.parametrize("T", [1, 2, 3])
def test_negative_control_stale_ghosts(T):
    p, pos, types, box = _ag(8)
    _, E0, F0, _ = _run(p, pos, types, box, T)
    _, E1, F1, _ = _run(p, pos, types, box, T, dd_grid=(2, 2, 2), stale=1)
    if T == 1:
        assert E1 == E0 and np.array_equal(F1, F0)
    else:
        assert abs(E1 - E0) > 1e-6 * max(1.0, abs(E0))
        assert np.abs(F1 - F0).max() > 1e-4


def test_ghost_bytes_per_layer_and_linear_total():
    p, pos, types, box = _ag(8)
    per_T = []
    for T in (1, 2, 3, 4):
        ctx, _, _, _ = _run(p, pos, types, box, T, dd_grid=(2, 2, 2))
        c = ctx.reann_get_counters()
        assert c.ghost_bytes_fwd == c.ghost_slots * p.D * 4
        assert c.ghost_bytes_bwd == c.ghost_slots * p.n_radial * 10 * 4
        # forward: one message refresh per layer t >= 1; backward: one dE/dA refresh per layer
        per_T.append((T - 1) * c.ghost_bytes_fwd + T * c.ghost_bytes_bwd)
        ghosts = c.ghost_slots
    d = np.diff(per_T)
    assert np.all(d == d[0])          # linear in T
    # the ghost set does not depend on T (one neighbour list for all layers)
    assert ghosts > 0


def test_dd_md_steps_match_monolithic():
    torch = torch_cuda()
    p, pos, types, box = _ag(8)
    v0 = synth.maxwell_boltzmann(p, types)
    out = []
    for grid in ((0, 0, 0), (2, 2, 2)):
        spec = reann.ModelSpec.from_preset(p, mlp_precision=0, dd_grid=grid)
        ctx = reann.Context(spec, synth.weight_blob(p))
        ctx.reann_build_neighbors(pos, types, box)
        x = torch.from_numpy(pos.astype(np.float64)).cuda()
        v = torch.from_numpy(v0.copy()).cuda()
        st = ctx.reann_md_step(5, 1.0, x, v, p.masses)
        out.append((x.cpu().numpy(), v.cpu().numpy(), st.e_pot))
    assert np.array_equal(out[0][0], out[1][0]) and np.array_equal(out[0][1], out[1][1])
    assert out[0][2] == out[1][2]


def test_full_size_ag_8x8x8_bit_identical():
    # the 1M-atom workload with 512 subdomains of ~2,048 local atoms, bf16 networks
    p = presets.get("ag1m")
    pos, types, box = synth.make_structure(p)
    _, E0, F0, _ = _run(p, pos, types, box, p.T, mlp_precision=1)
    ctx, E1, F1, _ = _run(p, pos, types, box, p.T, dd_grid=(8, 8, 8), mlp_precision=1)
    assert E1 == E0 and np.array_equal(F1, F0)
    c = ctx.reann_get_counters()
    # a ~7 A halo around a 32.7 A cube holds ~3,900 ghosts per subdomain
    assert 1.5e6 < c.ghost_slots < 2.5e6
