"""The pair-product density variant on the GPU (density_form = 1) against the
oracle: rho_(n,m,l) = sum_tau w_tau A_{n,tau} A_{m,tau} for n <= m, the density
dimension N_phi (N_phi+1)(L+1)/2 of section "REANN Architecture" of
"Efficient Parallelization of Message Passing Neural Network Potentials for
Large-Scale Molecular Dynamics".  Forces and atomic energies have the square
form's tolerances (fp32 networks).  The total energy per atom is held to
1e-5 of max(|E|/N, 0.1 eV): the synthetic weights scale forces to 1 eV/A RMS,
which makes 0.1 eV (1 eV/A x 0.1 A) the potential's natural per-atom energy
unit, while |E|/N itself is set by the arbitrary output bias and can sit near
zero; the coherent fp32 rounding of the 108 features of a crystal's
near-identical atoms leaves a bias of ~2e-7 eV/atom.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import E_TOL, F_TOL, assert_forces_close, cluster_around, gpu_eval, oracle_eval, torch_cuda
from helpers import model_for, small
from molecular_dynamics_b200 import presets, reann, synth

pytestmark = pytest.mark.gpu


def _energy_close(E, E_ref, n):
    tol = E_TOL[0] * max(abs(E_ref) / n, 0.1)
    assert abs(E - E_ref) / n <= tol, (E, E_ref, abs(E - E_ref) / n, tol)


def _atoms_close(Ei, Ei_ref):
    # worst atom against the same per-atom energy unit
    scale = max(float(np.sqrt(np.mean(Ei_ref ** 2))), 0.1)
    err = np.abs(Ei - Ei_ref).max() / scale
    assert err <= 10 * E_TOL[0], err


def test_pair_small_full_parity_and_features():
    p, pos, types, box = small("agp")
    ctx, E, F, Ei = gpu_eval(p, pos, types, box)
    ref = oracle_eval(p, pos, types, box, intermediates=True)
    n = len(pos)
    _energy_close(E, ref.energy, n)
    _atoms_close(Ei, ref.atom_energy)
    assert_forces_close(F, ref.forces)
    for t in range(p.T):
        rho, coef = ctx.reann_get_features(t)
        assert rho.shape == (n, 108)
        # fp32 features against fp64: relative to each layer's feature scale
        assert np.abs(rho - ref.rho[t]).max() <= 1e-5 * np.abs(ref.rho[t]).max()
        assert np.abs(coef - ref.coef[t]).max() <= 1e-4 * max(np.abs(ref.coef[t]).max(), 1.0)


def test_pair_larger_lattice_parity():
    # several tiles of 32 rows and a ragged tail (2,048 atoms = 64 tiles; 1,372 atoms ragged)
    for ncell in (8, 7):
        p = presets.scaled("ag1mp", ncell=ncell)
        pos, types, box = synth.make_structure(p)
        _, E, F, Ei = gpu_eval(p, pos, types, box)
        ref = oracle_eval(p, pos, types, box)
        _energy_close(E, ref.energy, len(pos))
        _atoms_close(Ei, ref.atom_energy)
        assert_forces_close(F, ref.forces)


@pytest.mark.parametrize("ncell", [8, 7])
def test_pair_tensor_core_networks_parity(ncell):
    # bf16 tensor-core networks (split activations, bf16-valued weights): the
    # bf16 force tolerance; tiles of 128 rows, ragged at 1,372 atoms
    p = presets.scaled("ag1mp", ncell=ncell)
    pos, types, box = synth.make_structure(p)
    _, E, F, Ei = gpu_eval(p, pos, types, box, mlp_precision=1)
    ref = oracle_eval(p, pos, types, box)
    _energy_close(E, ref.energy, len(pos))
    _atoms_close(Ei, ref.atom_energy)
    assert_forces_close(F, ref.forces, 1)


def test_pair_domain_decomposed_bit_identical():
    torch = torch_cuda()
    p = presets.scaled("ag1mp", ncell=8)
    pos, types, box = synth.make_structure(p)
    out = []
    for grid in ((0, 0, 0), (2, 2, 2)):
        spec = reann.ModelSpec.from_preset(p, dd_grid=grid)
        ctx = reann.Context(spec, synth.weight_blob(p))
        pos_d = torch.from_numpy(pos).cuda()
        ctx.reann_build_neighbors(pos_d, torch.from_numpy(types).cuda(), box)
        Fd = torch.empty_like(pos_d)
        out.append((ctx.reann_energy_forces(pos_d, Fd), Fd.cpu().numpy()))
    assert out[0][0] == out[1][0] and np.array_equal(out[0][1], out[1][1])


def test_pair_md_anchored_steps():
    torch = torch_cuda()
    p, pos, types, box = small("agp")
    v0 = synth.maxwell_boltzmann(p, types)
    x0 = pos.astype(np.float64)
    ctx = reann.Context(reann.ModelSpec.from_preset(p), synth.weight_blob(p))
    ctx.reann_build_neighbors(pos, types, box)
    x = torch.from_numpy(x0.copy()).cuda()
    v = torch.from_numpy(v0.copy()).cuda()
    st = ctx.reann_md_step(10, 1.0, x, v, p.masses)
    xo, vo, ep, ek = oracle.md_verlet(model_for(p), x0, v0, types, box, p.masses, 1.0, 10)
    d = x.cpu().numpy() - xo
    d -= box * np.rint(d / box)
    assert np.abs(d).max() < 1e-4
    assert np.abs(v.cpu().numpy() - vo).max() < 1e-5
    assert abs(st.e_pot - ep[-1]) / len(pos) < 1e-5


@pytest.mark.parametrize("prec", [1, 0])
def test_pair_full_size_sampled(prec):
    # the 1M-atom pair workload (its bf16 tensor-core networks, and fp32 ones):
    # sampled forces and atomic energies against the oracle on the cluster of
    # every atom within 2 T r_c; zero net force
    p = presets.get("ag1mp")
    pos, types, box = synth.make_structure(p)
    n = len(pos)
    w = synth.weight_blob(p)
    _, E, F, Ei = gpu_eval(p, pos, types, box, weights=w, mlp_precision=prec)
    assert np.abs(F.sum(0)).max() <= 1e-4 * np.sqrt(n) + 1e-3
    assert abs(Ei.sum() - E) <= 1e-6 * n + 1e-4 * abs(E)
    radius = 2 * p.T * p.r_cut + 0.5
    rng = np.random.default_rng(1007)
    for k in rng.choice(n, size=3, replace=False):
        cpos, ctypes_, cbox, _ = cluster_around(pos, types, box, k, radius)
        ref = oracle_eval(p, cpos, ctypes_, cbox, weights=w)
        assert np.abs(F[k] - ref.forces[0]).max() <= F_TOL[prec], (k, F[k], ref.forces[0])
        rel = abs(Ei[k] - ref.atom_energy[0]) / max(float(np.sqrt(np.mean(Ei ** 2))), 0.1)
        assert rel <= 10 * E_TOL[prec], (k, Ei[k], ref.atom_energy[0])


def test_pair_form_rejects_unsupported_configs():
    p = presets.get("ag256p")
    for spec in (reann.ModelSpec.from_preset(p.with_(hidden=(64, 128))),
                 reann.ModelSpec.from_preset(p.with_(n_radial=10))):
        with pytest.raises(reann.ReannError):
            reann.Context(spec, np.zeros(10, np.float32))
