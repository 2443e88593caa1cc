"""The oracle's pair-product density variant, pinned without its own code.

"Efficient Parallelization of Message Passing Neural Network Potentials for
Large-Scale Molecular Dynamics", section "REANN Architecture", gives the
density vector the dimension N_phi (N_phi+1)(L+1)/2; the variant reads it as
rho_{(n,m),l} = sum_{|tau|=l} l!/tau! A_{n,tau} A_{m,tau} for n <= m.  Pins:

  * a second formula with no Cartesian tuples (multinomial theorem):
    rho_{(n,m),l} = sum_{j,k} a_{j,n} a_{k,m} (d_ij . d_ik)^l, every layer;
  * its diagonal n = m is the square form of Eq. 1 (same coefficients);
  * a dimer: rho_{(n,m),l} = c_{n,l} c_{m,l} phi_n(r) phi_m(r) r^{2l};
  * forces are minus the gradient of the energy (central differences) and
    sum to zero.
"""
import math

import numpy as np
import pytest

import oracle
from helpers import model_for, small
from molecular_dynamics_b200 import presets, synth


def _phi(r, n, p):
    mu = p.r_cut * n / (p.n_radial - 1)
    return math.exp(-p.alpha * (r - mu) ** 2) * 0.5 * (math.cos(math.pi * r / p.r_cut) + 1.0)


def _pair(NP, n, m):
    # n <= m, row-major over the upper triangle
    return n * NP - n * (n - 1) // 2 + (m - n)


def test_pair_density_matches_pairwise_formula_every_layer():
    p, pos, types, box = small("agp")
    m = model_for(p)
    pairs = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    res = oracle.energy_forces(m, pos, types, box, pairs, forces=False, intermediates=True)
    assert res.rho.shape == (p.T, len(pos), 108)
    for t in range(p.T):
        rho2 = oracle.rho_pairwise(m, pos, box, res.coef[t], pairs)
        assert np.abs(rho2 - res.rho[t]).max() <= 1e-11 * np.abs(res.rho[t]).max()


def test_pair_diagonal_is_the_square_form():
    p, pos, types, box = small("agp")
    sq = p.with_(density_form=0)
    pairs = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    # layer 0 uses the element table c^0, drawn identically for both forms
    mp = oracle.Model.from_preset(p, synth.weight_blob(p, T=1, use_stored_norm=False), T=1)
    ms = oracle.Model.from_preset(sq, synth.weight_blob(sq, T=1, use_stored_norm=False), T=1)
    rp = oracle.energy_forces(mp, pos, types, box, pairs, forces=False, intermediates=True).rho[0]
    rs = oracle.energy_forces(ms, pos, types, box, pairs, forces=False, intermediates=True).rho[0]
    NP, P = p.n_radial, p.n_radial * (p.n_radial + 1) // 2
    for l in range(p.l_max + 1):
        for n in range(NP):
            assert np.array_equal(rp[:, l * P + _pair(NP, n, n)], rs[:, l * NP + n])


@pytest.mark.parametrize("r", [1.7, 3.1, 5.6])
def test_pair_dimer_closed_form(r):
    p = presets.get("ag256p")
    blob = synth.weight_blob(p, T=1, use_stored_norm=False)
    m = oracle.Model.from_preset(p, blob, T=1)
    C0 = blob[:p.D].astype(np.float64)
    d = np.array([0.6, 0.2, -0.77])
    d = d / np.linalg.norm(d) * r
    x = np.array([[10.0, 10.0, 10.0], [10.0, 10.0, 10.0] + d])
    types = np.array([0, 0], np.int32)
    box = np.array([30.0, 30.0, 30.0])
    rho = oracle.energy_forces(m, x, types, box, forces=False, intermediates=True).rho[0]
    NP, P = p.n_radial, p.n_radial * (p.n_radial + 1) // 2
    for l in range(p.l_max + 1):
        for n in range(NP):
            for k in range(n, NP):
                expect = C0[l * NP + n] * C0[l * NP + k] * _phi(r, n, p) * _phi(r, k, p) * r ** (2 * l)
                got = rho[0, l * P + _pair(NP, n, k)]
                assert got == pytest.approx(expect, rel=1e-12, abs=1e-300)


def test_pair_forces_match_central_differences():
    p, pos, types, box = small("agp")
    m = model_for(p)
    x = pos.astype(np.float64)
    pairs = oracle.pairs_brute(x, box, p.r_cut, p.skin)
    res = oracle.energy_forces(m, x, types, box, pairs)
    fscale = np.abs(res.forces).max()
    assert np.abs(res.forces.sum(0)).max() <= 1e-10 * len(x) * fscale
    rng = np.random.default_rng(11)
    h = 1e-4
    for _ in range(30):
        i, a = int(rng.integers(len(x))), int(rng.integers(3))

        def e(s):
            y = x.copy()
            y[i, a] += s
            return oracle.energy_forces(m, y, types, box, pairs, forces=False).energy

        fd = -(-e(2 * h) + 8 * e(h) - 8 * e(-h) + e(-2 * h)) / (12 * h)
        assert abs(fd - res.forces[i, a]) <= 1e-6 * max(abs(fd), 1e-2 * fscale)
