"""Pins of the oracle's embedded atom density (REANN-MPI paper, section
"REANN Architecture", Eq. 1) and of its network/feature layout.

  * multinomial theorem: sum_{|tau|=l} l!/tau! Y_tau(a) Y_tau(b) = (a.b)^l, so
    rho_{i,(n,l)} = sum_{j,k} a_j a_k (d_ij . d_ik)^l -- a second formula with
    no Cartesian tuples (oracle_rho_pairwise), compared layer by layer;
  * dimer closed form: one neighbour at distance r gives
    rho_{(n,l)} = (c_{(n,l)} phi_n(r))^2 r^(2l), with a distinct random c per
    feature so that a wrong feature index fails;
  * perfect FCC: inversion symmetry makes every l = 1 feature vanish;
  * T = 1 reduces REANN to the local EANN model (same section): the energy of
    a dimer equals the atomic network applied to the closed-form densities.
"""
import math

import numpy as np
import pytest

import oracle
from helpers import fcc_perfect, model_for, small
from molecular_dynamics_b200 import presets, synth


def _phi(r, n, p):
    mu = p.r_cut * n / (p.n_radial - 1)
    return math.exp(-p.alpha * (r - mu) ** 2) * 0.5 * (math.cos(math.pi * r / p.r_cut) + 1.0)


@pytest.mark.parametrize("key", ["ag256", "water", "hea", "chon"])
def test_density_matches_multinomial_formula_every_layer(key):
    p, pos, types, box = small(key)
    m = model_for(p)
    pairs = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    res = oracle.energy_forces(m, pos, types, box, pairs, forces=False, intermediates=True)
    for t in range(p.T):
        rho2 = oracle.rho_pairwise(m, pos, box, res.coef[t], pairs)
        scale = np.abs(res.rho[t]).max()
        assert np.abs(rho2 - res.rho[t]).max() <= 1e-11 * scale


@pytest.mark.parametrize("r", [1.3, 2.9, 4.4, 5.95])
def test_dimer_closed_form(r):
    p = presets.get("water3k")          # two elements, so c differs per species
    blob = synth.weight_blob(p, T=1)
    m = oracle.Model.from_preset(p, blob, T=1)
    C0 = blob[:p.n_elements * p.D].reshape(p.n_elements, p.D).astype(np.float64)
    d = np.array([0.3, -0.5, 0.8])
    d = d / np.linalg.norm(d) * r
    x = np.array([[10.0, 10.0, 10.0], [10.0, 10.0, 10.0] + d])
    types = np.array([0, 1], np.int32)
    box = np.array([30.0, 30.0, 30.0])
    res = oracle.energy_forces(m, x, types, box, forces=False, intermediates=True)
    rho = res.rho[0]
    for i, j in ((0, 1), (1, 0)):
        for l in range(p.l_max + 1):
            for n in range(p.n_radial):
                f = l * p.n_radial + n
                expect = (C0[types[j], f] * _phi(r, n, p)) ** 2 * r ** (2 * l)
                assert rho[i, f] == pytest.approx(expect, rel=1e-12, abs=1e-300)


def test_perfect_fcc_has_no_l1_density():
    p = presets.get("ag256")
    pos, box = fcc_perfect(4, 4.09)
    types = np.zeros(len(pos), np.int32)
    m = model_for(p)
    res = oracle.energy_forces(m, pos, types, box, forces=False, intermediates=True)
    NP = p.n_radial
    for t in range(p.T):
        l1 = res.rho[t][:, NP:2 * NP]
        assert np.abs(l1).max() <= 1e-12 * np.abs(res.rho[t]).max()


def test_t1_energy_is_the_local_eann_network_on_closed_form_density():
    p = presets.get("water3k")
    blob = synth.weight_blob(p, T=1)
    m = oracle.Model.from_preset(p, blob, T=1)
    lay = synth.blob_layout(p, 1)
    C0 = blob[:p.n_elements * p.D].reshape(p.n_elements, p.D).astype(np.float64)
    r = 2.37
    d = np.array([0.6, 0.64, -0.48]) * r
    x = np.array([[5.0, 5.0, 5.0], [5.0, 5.0, 5.0] + d])
    types = np.array([1, 0], np.int32)
    box = np.array([20.0, 20.0, 20.0])
    res = oracle.energy_forces(m, x, types, box, forces=False)

    def net(e, rho):
        g = lambda k: blob[lay["energy"][e][k][0]:lay["energy"][e][k][0] + int(np.prod(lay["energy"][e][k][1]))] \
            .reshape(lay["energy"][e][k][1]).astype(np.float64)
        xt = (rho - g("shift")) / g("scale")
        a1 = np.tanh(g("W1") @ xt + g("b1"))
        a2 = np.tanh(g("W2") @ a1 + g("b2"))
        return float((g("W3") @ a2 + g("b3"))[0])

    expect = 0.0
    for i, j in ((0, 1), (1, 0)):
        rho = np.array([(C0[types[j], l * p.n_radial + n] * _phi(r, n, p)) ** 2 * r ** (2 * l)
                        for l in range(p.l_max + 1) for n in range(p.n_radial)])
        e = net(types[i], rho)
        assert res.atom_energy[i] == pytest.approx(e, rel=1e-12)
        expect += e
    assert res.energy == pytest.approx(expect, rel=1e-12)


def _blob_net(blob, spec):
    """One network of the weight blob as a numpy function (row-major W, output
    index first; input standardised as (x - shift) / scale)."""
    g = lambda k: blob[spec[k][0]:spec[k][0] + int(np.prod(spec[k][1]))].reshape(spec[k][1]).astype(np.float64)

    def f(x):
        a1 = np.tanh(g("W1") @ ((x - g("shift")) / g("scale")) + g("b1"))
        a2 = np.tanh(g("W2") @ a1 + g("b2"))
        return g("W3") @ a2 + g("b3")
    return f


@pytest.mark.parametrize("T", [2, 3])
@pytest.mark.parametrize("types", [(0, 1), (1, 0)])
def test_message_passing_dimer_chain(T, types):
    """Eq. 2 (section "REANN Architecture"): c^{t+1}_i = M^t_{Z_i}(rho^t_i), one
    network per layer t and per element of the centre atom.  For a hetero
    dimer every layer's density has the closed form
    rho^t_{i,(n,l)} = (c^t_{j,(n,l)} phi_n(r))^2 r^(2l) of the partner j, so the
    whole chain c^0 -> rho^0 -> c^1 -> ... -> rho^{T-1} -> E_i is written out
    here with the networks read straight from the blob.  Using the networks
    in another layer order, or the partner's element (or one element for
    every atom), changes E_i."""
    p = presets.get("water3k")
    blob = synth.weight_blob(p, T=T)
    lay = synth.blob_layout(p, T)
    m = oracle.Model.from_preset(p, blob, T=T)
    NP, L = p.n_radial, p.l_max
    C0 = blob[:p.n_elements * p.D].reshape(p.n_elements, p.D).astype(np.float64)
    r = 2.61
    d = np.array([-0.36, 0.48, 0.8]) * r
    x = np.array([[7.0, 7.0, 7.0], [7.0, 7.0, 7.0] + d])
    z = np.array(types, np.int32)
    box = np.array([22.0, 22.0, 22.0])
    res = oracle.energy_forces(m, x, z, box, forces=False, intermediates=True)

    shape = np.array([_phi(r, n, p) ** 2 * r ** (2 * l) for l in range(L + 1) for n in range(NP)])
    c = [C0[z[0]], C0[z[1]]]
    for t in range(T):
        rho = [c[1] ** 2 * shape, c[0] ** 2 * shape]          # each atom's density from its partner
        for i in range(2):
            assert res.rho[t][i] == pytest.approx(rho[i], rel=1e-12, abs=1e-300)
        if t + 1 < T:
            c = [_blob_net(blob, lay["coef"][t][z[i]])(rho[i]) for i in range(2)]
            for i in range(2):
                assert res.coef[t + 1][i] == pytest.approx(c[i], rel=1e-12, abs=1e-14)
    e = [float(_blob_net(blob, lay["energy"][z[i]])(rho[i])[0]) for i in range(2)]
    for i in range(2):
        assert res.atom_energy[i] == pytest.approx(e[i], rel=1e-12)
    assert res.energy == pytest.approx(e[0] + e[1], rel=1e-12)
