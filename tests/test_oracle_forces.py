"""Pins of the oracle's energy and forces (REANN-MPI paper, section
"Parallelization Algorithm", Eqs. 3-5: F_k = -dE/dr_k through every
message-passing layer, with dc^0/dr = 0).

  * five-point central finite differences of the oracle's own energy;
  * zero net force; translation, cubic-group, SO(3) and permutation
    invariance of E (and the matching covariance of F);
  * two clusters farther apart than r_c: E(A u B) = E(A) + E(B);
  * T-hop receptive field: moving an atom more than T message-passing hops
    away leaves E_i bit-for-bit unchanged, and moving one exactly T hops away
    does change it (a skipped or extra layer fails);
  * perfect FCC: zero forces and equal atomic energies.
"""
import itertools

import numpy as np
import pytest

import oracle
from helpers import active_adjacency, fcc_perfect, graph_distance, model_for, small
from molecular_dynamics_b200 import presets, synth


def _fd(m, x, types, box, pairs, i, a, h=1e-4):
    """Five-point central difference of -E (truncation error O(h^4))."""
    def e(s):
        y = x.copy()
        y[i, a] += s
        return oracle.energy_forces(m, y, types, box, pairs, forces=False).energy
    return -(-e(2 * h) + 8 * e(h) - 8 * e(-h) + e(-2 * h)) / (12 * h)


@pytest.mark.parametrize("key,ncomp", [("ag256", 30), ("water", 30), ("hea", 30), ("chon", 30)])
def test_forces_match_central_differences(key, ncomp):
    p, pos, types, box = small(key)
    m = model_for(p)
    x = pos.astype(np.float64)
    pairs = oracle.pairs_brute(x, box, p.r_cut, p.skin)
    res = oracle.energy_forces(m, x, types, box, pairs)
    fscale = np.abs(res.forces).max()
    rng = np.random.default_rng(7)
    for _ in range(ncomp):
        i, a = int(rng.integers(len(x))), int(rng.integers(3))
        fd = _fd(m, x, types, box, pairs, i, a)
        assert abs(fd - res.forces[i, a]) <= 1e-6 * max(abs(fd), 1e-2 * fscale)


@pytest.mark.parametrize("key", ["ag256", "water", "hea", "chon"])
def test_zero_net_force(key):
    p, pos, types, box = small(key)
    res = oracle.energy_forces(model_for(p), pos, types, box)
    assert np.abs(res.forces.sum(0)).max() <= 1e-10 * len(pos) * max(1.0, np.abs(res.forces).max())


def test_translation_invariance():
    p, pos, types, box = small("water")
    m = model_for(p)
    a = oracle.energy_forces(m, pos, types, box)
    x2 = np.mod(pos.astype(np.float64) + np.array([3.3, -7.1, 12.9]), box)
    b = oracle.energy_forces(m, x2, types, box)
    assert b.energy == pytest.approx(a.energy, rel=1e-12)
    assert np.abs(b.forces - a.forces).max() <= 1e-10 * np.abs(a.forces).max()


def test_cubic_group_invariance_under_pbc():
    p, pos, types, box = small("hea")
    m = model_for(p)
    x = pos.astype(np.float64)
    ref = oracle.energy_forces(m, x, types, box)
    L = box[0]
    for perm in itertools.permutations(range(3)):
        for signs in itertools.product((1.0, -1.0), repeat=3):
            R = np.zeros((3, 3))
            for r, c in enumerate(perm):
                R[r, c] = signs[r]
            if perm == (0, 1, 2) and signs == (1.0, 1.0, 1.0):
                continue
            y = np.mod(x @ R.T, L)
            res = oracle.energy_forces(m, y, types, box)
            assert res.energy == pytest.approx(ref.energy, rel=1e-12)
            assert np.abs(res.forces - ref.forces @ R.T).max() <= 1e-10 * np.abs(ref.forces).max()


def test_so3_invariance_of_isolated_cluster():
    p = presets.get("water3k")
    m = model_for(p)
    rng = np.random.default_rng(3)
    # a 50-atom cluster of water-like geometry from the water recipe, centred in a padded box
    q, pos, types, box = small("water")
    x = pos.astype(np.float64)
    centre = x[0]
    d = x - centre
    d -= box * np.rint(d / box)
    sel = np.argsort((d * d).sum(1))[:50]
    cl = d[sel]
    ty = types[sel]
    L = 2 * (np.abs(cl).max() + p.r_cut + p.skin) + 1.0
    big = np.array([L, L, L])
    ref = oracle.energy_forces(m, cl + L / 2, ty, big)
    for _ in range(3):
        qv = rng.normal(size=4); qv /= np.linalg.norm(qv)
        w, a, b, c = qv
        R = np.array([[1 - 2 * (b * b + c * c), 2 * (a * b - w * c), 2 * (a * c + w * b)],
                      [2 * (a * b + w * c), 1 - 2 * (a * a + c * c), 2 * (b * c - w * a)],
                      [2 * (a * c - w * b), 2 * (b * c + w * a), 1 - 2 * (a * a + b * b)]])
        res = oracle.energy_forces(m, cl @ R.T + L / 2, ty, big)
        assert res.energy == pytest.approx(ref.energy, rel=1e-11)
        assert np.abs(res.forces - ref.forces @ R.T).max() <= 1e-9 * np.abs(ref.forces).max()


def test_permutation_invariance():
    p, pos, types, box = small("chon")
    m = model_for(p)
    ref = oracle.energy_forces(m, pos, types, box)
    perm = np.random.default_rng(5).permutation(len(pos))
    res = oracle.energy_forces(m, pos[perm], types[perm], box)
    assert res.energy == pytest.approx(ref.energy, rel=1e-12)
    assert np.abs(res.forces - ref.forces[perm]).max() <= 1e-10 * np.abs(ref.forces).max()
    assert np.abs(res.atom_energy - ref.atom_energy[perm]).max() <= 1e-12 * np.abs(ref.atom_energy).max()


def test_energy_additive_for_separated_clusters():
    p = presets.get("hea108k")
    m = model_for(p)
    q, pos, types, box = small("hea")
    x = pos.astype(np.float64)
    d = x - x[0]
    d -= box * np.rint(d / box)
    sel = np.argsort((d * d).sum(1))[:40]
    A, tA = d[sel], types[sel]
    B, tB = d[sel[::-1]] @ np.diag([1.0, -1.0, 1.0]), types[sel[::-1]]
    span = np.abs(A).max()
    L = 4 * span + 4 * (p.r_cut + p.skin)
    big = np.array([L, L, L])
    ea = oracle.energy_forces(m, A + L / 4, tA, big, forces=False).energy
    eb = oracle.energy_forces(m, B + 3 * L / 4, tB, big, forces=False).energy
    both = oracle.energy_forces(m, np.concatenate([A + L / 4, B + 3 * L / 4]), np.concatenate([tA, tB]), big,
                                forces=False).energy
    assert both == pytest.approx(ea + eb, rel=1e-13)


@pytest.mark.parametrize("T", [1, 2, 3])
def test_receptive_field_is_T_hops(T):
    # a sparse random gas so that graph distances span several hops
    p = presets.scaled("chon244k", n_mol=(320, 320, 16), box=40.0)
    pos, types, box = synth.make_structure(p)
    m = model_for(p, T=T)
    x = pos.astype(np.float64)
    adj, r = active_adjacency(x, box, p.r_cut)
    centre = 0
    hops = graph_distance(adj, centre)
    base = oracle.energy_forces(m, x, types, box, forces=False).atom_energy[centre]
    # choose movers whose small displacement does not change the active graph
    margin = np.min(np.abs(r - p.r_cut), axis=1)
    checked_far = checked_edge = 0
    for k in np.argsort(hops):
        if hops[k] == 0 or margin[k] < 1e-2:
            continue
        y = x.copy()
        y[k] += np.array([3e-3, -2e-3, 1e-3])
        e = oracle.energy_forces(m, y, types, box, forces=False).atom_energy[centre]
        if hops[k] > T or hops[k] < 0:
            assert e == base
            checked_far += 1
        elif hops[k] == T:
            assert e != base
            checked_edge += 1
        if checked_far >= 3 and checked_edge >= 3:
            break
    assert checked_far >= 3 and checked_edge >= 3


def test_perfect_fcc_zero_forces_equal_energies():
    p = presets.get("ag256")
    pos, box = fcc_perfect(4, 4.09)
    res = oracle.energy_forces(model_for(p), pos, np.zeros(len(pos), np.int32), box)
    assert np.abs(res.forces).max() <= 1e-10
    assert np.ptp(res.atom_energy) <= 1e-12 * np.abs(res.atom_energy).max()
