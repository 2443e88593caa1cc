"""The seeded synthetic inputs follow their stated recipe (readings 9-10 of the
input recipe: Maxwell-Boltzmann velocities at the stated temperature with
3N - 3 degrees of freedom and no centre-of-mass motion; FCC lattices of the
stated constant).  The checks use their own constants (CODATA values, the
FCC shell structure), not the generator's."""
import numpy as np
import pytest

from molecular_dynamics_b200 import presets, synth

KB = 8.617333262e-5                                  # eV/K (CODATA 2018, exact by definition of the SI)
AMU_A2_FS2_IN_EV = 1.66053906660e-27 * 1e-20 / 1e-30 / 1.602176634e-19   # 1 amu A^2/fs^2 in eV


def _kinetic_temperature(v, m):
    ke = 0.5 * float((m[:, None] * v * v).sum()) * AMU_A2_FS2_IN_EV
    return 2.0 * ke / ((3 * len(m) - 3) * KB)


@pytest.mark.parametrize("key,kw", [("ag1m", {"ncell": 6}), ("water3k", {"n_mol": (300,), "box": 20.8})])
def test_maxwell_boltzmann_velocities(key, kw):
    p = presets.scaled(key, **kw)
    _, types, _ = synth.make_structure(p)
    m = np.asarray(p.masses, np.float64)[types]
    for T in (300.0, 450.0):
        v = synth.maxwell_boltzmann(p, types, temperature=T)
        assert v.shape == (len(types), 3) and v.dtype == np.float64
        # no centre-of-mass motion, and exactly the temperature with 3N - 3 degrees of freedom
        assert np.abs((m[:, None] * v).sum(0)).max() <= 1e-12 * float((m[:, None] * np.abs(v)).sum())
        assert abs(_kinetic_temperature(v, m) - T) <= 1e-9 * T
    # seeded: the same seed repeats, another differs
    a = synth.maxwell_boltzmann(p, types, seed=7)
    assert np.array_equal(a, synth.maxwell_boltzmann(p, types, seed=7))
    assert not np.array_equal(a, synth.maxwell_boltzmann(p, types, seed=8))


def test_velocity_spread_scales_with_inverse_mass():
    # equipartition per species: <m v_x^2> is the same kT for H and O (within sampling error)
    p = presets.scaled("water3k", n_mol=(2000,), box=39.1)
    _, types, _ = synth.make_structure(p)
    v = synth.maxwell_boltzmann(p, types, temperature=300.0)
    m = np.asarray(p.masses, np.float64)
    per = [float((m[e] * v[types == e] ** 2).mean()) * AMU_A2_FS2_IN_EV for e in range(p.n_elements)]
    for e, x in enumerate(per):
        n = int((types == e).sum()) * 3
        assert abs(x / (KB * 300.0) - 1.0) < 5.0 * np.sqrt(2.0 / n) + 2.0 / n, (e, x, n)


def test_fcc_lattice_shells():
    a, nc = 4.09, 4
    x = synth.fcc_lattice(nc, a)
    assert x.shape == (4 * nc ** 3, 3)
    L = nc * a
    d = x[None, :, :] - x[:, None, :]
    d -= L * np.rint(d / L)
    r = np.sqrt((d * d).sum(-1))
    np.fill_diagonal(r, np.inf)
    # every atom: 12 nearest neighbours at a / sqrt(2), 6 next at a, nothing closer
    assert np.allclose(r.min(1), a / np.sqrt(2.0), rtol=1e-12)
    assert (np.isclose(r, a / np.sqrt(2.0), rtol=1e-9).sum(1) == 12).all()
    assert (np.isclose(r, a, rtol=1e-9).sum(1) == 6).all()


def test_structures_are_wrapped_typed_and_seeded():
    for key, kw in (("ag1m", {"ncell": 5}), ("hea108k", {"ncell": 4}), ("water3k", {"n_mol": (100,), "box": 14.41})):
        p = presets.scaled(key, **kw)
        pos, types, box = synth.make_structure(p)
        assert pos.dtype == np.float32 and types.dtype == np.int32 and box.shape == (3,)
        assert (pos >= 0).all() and (pos < box.astype(np.float32)).all()
        assert types.min() >= 0 and types.max() < p.n_elements
        pos2, types2, _ = synth.make_structure(p)
        assert np.array_equal(pos, pos2) and np.array_equal(types, types2)
