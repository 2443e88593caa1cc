"""The stored weight-recipe data: standardisation conditioning, energy scale,
and determinism of the seeded draws."""
import numpy as np
import pytest

from molecular_dynamics_b200 import presets, synth


@pytest.mark.parametrize("key", presets.ORDER)
def test_standardisation_is_well_conditioned(key):
    p = presets.get(key)
    shift, scale = synth.load_norm(p)
    assert shift.shape == (p.stats_depth, p.n_elements, p.D)
    assert np.all(scale > 0)
    # the recipe's floor bounds mean / scale by 20 (1 / 0.05)
    assert np.all(np.abs(shift) / scale <= 20.0 + 1e-3)


@pytest.mark.parametrize("key", presets.ORDER)
def test_energy_scale_present_and_signed(key):
    p = presets.get(key)
    lam = synth.load_energy_scale(p)
    assert 0 < abs(lam) < 10
    if p.kind != "fcc":
        assert lam > 0


def test_crystal_lies_below_its_thermal_structure():
    # the sign of the energy scale makes the perfect lattice the lower-energy
    # structure, so an MD run of the crystal stays in its basin
    import oracle
    p = presets.get("ag256")
    model = oracle.Model.from_preset(p, synth.weight_blob(p))
    e = []
    for q in (p, p.with_(sigma=0.0)):
        pos, types, box = synth.make_structure(q)
        e.append(oracle.energy_forces(model, pos, types, box, forces=False).energy / len(pos))
    assert e[0] > e[1] + 1e-3


def test_weight_blob_is_deterministic_and_sized():
    p = presets.get("hea108k")
    a, b = synth.weight_blob(p), synth.weight_blob(p)
    assert a.dtype == np.float32 and np.array_equal(a, b)
    assert len(a) == synth.blob_layout(p, p.T)["total"]


def test_energy_scale_multiplies_only_the_energy_output_layer():
    p = presets.get("water3k")
    a = synth.weight_blob(p, energy_scale=1.0)
    b = synth.weight_blob(p, energy_scale=2.0)
    lay = synth.blob_layout(p, p.T)
    diff = np.nonzero(a != b)[0]
    allowed = set()
    for net in lay["energy"]:
        for k in ("W3", "b3"):
            o, shape = net[k]
            allowed.update(range(o, o + int(np.prod(shape))))
    assert set(diff.tolist()) <= allowed
    for net in lay["energy"]:
        o, shape = net["W3"]
        m = int(np.prod(shape))
        assert np.allclose(b[o:o + m], 2 * a[o:o + m])


def test_thermostat_noise_has_the_stated_distributions():
    # R1 standard normal, S chi-squared with Nf - 1 = 3 n - 4 degrees of
    # freedom; seeded, so both sides of a parity test read the same numbers
    n, steps = 256, 20000
    z = synth.thermostat_noise(n, steps, seed=3)
    assert z.shape == (steps, 2)
    assert np.array_equal(z, synth.thermostat_noise(n, steps, seed=3))
    r1, s = z[:, 0], z[:, 1]
    k = 3 * n - 4
    assert abs(r1.mean()) < 4 / np.sqrt(steps) and abs(r1.std() - 1.0) < 0.02
    assert abs(s.mean() / k - 1.0) < 4 * np.sqrt(2.0 / k / steps)
    assert abs(s.var() / (2.0 * k) - 1.0) < 0.05
    assert np.all(s > 0)
