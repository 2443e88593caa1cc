"""Pins of the oracle's velocity-Verlet MD (the paper's production runs are
NVE/NVT MD driven by the REANN energy and forces; section "Strong Scaling"
mentions NVE energy conservation).

  * time reversal: k steps forward, negate v, k steps forward returns to the
    start (velocity Verlet is time-reversible);
  * second order: the NVE total-energy error over a fixed time shrinks about
    fourfold when dt is halved;
  * the first half-kick + drift agrees with x + v dt + F/(2m) dt^2.
"""
import numpy as np
import pytest

import oracle
from helpers import model_for, small
from molecular_dynamics_b200 import synth


def _setup():
    p, pos, types, box = small("water")
    m = model_for(p)
    v = synth.maxwell_boltzmann(p, types, temperature=100.0)
    return p, m, pos.astype(np.float64), v, types, box


def test_time_reversal():
    p, m, x0, v0, types, box = _setup()
    x1, v1, _, _ = oracle.md_verlet(m, x0, v0, types, box, p.masses, 0.25, 20)
    x2, v2, _, _ = oracle.md_verlet(m, x1, -v1, types, box, p.masses, 0.25, 20)
    d = x2 - x0
    d -= box * np.rint(d / box)
    assert np.abs(d).max() < 1e-8
    assert np.abs(v2 + v0).max() < 1e-8


def test_energy_error_is_second_order():
    p, m, x0, v0, types, box = _setup()
    errs = []
    for dt, n in ((0.2, 20), (0.1, 40)):
        _, _, ep, ek = oracle.md_verlet(m, x0, v0, types, box, p.masses, dt, n)
        et = ep + ek
        errs.append(np.abs(et - et[0]).max())
    ratio = errs[0] / errs[1]
    assert 3.0 < ratio < 5.0, ratio


def test_first_step_is_taylor_update():
    p, m, x0, v0, types, box = _setup()
    dt = 0.1
    f0 = oracle.energy_forces(m, x0, types, box).forces
    x1, _, _, _ = oracle.md_verlet(m, x0, v0, types, box, p.masses, dt, 1)
    acc = f0 / np.asarray(p.masses)[types][:, None] / synth.EV_PER_AMU_A2_FS2
    expect = np.mod(x0 + v0 * dt + 0.5 * acc * dt * dt, box)
    d = x1 - expect
    d -= box * np.rint(d / box)
    assert np.abs(d).max() < 1e-12


# ---------------------------------------------------------------------------
# NVT: stochastic velocity rescaling (Bussi, Donadio and Parrinello, J. Chem.
# Phys. 126, 014101 (2007)) with the per-step random numbers given as inputs.

def test_nvt_without_coupling_is_nve():
    # tau = infinity: c = 1, the rescaling factor is exactly 1 and the run is the
    # NVE run (to the oracle's run-to-run rounding: its threaded force sums are
    # reduced in schedule order)
    p, m, x0, v0, types, box = _setup()
    noise = synth.thermostat_noise(len(x0), 10, seed=5)
    xa, va, epa, eka = oracle.md_verlet(m, x0, v0, types, box, p.masses, 0.25, 10)
    xb, vb, epb, ekb, wk = oracle.md_nvt(m, x0, v0, types, box, p.masses, 0.25, 10, 300.0, np.inf, noise)
    assert np.abs(xa - xb).max() < 1e-12 and np.abs(va - vb).max() < 1e-12
    assert np.abs(epa - epb).max() < 1e-10 and np.abs(eka - ekb).max() < 1e-12
    assert np.all(wk == 0.0)


def test_nvt_effective_energy_is_conserved():
    # E_pot + E_kin minus the thermostat's accumulated work is conserved to the
    # integrator's own error (the NVE run with the same dt sets the scale)
    p, m, x0, v0, types, box = _setup()
    n = 80
    noise = synth.thermostat_noise(len(x0), n, seed=6)
    _, _, ep, ek, wk = oracle.md_nvt(m, x0, v0, types, box, p.masses, 0.2, n, 300.0, 20.0, noise)
    h = ep + ek - wk
    _, _, ep0, ek0 = oracle.md_verlet(m, x0, v0, types, box, p.masses, 0.2, n)
    nve = np.abs((ep0 + ek0) - (ep0[0] + ek0[0])).max()
    assert np.abs(h - h[0]).max() <= 3.0 * nve + 1e-9
    assert np.abs(wk).max() > 10.0 * nve           # the thermostat did work


def test_nvt_temperature_relaxes_to_target():
    p, pos, types, box = small("ag256")
    m = model_for(p)
    x0 = pos.astype(np.float64)
    v0 = synth.maxwell_boltzmann(p, types, temperature=300.0)
    n, target = 300, 600.0
    noise = synth.thermostat_noise(len(x0), n, seed=7)
    _, _, ep, ek, wk = oracle.md_nvt(m, x0, v0, types, box, p.masses, 1.0, n, target, 10.0, noise)
    nf = 3 * len(x0) - 3
    temp = 2.0 * ek / (nf * 8.617333262e-5)
    # kinetic temperature fluctuates by sqrt(2 / Nf) ~ 5 % per sample; over the
    # last half of the run its mean is within a few percent of the target
    assert abs(temp[n // 2:].mean() - target) < 0.1 * target, temp[n // 2:].mean()


def test_nvt_kinetic_energy_is_canonical():
    # the thermostat samples the canonical ensemble, where the kinetic energy
    # follows a Gamma distribution: mean Kt = Nf kB T / 2 and relative spread
    # sqrt(2 / Nf), whatever the potential.  Strong coupling (tau = dt) keeps
    # the correlation time to a few steps, so 800 samples after a 200-step
    # burn-in pin both moments; a wrong weight of either random term moves the
    # spread (halving the cross term gives ~0.77 of it)
    p, pos, types, box = small("ag256")
    m = model_for(p)
    x0 = pos.astype(np.float64)
    v0 = synth.maxwell_boltzmann(p, types, temperature=300.0)
    n = len(x0)
    nf = 3 * n - 3
    kt = 0.5 * nf * 8.617333262e-5 * 300.0
    noise = synth.thermostat_noise(n, 1000, seed=8)
    _, _, ep, ek, wk = oracle.md_nvt(m, x0, v0, types, box, p.masses, 1.0, 1000, 300.0, 1.0, noise)
    K = ek[200:]
    assert abs(K.mean() / kt - 1.0) < 0.01, K.mean() / kt
    ratio = K.std() / kt / np.sqrt(2.0 / nf)
    assert 0.85 < ratio < 1.15, ratio
