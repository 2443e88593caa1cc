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
