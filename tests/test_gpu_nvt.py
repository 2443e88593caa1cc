"""Canonical (NVT) MD on the GPU through reann_md_step_nvt: velocity Verlet
with stochastic velocity rescaling (Bussi, Donadio and Parrinello 2007), the
ensemble of the capsid run on the Tessera page (abstract).  The per-step
random numbers are inputs, so both sides take the same steps.

  * anchored parity with the oracle's md_nvt: positions, velocities, energies
    and the thermostat's work after a few coupled steps;
  * tau = 0 draws the kinetic energy afresh: K' = Kt (R1^2 + S) / Nf exactly;
  * tau = +inf is the NVE step bit for bit, with zero work;
  * the effective energy E_pot + E_kin - W is conserved;
  * a split call equals one call (continuation with the noise split);
  * invalid thermostat arguments are rejected;
  * the domain-decomposed checking mode runs the same NVT trajectory bit for bit;
  * at strong coupling the kinetic energy has the canonical moments.
"""
import ctypes as C

import numpy as np
import pytest

import oracle
from gpu_helpers import torch_cuda
from helpers import model_for, small
from molecular_dynamics_b200 import reann, synth

pytestmark = pytest.mark.gpu

KB = 8.617333262e-5


def _ctx(p, pos, types, box):
    ctx = reann.Context(reann.ModelSpec.from_preset(p, mlp_precision=0), synth.weight_blob(p))
    ctx.reann_build_neighbors(pos, types, box)
    return ctx


def _state(p, pos, types):
    torch = torch_cuda()
    x0 = pos.astype(np.float64)
    v0 = synth.maxwell_boltzmann(p, types)
    return x0, v0, torch.from_numpy(x0.copy()).cuda(), torch.from_numpy(v0.copy()).cuda()


def test_anchored_nvt_steps_match_oracle():
    p, pos, types, box = small("water")
    x0, v0, x, v = _state(p, pos, types)
    n = len(pos)
    noise = synth.thermostat_noise(n, 10, seed=11)
    ctx = _ctx(p, pos, types, box)
    st = ctx.reann_md_step_nvt(10, 0.5, 450.0, 5.0, noise, x, v, p.masses)
    assert st.steps == 10
    xo, vo, ep, ek, wk = oracle.md_nvt(model_for(p), x0, v0, types, box, p.masses, 0.5, 10, 450.0, 5.0, noise)
    d = x.cpu().numpy() - xo
    d -= box * np.rint(d / box)
    assert np.abs(d).max() < 1e-4
    assert np.abs(v.cpu().numpy() - vo).max() < 1e-5
    assert abs(st.e_pot - ep[-1]) / n < 1e-5
    assert abs(st.e_kin - ek[-1]) / n < 1e-5
    assert abs(st.e_thermostat - wk[-1]) / n < 1e-5
    # the coupling did something measurable at this tau
    assert abs(wk[-1]) / n > 1e-4


def test_full_resampling_sets_the_kinetic_energy():
    p, pos, types, box = small("water")
    _, _, x, v = _state(p, pos, types)
    n = len(pos)
    ctx = _ctx(p, pos, types, box)
    nf = 3 * n - 3
    kt = 0.5 * nf * KB * 300.0
    for seed in (1, 2, 3):
        noise = synth.thermostat_noise(n, 1, seed=seed)
        st = ctx.reann_md_step_nvt(1, 0.5, 300.0, 0.0, noise, x, v, p.masses)
        r1, s = noise[0]
        target = kt * (r1 * r1 + s) / nf
        # the device-side sum of m v^2 / 2 after scaling, against the exact target
        assert st.e_kin == pytest.approx(target, rel=1e-12)


def test_infinite_tau_is_the_nve_step():
    p, pos, types, box = small("water")
    _, _, x, v = _state(p, pos, types)
    x2, v2 = x.clone(), v.clone()
    noise = synth.thermostat_noise(len(pos), 20, seed=4)
    st = _ctx(p, pos, types, box).reann_md_step_nvt(20, 0.5, 300.0, np.inf, noise, x, v, p.masses)
    st2 = _ctx(p, pos, types, box).reann_md_step(20, 0.5, x2, v2, p.masses)
    assert st.e_thermostat == 0.0
    assert st.e_pot == st2.e_pot and st.e_kin == st2.e_kin
    assert bool((x == x2).all()) and bool((v == v2).all())


def test_effective_energy_is_conserved():
    # 400 steps of 0.25 fs with tau = 20 fs: E_pot + E_kin - W stays within a
    # few times the NVE run's own fluctuation while W itself moves far more
    p, pos, types, box = small("water")
    n = len(pos)
    _, _, x, v = _state(p, pos, types)
    x2, v2 = x.clone(), v.clone()
    noise = synth.thermostat_noise(n, 400, seed=9)
    ctx = _ctx(p, pos, types, box)
    h_nvt, h_nve, work = [], [], []
    for k in range(20):
        st = ctx.reann_md_step_nvt(20, 0.25, 300.0, 20.0, noise[20 * k:20 * (k + 1)], x, v, p.masses)
        work.append((work[-1] if work else 0.0) + st.e_thermostat)
        h_nvt.append(st.e_pot + st.e_kin - work[-1])
    ctx2 = _ctx(p, pos, types, box)
    for k in range(20):
        st = ctx2.reann_md_step(20, 0.25, x2, v2, p.masses)
        h_nve.append(st.e_pot + st.e_kin)
    spread_nvt = (max(h_nvt) - min(h_nvt)) / n
    spread_nve = (max(h_nve) - min(h_nve)) / n
    assert spread_nvt <= 3 * spread_nve + 1e-6, (spread_nvt, spread_nve)
    assert (max(work) - min(work)) / n > 10 * spread_nvt


def test_split_nvt_call_equals_one_call():
    p, pos, types, box = small("water")
    _, _, x, v = _state(p, pos, types)
    x2, v2 = x.clone(), v.clone()
    noise = synth.thermostat_noise(len(pos), 12, seed=3)
    st = _ctx(p, pos, types, box).reann_md_step_nvt(12, 0.5, 350.0, 10.0, noise, x, v, p.masses)
    ctx = _ctx(p, pos, types, box)
    a = ctx.reann_md_step_nvt(5, 0.5, 350.0, 10.0, noise[:5], x2, v2, p.masses)
    b = ctx.reann_md_step_nvt(7, 0.5, 350.0, 10.0, noise[5:], x2, v2, p.masses)
    assert bool((x == x2).all()) and bool((v == v2).all())
    assert st.e_pot == b.e_pot and st.e_kin == b.e_kin
    assert st.e_thermostat == pytest.approx(a.e_thermostat + b.e_thermostat, rel=1e-12, abs=1e-12)


def test_invalid_thermostat_arguments_are_rejected():
    p, pos, types, box = small("water")
    _, _, x, v = _state(p, pos, types)
    ctx = _ctx(p, pos, types, box)
    good = synth.thermostat_noise(len(pos), 2, seed=1)
    bad_s = good.copy()
    bad_s[1, 1] = -1.0
    bad_nan = good.copy()
    bad_nan[0, 0] = np.nan
    for T, tau, z in ((0.0, 10.0, good), (-5.0, 10.0, good), (np.inf, 10.0, good), (300.0, -1.0, good),
                      (300.0, np.nan, good), (300.0, 10.0, bad_s), (300.0, 10.0, bad_nan)):
        with pytest.raises(reann.ReannError) as e:
            ctx.reann_md_step_nvt(2, 0.5, T, tau, z, x, v, p.masses)
        assert e.value.status == 1
    # a device noise array is rejected by the library itself
    torch = torch_cuda()
    z = torch.from_numpy(good).cuda()
    m = (C.c_double * p.n_elements)(*p.masses)
    st = reann.MdStats()
    rc = ctx.lib.reann_md_step_nvt(ctx.h, 2, 0.5, 300.0, 10.0, C.cast(z.data_ptr(), C.POINTER(C.c_double)),
                                   x.data_ptr(), v.data_ptr(), m, C.byref(st), None)
    assert rc == 1


def test_domain_decomposed_nvt_is_bit_identical():
    # the single-GPU domain-decomposed mode gives the monolithic forces bit for
    # bit, and the thermostat reduces the same velocities in the same order
    torch = torch_cuda()
    from molecular_dynamics_b200 import presets
    p = presets.scaled("ag1m", ncell=8)
    pos, types, box = synth.make_structure(p)
    v0 = synth.maxwell_boltzmann(p, types)
    noise = synth.thermostat_noise(len(pos), 8, seed=21)
    out = []
    for grid in ((0, 0, 0), (2, 2, 2)):
        spec = reann.ModelSpec.from_preset(p, mlp_precision=0, dd_grid=grid)
        ctx = reann.Context(spec, synth.weight_blob(p))
        ctx.reann_build_neighbors(pos, types, box)
        x = torch.from_numpy(pos.astype(np.float64)).cuda()
        v = torch.from_numpy(v0.copy()).cuda()
        st = ctx.reann_md_step_nvt(8, 1.0, 500.0, 10.0, noise, x, v, p.masses)
        out.append((x.cpu().numpy(), v.cpu().numpy(), st.e_pot, st.e_kin, st.e_thermostat))
    assert np.array_equal(out[0][0], out[1][0]) and np.array_equal(out[0][1], out[1][1])
    assert out[0][2:] == out[1][2:]


def test_kinetic_energy_is_canonical():
    # the GPU thermostat on its own trajectory: at tau = dt the kinetic energy
    # has the canonical (Gamma) moments, mean Nf kB T / 2 and relative spread
    # sqrt(2 / Nf), over 800 steps after a 200-step burn-in
    p, pos, types, box = small("ag256")
    _, _, x, v = _state(p, pos, types)
    n = len(pos)
    nf = 3 * n - 3
    kt = 0.5 * nf * KB * 300.0
    noise = synth.thermostat_noise(n, 1000, seed=8)
    ctx = _ctx(p, pos, types, box)
    K = []
    for k in range(1000):
        st = ctx.reann_md_step_nvt(1, 1.0, 300.0, 1.0, noise[k:k + 1], x, v, p.masses)
        K.append(st.e_kin)
    K = np.array(K[200:])
    assert abs(K.mean() / kt - 1.0) < 0.01, K.mean() / kt
    ratio = K.std() / kt / np.sqrt(2.0 / nf)
    assert 0.85 < ratio < 1.15, ratio
