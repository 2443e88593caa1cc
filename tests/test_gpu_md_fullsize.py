"""The benchmark's workload as an MD run: 1,048,576 Ag atoms, bf16 networks,
200 velocity-Verlet steps of 1 fs from Maxwell-Boltzmann velocities at 300 K.

A chaotic trajectory cannot be compared with the oracle's over 200 steps, so
the oracle is anchored to the GPU state: after the run, the forces and atomic
energies of sampled atoms at the GPU's final positions are recomputed by the
oracle on the cluster that determines them (every atom within 2 T r_c).  The
run itself is checked by what holds for any correct velocity Verlet: the
total energy is conserved to a small fraction of the thermal energy, the
potential energy the MD call reports equals a fresh energy+force evaluation
at the returned positions, and the centre-of-mass velocity stays zero.
A second run couples the workload to a 450 K bath by stochastic velocity
rescaling (reann_md_step_nvt) and checks the thermostat step by step.
"""
import numpy as np
import pytest

from gpu_helpers import E_TOL, F_TOL, cluster_around, oracle_eval, torch_cuda
from molecular_dynamics_b200 import presets, reann, synth

pytestmark = pytest.mark.gpu

KB = 8.617333262e-5   # eV/K


def test_ag1m_run_anchored_to_oracle():
    torch = torch_cuda()
    p = presets.get("ag1m")
    pos, types, box = synth.make_structure(p)
    n = len(pos)
    v0 = synth.maxwell_boltzmann(p, types)
    w = synth.weight_blob(p)
    ctx = reann.Context(reann.ModelSpec.from_preset(p), w)      # the workload's bf16 networks
    ctx.reann_build_neighbors(pos, types, box)
    x = torch.from_numpy(pos.astype(np.float64)).cuda()
    v = torch.from_numpy(v0.copy()).cuda()
    m = np.asarray(p.masses)[types]
    ek0 = 0.5 * float((m[:, None] * v0 ** 2).sum()) * 103.6426965   # amu A^2/fs^2 -> eV
    etot, rebuilds = [], 0
    e_first = None
    for _ in range(4):
        st = ctx.reann_md_step(p.md_steps // 4, p.dt_fs, x, v, p.masses)
        if e_first is None:
            e_first = st.e_pot0 + ek0
        etot.append(st.e_pot + st.e_kin)
        rebuilds += st.rebuilds
    # energy conservation: drift within 1e-3 of the thermal energy 3/2 kT per atom
    drift = max(abs(e - e_first) for e in etot) / n
    assert drift < 1e-3 * 1.5 * KB * 300.0, (drift, etot, e_first)
    # momentum: the initial COM velocity is zero and Newton's third law holds pairwise
    vf = v.cpu().numpy()
    p_com = (m[:, None] * vf).sum(0) / m.sum()
    assert np.abs(p_com).max() < 1e-6
    # the reported potential energy is the energy at the returned positions
    xf = x.cpu().numpy()
    xw = np.mod(xf, box).astype(np.float32)
    pos_d = torch.from_numpy(xw).cuda()
    ctx.reann_build_neighbors(pos_d, torch.from_numpy(types).cuda(), box)
    F = torch.empty_like(pos_d)
    Ei = torch.empty(n, dtype=torch.float32, device="cuda")
    E = ctx.reann_energy_forces(pos_d, F, Ei)
    assert abs(E - st.e_pot) / n < E_TOL[1]
    F, Ei = F.cpu().numpy(), Ei.cpu().numpy()
    # anchored parity at the final state
    radius = 2 * p.T * p.r_cut + 0.5
    rng = np.random.default_rng(7)
    for k in rng.choice(n, size=3, replace=False):
        cpos, ctypes_, cbox, _ = cluster_around(xw, types, box, k, radius)
        ref = oracle_eval(p, cpos, ctypes_, cbox, weights=w)
        assert np.abs(F[k] - ref.forces[0]).max() <= F_TOL[1], (k, F[k], ref.forces[0])
        rel = abs(Ei[k] - ref.atom_energy[0]) / max(float(np.sqrt(np.mean(Ei ** 2))), 1e-2)
        assert rel <= 10 * E_TOL[1], (k, Ei[k], ref.atom_energy[0])
    print(f"ag1m 200 steps: drift/atom {drift:.3e} eV, rebuilds {rebuilds}, |p_com| {np.abs(p_com).max():.2e}")


def test_ag1m_nvt_rescaling_and_effective_energy():
    # the same workload coupled to 450 K (tau = 20 fs, 1 fs steps).  Each of the
    # first 20 steps runs as its own call, so the kinetic energy before the
    # rescaling (e_kin - e_thermostat) is known and the device's new kinetic
    # energy must be the thermostat's formula of it with that step's numbers
    # (the noise terms are tiny at this size: sqrt(2 / Nf) ~ 8e-4).  Then the
    # effective energy E_pot + E_kin - W is conserved over 200 steps like the
    # NVE run's total energy, the bath heats the crystal toward 450 K (the
    # kinetic temperature rings around the target while the potential energy
    # takes up its equipartition share: 477 K after 200 fs), and the global
    # scaling keeps the centre-of-mass velocity at zero
    torch = torch_cuda()
    p = presets.get("ag1m")
    pos, types, box = synth.make_structure(p)
    n = len(pos)
    v0 = synth.maxwell_boltzmann(p, types)
    ctx = reann.Context(reann.ModelSpec.from_preset(p), synth.weight_blob(p))
    ctx.reann_build_neighbors(pos, types, box)
    x = torch.from_numpy(pos.astype(np.float64)).cuda()
    v = torch.from_numpy(v0.copy()).cuda()
    target, tau, dt = 450.0, 20.0, 1.0
    noise = synth.thermostat_noise(n, 200, seed=31)
    nf = 3 * n - 3
    kt = 0.5 * nf * KB * target
    c = np.exp(-dt / tau)
    temps, heff, work = [], [], 0.0
    h0 = None
    for k in range(20):
        st = ctx.reann_md_step_nvt(1, dt, target, tau, noise[k:k + 1], x, v, p.masses)
        if h0 is None:
            h0 = st.e_pot0 + st.e_kin0
        K = st.e_kin - st.e_thermostat
        r1, s = noise[k]
        Kn = K + (1 - c) * (kt * (r1 * r1 + s) / nf - K) + 2 * r1 * np.sqrt(c * (1 - c) * K * kt / nf)
        assert st.e_kin == pytest.approx(Kn, rel=1e-9), (k, st.e_kin, Kn)
        work += st.e_thermostat
        heff.append(st.e_pot + st.e_kin - work)
        temps.append(2.0 * st.e_kin / (nf * KB))
    for k in range(9):
        st = ctx.reann_md_step_nvt(20, dt, target, tau, noise[20 + 20 * k:40 + 20 * k], x, v, p.masses)
        work += st.e_thermostat
        heff.append(st.e_pot + st.e_kin - work)
        temps.append(2.0 * st.e_kin / (nf * KB))
    drift = max(abs(h - h0) for h in heff) / n
    assert drift < 1e-3 * 1.5 * KB * 300.0, (drift, heff, h0)
    assert 0.85 * target < temps[-1] < 1.15 * target, temps
    assert work / n > 0.5 * 1.5 * KB * 150.0          # the bath put in heat: at least half the kinetic share
    m = np.asarray(p.masses)[types]
    vf = v.cpu().numpy()
    assert np.abs((m[:, None] * vf).sum(0) / m.sum()).max() < 1e-6
    print(f"ag1m NVT 200 steps: T {temps[-1]:.1f} K, work/atom {work / n:.4e} eV, |dH|/atom {drift:.3e} eV, "
          f"T every 20 fs {[round(t, 1) for t in [temps[19]] + temps[20:]]}")
