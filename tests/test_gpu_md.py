"""Velocity-Verlet MD on the GPU through reann_md_step.

  * anchored parity: a few steps from the same start as the oracle's own
    velocity Verlet (trajectories of a chaotic system diverge, so the horizon
    is short), positions within 1e-4 A and velocities within 1e-5 A/fs, on a
    water sample and on the whole 3,000-atom water workload;
  * the water workload's 1000 steps at 0.5 fs conserve total energy and
    rebuild the neighbour list as atoms cross skin/2;
  * splitting a run into two calls gives the same state as one call
    (the state round-trips through the caller's arrays);
  * host and device state arrays give identical trajectories.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import torch_cuda
from helpers import model_for, small
from molecular_dynamics_b200 import presets, reann, synth

pytestmark = pytest.mark.gpu


def _ctx(p, pos, types, box):
    ctx = reann.Context(reann.ModelSpec.from_preset(p, mlp_precision=0), synth.weight_blob(p))
    ctx.reann_build_neighbors(pos, types, box)
    return ctx


def _min_image(d, box):
    return d - box * np.rint(d / box)


@pytest.mark.parametrize("system", ["water300", "water3k"])
def test_anchored_steps_match_oracle(system):
    """10 steps of 0.5 fs from the same start as the oracle: a 300-atom water
    sample and the full 3,000-atom water workload."""
    torch = torch_cuda()
    if system == "water3k":
        p = presets.get("water3k")
        pos, types, box = synth.make_structure(p)
    else:
        p, pos, types, box = small("water")
    v0 = synth.maxwell_boltzmann(p, types)
    x0 = pos.astype(np.float64)
    ctx = _ctx(p, pos, types, box)
    x = torch.from_numpy(x0.copy()).cuda()
    v = torch.from_numpy(v0.copy()).cuda()
    st = ctx.reann_md_step(10, 0.5, x, v, p.masses)
    assert st.steps == 10
    xo, vo, ep, ek = oracle.md_verlet(model_for(p), x0, v0, types, box, p.masses, 0.5, 10)
    assert np.abs(_min_image(x.cpu().numpy() - xo, box)).max() < 1e-4
    assert np.abs(v.cpu().numpy() - vo).max() < 1e-5
    assert abs(st.e_pot - ep[-1]) / len(pos) < 1e-5
    assert abs(st.e_kin - ek[-1]) / len(pos) < 1e-5
    assert abs(st.e_pot0 - ep[0]) / len(pos) < 1e-5


def test_water_run_conserves_energy_and_rebuilds():
    torch = torch_cuda()
    p = presets.get("water3k")
    pos, types, box = synth.make_structure(p)
    v0 = synth.maxwell_boltzmann(p, types)
    ctx = _ctx(p, pos, types, box)
    x = torch.from_numpy(pos.astype(np.float64)).cuda()
    v = torch.from_numpy(v0).cuda()
    etot = []
    rebuilds = 0
    for chunk in range(10):
        st = ctx.reann_md_step(p.md_steps // 10, p.dt_fs, x, v, p.masses)
        if chunk == 0:
            etot.append(st.e_pot0 + st.e_kin0)
        etot.append(st.e_pot + st.e_kin)
        rebuilds += st.rebuilds
    etot = np.array(etot)
    ekin0 = 1.5 * len(pos) * synth.KB_EV * p.temperature
    # total-energy drift small against the thermal kinetic energy
    assert np.abs(etot - etot[0]).max() < 0.02 * ekin0, (etot - etot[0], ekin0)
    assert rebuilds >= 1


def test_split_run_equals_single_run():
    torch = torch_cuda()
    p, pos, types, box = small("hea")
    v0 = synth.maxwell_boltzmann(p, types)
    x1 = torch.from_numpy(pos.astype(np.float64)).cuda()
    v1 = torch.from_numpy(v0.copy()).cuda()
    _ctx(p, pos, types, box).reann_md_step(8, 1.0, x1, v1, p.masses)
    x2 = torch.from_numpy(pos.astype(np.float64)).cuda()
    v2 = torch.from_numpy(v0.copy()).cuda()
    ctx = _ctx(p, pos, types, box)
    ctx.reann_md_step(3, 1.0, x2, v2, p.masses)
    ctx.reann_md_step(5, 1.0, x2, v2, p.masses)
    assert torch.equal(x1, x2) and torch.equal(v1, v2)


def test_split_run_with_host_state_equals_single_run():
    # a continuing call starts from the resident state while the caller's host
    # arrays are moved in and compared on a second stream
    p, pos, types, box = small("hea")
    v0 = synth.maxwell_boltzmann(p, types)
    x1, v1 = pos.astype(np.float64).copy(), v0.copy()
    _ctx(p, pos, types, box).reann_md_step(8, 1.0, x1, v1, p.masses)
    x2, v2 = pos.astype(np.float64).copy(), v0.copy()
    ctx = _ctx(p, pos, types, box)
    for k in (3, 1, 4):
        ctx.reann_md_step(k, 1.0, x2, v2, p.masses)
    assert np.array_equal(x1, x2) and np.array_equal(v1, v2)


@pytest.mark.parametrize("changed", ["x", "v"])
@pytest.mark.parametrize("where", ["host", "device"])
def test_continuation_with_a_changed_state_starts_from_it(changed, where):
    # the caller passes back a state other than the one the last call returned:
    # the call must run from the caller's state, as a fresh context does
    torch = torch_cuda()
    p, pos, types, box = small("chon")
    v0 = synth.maxwell_boltzmann(p, types)
    ctx = _ctx(p, pos, types, box)
    x, v = pos.astype(np.float64).copy(), v0.copy()
    ctx.reann_md_step(3, 0.5, x, v, p.masses)
    if changed == "x":
        x[7] += np.array([0.013, -0.021, 0.008])
    else:
        v[11] *= -1.0
    xr, vr = x.copy(), v.copy()
    fresh = _ctx(p, xr.astype(np.float32), types, box)
    fresh.reann_md_step(4, 0.5, xr, vr, p.masses)
    if where == "host":
        ctx.reann_md_step(4, 0.5, x, v, p.masses)
        xo, vo = x, v
    else:
        xd, vd = torch.from_numpy(x).cuda(), torch.from_numpy(v).cuda()
        ctx.reann_md_step(4, 0.5, xd, vd, p.masses)
        xo, vo = xd.cpu().numpy(), vd.cpu().numpy()
    assert np.array_equal(xo, xr) and np.array_equal(vo, vr)


def test_zero_steps_return_the_state():
    # a call of zero steps returns the state it was given (wrapped into the
    # box), both as a continuation and after the caller changed it
    p, pos, types, box = small("water")
    v0 = synth.maxwell_boltzmann(p, types)
    ctx = _ctx(p, pos, types, box)
    x, v = pos.astype(np.float64).copy(), v0.copy()
    ctx.reann_md_step(2, 0.5, x, v, p.masses)
    x1, v1 = x.copy(), v.copy()
    st = ctx.reann_md_step(0, 0.5, x, v, p.masses)
    assert np.array_equal(x, x1) and np.array_equal(v, v1) and st.steps == 0
    x[3] += 0.01
    x2 = x - np.asarray(box) * np.floor(x / np.asarray(box))   # wrapped into [0, L)
    v2 = v.copy()
    ctx.reann_md_step(0, 0.5, x, v, p.masses)
    assert np.array_equal(x, x2) and np.array_equal(v, v2)
    # and the next call continues from it like a fresh context would
    xr, vr = x.copy(), v.copy()
    fresh = _ctx(p, xr.astype(np.float32), types, box)
    fresh.reann_md_step(3, 0.5, xr, vr, p.masses)
    ctx.reann_md_step(3, 0.5, x, v, p.masses)
    assert np.array_equal(x, xr) and np.array_equal(v, vr)


def test_host_state_equals_device_state():
    torch = torch_cuda()
    p, pos, types, box = small("chon")
    v0 = synth.maxwell_boltzmann(p, types)
    xd = torch.from_numpy(pos.astype(np.float64)).cuda()
    vd = torch.from_numpy(v0.copy()).cuda()
    sd = _ctx(p, pos, types, box).reann_md_step(6, 0.5, xd, vd, p.masses)
    xh = pos.astype(np.float64).copy()
    vh = v0.copy()
    sh = _ctx(p, pos, types, box).reann_md_step(6, 0.5, xh, vh, p.masses)
    assert np.array_equal(xd.cpu().numpy(), xh) and np.array_equal(vd.cpu().numpy(), vh)
    assert sd.e_pot == sh.e_pot


def _gpu_run(ctx, x, v, dt, n, p):
    torch = torch_cuda()
    xd = torch.from_numpy(x.copy()).cuda()
    vd = torch.from_numpy(v.copy()).cuda()
    st = ctx.reann_md_step(n, dt, xd, vd, p.masses)
    return xd.cpu().numpy(), vd.cpu().numpy(), st


def test_time_reversal_on_gpu():
    # k steps forward, negate v, k steps: velocity Verlet returns to the start;
    # with fp32 forces the return is exact up to their rounding
    p, pos, types, box = small("water")
    v0 = synth.maxwell_boltzmann(p, types, temperature=100.0)
    x0 = pos.astype(np.float64)
    ctx = _ctx(p, pos, types, box)
    x1, v1, _ = _gpu_run(ctx, x0, v0, 0.25, 20, p)
    x2, v2, _ = _gpu_run(ctx, x1, -v1, 0.25, 20, p)
    assert np.abs(_min_image(x2 - x0, box)).max() < 1e-5
    assert np.abs(v2 + v0).max() < 1e-5


def test_energy_error_is_second_order_on_gpu():
    # the NVE total-energy error over a fixed time shrinks about fourfold when dt halves
    p, pos, types, box = small("water")
    v0 = synth.maxwell_boltzmann(p, types, temperature=100.0)
    x0 = pos.astype(np.float64)
    errs = []
    for dt, n in ((0.4, 10), (0.2, 20)):
        ctx = _ctx(p, pos, types, box)
        et = []
        x, v = x0, v0
        for _ in range(n):
            x, v, st = _gpu_run(ctx, x, v, dt, 1, p)
            if not et:
                et.append(st.e_pot0 + st.e_kin0)
            et.append(st.e_pot + st.e_kin)
        errs.append(np.abs(np.array(et) - et[0]).max())
    ratio = errs[0] / errs[1]
    assert 3.0 < ratio < 5.0, (ratio, errs)


def test_graph_replay_matches_eager_launches(monkeypatch):
    # reann_md_step runs all steps but the last of a call as a device-side
    # loop (one graph launch per stretch between neighbour rebuilds); with
    # REANN_LOOP=0 it replays one graph per step, with REANN_GRAPHS=0 it
    # launches eagerly.  Same trajectory bit for bit in all three; the loop
    # adds its gate kernel once per looped step.
    torch = torch_cuda()
    p, pos, types, box = small("water")
    v0 = synth.maxwell_boltzmann(p, types)
    out = []
    nsteps = 30
    for graphs, loop in (("1", "1"), ("1", "0"), ("0", "1")):
        monkeypatch.setenv("REANN_GRAPHS", graphs)
        monkeypatch.setenv("REANN_LOOP", loop)
        ctx = _ctx(p, pos, types, box)
        x = torch.from_numpy(pos.astype(np.float64)).cuda()
        v = torch.from_numpy(v0.copy()).cuda()
        k0 = ctx.reann_get_counters().kernel_launches
        st = ctx.reann_md_step(nsteps, p.dt_fs, x, v, p.masses)
        out.append((x.cpu().numpy(), v.cpu().numpy(), st.e_pot, ctx.reann_get_counters().kernel_launches - k0,
                    st.rebuilds, st.steps))
    for o in out[1:]:
        assert np.array_equal(out[0][0], o[0]) and np.array_equal(out[0][1], o[1])
        assert out[0][2] == o[2] and out[0][4] == o[4] and o[5] == nsteps
    assert out[1][3] == out[2][3]
    assert out[0][3] == out[1][3] + (nsteps - 1)


@pytest.mark.parametrize("ensemble", ["nve", "nvt"])
def test_device_loop_across_rebuilds(monkeypatch, ensemble):
    # a hot water sample rebuilds its list several times within one call: the
    # device-side loop hands each rebuild to the host and resumes; trajectory,
    # energies, thermostat work and rebuild count equal the per-step graphs'
    torch = torch_cuda()
    p, pos, types, box = small("water")
    v0 = synth.maxwell_boltzmann(p, types, temperature=900.0)
    nsteps = 150
    noise = synth.thermostat_noise(len(pos), nsteps, seed=77)
    out = []
    for loop in ("1", "0"):
        monkeypatch.setenv("REANN_LOOP", loop)
        ctx = _ctx(p, pos, types, box)
        x = torch.from_numpy(pos.astype(np.float64)).cuda()
        v = torch.from_numpy(v0.copy()).cuda()
        if ensemble == "nve":
            st = ctx.reann_md_step(nsteps, p.dt_fs, x, v, p.masses)
        else:
            st = ctx.reann_md_step_nvt(nsteps, p.dt_fs, 300.0, 20.0, noise, x, v, p.masses)
        out.append((x.cpu().numpy(), v.cpu().numpy(), st))
    (x1, v1, s1), (x2, v2, s2) = out
    assert s1.rebuilds >= 2 and s1.rebuilds == s2.rebuilds
    assert np.array_equal(x1, x2) and np.array_equal(v1, v2)
    assert s1.e_pot == s2.e_pot and s1.e_kin == s2.e_kin and s1.e_thermostat == s2.e_thermostat
