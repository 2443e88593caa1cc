"""GPU path vs the fp64 oracle on the same seeded inputs, through the C ABI.

Sizes span several 32-row network tiles and 128-atom thread blocks with
ragged tails; one system has fewer than three cells per axis (the cell
stencil must not double count wrapped cells).  Pair lists must be
bit-identical as sets; energies and forces must meet the tolerances in
gpu_helpers.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import (assert_atom_energies_close, assert_energy_close, assert_forces_close, gpu_eval, oracle_eval,
                         torch_cuda)
from helpers import small
from molecular_dynamics_b200 import presets, reann, synth

pytestmark = pytest.mark.gpu

CASES = {
    "ag256": lambda: small("ag256"),                                           # 2 cells per axis
    "ag500": lambda: (lambda p: (p, *synth.make_structure(p)))(presets.scaled("ag1m", ncell=5)),
    "water300": lambda: small("water"),
    "water3k": lambda: (lambda p: (p, *synth.make_structure(p)))(presets.get("water3k")),
    "hea256": lambda: small("hea"),
    "hea1372": lambda: (lambda p: (p, *synth.make_structure(p)))(presets.scaled("hea108k", ncell=7)),
    "chon976": lambda: small("chon"),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_pair_list_bit_exact(case):
    p, pos, types, box = CASES[case]()
    ctx, _, _, _ = gpu_eval(p, pos, types, box)
    row, col = ctx.reann_get_neighbors()
    orow, ocol = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    assert np.array_equal(row, orow)
    assert np.array_equal(col, ocol)


@pytest.mark.parametrize("case", sorted(CASES))
def test_energy_forces_match_oracle(case):
    p, pos, types, box = CASES[case]()
    _, E, F, Ei = gpu_eval(p, pos, types, box)
    ref = oracle_eval(p, pos, types, box)
    assert_energy_close(E, ref.energy, len(pos))
    assert_atom_energies_close(Ei, ref.atom_energy)
    assert_forces_close(F, ref.forces)
    assert abs(Ei.sum() - E) <= 1e-4 * max(1.0, abs(E))


@pytest.mark.parametrize("case", ["water300", "hea1372", "chon976"])
def test_cuda_core_fp32_networks_match_oracle(case):
    # mlp_precision 2: the fp32 networks on the CUDA cores (the reference the
    # three-pass tf32 tensor-core networks of mlp_precision 0 are measured
    # against) meet the same tolerances
    p, pos, types, box = CASES[case]()
    _, E, F, Ei = gpu_eval(p, pos, types, box, mlp_precision=2)
    ref = oracle_eval(p, pos, types, box)
    assert_energy_close(E, ref.energy, len(pos))
    assert_atom_energies_close(Ei, ref.atom_energy)
    assert_forces_close(F, ref.forces)


@pytest.mark.parametrize("case", ["hea1372", "chon976"])
def test_tf32_and_cuda_core_networks_agree(case):
    # both fp32-accurate network paths on the same inputs: per-atom energies
    # and forces agree at the fp32 level, and the tensor-core path is
    # deterministic (fixed MMA order)
    p, pos, types, box = CASES[case]()
    _, E0, F0, Ei0 = gpu_eval(p, pos, types, box, mlp_precision=0)
    _, E0b, F0b, _ = gpu_eval(p, pos, types, box, mlp_precision=0)
    _, E2, F2, Ei2 = gpu_eval(p, pos, types, box, mlp_precision=2)
    assert E0 == E0b and np.array_equal(F0, F0b)
    scale = max(float(np.sqrt(np.mean(Ei2 ** 2))), 1e-2)
    assert np.abs(Ei0 - Ei2).max() <= 2e-5 * scale
    assert np.abs(F0 - F2).max() <= 5e-5


@pytest.mark.parametrize("case", ["ag500", "water300", "hea1372", "chon976"])
def test_every_layer_matches_oracle(case):
    # rho^t in the units the networks see, (rho - shift) / scale, and c^t
    # relative to each feature's largest value.  With fp64 orbital sums, rho
    # formed as rho - shift in fp64 and fp32-pair constants (fp32-accurate
    # paths) the layers stay within 4.3e-5 (rho) and 5.4e-6 (c); the
    # bf16-network Ag case within 9.0e-5 and 6.6e-6.  The bounds keep about 2x.
    p, pos, types, box = CASES[case]()
    ctx, _, _, _ = gpu_eval(p, pos, types, box)
    ref = oracle_eval(p, pos, types, box, intermediates=True)
    shift, scale = synth.load_norm(p)
    for t in range(p.T):
        rho, coef = ctx.reann_get_features(t)
        err_x = np.abs(rho - ref.rho[t]) / scale[t][types]
        scale_c = np.abs(ref.coef[t]).max(axis=0) + 1e-6
        err_c = (np.abs(coef - ref.coef[t]) / scale_c).max()
        print(f"\n{case} t={t}: rho err (standardised) {err_x.max():.3e}, c err (relative) {err_c:.3e}")
        assert err_x.max() <= 2e-4, (t, err_x.max())
        assert err_c <= 1.5e-5, (t, err_c)


def _rounding_sensitivity(p, pos, types, box, T, w, ref, draws=8):
    """The oracle's own response to perturbing the positions at fp32 rounding
    size (relative 2^-24, seeded normal draws): the largest |dE|/n and
    max|dF| over the draws.  It measures how strongly a model amplifies
    rounding-size input errors, independently of the GPU path."""
    rng = np.random.default_rng(2024)
    n = len(pos)
    dE = dF = 0.0
    for _ in range(draws):
        pp = pos.astype(np.float64) * (1.0 + rng.standard_normal(pos.shape) * 2.0 ** -24)
        r = oracle_eval(p, pp, types, box, T=T, weights=w)
        dE = max(dE, abs(r.energy - ref.energy) / n)
        dF = max(dF, float(np.abs(r.forces - ref.forces).max()))
    return dE, dF


ROUNDING_FACTOR = 30.0


@pytest.mark.parametrize("key,T", [("chon", 1), ("chon", 2), ("ag", 1), ("ag", 2), ("ag", 4), ("ag", 6)])
def test_depths_other_than_the_preset(key, T):
    # The Ag model's standardisation covers layers up to 6 (its T sweep).  Up
    # to the workloads' own depth (T <= 3) the stated tolerances apply.  Beyond
    # it the synthetic models' conditioning varies strongly with the depth
    # (the oracle's response to rounding-size input perturbations is ~10x
    # larger at T = 4 than at T = 3 or 5), and fp32 results of implementations
    # that differ only in rounding (cutoff polynomials, accurate library
    # cosine) were measured 1.4x apart there.  So for T > 3 the tolerance is
    # the stated one or ROUNDING_FACTOR times that oracle response, whichever
    # is larger: the GPU computes every intermediate in fp32, while the
    # perturbation rounds only the inputs (measured ratio 10-22).
    p, pos, types, box = small(key)
    w = synth.weight_blob(p, T=T)
    _, E, F, Ei = gpu_eval(p, pos, types, box, T=T, weights=w)
    ref = oracle_eval(p, pos, types, box, T=T, weights=w)
    n = len(pos)
    tol_E = 1e-5 * max(abs(ref.energy) / n, 1e-2)
    tol_F = 1e-4
    stated = (tol_E, tol_F)
    if T > 3:
        dE, dF = _rounding_sensitivity(p, pos, types, box, T, w, ref)
        tol_E = max(tol_E, ROUNDING_FACTOR * dE)
        tol_F = max(tol_F, ROUNDING_FACTOR * dF)
        # relative condition number of the forces: relative response per unit relative input change
        kappa = dF / float(np.sqrt((ref.forces ** 2).mean())) / 2.0 ** -24
        print(f"\n{key} T={T}: |dE|/N={abs(E - ref.energy) / n:.3e} (stated {stated[0]:.3e}), "
              f"max|dF|={np.abs(F - ref.forces).max():.3e} (stated {stated[1]:.1e}); oracle response to "
              f"2^-24 position noise: dE/N {dE:.3e}, dF {dF:.3e}; rms F {np.sqrt((ref.forces ** 2).mean()):.3f}, "
              f"force condition number {kappa:.0f}")
    assert abs(E - ref.energy) / n <= tol_E, (abs(E - ref.energy) / n, tol_E)
    assert np.abs(F - ref.forces).max() <= tol_F, (np.abs(F - ref.forces).max(), tol_F)


BF16_CASES = {
    "ag500": lambda: (lambda p: (p, *synth.make_structure(p)))(presets.scaled("ag1m", ncell=5)),
    "ag2048": lambda: (lambda p: (p, *synth.make_structure(p)))(presets.scaled("ag1m", ncell=8)),
    # five elements with N_phi = 10 and [128,128] networks: ragged 128-row tiles per element
    "hea1372_h128": lambda: (lambda p: (p, *synth.make_structure(p)))(
        presets.scaled("hea108k", ncell=7).with_(hidden=(128, 128), mlp_precision=1)),
}


@pytest.mark.parametrize("case", sorted(BF16_CASES))
def test_bf16_tensor_core_networks_match_oracle(case):
    p, pos, types, box = BF16_CASES[case]()
    w = synth.weight_blob(p)
    _, E, F, Ei = gpu_eval(p, pos, types, box, mlp_precision=1, weights=w)
    ref = oracle_eval(p, pos, types, box, weights=w)
    assert_energy_close(E, ref.energy, len(pos), prec=1)
    assert_atom_energies_close(Ei, ref.atom_energy, prec=1)
    assert_forces_close(F, ref.forces, prec=1)


def test_bf16_networks_are_deterministic():
    p, pos, types, box = BF16_CASES["ag500"]()
    _, E1, F1, _ = gpu_eval(p, pos, types, box, mlp_precision=1)
    _, E2, F2, _ = gpu_eval(p, pos, types, box, mlp_precision=1)
    assert E1 == E2 and np.array_equal(F1, F2)


def test_repeated_evaluation_is_bit_identical():
    p, pos, types, box = small("hea")
    ctx, E1, F1, Ei1 = gpu_eval(p, pos, types, box)
    torch = torch_cuda()
    pos_d = torch.from_numpy(pos).cuda()
    F2 = torch.empty_like(pos_d)
    E2 = ctx.reann_energy_forces(pos_d, F2)
    assert E1 == E2
    assert np.array_equal(F1, F2.cpu().numpy().astype(np.float64))


def test_host_and_device_arrays_give_identical_results():
    p, pos, types, box = small("water")
    ctx, E1, F1, Ei1 = gpu_eval(p, pos, types, box)
    F2 = np.zeros_like(pos)
    Ei2 = np.zeros(len(pos), np.float32)
    ctx2 = reann.Context(reann.ModelSpec.from_preset(p, mlp_precision=0), synth.weight_blob(p))
    ctx2.reann_build_neighbors(pos, types, box)
    E2 = ctx2.reann_energy_forces(pos, F2, Ei2)
    assert E1 == E2
    assert np.array_equal(F1, F2.astype(np.float64))
    assert np.array_equal(Ei1, Ei2.astype(np.float64))


def test_permuted_input_gives_permuted_output():
    p, pos, types, box = small("chon")
    _, E1, F1, _ = gpu_eval(p, pos, types, box)
    perm = np.random.default_rng(11).permutation(len(pos))
    _, E2, F2, _ = gpu_eval(p, pos[perm], types[perm], box)
    # the internal order is (element, cell, caller index): summation order may differ
    assert abs(E1 - E2) <= 1e-6 * max(1.0, abs(E1))
    assert np.abs(F2 - F1[perm]).max() <= 1e-4


def test_images_outside_the_box_are_accepted():
    p, pos, types, box = small("hea")
    shift = np.array([1, -2, 3], np.float32) * box.astype(np.float32)
    _, E1, F1, _ = gpu_eval(p, pos, types, box)
    _, E2, F2, _ = gpu_eval(p, pos + shift, types, box)
    ref = oracle_eval(p, pos + shift, types, box)
    assert_energy_close(E2, ref.energy, len(pos))
    assert_forces_close(F2, ref.forces)


def test_isolated_atom_and_pair():
    p = presets.get("water3k")
    box = np.array([30.0, 30.0, 30.0])
    for pos, types in ((np.array([[1.0, 2.0, 3.0]], np.float32), np.array([1], np.int32)),
                       (np.array([[5.0, 5.0, 5.0], [6.1, 5.3, 4.2]], np.float32), np.array([1, 0], np.int32))):
        _, E, F, Ei = gpu_eval(p, pos, types, box)
        ref = oracle_eval(p, pos, types, box)
        assert_energy_close(E, ref.energy, len(pos))
        assert_forces_close(F, ref.forces)


def test_empty_system():
    p = presets.get("ag256")
    ctx, E, F, Ei = gpu_eval(p, np.zeros((0, 3), np.float32), np.zeros(0, np.int32), np.array([20.0, 20.0, 20.0]))
    assert E == 0.0 and F.shape == (0, 3)


def test_error_statuses():
    torch = torch_cuda()
    p, pos, types, box = small("ag256")
    spec = reann.ModelSpec.from_preset(p, mlp_precision=0)
    ctx = reann.Context(spec, synth.weight_blob(p))
    with pytest.raises(reann.ReannError) as e:
        ctx.reann_energy_forces(pos)
    assert e.value.status == 6                                        # no list yet
    with pytest.raises(reann.ReannError) as e:
        ctx.reann_build_neighbors(pos, types, np.array([13.0, 20.0, 20.0]))
    assert e.value.status == 2                                        # box < 2 (r_c + skin)
    bad = types.copy()
    bad[3] = 5
    with pytest.raises(reann.ReannError) as e:
        ctx.reann_build_neighbors(pos, bad, box)
    assert e.value.status == 1                                        # type out of range
    nan = pos.copy()
    nan[7, 1] = np.nan
    with pytest.raises(reann.ReannError) as e:
        ctx.reann_build_neighbors(nan, types, box)
    assert e.value.status == 4                                        # non-finite
    ctx.reann_build_neighbors(pos, types, box)
    moved = pos.copy()
    moved[0] += np.float32(0.6)                                       # > skin / 2
    with pytest.raises(reann.ReannError) as e:
        ctx.reann_energy_forces(moved)
    assert e.value.status == 5
    ctx.reann_energy_forces(pos)                                      # context still usable
    with pytest.raises(reann.ReannError):
        ctx.reann_get_features(p.T)                                   # layer out of range
