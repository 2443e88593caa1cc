"""Writes the per-feature input standardisation of every atomic network.

    python -m oracle.make_norm_stats [workload ...]
    python -m oracle.make_norm_stats --sign-only [workload ...]

Part of the weight recipe, not of the model: the paper's trained weights are
not available, and random Xavier weights applied to raw embedded densities
(values up to ~1e3 with a spread of a few percent) would saturate tanh and
leave the forces near zero.  So each network sees (rho - shift) / scale,
with shift = mean(rho^t_f) and scale = std(rho^t_f) + 0.05 mean|rho^t_f|
+ 1e-6 (0.106 for the pair-product form, see floor()), measured per layer
t, per element of the centre atom and per feature f on the workload's own
seeded structure.  Layer t's statistics are
measured with the networks of layers < t already standardised.

The 0.05 mean|rho| floor bounds the conditioning mean|rho| / scale by 20.
For the FCC lattices the statistics are measured on the same lattice with
thermal displacements five times the workload's sigma: a fitted model's
normalisation spans the varied structures of its training set, far wider
than one thermal crystal, whose odd-l densities are small residuals of
cancelling neighbour sums.  Standardising by the crystal's own spread made
the synthetic model amplify the rounding of those residuals (measured:
1e-5 relative per-atom energy errors from fp32 arithmetic alone).  The
molecular workloads (liquid water, C/H/O/N gas) are already varied and use
their own structure.

The same script fixes the energy scale: the energy network's output layer
(W3, b3) is multiplied by lambda = +-1 / rms(F), with F the oracle forces of
the unscaled model on the same structure, so that the synthetic potential
has forces of physical size (RMS 1 eV/A) rather than the tens of eV/A that
random weights on standardised densities give.  The sign matters for the
FCC workloads: the perfect lattice is a stationary point of any such model
(every atom is a centre of inversion), and a random output layer makes it a
maximum or a minimum along the thermal displacements with equal odds; with
a maximum the crystal heats up in an MD run and, after ~100 fs at 1 fs steps,
throws atoms fast enough to break velocity Verlet.  A fitted potential has
its crystal at a minimum, so the sign is chosen to make the workload's
thermally displaced structure higher in energy than the perfect lattice.
Molecular workloads keep the positive sign.

Only the oracle and the seeded input generators run here; the output file
molecular_dynamics_b200/data/norm_<workload>.json is read by
molecular_dynamics_b200.synth.weight_blob.
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np

import oracle
from molecular_dynamics_b200 import presets, synth

FLOOR = 0.05


def floor(p):
    """The floor of the standardisation scale, as a fraction of mean|rho|.

    It bounds the conditioning mean|rho| / scale by 1 / floor, and with it how
    far the fp32 rounding of a feature moves the standardised input.  In a
    crystal that rounding is nearly the same in every atom, so its effect on
    the first layer's pre-activation adds up coherently over the features: the
    pair-product form (N_phi (N_phi+1)(L+1)/2 features instead of N_phi (L+1))
    takes the floor times sqrt(features / N_phi (L+1)), which keeps that sum at
    the square form's level (0.05 -> 0.106 for N_phi = 8)."""
    return FLOOR * float(np.sqrt(p.DR / p.D))


OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "molecular_dynamics_b200", "data")


STATS_SIGMA_FACTOR = 5.0
ENERGY_SCALE_RECIPE = ("energy network output layer multiplied by +-1/rms(F) of the unscaled model; FCC workloads "
                       "take the sign that puts the perfect lattice below the workload's thermal structure")


def stats_lattice(p):
    """FCC workloads: the lattice the statistics and the energy scale are
    measured on -- the workload's own, or a smaller one of the same recipe
    (stats_ncell) where the per-feature statistics of the periodic crystal are
    the same and the oracle is cheaper."""
    return p.with_(ncell=p.stats_ncell) if p.kind == "fcc" and p.stats_ncell else p


def stats_structure(p):
    """The structure the statistics are measured on (see the module text)."""
    if p.kind == "fcc":
        return synth.make_structure(stats_lattice(p).with_(sigma=STATS_SIGMA_FACTOR * p.sigma))
    return synth.make_structure(p)


def measure(p, verbose=True):
    pos, types, box = stats_structure(p)
    n = len(pos)
    t0 = time.time()
    if n <= 20000:
        pairs = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    else:
        pairs = oracle.pairs_cells(pos, box, p.r_cut, p.skin)
    depth = p.stats_depth
    ne, D = p.n_elements, p.DR
    shift = np.zeros((depth, ne, D))
    scale = np.ones((depth, ne, D))
    sat = []
    for t in range(depth):
        T = t + 1
        blob = synth.weight_blob(p, T=T, norm=(shift[:t], scale[:t]), use_stored_norm=False)
        model = oracle.Model.from_preset(p, blob, T=T)
        res = oracle.energy_forces(model, pos, types, box, pairs, forces=False, intermediates=True)
        rho = res.rho[t]
        for e in range(ne):
            sel = types == e
            r = rho[sel]
            mu = r.mean(0)
            sd = r.std(0) + floor(p) * np.abs(r).mean(0) + 1e-6
            shift[t, e] = np.float32(mu)
            scale[t, e] = np.float32(sd)
            # diagnostic: fraction of first-layer pre-activations beyond |3|
            layer = t if t < p.T - 1 else synth.ENERGY_LAYER
            raw = synth.raw_network(p, layer, e)
            z = ((r - shift[t, e]) / scale[t, e]) @ raw["W1"].T + raw["b1"]
            sat.append(float((np.abs(z) > 3).mean()))
        if verbose:
            print(f"  {p.key} layer {t}: {time.time() - t0:.1f}s, saturated fraction {sat[-1]:.3f}", flush=True)
    # energy scale from the unscaled model at the workload's own depth T
    blob = synth.weight_blob(p, T=p.T, norm=(shift, scale), use_stored_norm=False, energy_scale=1.0)
    model = oracle.Model.from_preset(p, blob, T=p.T)
    res = oracle.energy_forces(model, pos, types, box, pairs)
    lam = float(np.float32(1.0 / np.sqrt(np.mean(res.forces ** 2))))
    lam *= energy_sign(p, shift, scale, lam, verbose)
    if verbose:
        print(f"  {p.key} energy scale {lam:.6g} ({time.time() - t0:.1f}s)", flush=True)
    return shift, scale, sat, lam


def energy_sign(p, shift, scale, lam, verbose=True):
    """+1 or -1 for the energy scale (see the module text): FCC workloads get
    the sign that puts the perfect lattice below the workload's structure."""
    if p.kind != "fcc":
        return 1.0
    blob = synth.weight_blob(p, T=p.T, norm=(shift, scale), use_stored_norm=False, energy_scale=abs(lam))
    model = oracle.Model.from_preset(p, blob, T=p.T)
    per_atom = []
    base = stats_lattice(p)
    for q in (base, base.with_(sigma=0.0)):
        pos, types, box = synth.make_structure(q)
        pairs = oracle.pairs_brute(pos, box, q.r_cut, q.skin) if len(pos) <= 20000 else \
            oracle.pairs_cells(pos, box, q.r_cut, q.skin)
        per_atom.append(oracle.energy_forces(model, pos, types, box, pairs, forces=False).energy / len(pos))
    sign = 1.0 if per_atom[0] > per_atom[1] else -1.0
    if verbose:
        print(f"  {p.key} E/atom thermal {per_atom[0]:.6f}, perfect lattice {per_atom[1]:.6f} "
              f"(positive scale) -> sign {sign:+.0f}", flush=True)
    return sign


def resign(keys):
    """Recompute only the sign of the stored energy scales (the standardisation
    and |lambda| do not depend on it)."""
    for k in keys:
        p = presets.get(k)
        path = os.path.join(OUT, f"norm_{k}.json")
        with open(path) as f:
            d = json.load(f)
        shift = np.asarray(d["shift"], np.float64)
        scale = np.asarray(d["scale"], np.float64)
        lam = abs(float(d["energy_scale"]))
        d["energy_scale"] = lam * energy_sign(p, shift[:p.T], scale[:p.T], lam)
        d["energy_scale_recipe"] = ENERGY_SCALE_RECIPE
        with open(path, "w") as f:
            json.dump(d, f)
        print(f"wrote norm_{k}.json  energy scale {d['energy_scale']:.6g}")


def main(keys):
    os.makedirs(OUT, exist_ok=True)
    for k in keys:
        p = presets.get(k)
        shift, scale, sat, lam = measure(p)
        out = {
            "workload": k,
            "recipe": "shift = mean(rho^t_f), scale = std(rho^t_f) + 0.05 mean|rho^t_f| + 1e-6, per layer t, "
                      "element of the centre atom and feature f, on the workload's seeded structure (FCC lattices: "
                      "thermal displacements 5x the workload's sigma)",
            "shift": shift.tolist(),
            "scale": scale.tolist(),
            "saturated_fraction": sat,
            "energy_scale": lam,
            "energy_scale_recipe": ENERGY_SCALE_RECIPE,
        }
        with open(os.path.join(OUT, f"norm_{k}.json"), "w") as f:
            json.dump(out, f)
        print(f"wrote norm_{k}.json  max saturated fraction {max(sat):.3f}")


if __name__ == "__main__":
    args = sys.argv[1:]
    if args and args[0] == "--sign-only":
        resign(args[1:] or list(presets.ORDER))
    else:
        main(args or list(presets.ORDER))
