"""Helpers for the GPU tests: run the CUDA path through the C ABI, run the
oracle on the same inputs, and compare with the stated tolerances.

Tolerances (fp32 path): total energy |E_gpu - E_ref| / N <= 1e-5 max(|E_ref| / N,
1e-2 eV); the worst atom's |dE_i| <= 1e-4 of the RMS per-atom energy; forces
max-abs <= 1e-4 eV/A.  BF16-network path: forces max-abs <= 5e-3 eV/A, the
same energy tolerances (the split-bf16 networks keep 16 significant bits).
"""
from __future__ import annotations

import numpy as np

import oracle
from molecular_dynamics_b200 import reann, synth

F_TOL = {0: 1e-4, 1: 5e-3}
E_TOL = {0: 1e-5, 1: 1e-5}


def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU tests need CUDA")
    return torch


def gpu_eval(p, pos, types, box, T=None, mlp_precision=0, weights=None):
    torch = torch_cuda()
    T = p.T if T is None else T
    w = synth.weight_blob(p, T=T) if weights is None else weights
    ctx = reann.Context(reann.ModelSpec.from_preset(p, T=T, mlp_precision=mlp_precision), w)
    pos_d = torch.from_numpy(np.ascontiguousarray(pos, np.float32)).cuda()
    types_d = torch.from_numpy(np.ascontiguousarray(types, np.int32)).cuda()
    ctx.reann_build_neighbors(pos_d, types_d, box)
    F = torch.empty_like(pos_d)
    Ei = torch.empty(len(pos), dtype=torch.float32, device="cuda")
    E = ctx.reann_energy_forces(pos_d, F, Ei)
    torch.cuda.synchronize()
    return ctx, E, F.cpu().numpy().astype(np.float64), Ei.cpu().numpy().astype(np.float64)


def oracle_eval(p, pos, types, box, T=None, weights=None, intermediates=False):
    T = p.T if T is None else T
    w = synth.weight_blob(p, T=T) if weights is None else weights
    return oracle.energy_forces(oracle.Model.from_preset(p, w, T=T), pos, types, box, intermediates=intermediates)


def assert_energy_close(E_gpu, E_ref, n, prec=0):
    tol = E_TOL[prec] * max(abs(E_ref) / n, 1e-2)
    assert abs(E_gpu - E_ref) / n <= tol, (E_gpu, E_ref, abs(E_gpu - E_ref) / n, tol)


def assert_forces_close(F_gpu, F_ref, prec=0):
    err = np.abs(F_gpu - F_ref).max()
    assert err <= F_TOL[prec], (err, F_TOL[prec], np.abs(F_ref).max())


def assert_atom_energies_close(Ei_gpu, Ei_ref, prec=0):
    # worst atom against the system's per-atom energy scale (RMS of E_i): the
    # per-atom figure is reported beside the total-energy tolerance, and an
    # atom whose own E_i happens to be near zero is not a scale
    scale = max(float(np.sqrt(np.mean(Ei_ref ** 2))), 1e-2)
    err = np.abs(Ei_gpu - Ei_ref).max() / scale
    assert err <= 10 * E_TOL[prec], err


def cluster_around(pos, types, box, k, radius):
    """Atoms within `radius` of atom k (minimum image), unwrapped around k and
    placed in an open box large enough that no periodic image interacts."""
    x = pos.astype(np.float64)
    d = x - x[k]
    d -= box * np.rint(d / box)
    r = np.sqrt((d * d).sum(1))
    sel = np.nonzero(r < radius)[0]
    order = np.argsort(sel != k, kind="stable")        # atom k first
    sel = sel[order]
    L = 2 * radius + 4 * 8.0
    return d[sel] + L / 2, types[sel], np.array([L, L, L]), sel
