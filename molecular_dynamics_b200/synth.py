"""Seeded synthetic inputs: structures, velocities and model weights.

This module is shared by the CUDA path, the benchmark and the tests.  It
draws random numbers and lays them out; it evaluates nothing of the model
itself (no orbital, density, network or force arithmetic lives here).

Structures follow the workloads of "Efficient Parallelization of Message
Passing Neural Network Potentials for Large-Scale Molecular Dynamics"
(Results): perturbed FCC silver and high-entropy-alloy lattices, a
liquid-water-like box and a C2H2/O2/N2 gas mixture.  The datasets and
trained weights of the paper are not available, so seeded stand-ins of the
same shape are produced here.

Readings of unstated recipe details:
  * thermal displacements are i.i.d. N(0, sigma^2) per Cartesian component,
    applied once to the ideal lattice, then wrapped into [0, L);
  * water: oxygen centres are placed by random sequential addition with a
    2.5 A minimum O-O image distance, orientations are uniform on SO(3), and
    each molecule has O-H 0.96 A and H-O-H 104.5 deg;
  * C/H/O/N: linear molecules (C-C 1.20 A, C-H 1.06 A, O-O 1.21 A,
    N-N 1.10 A) with uniform random axes; a molecule overlapping an earlier
    one (any intermolecular atom pair closer than 2.0 A) is redrawn, and the
    molecule kinds are interleaved in a seeded random order;
  * Maxwell-Boltzmann velocities: Gaussian per component with variance
    kT/m, centre-of-mass velocity removed, rescaled to exactly the target
    temperature with 3N-3 degrees of freedom;
  * workloads with bf16 networks store their matrices as bf16 values;
  * weights: Xavier-uniform matrices, U(-0.1, 0.1) biases, U(-1, 1) initial
    element coefficients c^0, and a per-feature input standardisation
    (shift = mean, scale = std + 0.05 mean|.|, so that mean/scale <= 20) in
    front of every atomic network; the energy
    network's output layer is multiplied by an energy scale that gives
    forces of RMS 1 eV/A.  Shift, scale and energy scale are measured once
    on each workload's own structure (FCC lattices: with five times the
    thermal displacement, a training-set-like spread) and stored in
    molecular_dynamics_b200/data/norm_<workload>.json.

Positions are returned as float32 values wrapped into [0, L): both the GPU
library and the fp64 oracle consume exactly these values.
"""
from __future__ import annotations

import json
import os
from typing import Dict, Optional, Tuple

import numpy as np

from .presets import Preset

KB_EV = 8.617333262e-5            # Boltzmann constant, eV/K
EV_PER_AMU_A2_FS2 = 103.6426965   # 1 amu*A^2/fs^2 in eV
ACC_UNIT = 1.0 / EV_PER_AMU_A2_FS2  # eV/(A*amu) -> A/fs^2 (= 9.648533e-3)

_DATA = os.path.join(os.path.dirname(os.path.abspath(__file__)), "data")


def seeds(p: Preset) -> Tuple[int, int, int]:
    """(structure, weights, velocities) seeds of workload number k: 1000k+1..3."""
    k = p.index
    return 1000 * k + 1, 1000 * k + 2, 1000 * k + 3


# ----------------------------------------------------------------------------
# structures

def _wrap32(pos: np.ndarray, L: float) -> np.ndarray:
    pos = np.mod(pos, L)
    p32 = pos.astype(np.float32)
    L32 = np.float32(L)
    p32[p32 >= L32] = np.float32(0.0)
    p32[p32 < 0] = np.float32(0.0)
    return p32


def fcc_lattice(ncell: int, a: float) -> np.ndarray:
    basis = np.array([[0, 0, 0], [0.5, 0.5, 0], [0.5, 0, 0.5], [0, 0.5, 0.5]])
    g = np.arange(ncell)
    cells = np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3)
    return ((cells[:, None, :] + basis[None]) * a).reshape(-1, 3)


def _random_rotations(rng: np.random.Generator, n: int) -> np.ndarray:
    """Uniform SO(3) rotations from uniform unit quaternions."""
    q = rng.normal(size=(n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    w, x, y, z = q.T
    return np.stack([
        np.stack([1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)], -1),
        np.stack([2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)], -1),
        np.stack([2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)], -1),
    ], 1)


def _random_axes(rng: np.random.Generator, n: int) -> np.ndarray:
    v = rng.normal(size=(n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def _resolve_overlaps(L, atoms_of, owner, n_mol, redraw, gap, check_mask=None, max_rounds=100000):
    """Redraw molecules until no two atoms of different molecules (among the
    atoms selected by check_mask) are closer than `gap` (minimum image).  Of an
    overlapping pair of molecules the one with the larger index is redrawn
    first; afterwards a redrawn molecule is redrawn again while it overlaps
    any other molecule."""
    from scipy.spatial import cKDTree

    sel = np.arange(len(owner)) if check_mask is None else np.nonzero(check_mask)[0]
    own = owner[sel]
    redo = None
    for _ in range(max_rounds):
        pts = np.mod(atoms_of()[sel], L)
        tree = cKDTree(pts, boxsize=L)
        if redo is None:
            pairs = tree.query_pairs(gap, output_type="ndarray")
            if len(pairs):
                mi, mj = own[pairs[:, 0]], own[pairs[:, 1]]
                inter = mi != mj
                redo = np.unique(np.maximum(mi[inter], mj[inter]))
            else:
                redo = np.zeros(0, dtype=np.int64)
        else:
            q = np.nonzero(np.isin(own, redo))[0]
            bad = set()
            for a, hs in zip(q, tree.query_ball_point(pts[q], gap)):
                if any(own[b] != own[a] for b in hs):
                    bad.add(int(own[a]))
            redo = np.array(sorted(bad), dtype=np.int64)
        if len(redo) == 0:
            return
        redraw(redo)
    raise RuntimeError("molecular placement did not converge")


def water_box(n_h2o: int, L: float, rng: np.random.Generator):
    """Returns (positions [3n,3], types) with per-molecule order O, H, H."""
    theta = np.deg2rad(104.5)
    r_oh = 0.96
    body = np.array([[0.0, 0.0, 0.0],
                     [r_oh * np.sin(theta / 2), r_oh * np.cos(theta / 2), 0.0],
                     [-r_oh * np.sin(theta / 2), r_oh * np.cos(theta / 2), 0.0]])
    centres = rng.uniform(0.0, L, size=(n_h2o, 3))
    rot = _random_rotations(rng, n_h2o)

    def redraw(ix):
        centres[ix] = rng.uniform(0.0, L, size=(len(ix), 3))
        rot[ix] = _random_rotations(rng, len(ix))

    def atoms_of():
        return (centres[:, None, :] + np.einsum("mij,kj->mki", rot, body)).reshape(-1, 3)

    owner = np.repeat(np.arange(n_h2o), 3)
    # only the oxygen atoms (first atom of each molecule) enter the overlap test
    _resolve_overlaps(L, atoms_of, owner, n_h2o, redraw, 2.5, check_mask=(np.arange(3 * n_h2o) % 3 == 0))
    types = np.tile(np.array([1, 0, 0], dtype=np.int32), n_h2o)   # O=1, H=0
    return atoms_of(), types


def chon_box(n_c2h2: int, n_o2: int, n_n2: int, L: float, rng: np.random.Generator):
    """Returns (positions, types); elements (H, C, N, O) -> 0, 1, 2, 3."""
    kinds = np.concatenate([np.zeros(n_c2h2, int), np.ones(n_o2, int), np.full(n_n2, 2)])
    rng.shuffle(kinds)
    n_mol = len(kinds)
    # atom offsets along the molecular axis; every molecule has 4 slots and a
    # diatomic repeats its two atoms (repeats never overlap another molecule
    # in a way its real atoms do not, and are dropped at the end)
    along = {0: [-(0.60 + 1.06), -0.60, 0.60, 0.60 + 1.06],
             1: [-0.605, 0.605, -0.605, 0.605],
             2: [-0.55, 0.55, -0.55, 0.55]}
    offs = np.array([along[k] for k in range(3)])[kinds]          # [n_mol, 4]
    centres = rng.uniform(0.0, L, size=(n_mol, 3))
    axes = _random_axes(rng, n_mol)

    def redraw(ix):
        centres[ix] = rng.uniform(0.0, L, size=(len(ix), 3))
        axes[ix] = _random_axes(rng, len(ix))

    def atoms_of():
        return (centres[:, None, :] + offs[:, :, None] * axes[:, None, :]).reshape(-1, 3)

    owner = np.repeat(np.arange(n_mol), 4)
    _resolve_overlaps(L, atoms_of, owner, n_mol, redraw, 2.0)
    slot_types = np.array([[0, 1, 1, 0], [3, 3, -1, -1], [2, 2, -1, -1]])[kinds].reshape(-1)
    keep = slot_types >= 0
    return atoms_of()[keep], slot_types[keep].astype(np.int32)


def make_structure(p: Preset, seed: Optional[int] = None):
    """Returns (pos float32 [N,3] in [0,L), types int32 [N], box float64 [3])."""
    s = seeds(p)[0] if seed is None else seed
    rng = np.random.default_rng(s)
    L = p.box_edge
    if p.kind == "fcc":
        pos = fcc_lattice(p.ncell, p.a)
        if p.sigma > 0:
            pos = pos + rng.normal(0.0, p.sigma, size=pos.shape)
        if p.n_elements > 1:
            types = rng.integers(0, p.n_elements, size=len(pos)).astype(np.int32)
        else:
            types = np.zeros(len(pos), dtype=np.int32)
    elif p.kind == "water":
        pos, types = water_box(p.n_mol[0], L, rng)
    elif p.kind == "chon":
        pos, types = chon_box(*p.n_mol, L, rng)
    else:
        raise ValueError(p.kind)
    return _wrap32(pos, L), types, np.array([L, L, L], dtype=np.float64)


def maxwell_boltzmann(p: Preset, types: np.ndarray, seed: Optional[int] = None,
                      temperature: Optional[float] = None) -> np.ndarray:
    """Velocities in A/fs, fp64 [N,3]."""
    s = seeds(p)[2] if seed is None else seed
    Tk = p.temperature if temperature is None else temperature
    rng = np.random.default_rng(s)
    m = np.asarray(p.masses)[types]
    std = np.sqrt(KB_EV * Tk / m * ACC_UNIT)
    v = rng.normal(size=(len(types), 3)) * std[:, None]
    v -= (m[:, None] * v).sum(0) / m.sum()
    ke = 0.5 * (m[:, None] * v * v).sum() * EV_PER_AMU_A2_FS2
    dof = 3 * len(types) - 3
    t_now = 2.0 * ke / (dof * KB_EV)
    return v * np.sqrt(Tk / t_now)


def thermostat_noise(n_atoms: int, nsteps: int, seed: int) -> np.ndarray:
    """The random numbers of stochastic velocity rescaling, two per step:
    R1 ~ N(0, 1) and S = a sum of Nf - 1 squared standard normals
    (Nf = 3 n - 3), drawn as a chi-squared variate; [nsteps][2]."""
    rng = np.random.default_rng(seed)
    nf = 3 * n_atoms - 3
    return np.stack([rng.standard_normal(nsteps), rng.chisquare(nf - 1, nsteps)], axis=1)


# ----------------------------------------------------------------------------
# weights

_KIND = {"W1": 1, "b1": 2, "W2": 3, "b2": 4, "W3": 5, "b3": 6}
ENERGY_LAYER = 100


def to_bf16_values(a) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float32."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def _xavier(rng, fan_out, fan_in):
    b = np.sqrt(6.0 / (fan_in + fan_out))
    return rng.uniform(-b, b, size=(fan_out, fan_in))


def raw_network(p: Preset, layer: int, element: int) -> Dict[str, np.ndarray]:
    """Random draws of one atomic network; layer = t for the coefficient network
    M^t (rho^t -> c^{t+1}), or ENERGY_LAYER for the energy network."""
    seed = seeds(p)[1]
    D, DR, (H1, H2) = p.D, p.DR, p.hidden
    n_out = 1 if layer == ENERGY_LAYER else D
    g = lambda k: np.random.default_rng([seed, layer, element, _KIND[k]])
    return {
        "W1": _xavier(g("W1"), H1, DR), "b1": g("b1").uniform(-0.1, 0.1, H1),
        "W2": _xavier(g("W2"), H2, H1), "b2": g("b2").uniform(-0.1, 0.1, H2),
        "W3": _xavier(g("W3"), n_out, H2), "b3": g("b3").uniform(-0.1, 0.1, n_out),
    }


def raw_c0(p: Preset) -> np.ndarray:
    return np.random.default_rng([seeds(p)[1], 999]).uniform(-1.0, 1.0, size=(p.n_elements, p.D))


def _load_data(p: Preset):
    path = os.path.join(_DATA, f"norm_{p.key}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        return json.load(f)


def load_norm(p: Preset):
    """Standardisation (shift, scale) per layer t, element and feature, or None."""
    d = _load_data(p)
    if d is None:
        return None
    return np.asarray(d["shift"], np.float64), np.asarray(d["scale"], np.float64)


def load_energy_scale(p: Preset) -> float:
    d = _load_data(p)
    if d is None or "energy_scale" not in d:
        raise FileNotFoundError(f"no energy scale for workload {p.key}")
    return float(d["energy_scale"])


def blob_layout(p: Preset, T: int):
    """Offsets (in float32 elements) of every tensor in the weight blob.

    Layout: C0[n_el][D]; then for t = 0..T-2 and each element the coefficient
    network M^t; then for each element the energy network.  Each network is
    shift[DR], scale[DR], W1[H1][DR], b1[H1], W2[H2][H1], b2[H2], W3[n_out][H2],
    b3[n_out] (matrices row-major, output index first); DR is the density
    feature count (D for the square form), n_out = D or 1.
    """
    D, DR, (H1, H2), ne = p.D, p.DR, p.hidden, p.n_elements
    off = 0
    lay = {"C0": (off, (ne, D))}
    off += ne * D

    def net(n_out):
        nonlocal off
        d = {}
        for name, shape in (("shift", (DR,)), ("scale", (DR,)), ("W1", (H1, DR)), ("b1", (H1,)),
                            ("W2", (H2, H1)), ("b2", (H2,)), ("W3", (n_out, H2)), ("b3", (n_out,))):
            d[name] = (off, shape)
            off += int(np.prod(shape))
        return d

    lay["coef"] = [[net(D) for _ in range(ne)] for _ in range(T - 1)]
    lay["energy"] = [net(1) for _ in range(ne)]
    lay["total"] = off
    return lay


def weight_blob(p: Preset, T: Optional[int] = None, norm=None, use_stored_norm: bool = True,
                energy_scale: Optional[float] = None) -> np.ndarray:
    """The float32 weight blob read by both the GPU library and the oracle.

    energy_scale multiplies the energy network's output layer (W3, b3); by
    default the stored per-workload value is used."""
    T = p.T if T is None else T
    if norm is None and use_stored_norm:
        norm = load_norm(p)
        if norm is None:
            raise FileNotFoundError(f"no standardisation data for workload {p.key}")
    if energy_scale is None:
        energy_scale = load_energy_scale(p) if use_stored_norm else 1.0
    lay = blob_layout(p, T)
    blob = np.zeros(lay["total"], dtype=np.float32)

    def put(entry, arr):
        o, shape = entry
        blob[o:o + int(np.prod(shape))] = np.asarray(arr, np.float64).reshape(-1).astype(np.float32)

    put(lay["C0"], raw_c0(p))

    def fill(net, layer, t_in, e):
        raw = raw_network(p, layer, e)
        if layer == ENERGY_LAYER:
            raw["W3"] = raw["W3"] * energy_scale
            raw["b3"] = raw["b3"] * energy_scale
        if p.mlp_precision == 1:
            # bf16 networks: the matrices are stored as bf16 values, as bf16
            # inference stores them (biases and standardisation stay fp32)
            for k in ("W1", "W2", "W3"):
                raw[k] = to_bf16_values(raw[k])
        if norm is not None and t_in < norm[0].shape[0]:
            put(net["shift"], norm[0][t_in, e])
            put(net["scale"], norm[1][t_in, e])
        else:
            put(net["shift"], np.zeros(p.DR))
            put(net["scale"], np.ones(p.DR))
        for k in ("W1", "b1", "W2", "b2", "W3", "b3"):
            put(net[k], raw[k])

    for t in range(T - 1):
        for e in range(p.n_elements):
            fill(lay["coef"][t][e], t, t, e)
    for e in range(p.n_elements):
        fill(lay["energy"][e], ENERGY_LAYER, T - 1, e)
    return blob


def workload(p: Preset, T: Optional[int] = None, with_velocities: bool = False):
    """Everything one evaluation needs: dict of pos, types, box, weights (+ v)."""
    pos, types, box = make_structure(p)
    out = {"pos": pos, "types": types, "box": box, "weights": weight_blob(p, T)}
    if with_velocities:
        out["vel"] = maxwell_boltzmann(p, types)
    return out
