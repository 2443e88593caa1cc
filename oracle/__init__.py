"""fp64 CPU oracle of the REANN energy+force evaluation (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
CPU-baseline leg use this package; the product path (the CUDA library and
its binding) never imports, links or calls it, and it imports nothing from
the product path.  It evaluates what "Efficient Parallelization of Message
Passing Neural Network Potentials for Large-Scale Molecular Dynamics"
defines in section "REANN Architecture" (Eqs. 1-2) and section
"Parallelization Algorithm" (Eqs. 3-5); the readings of details the paper
leaves open are listed at the top of reann_oracle.c.

Every function here is pinned by tests/test_oracle_*.py to facts that do not
come from the oracle itself: finite differences, invariances, closed forms,
the multinomial identity, brute force against a second pair search, energy
additivity and the T-hop receptive field.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "reann_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

OK, ERR_ARG, ERR_BOX, ERR_CAPACITY, ERR_MEM = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile reann_oracle.c with gcc (fp64, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-std=c99", "-D_DEFAULT_SOURCE",
                               "-Wall", "-shared", "-fPIC", "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


class Cfg(C.Structure):
    _fields_ = [("n_elements", C.c_int32), ("T", C.c_int32), ("n_radial", C.c_int32), ("l_max", C.c_int32),
                ("hidden1", C.c_int32), ("hidden2", C.c_int32), ("r_cut", C.c_double), ("skin", C.c_double),
                ("alpha", C.c_double), ("density_form", C.c_int32)]


_lib = None


def _bind(cdll):
    _bind_signatures(cdll)
    return cdll


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(C.CDLL(build()))
    return _lib


class use_library:
    """Temporarily route every oracle call through another build of the C
    source (the planted-mistake tests compile deliberately broken copies)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = _bind(C.CDLL(self.path))
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved


def compile_source(src: str, out: str) -> str:
    """Compile an oracle C source with the oracle's own flags."""
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-std=c99", "-D_DEFAULT_SOURCE",
                           "-shared", "-fPIC", "-o", out, src, "-lm"])
    return out


def _bind_signatures(cdll):
    P = C.c_void_p
    cdll.oracle_pairs_brute.argtypes = [C.c_int64, P, P, C.c_double, C.c_double, C.c_int64, P, C.c_int64, P, P, P]
    cdll.oracle_pairs_cells.argtypes = [C.c_int64, P, P, C.c_double, C.c_double, C.c_int64, P, P, P]
    cdll.oracle_energy_forces.argtypes = [P, P, C.c_int64, C.c_int64, P, P, P, P, P, P, P, P, P, P, P]
    cdll.oracle_rho_pairwise.argtypes = [P, C.c_int64, P, P, P, P, P, P]
    cdll.oracle_md_verlet.argtypes = [P, P, C.c_int64, C.c_int64, P, P, P, P, P, C.c_double, C.c_int32, P, P]
    cdll.oracle_md_nvt.argtypes = [P, P, C.c_int64, C.c_int64, P, P, P, P, P, C.c_double, C.c_int32, P, P, P, P,
                                   P]
    cdll.oracle_weight_count.argtypes = [P]
    cdll.oracle_weight_count.restype = C.c_int64
    cdll.oracle_num_threads.restype = C.c_int


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


@dataclass
class Model:
    """Hyperparameters + float32 weight blob of one REANN model."""
    n_elements: int
    T: int
    n_radial: int
    l_max: int
    hidden: Sequence[int]
    r_cut: float
    skin: float
    alpha: float
    weights: np.ndarray
    density_form: int = 0

    @classmethod
    def from_preset(cls, p, weights: np.ndarray, T: Optional[int] = None) -> "Model":
        return cls(p.n_elements, p.T if T is None else T, p.n_radial, p.l_max, tuple(p.hidden), p.r_cut, p.skin,
                   p.alpha, np.ascontiguousarray(weights, dtype=np.float32), getattr(p, "density_form", 0))

    @property
    def D(self) -> int:
        """coefficients per atom: one per (n, l)"""
        return self.n_radial * (self.l_max + 1)

    @property
    def DR(self) -> int:
        """density features per atom (network input width)"""
        pairs = self.n_radial * (self.n_radial + 1) // 2 if self.density_form == 1 else self.n_radial
        return pairs * (self.l_max + 1)

    @property
    def n_tuples(self) -> int:
        return (self.l_max + 1) * (self.l_max + 2) * (self.l_max + 3) // 6

    def cfg(self) -> Cfg:
        return Cfg(self.n_elements, self.T, self.n_radial, self.l_max, self.hidden[0], self.hidden[1], self.r_cut,
                   self.skin, self.alpha, self.density_form)


def _check(rc: int, what: str):
    if rc != OK:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def pairs_brute(x, box, r_cut: float, skin: float, centres=None):
    """Brute-force O(N^2) pair list. Returns (row_ptr int64 [rows+1], col int32)."""
    x, box = _f64(x), _f64(box)
    n = len(x)
    cen = None if centres is None else np.ascontiguousarray(centres, dtype=np.int64)
    rows = n if cen is None else len(cen)
    counts = np.zeros(rows + 1, np.int64)
    nnz = np.zeros(1, np.int64)
    L = lib()
    _check(L.oracle_pairs_brute(n, _p(x), _p(box), r_cut, skin, rows, _p(cen), 0, _p(counts), None, _p(nnz)),
           "pairs_brute(count)")
    col = np.zeros(max(int(nnz[0]), 1), np.int32)
    _check(L.oracle_pairs_brute(n, _p(x), _p(box), r_cut, skin, rows, _p(cen), int(nnz[0]), _p(counts), _p(col),
                                _p(nnz)), "pairs_brute")
    row = np.zeros(rows + 1, np.int64)
    np.cumsum(counts[:rows], out=row[1:])
    return row, col[:int(nnz[0])]


def pairs_cells(x, box, r_cut: float, skin: float):
    """Independent cell-list pair search (used to pin pairs_brute)."""
    x, box = _f64(x), _f64(box)
    n = len(x)
    counts = np.zeros(n + 1, np.int64)
    nnz = np.zeros(1, np.int64)
    L = lib()
    _check(L.oracle_pairs_cells(n, _p(x), _p(box), r_cut, skin, 0, _p(counts), None, _p(nnz)), "pairs_cells(count)")
    col = np.zeros(max(int(nnz[0]), 1), np.int32)
    _check(L.oracle_pairs_cells(n, _p(x), _p(box), r_cut, skin, int(nnz[0]), _p(counts), _p(col), _p(nnz)),
           "pairs_cells")
    row = np.zeros(n + 1, np.int64)
    np.cumsum(counts[:n], out=row[1:])
    return row, col[:int(nnz[0])]


@dataclass
class Result:
    energy: float
    atom_energy: np.ndarray
    forces: Optional[np.ndarray]
    rho: Optional[np.ndarray] = None      # [T, N, DR]
    coef: Optional[np.ndarray] = None     # [T, N, D]
    A: Optional[np.ndarray] = None        # [T, N, N_phi * n_tuples]


def energy_forces(model: Model, x, types, box, pairs=None, forces: bool = True, intermediates: bool = False) -> Result:
    x, box = _f64(x), _f64(box)
    types = np.ascontiguousarray(types, dtype=np.int32)
    n = len(x)
    if pairs is None:
        pairs = pairs_brute(x, box, model.r_cut, model.skin)
    row, col = np.ascontiguousarray(pairs[0], np.int64), np.ascontiguousarray(pairs[1], np.int32)
    cfg = model.cfg()
    w = model.weights
    E = np.zeros(1)
    Ei = np.zeros(n)
    F = np.zeros((n, 3)) if forces else None
    rho = coef = A = None
    if intermediates:
        rho = np.zeros((model.T, n, model.DR))
        coef = np.zeros((model.T, n, model.D))
        A = np.zeros((model.T, n, model.n_radial * model.n_tuples))
    _check(lib().oracle_energy_forces(C.byref(cfg), _p(w), len(w), n, _p(x), _p(types), _p(box), _p(row),
                                      _p(col if len(col) else np.zeros(1, np.int32)), _p(E), _p(Ei), _p(F),
                                      _p(rho), _p(coef), _p(A)), "energy_forces")
    return Result(float(E[0]), Ei, F, rho, coef, A)


def rho_pairwise(model: Model, x, box, coef, pairs=None) -> np.ndarray:
    """rho of one layer by the multinomial-theorem formula (pins the density)."""
    x, box = _f64(x), _f64(box)
    coef = _f64(coef)
    n = len(x)
    if pairs is None:
        pairs = pairs_brute(x, box, model.r_cut, model.skin)
    row, col = np.ascontiguousarray(pairs[0], np.int64), np.ascontiguousarray(pairs[1], np.int32)
    rho = np.zeros((n, model.DR))
    cfg = model.cfg()
    _check(lib().oracle_rho_pairwise(C.byref(cfg), n, _p(x), _p(box), _p(row),
                                     _p(col if len(col) else np.zeros(1, np.int32)), _p(coef), _p(rho)),
           "rho_pairwise")
    return rho


def md_verlet(model: Model, x, v, types, box, masses, dt: float, nsteps: int):
    """Velocity Verlet; returns (x, v, epot[nsteps+1], ekin[nsteps+1])."""
    x, v, box = _f64(x).copy(), _f64(v).copy(), _f64(box)
    types = np.ascontiguousarray(types, dtype=np.int32)
    m = _f64(masses)
    ep = np.zeros(nsteps + 1)
    ek = np.zeros(nsteps + 1)
    cfg = model.cfg()
    _check(lib().oracle_md_verlet(C.byref(cfg), _p(model.weights), len(model.weights), len(x), _p(x), _p(v),
                                  _p(types), _p(box), _p(m), dt, nsteps, _p(ep), _p(ek)), "md_verlet")
    return x, v, ep, ek


def md_nvt(model: Model, x, v, types, box, masses, dt: float, nsteps: int, temperature: float, tau: float,
           noise):
    """Velocity Verlet with stochastic velocity rescaling (see reann_oracle.c);
    noise [nsteps][2] = (R1, S) per step.  Returns (x, v, epot, ekin, work),
    each energy array of length nsteps + 1."""
    x, v, box = _f64(x).copy(), _f64(v).copy(), _f64(box)
    types = np.ascontiguousarray(types, dtype=np.int32)
    m = _f64(masses)
    noise = _f64(noise).reshape(-1)
    if len(noise) < 2 * nsteps:
        raise ValueError("noise needs two numbers per step")
    ep, ek, wk = np.zeros(nsteps + 1), np.zeros(nsteps + 1), np.zeros(nsteps + 1)
    thermo = np.array([temperature, tau], np.float64)
    cfg = model.cfg()
    _check(lib().oracle_md_nvt(C.byref(cfg), _p(model.weights), len(model.weights), len(x), _p(x), _p(v), _p(types),
                               _p(box), _p(m), dt, nsteps, _p(thermo), _p(noise), _p(ep), _p(ek), _p(wk)), "md_nvt")
    return x, v, ep, ek, wk


def pairs_as_set(row, col) -> np.ndarray:
    """(i, j) pairs as one sorted int64 key array i * 2^32 + j."""
    i = np.repeat(np.arange(len(row) - 1, dtype=np.int64), np.diff(row))
    return np.sort(i * (1 << 32) + col.astype(np.int64))
