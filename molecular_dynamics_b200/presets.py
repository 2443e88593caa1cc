"""Named workloads and model hyperparameters.

Each preset fixes the synthetic structure recipe (lattice or random
molecular placement), the REANN hyperparameters (message-passing depth T,
cutoff r_c, number of primitive Gaussian radial orbitals N_phi with their
width alpha, maximum angular momentum L, atomic-NN hidden widths) and the MD
settings.  The five presets are the workloads the REANN-MPI paper
benchmarks on ("Efficient Parallelization of Message Passing Neural Network
Potentials for Large-Scale Molecular Dynamics", Results: silver, liquid
water, the five-element high-entropy alloy, the C/H/O/N reactive mixture),
rebuilt as seeded synthetic inputs of the same shape.

Readings fixed here (the paper leaves them to its absent Supporting
Information): radial centres mu_n = r_c * n / (N_phi - 1), alpha = 1.0 A^-2,
a 1.0 A Verlet skin for every workload, tanh hidden layers, and the HEA
species Cr, Mn, Fe, Co, Ni.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Tuple

# atomic masses in amu (standard atomic weights)
MASS = {
    "H": 1.008, "C": 12.011, "N": 14.007, "O": 15.999, "Ag": 107.8682,
    "Cr": 51.996, "Mn": 54.938, "Fe": 55.845, "Co": 58.933, "Ni": 58.693,
}


@dataclass(frozen=True)
class Preset:
    key: str                    # short name, e.g. "ag256"
    index: int                  # 1-based workload number, used for seeds
    description: str
    elements: Tuple[str, ...]
    T: int                      # message-passing layers
    r_cut: float                # A
    n_radial: int               # N_phi
    l_max: int = 2              # L
    alpha: float = 1.0          # Gaussian width, A^-2
    skin: float = 1.0           # Verlet skin, A
    hidden: Tuple[int, int] = (64, 64)
    mlp_precision: int = 0      # 0 = fp32 accuracy (3xTF32 tensor cores for [64,64]), 1 = bf16 GEMMs, 2 = fp32 CUDA cores
    # structure recipe
    kind: str = "fcc"           # fcc | water | chon
    ncell: int = 0              # fcc: conventional cells per axis
    a: float = 0.0              # fcc lattice constant, A
    sigma: float = 0.0          # fcc thermal displacement, A
    n_mol: Tuple[int, ...] = ()  # water: (n_h2o,), chon: (n_c2h2, n_o2, n_n2)
    box: float = 0.0            # molecular systems: cubic box edge, A
    # MD recipe (0 steps = single energy+force evaluation)
    md_steps: int = 0
    dt_fs: float = 1.0
    temperature: float = 300.0
    # largest T the standardisation statistics cover (T sweeps)
    t_stats: int = 0
    # density features: 0 = sum_tau w A_{n,tau}^2 per (n, l) (Eq. 1);
    # 1 = sum_tau w A_{n,tau} A_{m,tau} per (n <= m, l), N_phi (N_phi+1)(L+1)/2 features
    density_form: int = 0
    # FCC: cells per axis of the lattice the standardisation statistics are
    # measured on (0 = the workload's own lattice)
    stats_ncell: int = 0

    @property
    def n_elements(self) -> int:
        return len(self.elements)

    @property
    def D(self) -> int:
        """orbital coefficients per atom, one per (n, l)"""
        return self.n_radial * (self.l_max + 1)

    @property
    def DR(self) -> int:
        """density features per atom (the networks' input width)"""
        pairs = self.n_radial * (self.n_radial + 1) // 2 if self.density_form == 1 else self.n_radial
        return pairs * (self.l_max + 1)

    @property
    def masses(self) -> Tuple[float, ...]:
        return tuple(MASS[e] for e in self.elements)

    @property
    def n_atoms(self) -> int:
        if self.kind == "fcc":
            return 4 * self.ncell ** 3
        if self.kind == "water":
            return 3 * self.n_mol[0]
        c2h2, o2, n2 = self.n_mol
        return 4 * c2h2 + 2 * o2 + 2 * n2

    @property
    def box_edge(self) -> float:
        return self.ncell * self.a if self.kind == "fcc" else self.box

    @property
    def stats_depth(self) -> int:
        return max(self.T, self.t_stats)

    def with_(self, **kw) -> "Preset":
        return replace(self, **kw)


PRESETS = {
    "ag256": Preset(
        key="ag256", index=1,
        description="Ag FCC 4x4x4 cells (256 atoms), a=4.09 A, sigma=0.05 A; single E+F",
        elements=("Ag",), T=2, r_cut=6.0, n_radial=8, hidden=(64, 64),
        kind="fcc", ncell=4, a=4.09, sigma=0.05),
    "water3k": Preset(
        key="water3k", index=2,
        description="1000 H2O at 1.0 g/cm^3 in a 31.04 A cube; 1000 velocity-Verlet steps of 0.5 fs at 300 K",
        elements=("H", "O"), T=3, r_cut=6.0, n_radial=8, hidden=(64, 64),
        kind="water", n_mol=(1000,), box=31.04, md_steps=1000, dt_fs=0.5),
    "hea108k": Preset(
        key="hea108k", index=3,
        description="5-element HEA, FCC 30x30x30 cells (108,000 atoms), a=3.60 A, sigma=0.10 A; E+F throughput",
        elements=("Cr", "Mn", "Fe", "Co", "Ni"), T=3, r_cut=5.5, n_radial=10,
        hidden=(64, 64), kind="fcc", ncell=30, a=3.60, sigma=0.10),
    "ag1m": Preset(
        key="ag1m", index=4,
        description="Ag FCC 64x64x64 cells (1,048,576 atoms), a=4.09 A, sigma=0.05 A; 200 velocity-Verlet steps of 1 fs",
        elements=("Ag",), T=3, r_cut=6.0, n_radial=8, hidden=(128, 128),
        mlp_precision=1, kind="fcc", ncell=64, a=4.09, sigma=0.05,
        md_steps=200, dt_fs=1.0, t_stats=6),
    "chon244k": Preset(
        key="chon244k", index=5,
        description="40,000 C2H2 + 40,000 O2 + 2,000 N2 (244,000 atoms) in a 200 A cube, 2.0 A gap; E+F throughput",
        elements=("H", "C", "N", "O"), T=3, r_cut=5.0, n_radial=8, hidden=(64, 64),
        kind="chon", n_mol=(40000, 40000, 2000), box=200.0),
    # pair-product density variant (D_rho = N_phi (N_phi+1)(L+1)/2 = 108 features)
    "ag256p": Preset(
        key="ag256p", index=6,
        description="Ag FCC 4x4x4 cells (256 atoms), a=4.09 A, sigma=0.05 A, pair-product densities; single E+F",
        elements=("Ag",), T=2, r_cut=6.0, n_radial=8, hidden=(64, 64),
        kind="fcc", ncell=4, a=4.09, sigma=0.05, density_form=1),
    "ag1mp": Preset(
        key="ag1mp", index=7,
        description="Ag FCC 64x64x64 cells (1,048,576 atoms), a=4.09 A, sigma=0.05 A, pair-product densities; "
                    "200 velocity-Verlet steps of 1 fs",
        elements=("Ag",), T=3, r_cut=6.0, n_radial=8, hidden=(128, 128), mlp_precision=1,
        kind="fcc", ncell=64, a=4.09, sigma=0.05, md_steps=200, dt_fs=1.0, density_form=1, stats_ncell=16),
}

ORDER = ("ag256", "water3k", "hea108k", "ag1m", "chon244k")
VARIANTS = ("ag256p", "ag1mp")
ALL = ORDER + VARIANTS


def get(key: str) -> Preset:
    return PRESETS[key]


def scaled(key: str, ncell: int | None = None, n_mol: Tuple[int, ...] | None = None,
           box: float | None = None) -> Preset:
    """A smaller structure with the same model and recipe (parity-test sizes)."""
    p = PRESETS[key]
    kw = {}
    if ncell is not None:
        kw["ncell"] = ncell
    if n_mol is not None:
        kw["n_mol"] = tuple(n_mol)
    if box is not None:
        kw["box"] = box
    return p.with_(**kw)
