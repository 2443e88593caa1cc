"""ctypes binding of libreann.so (argument marshalling only).

Every entry point of include/reann.h has a method of the same name here.
Arrays may be torch tensors (CUDA or CPU; contiguous) or numpy arrays (host);
the library copies host arrays itself.  Streams default to torch's current
CUDA stream.  There is no fallback: if the library is missing, load() raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libreann.so")
CHECKED_LIB_PATH = os.path.join(HERE, "libreann_checked.so")   # built with `build --checked`

STATUS = {
    0: "REANN_OK", 1: "REANN_ERR_ARG", 2: "REANN_ERR_BOX", 3: "REANN_ERR_CAPACITY", 4: "REANN_ERR_NONFINITE",
    5: "REANN_ERR_SKIN", 6: "REANN_ERR_STATE", 7: "REANN_ERR_CUDA", 8: "REANN_ERR_TIMEOUT", 9: "REANN_ERR_UNSUPPORTED",
    10: "REANN_ERR_INDEX",
}

EXPORTS = ("reann_create", "reann_destroy", "reann_build_neighbors", "reann_energy_forces", "reann_md_step",
           "reann_md_step_nvt", "reann_get_counters", "reann_last_error", "reann_get_neighbors", "reann_get_features", "reann_profile",
           "reann_profile_read", "reann_pair_list_noalloc", "reann_halo_plan", "reann_energy_forces_halo",
           "reann_checked", "reann_debug_set_neighbor")

# kinds of the exchange function (include/reann.h)
EXCHANGE_COEF, EXCHANGE_COEF_GRAD, EXCHANGE_FORCE = 0, 1, 2
ExchangeFn = C.CFUNCTYPE(C.c_int32, C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_int64, C.c_void_p, C.c_int64,
                         C.c_int32, C.c_void_p)

KERNEL_GROUPS = ("active", "density", "mlp_fwd", "mlp_energy", "edge_bwd", "mlp_bwd", "energy_sum", "integrate",
                 "neighbors", "other", "ghost")


class ReannError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Config(C.Structure):
    _fields_ = [("n_elements", C.c_int32), ("T", C.c_int32), ("n_radial", C.c_int32), ("l_max", C.c_int32),
                ("hidden", C.c_int32 * 2), ("r_cut", C.c_double), ("skin", C.c_double), ("alpha", C.c_double),
                ("mlp_precision", C.c_int32), ("dd_grid", C.c_int32 * 3), ("dd_stale_ghosts", C.c_int32),
                ("density_form", C.c_int32)]


class MdStats(C.Structure):
    _fields_ = [("e_pot", C.c_double), ("e_kin", C.c_double), ("e_pot0", C.c_double), ("e_kin0", C.c_double),
                ("rebuilds", C.c_int64), ("steps", C.c_int64), ("e_thermostat", C.c_double)]


class Counters(C.Structure):
    _fields_ = [("n_atoms", C.c_int64), ("nnz", C.c_int64), ("capacity", C.c_int64), ("max_row", C.c_int64),
                ("active_pairs", C.c_int64), ("builds", C.c_int64), ("evaluations", C.c_int64),
                ("ghost_slots", C.c_int64), ("ghost_bytes_fwd", C.c_int64), ("ghost_bytes_bwd", C.c_int64),
                ("kernel_launches", C.c_int64), ("cells", C.c_int32 * 3), ("reserved", C.c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Loads libreann.so; raises if it is missing (no CPU fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m molecular_dynamics_b200.build`")
    lib = C.CDLL(path)
    P, I64, I32, D = C.c_void_p, C.c_int64, C.c_int32, C.c_double
    lib.reann_create.argtypes = [C.POINTER(Config), P, C.c_size_t, C.c_int, C.POINTER(P)]
    lib.reann_destroy.argtypes = [P]
    lib.reann_build_neighbors.argtypes = [P, I64, P, P, C.POINTER(D), P]
    lib.reann_energy_forces.argtypes = [P, P, C.POINTER(D), P, P, P]
    lib.reann_md_step.argtypes = [P, I32, D, P, P, C.POINTER(D), C.POINTER(MdStats), P]
    lib.reann_md_step_nvt.argtypes = [P, I32, D, D, D, C.POINTER(D), P, P, C.POINTER(D), C.POINTER(MdStats), P]
    lib.reann_get_counters.argtypes = [P, C.POINTER(Counters)]
    lib.reann_last_error.argtypes = [P]
    lib.reann_last_error.restype = C.c_char_p
    lib.reann_get_neighbors.argtypes = [P, P, P, I64, P]
    lib.reann_get_features.argtypes = [P, I32, P, P, P]
    lib.reann_profile.argtypes = [P, I32]
    lib.reann_pair_list_noalloc.argtypes = [I64, P, C.POINTER(D), D, D, P, P, I64, C.POINTER(I64), P]
    lib.reann_profile_read.argtypes = [P, I32, C.POINTER(D), C.POINTER(I64)]
    lib.reann_halo_plan.argtypes = [P, I64, I64, P, I64]
    lib.reann_energy_forces_halo.argtypes = [P, P, C.POINTER(D), P, P, ExchangeFn, P, P]
    lib.reann_checked.argtypes = []
    lib.reann_debug_set_neighbor.argtypes = [P, I64, I32]
    for name in EXPORTS:
        if name != "reann_last_error":
            getattr(lib, name).restype = C.c_int
    _lib = lib
    return lib


def _ptr(a) -> Optional[int]:
    """Data pointer of a contiguous torch tensor or numpy array (None passes through)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        if not a.flags.c_contiguous:
            raise ValueError("arrays must be C-contiguous")
        return a.ctypes.data
    if hasattr(a, "data_ptr"):
        if not a.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return a.data_ptr()
    raise TypeError(f"unsupported array type {type(a)}")


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return int(stream)
    try:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
    except ImportError:
        pass
    return None


def reann_checked() -> bool:
    """True when the loaded library is the checked build (every internal index tested before use)."""
    return bool(load().reann_checked())


def reann_pair_list_noalloc(pos, box, r_cut: float, skin: float, row, col, stream=None) -> int:
    """Allocation-free pair list into caller buffers (device tensors): row
    int32 [n+1], col int32 [cap].  Returns the list length."""
    lib = load()
    n = int(pos.shape[0])
    b = (C.c_double * 3)(*[float(x) for x in box])
    nnz = C.c_int64(0)
    st = lib.reann_pair_list_noalloc(n, _ptr(pos), b, float(r_cut), float(skin), _ptr(row), _ptr(col),
                                     int(col.shape[0]), C.byref(nnz), _stream(stream))
    if st:
        raise ReannError(st, lib.reann_last_error(None).decode())
    return nnz.value


@dataclass
class ModelSpec:
    n_elements: int
    T: int
    n_radial: int
    l_max: int
    hidden: Sequence[int]
    r_cut: float
    skin: float
    alpha: float
    mlp_precision: int = 0
    dd_grid: Sequence[int] = (0, 0, 0)
    dd_stale_ghosts: int = 0
    density_form: int = 0

    @classmethod
    def from_preset(cls, p, T: Optional[int] = None, mlp_precision: Optional[int] = None, dd_grid=(0, 0, 0),
                    dd_stale_ghosts: int = 0):
        return cls(p.n_elements, p.T if T is None else T, p.n_radial, p.l_max, tuple(p.hidden), p.r_cut, p.skin,
                   p.alpha, p.mlp_precision if mlp_precision is None else mlp_precision, tuple(dd_grid),
                   dd_stale_ghosts, getattr(p, "density_form", 0))

    @property
    def DR(self) -> int:
        """density features per atom"""
        pairs = self.n_radial * (self.n_radial + 1) // 2 if self.density_form == 1 else self.n_radial
        return pairs * (self.l_max + 1)

    def config(self) -> Config:
        c = Config()
        c.n_elements, c.T, c.n_radial, c.l_max = self.n_elements, self.T, self.n_radial, self.l_max
        c.hidden[0], c.hidden[1] = self.hidden
        c.r_cut, c.skin, c.alpha = self.r_cut, self.skin, self.alpha
        c.mlp_precision = self.mlp_precision
        for k in range(3):
            c.dd_grid[k] = self.dd_grid[k]
        c.dd_stale_ghosts = self.dd_stale_ghosts
        c.density_form = self.density_form
        return c


class _DeviceRows:
    """A float32 [rows][width] device array at a raw address, for torch.as_tensor."""

    def __init__(self, ptr: int, rows: int, width: int):
        self.__cuda_array_interface__ = {"shape": (int(rows), int(width)), "typestr": "<f4",
                                         "data": (int(ptr), False), "version": 3, "strides": None}


class Context:
    """One reann_ctx.  Methods mirror the C entry points."""

    def __init__(self, spec: ModelSpec, weights: np.ndarray, device: int = 0):
        self.lib = load()
        self.spec = spec
        w = np.ascontiguousarray(weights, dtype=np.float32)
        cfg = spec.config()
        h = C.c_void_p()
        st = self.lib.reann_create(C.byref(cfg), w.ctypes.data, w.nbytes, device, C.byref(h))
        if st:
            raise ReannError(st, self.lib.reann_last_error(None).decode())
        self.h = h
        self.n = 0

    def close(self):
        if getattr(self, "h", None):
            self.lib.reann_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _check(self, st: int):
        if st:
            raise ReannError(st, self.lib.reann_last_error(self.h).decode())

    def reann_build_neighbors(self, pos, types, box, stream=None):
        n = int(pos.shape[0])
        b = (C.c_double * 3)(*[float(x) for x in box])
        self._check(self.lib.reann_build_neighbors(self.h, n, _ptr(pos), _ptr(types), b, _stream(stream)))
        self.n = n

    def reann_energy_forces(self, pos, forces=None, atom_energy=None, stream=None) -> float:
        e = C.c_double(0.0)
        self._check(self.lib.reann_energy_forces(self.h, _ptr(pos), C.byref(e), _ptr(forces), _ptr(atom_energy),
                                                 _stream(stream)))
        return e.value

    def reann_halo_plan(self, n_local: int, n_ghost: int, send_index):
        """send_index: own atoms (caller indices < n_local) in send order, host int array."""
        idx = np.ascontiguousarray(np.asarray(send_index, np.int32).reshape(-1))
        self._check(self.lib.reann_halo_plan(self.h, int(n_local), int(n_ghost), idx.ctypes.data if len(idx) else None,
                                             len(idx)))

    def reann_energy_forces_halo(self, pos, exchange, forces=None, atom_energy=None, stream=None) -> float:
        """exchange(kind, layer, send, recv, stream): send and recv are torch
        CUDA tensors [rows][width] viewing the library's exchange buffers; it
        must fill recv (in stream order) and return nothing.  Exceptions abort
        the evaluation."""
        import torch

        errors = []

        def view(ptr, rows, width):
            if rows == 0:
                return torch.empty((0, width), dtype=torch.float32, device="cuda")
            return torch.as_tensor(_DeviceRows(ptr, rows, width), device="cuda")

        def cb(user, kind, layer, send, send_rows, recv, recv_rows, width, strm):
            try:
                exchange(kind, layer, view(send, send_rows, width), view(recv, recv_rows, width), strm)
                return 0
            except Exception as exc:   # reported after the library returns
                errors.append(exc)
                return 1

        fn = ExchangeFn(cb)
        e = C.c_double(0.0)
        st = self.lib.reann_energy_forces_halo(self.h, _ptr(pos), C.byref(e), _ptr(forces), _ptr(atom_energy), fn,
                                               None, _stream(stream))
        if errors:
            raise errors[0]
        self._check(st)
        return e.value

    def reann_md_step(self, nsteps: int, dt_fs: float, x, v, masses, stream=None) -> MdStats:
        m = (C.c_double * self.spec.n_elements)(*[float(a) for a in masses])
        st = MdStats()
        self._check(self.lib.reann_md_step(self.h, int(nsteps), float(dt_fs), _ptr(x), _ptr(v), m, C.byref(st),
                                           _stream(stream)))
        return st

    def reann_md_step_nvt(self, nsteps: int, dt_fs: float, temperature: float, tau_fs: float, noise, x, v, masses,
                          stream=None) -> MdStats:
        """noise: host array [nsteps][2] of (R1, S) per step (synth.thermostat_noise draws them)."""
        m = (C.c_double * self.spec.n_elements)(*[float(a) for a in masses])
        z = np.ascontiguousarray(np.asarray(noise, np.float64).reshape(-1))
        if len(z) < 2 * int(nsteps):
            raise ValueError("noise needs two numbers per step")
        st = MdStats()
        self._check(self.lib.reann_md_step_nvt(self.h, int(nsteps), float(dt_fs), float(temperature), float(tau_fs),
                                               z.ctypes.data_as(C.POINTER(C.c_double)), _ptr(x), _ptr(v), m,
                                               C.byref(st), _stream(stream)))
        return st

    def reann_get_counters(self) -> Counters:
        c = Counters()
        self._check(self.lib.reann_get_counters(self.h, C.byref(c)))
        return c

    def reann_last_error(self) -> str:
        return self.lib.reann_last_error(self.h).decode()

    def reann_get_neighbors(self, stream=None):
        """(row int64 [n+1], col int32 [nnz]) in the caller's order, as numpy arrays."""
        nnz = self.reann_get_counters().nnz
        row = np.zeros(self.n + 1, np.int64)
        col = np.zeros(max(nnz, 1), np.int32)
        self._check(self.lib.reann_get_neighbors(self.h, row.ctypes.data, col.ctypes.data, nnz, _stream(stream)))
        return row, col[:nnz]

    def reann_debug_set_neighbor(self, k: int, j: int):
        """Checked build only: writes j into entry k of the neighbour list (host-side fault injection)."""
        self._check(self.lib.reann_debug_set_neighbor(self.h, int(k), int(j)))

    def reann_profile(self, enable: bool = True):
        self._check(self.lib.reann_profile(self.h, 1 if enable else 0))

    def reann_profile_read(self):
        """{group name: (total ms, launches)} since the last reann_profile(True)."""
        out = {}
        for g, name in enumerate(KERNEL_GROUPS):
            ms, n = C.c_double(0.0), C.c_int64(0)
            self._check(self.lib.reann_profile_read(self.h, g, C.byref(ms), C.byref(n)))
            out[name] = (ms.value, n.value)
        return out

    def reann_get_features(self, t: int, stream=None):
        """(rho^t [n][Dr], c^t [n][D]), float32, caller order, numpy."""
        D = self.spec.n_radial * (self.spec.l_max + 1)
        rho = np.zeros((self.n, self.spec.DR), np.float32)
        coef = np.zeros((self.n, D), np.float32)
        self._check(self.lib.reann_get_features(self.h, int(t), rho.ctypes.data, coef.ctypes.data, _stream(stream)))
        return rho, coef
