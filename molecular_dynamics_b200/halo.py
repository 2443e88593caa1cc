"""Energy and forces of one system spread over several processes (GPUs): the
spatial decomposition and per-layer halo exchange of "Efficient
Parallelization of Message Passing Neural Network Potentials for Large-Scale
Molecular Dynamics", section "Parallelization Algorithm" (Figs. 3-4, Eqs. 3-5).

The box is cut into a grid of regions, one per process.  A process owns the
atoms inside its region and keeps ghost copies of the other processes' atoms
within the list radius (r_cut + skin) of its region.  Per message-passing
layer the owners send their atoms' new coefficients c^t to the processes
holding them as ghosts; in the backward sweep the partial gradients dE/dc^t
and, once, the partial forces that a process computed for its ghosts go back
to the owners and are added there.  The library (reann_halo_plan,
reann_energy_forces_halo) does the arithmetic and the row packing; this
module decides ownership and ghosts and moves the rows with torch.distributed
point-to-point messages (NCCL between GPUs, or gloo with host staging).

Nothing here computes the method: it selects atoms and moves rows.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import numpy as np

EXCHANGE_COEF, EXCHANGE_COEF_GRAD, EXCHANGE_FORCE = 0, 1, 2


class Grid:
    """A px x py x pz grid of equal regions over an orthorhombic periodic box;
    region r has coordinates (r // (py pz), (r // pz) % py, r % pz)."""

    def __init__(self, box: Sequence[float], dims: Sequence[int]):
        self.box = np.asarray(box, np.float64)
        self.dims = np.asarray(dims, np.int64)
        if self.box.shape != (3,) or self.dims.shape != (3,) or (self.dims < 1).any():
            raise ValueError("box and dims are three positive numbers")
        self.size = int(np.prod(self.dims))

    def coords(self, r: int) -> np.ndarray:
        py, pz = self.dims[1], self.dims[2]
        return np.array([r // (py * pz), (r // pz) % py, r % pz])

    def bounds(self, r: int):
        w = self.box / self.dims
        lo = self.coords(r) * w
        return lo, lo + w

    def owner(self, pos) -> np.ndarray:
        """Region of every position (wrapped into the box first)."""
        x = np.mod(np.asarray(pos, np.float64), self.box)
        c = np.minimum((x / (self.box / self.dims)).astype(np.int64), self.dims - 1)
        return (c[:, 0] * self.dims[1] + c[:, 1]) * self.dims[2] + c[:, 2]

    def distance2(self, pos, r: int) -> np.ndarray:
        """Squared periodic distance from each position to region r (0 inside)."""
        lo, hi = self.bounds(r)
        x = np.asarray(pos, np.float64)
        d2 = np.zeros(len(x))
        for a in range(3):
            L, w = self.box[a], hi[a] - lo[a]
            u = np.mod(x[:, a] - lo[a], L)            # offset from the region's lower face, [0, L)
            out = np.where(u < w, 0.0, np.minimum(u - w, L - u))
            d2 += out * out
        return d2


@dataclass
class Plan:
    """One process's halo: which own atoms go to which peer and how many
    ghosts come from each (peer order: ascending rank)."""
    n_local: int
    n_ghost: int
    send_index: np.ndarray          # own atoms, concatenated over peers
    send_counts: List[int]          # rows sent to each rank
    recv_counts: List[int]          # ghosts received from each rank


class Transport:
    """Row messages between processes with torch.distributed point-to-point
    operations.  With the gloo backend, CUDA rows are staged through host
    memory; with NCCL they move between GPUs directly, ordered on the
    current CUDA stream."""

    def __init__(self, rank: int, world: int, backend: str, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.rank, self.world, self.group = rank, world, group
        self.stage = backend == "gloo"

    def alltoallv(self, send, send_counts, recv, recv_counts):
        """recv[block q] <- what rank q sends to this rank; send[block q] -> rank q."""
        import torch
        dist = self.dist
        dev = send.device
        s = send.cpu() if (self.stage and dev.type == "cuda") else send
        r = torch.empty(recv.shape, dtype=recv.dtype) if (self.stage and dev.type == "cuda") else recv
        so = np.concatenate([[0], np.cumsum(send_counts)]).astype(np.int64)
        ro = np.concatenate([[0], np.cumsum(recv_counts)]).astype(np.int64)
        # own block: a local copy (a region next to itself through the periodic box sends nothing)
        if send_counts[self.rank]:
            r[ro[self.rank]:ro[self.rank + 1]] = s[so[self.rank]:so[self.rank + 1]]
        ops = []
        for q in range(self.world):
            if q == self.rank:
                continue
            if send_counts[q]:
                ops.append(dist.P2POp(dist.isend, s[so[q]:so[q + 1]].contiguous(), q, self.group))
            if recv_counts[q]:
                ops.append(dist.P2POp(dist.irecv, r[ro[q]:ro[q + 1]], q, self.group))
        if ops:
            for w in dist.batch_isend_irecv(ops):
                w.wait()
        if r is not recv:
            recv.copy_(r)

    def counts(self, mine: List[int]) -> List[int]:
        """All-to-all of one integer per peer: how many rows each rank sends here."""
        import torch
        dev = "cpu" if self.stage else "cuda"
        send = torch.tensor(mine, dtype=torch.int64, device=dev).reshape(-1, 1)
        recv = torch.empty_like(send)
        self.alltoallv(send, [1] * self.world, recv, [1] * self.world)
        return [int(v) for v in recv.reshape(-1).tolist()]


def make_plan(grid: Grid, rank: int, pos_own, r_list: float, transport: Transport) -> Plan:
    """Own atoms within r_list of every other region go there as ghosts."""
    send_idx = []
    for q in range(grid.size):
        if q == rank:
            send_idx.append(np.zeros(0, np.int64))
            continue
        send_idx.append(np.nonzero(grid.distance2(pos_own, q) <= r_list * r_list)[0])
    send_counts = [len(s) for s in send_idx]
    recv_counts = transport.counts(send_counts)
    return Plan(len(pos_own), int(sum(recv_counts)), np.concatenate(send_idx).astype(np.int32), send_counts,
                recv_counts)


class HaloEvaluator:
    """Energy and forces of a decomposed system from one process.

    `engine` evaluates the process's share: reann_halo_plan(n_local, n_ghost,
    send_index), reann_build_neighbors(pos, types, box) and
    reann_energy_forces_halo(pos, exchange, forces) -> own energy (the
    library's Context has these).  setup() takes this process's own atoms;
    energy_forces() returns the total energy of the system (summed over
    processes) and the forces on the own atoms."""

    def __init__(self, engine, grid: Grid, rank: int, r_list: float, transport: Transport):
        self.engine, self.grid, self.rank, self.r_list, self.t = engine, grid, rank, r_list, transport
        self.plan: Optional[Plan] = None
        self.exchanges = 0

    def _ghost_rows(self, own):
        """Ghost rows for own rows (positions, types): the send-list rows go out."""
        import torch
        p = self.plan
        sent = own[torch.as_tensor(p.send_index, dtype=torch.long, device=own.device)]
        ghost = own.new_empty((p.n_ghost,) + tuple(own.shape[1:]))
        self.t.alltoallv(sent, p.send_counts, ghost, p.recv_counts)
        return ghost

    def setup(self, pos_own, types_own):
        """pos_own: torch [n_own][3] float32, types_own: torch [n_own] int32 (own atoms)."""
        import torch
        self.plan = make_plan(self.grid, self.rank, pos_own.cpu().numpy(), self.r_list, self.t)
        p = self.plan
        self.types_all = torch.cat([types_own, self._ghost_rows(types_own.reshape(-1, 1)).reshape(-1)])
        pos_all = torch.cat([pos_own, self._ghost_rows(pos_own)])
        self.engine.reann_halo_plan(p.n_local, p.n_ghost, p.send_index)
        self.engine.reann_build_neighbors(pos_all, self.types_all, self.grid.box)
        return pos_all

    def exchange(self, kind, layer, send, recv, stream=None):
        p = self.plan
        self.exchanges += 1
        if kind == EXCHANGE_COEF:
            self.t.alltoallv(send, p.send_counts, recv, p.recv_counts)
        else:
            self.t.alltoallv(send, p.recv_counts, recv, p.send_counts)

    def energy_forces(self, pos_own, forces_own):
        """Total energy of the system (all processes) and this process's forces."""
        import torch
        pos_all = torch.cat([pos_own, self._ghost_rows(pos_own)])
        e_own = self.engine.reann_energy_forces_halo(pos_all, self.exchange, forces=forces_own)
        dev = "cpu" if self.t.stage else pos_own.device
        tot = torch.tensor([e_own], dtype=torch.float64, device=dev)
        self.t.dist.all_reduce(tot, group=self.t.group)
        return float(tot.item())


def partition(grid: Grid, pos, rank: int) -> np.ndarray:
    """Indices (in the given order) of the atoms region `rank` owns."""
    return np.nonzero(grid.owner(pos) == rank)[0]
