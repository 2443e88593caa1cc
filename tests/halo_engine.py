"""An fp64 numpy stand-in for the library's share of a decomposed evaluation
(reann_halo_plan / reann_build_neighbors / reann_energy_forces_halo), so that
the multi-process halo driver can be run as gloo ranks on the CPU.

TEST INFRASTRUCTURE ONLY.  It evaluates a process's own atoms the way the
method prescribes ("Efficient Parallelization of Message Passing Neural
Network Potentials for Large-Scale Molecular Dynamics", section "REANN
Architecture", Eqs. 1-2; section "Parallelization Algorithm", Eqs. 3-5):
densities of own atoms from own and ghost neighbours, coefficient networks of
own atoms, and a scatter-form backward over the edges from own atoms, whose
ghost-side gradients are handed to the exchange function -- at the same
points and in the same row layout as the library.  It shares no code with the
oracle or the CUDA path; the weights come from the blob layout.
"""
from __future__ import annotations

import numpy as np
import torch

from molecular_dynamics_b200 import synth

TUPLES = [(0, 0, 0), (1, 0, 0), (0, 1, 0), (0, 0, 1), (2, 0, 0), (0, 2, 0), (0, 0, 2), (1, 1, 0), (1, 0, 1), (0, 1, 1)]
L_OF = np.array([sum(t) for t in TUPLES])
W_TAU = np.array([1, 1, 1, 1, 1, 1, 1, 2, 2, 2], np.float64)   # l!/(lx! ly! lz!)
EXCHANGE_COEF, EXCHANGE_COEF_GRAD, EXCHANGE_FORCE = 0, 1, 2


class _Net:
    def __init__(self, blob, spec):
        g = lambda k: blob[spec[k][0]:spec[k][0] + int(np.prod(spec[k][1]))].reshape(spec[k][1]).astype(np.float64)
        self.shift, self.scale = g("shift"), g("scale")
        self.W1, self.b1, self.W2, self.b2, self.W3, self.b3 = g("W1"), g("b1"), g("W2"), g("b2"), g("W3"), g("b3")

    def forward(self, x):
        """x [m][Dr] -> (y [m][n_out], cache)"""
        xt = (x - self.shift) / self.scale
        a1 = np.tanh(xt @ self.W1.T + self.b1)
        a2 = np.tanh(a1 @ self.W2.T + self.b2)
        return a2 @ self.W3.T + self.b3, (a1, a2)

    def vjp(self, cache, gy):
        a1, a2 = cache
        g2 = (gy @ self.W3) * (1 - a2 * a2)
        g1 = (g2 @ self.W2) * (1 - a1 * a1)
        return (g1 @ self.W1) / self.scale


class NumpyHaloEngine:
    def __init__(self, p, weights, T=None):
        self.p, self.T = p, p.T if T is None else T
        self.NP, self.D, self.ne = p.n_radial, p.D, p.n_elements
        lay = synth.blob_layout(p, self.T)
        w = np.asarray(weights)
        self.C0 = w[:self.ne * self.D].reshape(self.ne, self.D).astype(np.float64)
        self.coef = [[_Net(w, lay["coef"][t][e]) for e in range(self.ne)] for t in range(self.T - 1)]
        self.energy = [_Net(w, lay["energy"][e]) for e in range(self.ne)]
        self.exchanges = []

    def reann_halo_plan(self, n_local, n_ghost, send_index):
        self.n_local, self.n_ghost = int(n_local), int(n_ghost)
        self.send_index = np.asarray(send_index, np.int64)

    def reann_build_neighbors(self, pos, types, box):
        self.types = np.asarray(types.cpu() if hasattr(types, "cpu") else types, np.int64).reshape(-1)
        self.box = np.asarray(box, np.float64)

    def _nets(self, nets, types, x):
        """per-element networks over rows x: outputs and caches"""
        out, caches = None, {}
        for e in range(self.ne):
            m = types == e
            if not m.any():
                continue
            y, cache = nets[e].forward(x[m])
            if out is None:
                out = np.zeros((len(x), y.shape[1]))
            out[m] = y
            caches[e] = (m, cache)
        return out, caches

    def _vjp(self, nets, caches, gy, width):
        g = np.zeros((len(gy), width))
        for e, (m, cache) in caches.items():
            g[m] = nets[e].vjp(cache, gy[m])
        return g

    def reann_energy_forces_halo(self, pos, exchange, forces=None, **_):
        p, NP, D, T, nl = self.p, self.NP, self.D, self.T, self.n_local
        x = np.asarray(pos.cpu() if hasattr(pos, "cpu") else pos, np.float64)
        n = len(x)
        # edges from own atoms to every atom closer than r_cut (minimum image)
        d = x[None, :, :] - x[:nl, None, :]
        d -= self.box * np.rint(d / self.box)
        r = np.sqrt((d * d).sum(-1))
        ii, jj = np.nonzero(r < p.r_cut)
        keep = ii != jj
        ii, jj = ii[keep], jj[keep]
        dv, rv = d[ii, jj], r[ii, jj]
        mu = p.r_cut * np.arange(NP) / (NP - 1)
        fc = 0.5 * (np.cos(np.pi * rv / p.r_cut) + 1)
        dfc = -0.5 * np.pi / p.r_cut * np.sin(np.pi * rv / p.r_cut)
        gs = np.exp(-p.alpha * (rv[:, None] - mu) ** 2)
        phi = gs * fc[:, None]
        dphi = gs * (-2 * p.alpha * (rv[:, None] - mu) * fc[:, None] + dfc[:, None])
        ex = np.array(TUPLES)
        Y = np.prod(dv[:, None, :] ** ex[None], axis=2)                      # [e][tau]
        dY = np.zeros(Y.shape + (3,))
        for a in range(3):
            e2 = ex.copy()
            e2[:, a] = np.maximum(e2[:, a] - 1, 0)
            dY[:, :, a] = ex[:, a] * np.prod(dv[:, None, :] ** e2[None], axis=2)
        feat = L_OF[None, :] * NP + np.arange(NP)[:, None]                   # [n][tau] -> feature index

        c = np.zeros((T, n, D))
        c[0] = self.C0[self.types]
        A, rho, caches = [], [], []
        own_types = self.types[:nl]
        for t in range(T):
            Ai = np.zeros((nl, NP, len(TUPLES)))
            contrib = c[t][jj][:, feat] * phi[:, :, None] * Y[:, None, :]    # [e][n][tau]
            np.add.at(Ai, ii, contrib)
            rh = np.zeros((nl, D))
            for n_ in range(NP):
                for tau in range(len(TUPLES)):
                    rh[:, L_OF[tau] * NP + n_] += W_TAU[tau] * Ai[:, n_, tau] ** 2
            A.append(Ai)
            rho.append(rh)
            if t + 1 < T:
                y, cache = self._nets(self.coef[t], own_types, rh)
                caches.append(cache)
                c[t + 1][:nl] = y
                recv = np.zeros((self.n_ghost, D))
                exchange(EXCHANGE_COEF, t + 1, torch.from_numpy(np.ascontiguousarray(c[t + 1][self.send_index])),
                         torch.from_numpy(recv), None)
                c[t + 1][nl:] = recv
        Ei, ecache = self._nets(self.energy, own_types, rho[T - 1])
        g = self._vjp(self.energy, ecache, np.ones((nl, 1)), D)             # dE/drho^{T-1}
        gx = np.zeros((n, 3))
        for t in range(T - 1, -1, -1):
            G = 2 * W_TAU[None, None, :] * A[t] * g[:, feat]                   # dE/dA [own][n][tau]
            Ge = G[ii]                                                         # [e][n][tau]
            dc = np.zeros((n, D))
            np.add.at(dc, (jj[:, None, None], feat[None]), Ge * phi[:, :, None] * Y[:, None, :])
            cj = c[t][jj][:, feat]
            V = ((Ge * cj)[..., None] * (dphi[:, :, None, None] * (dv / rv[:, None])[:, None, None, :] * Y[:, None, :, None]
                                          + phi[:, :, None, None] * dY[:, None, :, :])).sum(axis=(1, 2))
            np.add.at(gx, jj, V)
            np.add.at(gx, ii, -V)
            if t >= 1:
                recv = np.zeros((len(self.send_index), D))
                exchange(EXCHANGE_COEF_GRAD, t, torch.from_numpy(np.ascontiguousarray(dc[nl:])), torch.from_numpy(recv),
                         None)
                np.add.at(dc, self.send_index, recv)
                g = self._vjp(self.coef[t - 1], caches[t - 1], dc[:nl], D)
        F = -gx
        recv = np.zeros((len(self.send_index), 3))
        exchange(EXCHANGE_FORCE, 0, torch.from_numpy(np.ascontiguousarray(F[nl:])), torch.from_numpy(recv), None)
        np.add.at(F, self.send_index, recv)
        if forces is not None:
            forces[:] = torch.from_numpy(F[:nl])
        return float(Ei.sum())
