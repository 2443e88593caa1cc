"""Shared test helpers: small seeded systems and hand-made models."""
from __future__ import annotations

import numpy as np

import oracle
from molecular_dynamics_b200 import presets, synth


def small(key: str):
    """A seeded structure of the workload's recipe, small enough for brute force."""
    if key == "ag256":
        p = presets.get("ag256")
    elif key == "water":
        p = presets.scaled("water3k", n_mol=(100,), box=14.41)
    elif key == "hea":
        p = presets.scaled("hea108k", ncell=4)
    elif key == "chon":
        p = presets.scaled("chon244k", n_mol=(160, 160, 8), box=31.7)
    elif key == "ag":
        p = presets.scaled("ag1m", ncell=4)
    elif key == "agp":
        p = presets.get("ag256p")
    else:
        raise KeyError(key)
    pos, types, box = synth.make_structure(p)
    return p, pos, types, box


def model_for(p, T=None):
    T = p.T if T is None else T
    return oracle.Model.from_preset(p, synth.weight_blob(p, T=T), T=T)


def active_adjacency(pos, box, r_cut):
    """Boolean adjacency of pairs closer than r_cut (numpy, minimum image)."""
    x = pos.astype(np.float64)
    d = x[None, :, :] - x[:, None, :]
    d -= box * np.rint(d / box)
    r = np.sqrt((d * d).sum(-1))
    adj = r < r_cut
    np.fill_diagonal(adj, False)
    return adj, r


def graph_distance(adj, src):
    n = len(adj)
    dist = np.full(n, -1)
    dist[src] = 0
    frontier = [src]
    k = 0
    while frontier:
        k += 1
        nxt = np.nonzero(adj[frontier].any(0) & (dist < 0))[0]
        dist[nxt] = k
        frontier = list(nxt)
    return dist


def fcc_perfect(ncell, a):
    pos = synth.fcc_lattice(ncell, a)
    L = ncell * a
    return pos, np.array([L, L, L])
