"""Pins of the oracle's brute-force pair search.

The pair list is defined in the REANN-MPI paper only as "a full set of
neighbor lists" computed once and reused by every message-passing layer
(section "Parallelization Algorithm", Fig. 2 and Fig. 3a).  Pins: a second,
independent search (cell list) must give the same set; perfect FCC lattices
must give the coordination shells fixed by geometry; rows must be symmetric,
sorted and free of self pairs; a box smaller than twice the list radius is
an error.
"""
import os

import numpy as np
import pytest

import oracle
from helpers import fcc_perfect, small


@pytest.mark.parametrize("key", ["ag256", "water", "hea", "chon"])
def test_brute_equals_cell_list(key):
    p, pos, types, box = small(key)
    rb = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    rc = oracle.pairs_cells(pos, box, p.r_cut, p.skin)
    assert np.array_equal(rb[0], rc[0])
    assert np.array_equal(rb[1], rc[1])


def test_cell_list_with_many_cells():
    # 8 cells per axis: the cell stencil is the generic 27-cell one
    from molecular_dynamics_b200 import presets, synth
    q = presets.scaled("ag1m", ncell=14)
    pos, types, box = synth.make_structure(q)
    rb = oracle.pairs_brute(pos, box, q.r_cut, q.skin)
    rc = oracle.pairs_cells(pos, box, q.r_cut, q.skin)
    assert np.array_equal(rb[0], rc[0]) and np.array_equal(rb[1], rc[1])


def _fcc_shells():
    """(n, sites) of the FCC neighbour shells at squared radius n a^2 / 2, from
    the cited fixture tests/golden/fcc_shells.txt."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fcc_shells.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    return [(int(n), int(k)) for n, k in rows]


def _sites_within(a, r):
    return sum(k for n, k in _fcc_shells() if n * a * a / 2.0 < r * r)


@pytest.mark.parametrize("a,rc,listed,active", [
    (4.09, 6.0, 78, 54),   # Ag: shells below 7.0 A: 12+6+24+12+24; below 6.0 A: 12+6+24+12
    (3.60, 5.5, 86, 54),   # HEA: shells below 6.5 A add the 8 at 6.235 A; below 5.5 A: 12+6+24+12
])
def test_fcc_shell_counts(a, rc, listed, active):
    # the expected counts follow from the lattice's shells (skin 1.0 A)
    assert _sites_within(a, rc + 1.0) == listed and _sites_within(a, rc) == active
    pos, box = fcc_perfect(6, a)
    row, col = oracle.pairs_brute(pos, box, rc, 1.0)
    assert np.all(np.diff(row) == listed)
    x = pos.astype(np.float64)
    i = np.repeat(np.arange(len(x)), np.diff(row))
    d = x[col] - x[i]
    d -= box * np.rint(d / box)
    r = np.sqrt((d * d).sum(1))
    assert np.all(np.bincount(i[r < rc], minlength=len(x)) == active)


def test_rows_sorted_symmetric_no_self():
    p, pos, types, box = small("water")
    row, col = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    keys = oracle.pairs_as_set(row, col)
    i, j = keys >> 32, keys & 0xffffffff
    assert np.all(i != j)
    for a in range(len(pos)):
        r = col[row[a]:row[a + 1]]
        assert np.all(np.diff(r) > 0)
    rev = np.sort(j * (1 << 32) + i)
    assert np.array_equal(rev, keys)


def test_centre_subset_rows_match_full():
    p, pos, types, box = small("hea")
    row, col = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    cen = np.array([5, 0, 77, len(pos) - 1])
    rs, cs = oracle.pairs_brute(pos, box, p.r_cut, p.skin, centres=cen)
    for k, c in enumerate(cen):
        assert np.array_equal(cs[rs[k]:rs[k + 1]], col[row[c]:row[c + 1]])


def test_box_too_small_is_an_error():
    pos, box = fcc_perfect(3, 4.09)     # 12.27 A < 2 * 7.0 A
    with pytest.raises(RuntimeError):
        oracle.pairs_brute(pos, box, 6.0, 1.0)
    with pytest.raises(RuntimeError):
        oracle.pairs_cells(pos, box, 6.0, 1.0)


def test_threshold_is_strict_and_uses_the_fp64_expression():
    # two atoms exactly at the list radius apart are not listed; a hair closer are
    L = 20.0
    for dx, expect in ((7.0, 0), (np.nextafter(7.0, 0.0), 2)):
        x = np.array([[0.0, 1.0, 1.0], [dx, 1.0, 1.0]])
        row, col = oracle.pairs_brute(x, np.array([L, L, L]), 6.0, 1.0)
        assert len(col) == expect
