"""reann_pair_list_noalloc: the allocation-free pair list for callers that
cannot allocate device memory (programs that own the device through their own
pool or a fixed budget, and loops that must not call cudaMalloc/cudaFree,
which can synchronise the whole device).  Its scratch is a fixed device array
inside the library, so the caller only passes inputs and outputs.

The list must be bit-identical to the one the context API builds
(reann_build_neighbors + reann_get_neighbors) and to the oracle's brute-force
list, on two calls in a row with different systems (the second call must not
see the first call's leftovers), on a sparse box whose cell grid exceeds the
scratch (coarser cells) and on an empty system.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import torch_cuda
from helpers import small
from molecular_dynamics_b200 import presets, reann, synth

pytestmark = pytest.mark.gpu


def _context_list(p, pos, types, box):
    ctx = reann.Context(reann.ModelSpec.from_preset(p, mlp_precision=0), synth.weight_blob(p))
    ctx.reann_build_neighbors(pos, types, box)
    return ctx.reann_get_neighbors()


def _noalloc_list(torch, p, pos, box, cap):
    pos_d = torch.from_numpy(np.ascontiguousarray(pos, np.float32)).cuda()
    row = torch.full((len(pos) + 1,), -1, dtype=torch.int32, device="cuda")
    col = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    nnz = reann.reann_pair_list_noalloc(pos_d, box, p.r_cut, p.skin, row, col)
    torch.cuda.synchronize()
    return nnz, row.cpu().numpy().astype(np.int64), col.cpu().numpy()[:nnz]


def test_two_calls_match_the_context_api():
    torch = torch_cuda()
    big = presets.scaled("hea108k", ncell=7)                 # 1,372 atoms, 5 elements
    cases = [(big, *synth.make_structure(big)), small("chon")]  # then 976 gas atoms
    for p, pos, types, box in cases:
        row_ref, col_ref = _context_list(p, pos, types, box)
        nnz, row, col = _noalloc_list(torch, p, pos, box, cap=len(col_ref) + 64)
        assert nnz == len(col_ref)
        assert np.array_equal(row, row_ref)
        assert np.array_equal(col, col_ref)
        row_o, col_o = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
        assert np.array_equal(row, row_o)
        assert np.array_equal(col, col_o)


def test_sparse_box_with_coarsened_cells_and_empty_input():
    """400 atoms in 40 tight clusters (some across the periodic faces) in a
    250 A cube: 35 cells of 7 A per axis exceed the scratch's cell count, so
    the call halves the widest axis; the list must still equal brute force.
    Then n = 0: row[0] = 0 and an empty list."""
    torch = torch_cuda()
    p = presets.get("chon244k")
    rng = np.random.default_rng(7001)
    L = 250.0
    centres = rng.uniform(0.0, L, (40, 3))
    centres[:8, 0] = rng.uniform(-1.0, 1.0, 8)              # straddling x = 0 / L
    pos = (centres[:, None, :] + rng.normal(0.0, 2.0, (40, 10, 3))).reshape(-1, 3)
    pos = np.mod(pos, L).astype(np.float32)
    box = np.array([L, L, L])
    row_o, col_o = oracle.pairs_brute(pos, box, p.r_cut, p.skin)
    assert len(col_o) > 1000
    nnz, row, col = _noalloc_list(torch, p, pos, box, cap=len(col_o) + 8)
    assert nnz == len(col_o)
    assert np.array_equal(row, row_o)
    assert np.array_equal(col, col_o)

    row0 = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    col0 = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    pos0 = torch.zeros((0, 3), dtype=torch.float32, device="cuda")
    assert reann.reann_pair_list_noalloc(pos0, box, p.r_cut, p.skin, row0, col0) == 0
    torch.cuda.synchronize()
    assert int(row0.item()) == 0
    assert (col0.cpu().numpy() == -1).all()


def test_rejects_lists_beyond_int32_offsets():
    """70,000 atoms in a 14 A cube (twice the list radius): about half of all
    ordered pairs, 2.5e9 entries, lie within 7 A -- more than int32 row offsets
    can address.  The call must say so before writing col."""
    torch = torch_cuda()
    rng = np.random.default_rng(7002)
    pos = torch.from_numpy(rng.uniform(0.0, 14.0, (70000, 3)).astype(np.float32)).cuda()
    row = torch.zeros(70001, dtype=torch.int32, device="cuda")
    col = torch.full((16,), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(reann.ReannError) as e:
        reann.reann_pair_list_noalloc(pos, [14.0, 14.0, 14.0], 6.0, 1.0, row, col)
    assert e.value.status == 3 and "2^31-1" in str(e.value)
    assert (col.cpu().numpy() == -1).all()


def test_rejects_sizes_beyond_the_maximum():
    torch = torch_cuda()
    pos = torch.zeros((131073, 3), dtype=torch.float32, device="cuda")
    row = torch.zeros(131074, dtype=torch.int32, device="cuda")
    col = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(reann.ReannError) as e:
        reann.reann_pair_list_noalloc(pos, [300.0, 300.0, 300.0], 6.0, 1.0, row, col)
    assert e.value.status == 3 and "at most 131072 atoms" in str(e.value)


def test_short_output_reports_the_needed_length():
    torch = torch_cuda()
    p, pos, types, box = small("water")
    row_ref, col_ref = _context_list(p, pos, types, box)
    pos_d = torch.from_numpy(pos).cuda()
    row = torch.zeros(len(pos) + 1, dtype=torch.int32, device="cuda")
    col = torch.zeros(10, dtype=torch.int32, device="cuda")
    with pytest.raises(reann.ReannError) as e:
        reann.reann_pair_list_noalloc(pos_d, box, p.r_cut, p.skin, row, col)
    assert e.value.status == 3 and str(len(col_ref)) in str(e.value)
