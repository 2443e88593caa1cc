"""reann_pair_list_noalloc: the allocation-free pair list for callers that
cannot allocate device memory (programs that own the device through their own
pool or a fixed budget, and loops that must not call cudaMalloc/cudaFree,
which can synchronise the whole device).  Its scratch is a fixed device array
inside the library, so the caller only passes inputs and outputs.

The list must be bit-identical to the one the context API builds
(reann_build_neighbors + reann_get_neighbors), on two calls in a row with
different systems (the second call must not see the first call's leftovers).
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

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
