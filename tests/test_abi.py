"""The C ABI library builds, loads and exports every symbol include/reann.h
declares; argument validation that needs no GPU returns the documented
status codes.  No compute call is made here (this file runs without a GPU).
"""
import ctypes as C
import os
import re

import numpy as np
import pytest

from molecular_dynamics_b200 import build, presets, reann, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "reann.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(reann_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return reann.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("reann_create", "reann_destroy", "reann_build_neighbors", "reann_energy_forces",
                     "reann_md_step", "reann_get_counters", "reann_last_error"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(reann.EXPORTS)


def test_normal_build_is_unchecked_and_refuses_fault_injection(lib):
    assert lib.reann_checked() == 0
    assert lib.reann_debug_set_neighbor(None, 0, 0) == 1


def test_checked_build_exports_the_same_symbols():
    path = build.build(checked=True)
    clib = C.CDLL(path)
    for name in declared_functions():
        assert hasattr(clib, name), name
    clib.reann_checked.restype = C.c_int32
    assert clib.reann_checked() == 1


def test_create_rejects_bad_blob_size_without_touching_the_gpu(lib):
    p = presets.get("ag256")
    w = synth.weight_blob(p)
    cfg = reann.ModelSpec.from_preset(p).config()
    h = C.c_void_p()
    st = lib.reann_create(C.byref(cfg), w.ctypes.data, w.nbytes - 4, 0, C.byref(h))
    assert st == 1 and not h.value
    assert b"weight blob size" in lib.reann_last_error(None)


def test_create_rejects_unsupported_and_invalid_configs(lib):
    p = presets.get("ag256")
    w = synth.weight_blob(p)
    for field, value, expect in (("n_radial", 7, 9), ("l_max", 1, 9), ("T", 0, 1), ("n_elements", 0, 1),
                                 ("mlp_precision", 3, 1), ("mlp_precision", -1, 1)):
        cfg = reann.ModelSpec.from_preset(p).config()
        setattr(cfg, field, value)
        h = C.c_void_p()
        assert lib.reann_create(C.byref(cfg), w.ctypes.data, w.nbytes, 0, C.byref(h)) == expect, field
        assert not h.value


def test_null_context_is_rejected(lib):
    assert lib.reann_destroy(None) == 0
    assert lib.reann_get_counters(None, None) == 1
    m = (C.c_double * 1)(107.8682)
    noise = (C.c_double * 2)(0.0, 1.0)
    assert lib.reann_md_step(None, 1, 1.0, None, None, m, None, None) == 1
    assert lib.reann_md_step_nvt(None, 1, 1.0, 300.0, 10.0, noise, None, None, m, None, None) == 1


def test_md_stats_layout_matches_the_header():
    # the ctypes mirror of reann_md_stats has the header's fields in order
    import re
    from pathlib import Path
    hdr = (Path(__file__).resolve().parent.parent / "include" / "reann.h").read_text()
    block = re.search(r"typedef struct \{([^}]*)\} reann_md_stats;", hdr).group(1)
    names = re.findall(r"^\s*(?:double|int64_t)\s+(\w+);", block, re.M)
    assert names == [f[0] for f in reann.MdStats._fields_]


def test_blob_layout_matches_the_header(lib):
    # the size formula of include/reann.h and synth.blob_layout agree
    for key in presets.ORDER:
        p = presets.get(key)
        lay = synth.blob_layout(p, p.T)
        D, (H1, H2), ne = p.D, p.hidden, p.n_elements
        net = lambda o: 2 * D + H1 * D + H1 + H2 * H1 + H2 + o * H2 + o
        assert lay["total"] == ne * D + (p.T - 1) * ne * net(D) + ne * net(1)
