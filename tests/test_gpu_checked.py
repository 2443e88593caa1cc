"""The checked build (libreann_checked.so, REANN_CHECKED: every index read
from a neighbour list, permutation, ghost map or halo list is tested before
use) gives bit-identical energies, forces, per-atom energies and MD
trajectories to the normal build on valid inputs, and a damaged neighbour
list (host-side fault injection through reann_debug_set_neighbor; nothing
faults on the device) is reported as REANN_ERR_INDEX, after which a rebuilt
list gives the clean result again.  Each build runs in its own process
(tests/checked_worker.py).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

from molecular_dynamics_b200 import build, reann

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def _run(lib, out, *extra):
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_worker.py"), lib, out, *extra],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return dict(np.load(out))


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    d = tmp_path_factory.mktemp("checked")
    normal = _run(build.build(), str(d / "normal.npz"))
    checked = _run(build.build(checked=True), str(d / "checked.npz"), "--inject")
    return normal, checked


def test_builds_identify_themselves(results):
    normal, checked = results
    assert int(normal["checked"]) == 0 and int(checked["checked"]) == 1


def test_checked_build_is_bit_identical_on_valid_inputs(results):
    normal, checked = results
    keys = [k for k in normal if k != "checked"]
    assert len(keys) >= 20
    for k in keys:
        assert np.array_equal(normal[k], checked[k]), k


def test_damaged_list_is_reported_and_a_rebuild_recovers(results):
    _, checked = results
    assert int(checked["inj_status"]) == 10, reann.STATUS.get(int(checked["inj_status"]))
    assert np.array_equal(checked["inj_after_E"], checked["inj_clean_E"])
    assert np.array_equal(checked["inj_after_F"], checked["inj_clean_F"])
