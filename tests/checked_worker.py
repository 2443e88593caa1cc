"""Runs a fixed set of small energy+force, domain-decomposed and MD cases
through one build of the library and saves every output (test helper for
test_gpu_checked.py; one process per build, since a process loads one
library).

    python tests/checked_worker.py <library.so> <out.npz> [--inject]

--inject (checked build only): damages one neighbour-list entry through
reann_debug_set_neighbor and records the status of the next evaluation,
then the outputs after the list is rebuilt.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import numpy as np  # noqa: E402


def main(lib_path, out_path, inject):
    import torch
    from helpers import small
    from molecular_dynamics_b200 import reann, synth
    reann.load(lib_path)
    out = {"checked": np.array(int(reann.reann_checked()))}

    def run(tag, p, pos, types, box, mlp_precision=0, dd_grid=(0, 0, 0)):
        spec = reann.ModelSpec.from_preset(p, mlp_precision=mlp_precision, dd_grid=dd_grid)
        ctx = reann.Context(spec, synth.weight_blob(p))
        pd = torch.from_numpy(np.ascontiguousarray(pos, np.float32)).cuda()
        td = torch.from_numpy(np.ascontiguousarray(types, np.int32)).cuda()
        ctx.reann_build_neighbors(pd, td, box)
        F = torch.empty_like(pd)
        Ei = torch.empty(len(pos), dtype=torch.float32, device="cuda")
        E = ctx.reann_energy_forces(pd, F, Ei)
        out[tag + "_E"] = np.array(E)
        out[tag + "_F"] = F.cpu().numpy()
        out[tag + "_Ei"] = Ei.cpu().numpy()
        return ctx, pd, td, F, Ei

    for key, prec in (("ag", 0), ("ag", 1), ("water", 0), ("hea", 0), ("chon", 0)):
        p, pos, types, box = small(key)
        run(f"{key}{prec}", p, pos, types, box, mlp_precision=prec)
    p, pos, types, box = small("ag")
    run("ag_dd", p, pos, types, box, dd_grid=(2, 2, 2))

    # a few velocity-Verlet steps
    spec = reann.ModelSpec.from_preset(p)
    ctx = reann.Context(spec, synth.weight_blob(p))
    pd = torch.from_numpy(np.ascontiguousarray(pos, np.float32)).cuda()
    ctx.reann_build_neighbors(pd, torch.from_numpy(types).cuda(), box)
    x = torch.from_numpy(pos.astype(np.float64)).cuda()
    v = torch.from_numpy(synth.maxwell_boltzmann(p, types)).cuda()
    st = ctx.reann_md_step(5, 1.0, x, v, p.masses)
    out["md_x"], out["md_v"] = x.cpu().numpy(), v.cpu().numpy()
    out["md_E"] = np.array([st.e_pot, st.e_kin])

    if inject:
        ctx, pd, td, F, Ei = run("inj_clean", p, pos, types, box)
        n = len(pos)
        ctx.reann_debug_set_neighbor(5, n + 1000)
        try:
            ctx.reann_energy_forces(pd, F, Ei)
            out["inj_status"] = np.array(0)
        except reann.ReannError as e:
            out["inj_status"] = np.array(e.status)
        ctx.reann_build_neighbors(pd, td, box)
        E = ctx.reann_energy_forces(pd, F, Ei)
        out["inj_after_E"] = np.array(E)
        out["inj_after_F"] = F.cpu().numpy()
    torch.cuda.synchronize()
    np.savez(out_path, **out)


if __name__ == "__main__":
    main(sys.argv[1], sys.argv[2], "--inject" in sys.argv[3:])
