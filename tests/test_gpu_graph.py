"""CUDA-graph record/replay of mp_energy_forces: a replay (same buffers, new contents) gives the
same bits as plain launches, and counts the kernels it runs."""
import numpy as np
import pytest
import torch

from atomistic_neighbor_list_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as m
    return m


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_energy_forces_graph_replay_matches_plain_launches(mp, dtype):
    import dataclasses
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], 3000), dtype=dtype)
    pos0, _ = synth.positions_for(wl)
    n = len(pos0)
    types = torch.from_numpy(synth.atom_types(n, wl.n_types)).to(DEV)
    w = synth.make_weights(wl)
    pos = torch.from_numpy(pos0).to(DEV)
    rp, ci = mp.neighbor_csr(pos, wl.r_c)
    ctx_g = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=ci.numel())
    ctx_p = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=ci.numel())
    ctx_p.set_graphs(False)
    side = torch.cuda.Stream()
    e_g = torch.empty(1, device=DEV)
    f_g = torch.empty(n, 3, device=DEV)
    e_p = torch.empty(1, device=DEV)
    f_p = torch.empty(n, 3, device=DEV)
    shift = torch.from_numpy(np.random.default_rng(5).normal(scale=0.02, size=(n, 3)).astype(
        np.float32)).to(DEV)
    with torch.cuda.stream(side):
        for it in range(3):  # record, then replay twice with moved atoms (same CSR still valid)
            if it > 0:
                pos.add_(shift)
            l0 = ctx_g.launch_count()
            ctx_g.energy_forces(pos, types, rp, ci, energy=e_g, forces=f_g)
            lg = ctx_g.launch_count() - l0
            l1 = ctx_p.launch_count()
            ctx_p.energy_forces(pos, types, rp, ci, energy=e_p, forces=f_p)
            lp = ctx_p.launch_count() - l1
            side.synchronize()
            assert lg == lp > 0
            assert torch.equal(e_g, e_p) and torch.equal(f_g, f_p), it
            assert torch.isfinite(f_g).all()
    ctx_g.status_sync()
    ctx_p.status_sync()
