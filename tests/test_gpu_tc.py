"""Tensor-core (tcgen05) fused cfconv: layout self-check and the cases its tiling creates.

A tile holds 128 edges in CSR order; rows longer than a tile are carried across tiles, a tile with
more than 64 destination rows takes two segment-sum passes, rows without edges must come out zero.
Each case is compared with the fp64 oracle fed the bf16 values the library holds.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from atomistic_neighbor_list_b200 import synth
from helpers import TOL_BF16_FEAT, features_for, normwise, oracle_csr, oracle_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as _mp
    return _mp


def test_layout_selftest(mp):
    assert mp.selftest_tc() == (0, 0)


def run_case(mp, pos, r_c=5.0, n_rbf=50, block=0, seed=0):
    wl = dataclasses.replace(synth.WORKLOADS["cfg2"], n_atoms=len(pos), r_c=r_c, n_rbf=n_rbf,
                             n_blocks=2)
    w = synth.make_weights(wl, seed=seed + 2)
    pos_d = torch.from_numpy(np.ascontiguousarray(pos, dtype=np.float32)).cuda()
    rp, ci = mp.neighbor_csr(pos_d, r_c)
    n = len(pos)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=max(ci.numel(), 1))
    x_t, x_ref = features_for(synth.node_features(n, wl.F, seed=seed + 3), "bf16")
    out = ctx.cfconv_fwd(block, pos_d, rp, ci, x_t.cuda())
    torch.cuda.synchronize()
    ctx.status_sync()
    model = oracle.Model.from_workload(wl, oracle_weights(w, "bf16"))
    orp, oci = oracle_csr(pos, r_c, rp, ci)
    ref = oracle.cfconv(model, block, pos, orp, oci, x_ref)
    got = out.float().cpu().numpy()
    return got, ref, orp


def test_rows_longer_than_a_tile(mp):
    # r_c = 10 A at 0.1 atoms/A^3: about 400 neighbors per interior atom (3+ tiles per row)
    pos = synth.uniform_positions(2500, seed=4)
    got, ref, rp = run_case(mp, pos, r_c=10.0)
    assert np.diff(rp).max() > 3 * 128
    assert normwise(got, ref) <= TOL_BF16_FEAT


def test_two_edges_per_row_two_segment_passes(mp):
    # a straight line, spacing 4 A, cutoff 5 A: each row has at most 2 edges (64+ rows per tile)
    n = 1000
    pos = np.zeros((n, 3), dtype=np.float32)
    pos[:, 0] = 4.0 * np.arange(n)
    got, ref, rp = run_case(mp, pos)
    assert np.diff(rp).max() == 2
    assert normwise(got, ref) <= TOL_BF16_FEAT


def test_one_edge_per_row_dimers_and_isolated(mp):
    # dimers 3 A apart, dimers 50 A from each other, plus isolated atoms (empty rows)
    rng = np.random.default_rng(0)
    pos = []
    for k in range(300):
        base = np.array([50.0 * (k % 20), 50.0 * (k // 20), 0.0])
        pos.append(base)
        if k % 7 != 3:
            pos.append(base + rng.normal(size=3) * 0.3 + np.array([3.0, 0, 0]))
    pos.append(np.array([-500.0, 0, 0]))  # trailing empty row
    pos = np.array(pos, dtype=np.float32)
    got, ref, rp = run_case(mp, pos, seed=1)
    assert np.diff(rp).min() == 0 and np.diff(rp).max() == 1
    assert np.all(got[np.diff(rp) == 0] == 0)
    assert normwise(got, ref) <= TOL_BF16_FEAT


@pytest.mark.parametrize("n", [1, 2, 3, 37, 129, 700])
def test_small_and_ragged(mp, n):
    pos = synth.uniform_positions(n, seed=n)
    got, ref, rp = run_case(mp, pos, seed=2)
    if np.abs(ref).max() == 0:
        assert np.all(got == 0)
    else:
        assert normwise(got, ref) <= TOL_BF16_FEAT


def test_sixty_four_radial_functions(mp):
    pos, _ = synth.chain_replicas(4, 300, seed=3)
    got, ref, rp = run_case(mp, pos, r_c=10.0, n_rbf=64, block=1)
    assert normwise(got, ref) <= TOL_BF16_FEAT


def test_deterministic(mp):
    wl = synth.WORKLOADS["cfg2"]
    pos = synth.uniform_positions(5000, seed=9)
    w = synth.make_weights(wl)
    pos_d = torch.from_numpy(pos).cuda()
    rp, ci = mp.neighbor_csr(pos_d, wl.r_c)
    ctx = mp.Context.from_workload(wl, w, max_atoms=5000, max_edges=ci.numel())
    x = torch.from_numpy(synth.node_features(5000, wl.F)).cuda().to(torch.bfloat16)
    a = ctx.cfconv_fwd(0, pos_d, rp, ci, x)
    b = ctx.cfconv_fwd(0, pos_d, rp, ci, x)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ----------------------------------------------------------------------------- backward (forces)
def run_ef(mp, pos, r_c=5.0, n_rbf=50, seed=0):
    from helpers import TOL_BF16_FORCE, rel_rms
    wl = dataclasses.replace(synth.WORKLOADS["cfg2"], n_atoms=len(pos), r_c=r_c, n_rbf=n_rbf,
                             n_blocks=2)
    w = synth.make_weights(wl, seed=seed + 2)
    n = len(pos)
    types = synth.atom_types(n, wl.n_types, seed=seed + 1)
    pos_d = torch.from_numpy(np.ascontiguousarray(pos, dtype=np.float32)).cuda()
    rp, ci = mp.neighbor_csr(pos_d, r_c)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=max(ci.numel(), 1))
    E, F = ctx.energy_forces(pos_d, torch.from_numpy(types).cuda(), rp, ci)
    torch.cuda.synchronize()
    ctx.status_sync()
    model = oracle.Model.from_workload(wl, oracle_weights(w, "bf16"))
    orp, oci = oracle_csr(pos, r_c, rp, ci)
    Eref, Fref, e_atom = oracle.energy_forces(model, pos, types, orp, oci,
                                              return_atom_energy=True)
    e_err = abs(float(E[0]) - Eref[0]) / np.abs(e_atom).sum()
    return e_err, rel_rms(F.cpu().numpy(), Fref), TOL_BF16_FORCE


def test_forces_rows_longer_than_a_tile(mp):
    e_err, f_err, tol = run_ef(mp, synth.uniform_positions(1500, seed=4), r_c=10.0)
    assert e_err <= TOL_BF16_FEAT and f_err <= tol


def test_forces_sparse_rows_and_empty_rows(mp):
    n = 600
    pos = np.zeros((n, 3), dtype=np.float32)
    pos[:, 0] = 4.0 * np.arange(n)
    pos[::50, 1] = 300.0  # every 50th atom isolated: empty rows
    e_err, f_err, tol = run_ef(mp, pos, seed=1)
    assert e_err <= TOL_BF16_FEAT and f_err <= tol


@pytest.mark.parametrize("n", [2, 5, 130])
def test_forces_small(mp, n):
    pos = synth.uniform_positions(n, seed=n + 1)
    pos = pos * (0.5 if n < 10 else 1.0)
    e_err, f_err, tol = run_ef(mp, pos, seed=3)
    assert e_err <= TOL_BF16_FEAT and f_err <= tol


def test_forces_sixty_four_radial_functions(mp):
    pos, _ = synth.chain_replicas(3, 250, seed=2)
    e_err, f_err, tol = run_ef(mp, pos, r_c=10.0, n_rbf=64)
    assert e_err <= TOL_BF16_FEAT and f_err <= tol


# ----------------------------------------------------------------------------- bounded waits
def test_bounded_wait_timeout_is_reported_and_the_context_recovers(mp):
    """The warp-specialised cfconv kernels hand tiles between warp roles through shared-memory
    barriers, every wait bounded by the context's budget. With a zero budget the waits give up at
    once: the kernels stop their roles in order, free their tensor memory and return, and the
    status word reports MP_ERR_TIMEOUT (no trap, no fault, no hang). With the default budget
    restored the next call on the same context matches the oracle."""
    from helpers import TOL_BF16_FORCE, rel_rms
    wl = synth.scaled(synth.WORKLOADS["cfg2"], 400)
    pos = synth.uniform_positions(400, seed=21)
    types = synth.atom_types(400, wl.n_types, seed=22)
    w = synth.make_weights(wl)
    pos_d = torch.from_numpy(pos).cuda()
    types_d = torch.from_numpy(types).cuda()
    rp, ci = mp.neighbor_csr(pos_d, wl.r_c)
    ctx = mp.Context.from_workload(wl, w, max_atoms=400, max_edges=ci.numel())
    ctx.set_wait_budget(0)
    for _ in range(2):  # both cfconv directions run; a second call finds a clean context too
        ctx.energy_forces(pos_d, types_d, rp, ci)
        torch.cuda.synchronize()
        with pytest.raises(mp.MpError) as e:
            ctx.status_sync()
        assert e.value.name == "MP_ERR_TIMEOUT"
    ctx.set_wait_budget(2_000_000_000)
    E, F = ctx.energy_forces(pos_d, types_d, rp, ci)
    torch.cuda.synchronize()
    ctx.status_sync()
    model = oracle.Model.from_workload(wl, oracle_weights(w, "bf16"))
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci)
    Eref, Fref, e_atom = oracle.energy_forces(model, pos, types, orp, oci, return_atom_energy=True)
    assert abs(float(E[0]) - Eref[0]) / np.abs(e_atom).sum() <= TOL_BF16_FEAT
    assert rel_rms(F.cpu().numpy(), Fref) <= TOL_BF16_FORCE


def test_sixty_four_radial_functions_run_warp_specialised(mp):
    """The chain workload's 64 radial functions (a 16-bit Gaussian operand of 80 columns, the
    widest the tensor-core kernels take) run on the warp-specialised forward and backward."""
    wl = synth.WORKLOADS["cfg3"]
    pos, gp = synth.chain_replicas(4, 200, seed=3)
    n = len(pos)
    pos_d = torch.from_numpy(pos).cuda()
    gp_d = torch.from_numpy(gp).cuda()
    rp, ci = mp.neighbor_csr(pos_d, wl.r_c, graph_ptr=gp_d)
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=n, max_edges=ci.numel(),
                                   max_graphs=4)
    types = torch.from_numpy(synth.atom_types(n, wl.n_types)).cuda()
    ctx.profile_begin()
    ctx.energy_forces(pos_d, types, rp, ci, gp_d)
    prof = ctx.profile_end()
    ctx.status_sync()
    assert "cfconv_fwd_tc" in prof and "cfconv_bwd_tc" in prof, prof


def test_few_radial_functions_run_on_the_cuda_cores(mp):
    """Eight radial functions (a 16-column operand, below the tensor-core kernels' 32 to 80) take
    the bf16 path on the CUDA-core kernels, and energy and forces match the oracle."""
    pos = synth.uniform_positions(600, seed=6)
    wl = dataclasses.replace(synth.WORKLOADS["cfg2"], n_atoms=600, n_rbf=8)
    rp, ci = mp.neighbor_csr(torch.from_numpy(pos).cuda(), wl.r_c)
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=600, max_edges=ci.numel())
    ctx.profile_begin()
    ctx.energy_forces(torch.from_numpy(pos).cuda(),
                      torch.from_numpy(synth.atom_types(600, wl.n_types)).cuda(), rp, ci)
    prof = ctx.profile_end()
    ctx.status_sync()
    assert "cfconv_fwd_simt" in prof and "cfconv_fwd_tc" not in prof, prof
    e_err, f_err, tol = run_ef(mp, pos, n_rbf=8)
    assert e_err <= TOL_BF16_FEAT and f_err <= tol
