"""Undirected-pair cfconv (mp_pair_plan + mp_cfconv_fwd_pairs) against the fp64 oracle.

The pair path evaluates the filter once per pair {i, j} and sends both messages from it; its rows
are the directed cfconv's sums. The oracle side is oracle.cfconv_pairs (the same definition
written per pair, pinned against the directed form) on the whole system, or oracle.cfconv on
sampled rows where the system is too large for it; inputs are the seeded generator's, the neighbor
list is checked bit for bit against the oracle's own. Tolerance: the bf16 feature bound
(normwise 2e-2). Also: empty rows, a ragged last 128-atom block, atoms in no spatial order (many
block pairs), a list with no pairs, bitwise repeatability, and the plan's error paths.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from atomistic_neighbor_list_b200 import synth
from helpers import TOL_BF16_FEAT, features_for, normwise, oracle_csr, oracle_weights

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as _mp
    return _mp


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def system(mp, key, n, order=True, seed=0):
    wl = dataclasses.replace(synth.WORKLOADS[key], dtype="bf16")
    pos, gp = synth.positions_for(synth.scaled(wl, n) if wl.geometry == "uniform" else wl, seed)
    gpd = dev(gp) if len(gp) > 2 else None
    if order:
        perm = mp.spatial_order(dev(pos), wl.r_c, graph_ptr=gpd).cpu().numpy()
        pos = np.ascontiguousarray(pos[perm])
    rp, ci = mp.neighbor_csr(dev(pos), wl.r_c, graph_ptr=gpd)
    return wl, pos, gp, rp, ci


def run_pairs(mp, wl, pos, rp, ci, block=0, seed=0, validate=False):
    n = len(pos)
    w = synth.make_weights(wl)
    ctx = mp.Context.from_workload(wl, w, max_atoms=max(n, 1), max_edges=max(ci.numel(), 1),
                                   validate=validate)
    ctx.pair_plan(rp, ci)
    x_t, x_ref = features_for(synth.node_features(n, wl.F, seed=seed), wl.dtype)
    out = ctx.cfconv_fwd_pairs(block, dev(pos), x_t.to(DEV))
    torch.cuda.synchronize()
    ctx.status_sync()
    return ctx, w, x_t, x_ref, out


@pytest.mark.parametrize("key,n,order", [("cfg2", 700, True), ("cfg2", 3000, True),
                                         ("cfg2", 10_000, True), ("cfg2", 3000, False)])
def test_pair_cfconv_matches_oracle(mp, key, n, order):
    wl, pos, gp, rp, ci = system(mp, key, n, order)
    ctx, w, x_t, x_ref, out = run_pairs(mp, wl, pos, rp, ci, block=1)
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    ref = oracle.cfconv_pairs(model, 1, pos, orp, oci, x_ref)
    assert normwise(out.float().cpu().numpy(), ref) <= TOL_BF16_FEAT
    # and the directed kernel on the same list gives the same rows within the same bound
    d = ctx.cfconv_fwd(1, dev(pos), rp, ci, x_t.to(DEV))
    torch.cuda.synchronize()
    assert normwise(out.float().cpu().numpy(), d.float().cpu().numpy()) <= TOL_BF16_FEAT


def test_pair_cfconv_full_100k_sampled(mp):
    wl, pos, gp, rp, ci = system(mp, "cfg5", 100_000)
    ctx, w, x_t, x_ref, out = run_pairs(mp, wl, pos, rp, ci, block=2)
    rows = np.sort(np.random.default_rng(7).choice(len(pos), 3000, replace=False))
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    ref = oracle.cfconv(model, 2, pos, orp, oci, x_ref, rows=rows)
    assert normwise(out.float().cpu().numpy()[rows], ref) <= TOL_BF16_FEAT


def test_pair_cfconv_chains_sixty_four_radial_functions(mp):
    # 64 chains of 1,000 beads, n_rbf = 64 (the wider Gaussian operand, one buffer), sampled rows
    wl, pos, gp, rp, ci = system(mp, "cfg3", 64_000)
    ctx, w, x_t, x_ref, out = run_pairs(mp, wl, pos, rp, ci, block=1)
    rows = np.sort(np.random.default_rng(8).choice(len(pos), 4000, replace=False))
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci, gp)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    ref = oracle.cfconv(model, 1, pos, orp, oci, x_ref, rows=rows)
    assert normwise(out.float().cpu().numpy()[rows], ref) <= TOL_BF16_FEAT


def test_pair_cfconv_deterministic_and_empty_rows(mp):
    wl = dataclasses.replace(synth.WORKLOADS["cfg2"], dtype="bf16")
    pos = synth.uniform_positions(300, seed=2) * np.float32(0.6)
    pos[5] = [900.0, 900.0, 900.0]   # isolated: an empty row inside the first block
    pos[299] = [-900.0, 0.0, 0.0]    # isolated last atom of the ragged last block
    rp, ci = mp.neighbor_csr(dev(pos), wl.r_c)
    ctx, w, x_t, x_ref, o1 = run_pairs(mp, wl, pos, rp, ci)
    o2 = ctx.cfconv_fwd_pairs(0, dev(pos), x_t.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.all(o1[5] == 0) and torch.all(o1[299] == 0)
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    ref = oracle.cfconv_pairs(model, 0, pos, orp, oci, x_ref)
    assert normwise(o1.float().cpu().numpy(), ref) <= TOL_BF16_FEAT


def test_pair_cfconv_list_without_pairs(mp):
    wl = dataclasses.replace(synth.WORKLOADS["cfg2"], dtype="bf16")
    pos = (np.arange(200 * 3, dtype=np.float32).reshape(200, 3) * 10.0)  # all farther than r_c
    rp, ci = mp.neighbor_csr(dev(pos), wl.r_c)
    assert ci.numel() == 0
    ctx, w, x_t, x_ref, out = run_pairs(mp, wl, pos, rp, ci)
    assert torch.all(out == 0)


def test_pair_plan_checks(mp):
    wl, pos, gp, rp, ci = system(mp, "cfg2", 500)
    w = synth.make_weights(wl)
    ctx = mp.Context.from_workload(wl, w, max_atoms=600, max_edges=ci.numel() + 8, validate=True)
    x = dev(synth.node_features(500, wl.F)).to(torch.bfloat16)
    with pytest.raises(mp.MpError) as e:  # no plan yet
        ctx.cfconv_fwd_pairs(0, dev(pos), x)
    assert e.value.name == "MP_ERR_INVALID_ARG"
    # an edge whose reverse is missing: the symmetric-list contract, checked under validate
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy()
    keep = np.ones(len(ci_h), dtype=bool)
    keep[0] = False
    rp_b = rp_h.copy()
    rp_b[1:] -= 1
    with pytest.raises(mp.MpError) as e:
        ctx.pair_plan(dev(rp_b), dev(ci_h[keep]))
    assert e.value.name == "MP_ERR_CSR_NOT_SYMMETRIC"
    ctx.pair_plan(rp, ci)
    ctx.cfconv_fwd_pairs(0, dev(pos), x)
    with pytest.raises(mp.MpError) as e:  # a plan of another N
        ctx.cfconv_fwd_pairs(0, dev(pos[:400]), x[:400])
    assert e.value.name == "MP_ERR_INVALID_ARG"


def test_pair_cfconv_needs_the_tensor_core_configuration(mp):
    wl = synth.WORKLOADS["cfg1"]  # fp32, F = 64
    pos = synth.uniform_positions(100, seed=1)
    rp, ci = mp.neighbor_csr(dev(pos), wl.r_c)
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=100,
                                   max_edges=ci.numel())
    ctx.pair_plan(rp, ci)
    with pytest.raises(mp.MpError) as e:
        ctx.cfconv_fwd_pairs(0, dev(pos), dev(synth.node_features(100, wl.F)))
    assert e.value.name == "MP_ERR_UNIMPLEMENTED"


def test_energy_forces_uses_the_plan_of_its_own_list(mp):
    # with a plan of the very buffers it is given, energy + forces run the pair forward (the
    # profile shows it) and agree with the oracle; on a copy of the list they run the directed
    # kernels and repeat the plan-free result bit for bit
    from helpers import TOL_BF16_FORCE, rel_rms
    wl, pos, gp, rp, ci = system(mp, "cfg2", 3000)
    n = len(pos)
    w = synth.make_weights(wl)
    types = synth.atom_types(n, wl.n_types)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=ci.numel())
    pd, td = dev(pos), dev(types)
    e0, f0 = ctx.energy_forces(pd, td, rp, ci)
    e0, f0 = e0.clone(), f0.clone()
    ctx.pair_plan(rp, ci)
    ctx.profile_begin()
    e1, f1 = ctx.energy_forces(pd, td, rp, ci)
    prof = ctx.profile_end()
    e1, f1 = e1.clone(), f1.clone()
    assert "cfconv_pair_tc" in prof and "cfconv_fwd_tc" not in prof
    rp2, ci2 = rp.clone(), ci.clone()
    ctx.profile_begin()
    e2, f2 = ctx.energy_forces(pd, td, rp2, ci2)
    prof2 = ctx.profile_end()
    torch.cuda.synchronize()
    ctx.status_sync()
    assert "cfconv_fwd_tc" in prof2 and "cfconv_pair_tc" not in prof2
    assert torch.equal(e2, e0) and torch.equal(f2, f0)
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    Eref, Fref, e_atom = oracle.energy_forces(model, pos, types, orp, oci, return_atom_energy=True)
    assert abs(float(e1[0]) - Eref[0]) <= 2e-2 * np.abs(e_atom).sum()
    assert rel_rms(f1.cpu().numpy(), Fref) <= TOL_BF16_FORCE


def test_pair_plan_reports_a_block_with_too_many_pairs(mp):
    # a complete graph on 800 atoms: rows 0-127 hold 94,144 upper pairs, more than one block's
    # sort holds; the plan reports the capacity error, leaves no plan behind, and the context goes
    # on (its status word clear)
    n = 800
    rows = [np.delete(np.arange(n), i) for i in range(n)]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    wl = dataclasses.replace(synth.WORKLOADS["cfg2"], dtype="bf16")
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=n, max_edges=len(ci))
    with pytest.raises(mp.MpError) as e:
        ctx.pair_plan(dev(rp), dev(ci))
    assert e.value.name == "MP_ERR_CAPACITY"
    with pytest.raises(mp.MpError) as e:
        ctx.cfconv_fwd_pairs(0, dev(synth.uniform_positions(n, seed=1)),
                             dev(synth.node_features(n, wl.F)).to(torch.bfloat16))
    assert e.value.name == "MP_ERR_INVALID_ARG"
    ctx.status_sync()


def test_pair_kernel_bounded_waits_report_a_timeout_and_recover(mp):
    # with a zero wait budget every hand-off wait of the pair kernel gives up at once: the kernel
    # drains what it issued and returns, the status word reports MP_ERR_TIMEOUT; with the default
    # budget the same context's next call matches the oracle
    wl, pos, gp, rp, ci = system(mp, "cfg2", 1200)
    ctx, w, x_t, x_ref, _ = run_pairs(mp, wl, pos, rp, ci)
    ctx.set_wait_budget(0)
    ctx.cfconv_fwd_pairs(0, dev(pos), x_t.to(DEV))
    torch.cuda.synchronize()
    with pytest.raises(mp.MpError) as e:
        ctx.status_sync()
    assert e.value.name == "MP_ERR_TIMEOUT"
    ctx.set_wait_budget(2_000_000_000)
    out = ctx.cfconv_fwd_pairs(0, dev(pos), x_t.to(DEV))
    torch.cuda.synchronize()
    ctx.status_sync()
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    ref = oracle.cfconv_pairs(model, 0, pos, orp, oci, x_ref)
    assert normwise(out.float().cpu().numpy(), ref) <= TOL_BF16_FEAT


def test_pair_cfconv_high_degree(mp):
    # r_c = 10 A at the workloads' density in a 25 A box: about 250 neighbors per atom, some 16 k
    # upper pairs per 128-atom block, block pairs of many tiles each
    wl = dataclasses.replace(synth.WORKLOADS["cfg2"], dtype="bf16", r_c=10.0, n_atoms=1500)
    pos = synth.uniform_positions(1500, seed=4)
    perm = mp.spatial_order(dev(pos), wl.r_c).cpu().numpy()
    pos = np.ascontiguousarray(pos[perm])
    rp, ci = mp.neighbor_csr(dev(pos), wl.r_c)
    assert ci.numel() > 200 * 1500
    ctx, w, x_t, x_ref, out = run_pairs(mp, wl, pos, rp, ci, block=2)
    orp, oci = oracle_csr(pos, wl.r_c, rp, ci)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    ref = oracle.cfconv_pairs(model, 2, pos, orp, oci, x_ref)
    assert normwise(out.float().cpu().numpy(), ref) <= TOL_BF16_FEAT
