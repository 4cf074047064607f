"""Cell-list neighbor construction vs the oracle's exact rule, bit for bit, on geometries that
stress the cell grid: coincident atoms, flat and linear systems, far-apart clusters (grids capped
and coarsened), large coordinate offsets, pairs exactly at the cutoff on cell boundaries, empty
graphs, rows with more hits than the on-chip staging, and capped padded lists."""
import numpy as np
import pytest
import torch

import oracle
from atomistic_neighbor_list_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def check_csr(mp, pos, r_c, gp=None):
    pos = np.ascontiguousarray(pos, dtype=np.float32)
    gp_np = None if gp is None else np.asarray(gp, dtype=np.int32)
    rp, ci = mp.neighbor_csr(dev(pos), r_c, graph_ptr=None if gp is None else dev(gp_np))
    orp, oci = oracle.neighbor_csr(pos, r_c, gp_np)
    assert np.array_equal(rp.cpu().numpy(), orp)
    assert np.array_equal(ci.cpu().numpy(), oci)
    return orp, oci


def geometry(name, rng):
    if name == "coincident":
        return np.zeros((40, 3)) + 1.5
    if name == "plane":
        p = rng.uniform(0, 30, size=(700, 3))
        p[:, 2] = 2.0
        return p
    if name == "line":
        p = np.zeros((300, 3))
        p[:, 0] = rng.uniform(0, 200, size=300)
        return p
    if name == "far_clusters":  # two blobs 1e4 A apart: the grid is capped and coarsened
        a = rng.uniform(0, 12, size=(300, 3))
        b = rng.uniform(0, 12, size=(300, 3)) + 1.0e4
        return np.concatenate([a, b])
    if name == "offset":  # large coordinates: cells from exact float64 differences
        return synth.uniform_positions(800, seed=3).astype(np.float64) + 7.0e3
    if name == "lattice_at_cutoff":  # spacing exactly r_c: those pairs are excluded
        g = np.arange(6) * 5.0
        return np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3)
    if name == "lattice_below_cutoff":  # spacing one float below r_c: those pairs are kept
        s = float(np.nextafter(np.float32(5.0), np.float32(0.0)))
        g = np.arange(6) * s
        return np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3)
    raise KeyError(name)


@pytest.mark.parametrize("name", ["coincident", "plane", "line", "far_clusters", "offset",
                                  "lattice_at_cutoff", "lattice_below_cutoff"])
def test_csr_geometries(mp, name):
    rng = np.random.default_rng(11)
    pos = geometry(name, rng).astype(np.float32)
    orp, oci = check_csr(mp, pos, 5.0)
    if name == "coincident":
        assert len(oci) == 40 * 39
    if name == "lattice_at_cutoff":
        assert len(oci) == 0
    if name == "lattice_below_cutoff":
        assert len(oci) > 0  # the float32 lattice rounds some spacings up to r_c, some not


def test_csr_graphs_with_empty_ranges(mp):
    pos = synth.uniform_positions(400, seed=5)
    gp = [0, 0, 120, 120, 121, 400, 400]
    check_csr(mp, pos, 5.0, gp)


def test_csr_overlapping_replicas(mp):
    """Replicas on top of each other in space: only pairs inside one graph are neighbors."""
    one = synth.uniform_positions(500, seed=6)
    pos = np.concatenate([one, one + 0.01, one - 0.02])
    check_csr(mp, pos, 5.0, [0, 500, 1000, 1500])


def test_csr_rows_beyond_staging(mp):
    """1500 atoms within a 3 A cube: every row has 1499 hits, more than the staging holds, so
    every row is filled by the ordered scan over its graph."""
    pos = np.random.default_rng(7).uniform(0, 3.0, size=(1500, 3)).astype(np.float32)
    orp, oci = check_csr(mp, pos, 5.0)
    assert len(oci) == 1500 * 1499


def test_csr_mixed_dense_and_sparse_rows(mp):
    rng = np.random.default_rng(8)
    dense = rng.uniform(0, 2.5, size=(1100, 3))
    sparse = synth.uniform_positions(3000, seed=8).astype(np.float64) + 40.0
    check_csr(mp, np.concatenate([dense, sparse]).astype(np.float32), 5.0)


@pytest.mark.parametrize("K", [1, 16, 64])
def test_padded_dense_cluster(mp, K):
    rng = np.random.default_rng(9)
    pos = np.concatenate([rng.uniform(0, 6, size=(400, 3)),
                          synth.uniform_positions(600, seed=9) + 30.0]).astype(np.float32)
    nbr, mask = mp.neighbor_padded(dev(pos), 5.0, K)
    onbr, omask = oracle.neighbor_padded(pos, 5.0, K)
    assert np.array_equal(mask.cpu().numpy(), omask)
    assert np.array_equal(nbr.cpu().numpy(), onbr)


def test_padded_graphs_and_ties(mp):
    """Equal distances (a lattice) are broken by the source index; graphs are respected."""
    g = np.arange(5) * 2.0
    lat = np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3)
    pos = np.concatenate([lat, lat + 0.5]).astype(np.float32)
    gp = np.array([0, 125, 250], dtype=np.int32)
    nbr, mask = mp.neighbor_padded(dev(pos), 5.0, 12, graph_ptr=dev(gp))
    onbr, omask = oracle.neighbor_padded(pos, 5.0, 12, gp)
    assert np.array_equal(mask.cpu().numpy(), omask)
    assert np.array_equal(nbr.cpu().numpy(), onbr)


def test_padded_row_beyond_staging_is_a_capacity_error(mp):
    pos = np.random.default_rng(10).uniform(0, 2.0, size=(1100, 3)).astype(np.float32)
    with pytest.raises(mp.MpError) as e:
        mp.neighbor_padded(dev(pos), 5.0, 8)
    assert e.value.name == "MP_ERR_CAPACITY"


def test_spatial_order_is_a_graph_preserving_permutation(mp):
    """mp_spatial_order: a permutation that keeps every atom inside its graph's range and places
    neighbors close together; the energy and forces of the relabelled system are the original
    ones, relabelled."""
    wl = synth.WORKLOADS["cfg3"]
    import dataclasses
    wl = dataclasses.replace(wl, n_atoms=4 * 300, replicas=4)
    pos, gp = synth.positions_for(wl)
    perm = mp.spatial_order(dev(pos), wl.r_c, graph_ptr=dev(gp)).cpu().numpy()
    assert np.array_equal(np.sort(perm), np.arange(len(pos)))
    for g in range(len(gp) - 1):
        seg = perm[gp[g]:gp[g + 1]]
        assert seg.min() >= gp[g] and seg.max() < gp[g + 1]
    # locality: consecutive atoms of the new order are much closer than in the old one
    p2 = pos[perm]
    step_new = np.linalg.norm(np.diff(p2, axis=0), axis=1).mean()
    u = synth.uniform_positions(5000, seed=3)
    pu = u[mp.spatial_order(dev(u), 5.0).cpu().numpy()]
    assert np.linalg.norm(np.diff(pu, axis=0), axis=1).mean() < 0.25 * np.linalg.norm(
        np.diff(u, axis=0), axis=1).mean()
    assert np.isfinite(step_new)


def test_spatial_order_relabels_energy_and_forces(mp):
    import dataclasses
    wl = dataclasses.replace(synth.scaled(synth.WORKLOADS["cfg2"], 2000), dtype="fp32")
    pos, _ = synth.positions_for(wl)
    types = synth.atom_types(len(pos), wl.n_types)
    perm = mp.spatial_order(dev(pos), wl.r_c).cpu().numpy()
    out = []
    for p, t in ((pos, types), (pos[perm], types[perm])):
        pd = dev(np.ascontiguousarray(p))
        rp, ci = mp.neighbor_csr(pd, wl.r_c)
        ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=len(p),
                                       max_edges=ci.numel())
        e, f = ctx.energy_forces(pd, dev(np.ascontiguousarray(t)), rp, ci)
        torch.cuda.synchronize()
        out.append((float(e[0]), f.cpu().numpy()))
    (e0, f0), (e1, f1) = out
    assert abs(e0 - e1) <= 1e-5 * abs(e0)
    assert np.abs(f1 - f0[perm]).max() <= 1e-4 * np.abs(f0).max()
