"""Pins for the fp64 oracle: each test ties it to something other than itself.

Brute-force enumeration, closed forms, hand calculations with the ``math`` module, reduction to a
dense matrix product, central finite differences, symmetry (translation, rotation, permutation),
replica additivity and the exact zero at the cutoff. A plausible mistake in the oracle (a dropped
bias, a wrong sign, a transposed weight, a missed neighbor) fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import schnet
from atomistic_neighbor_list_b200 import synth


def small_model(F=8, R=6, n_blocks=2, r_c=5.0, seed=7, n_heads=2, head_dim=4, n_types=3):
    wl = synth.Workload("t", "energy_forces", 0, r_c, R, F, "fp32", n_blocks=n_blocks,
                        n_types=n_types, n_heads=n_heads, head_dim=head_dim)
    w = synth.make_weights(wl, seed=seed)
    return oracle.Model.from_workload(wl, w), w, wl


# ----------------------------------------------------------------------------- neighbor list
def brute_csr(pos, r_c, graph_ptr=None):
    """O(N^2) enumeration with plain Python floats (IEEE double, same operation order)."""
    pos = np.asarray(pos, dtype=np.float32)
    n = len(pos)
    gp = [0, n] if graph_ptr is None else list(graph_ptr)
    graph_of = np.zeros(n, dtype=np.int64)
    for g in range(len(gp) - 1):
        graph_of[gp[g]:gp[g + 1]] = g
    rc = float(np.float32(r_c))
    rc2 = rc * rc
    P = [tuple(float(c) for c in p) for p in pos]
    row_ptr, cols = [0], []
    for i in range(n):
        xi, yi, zi = P[i]
        for j in range(n):
            if j == i or graph_of[j] != graph_of[i]:
                continue
            xj, yj, zj = P[j]
            dx, dy, dz = xj - xi, yj - yi, zj - zi
            if (dx * dx + dy * dy) + dz * dz < rc2:
                cols.append(j)
        row_ptr.append(len(cols))
    return np.array(row_ptr, dtype=np.int32), np.array(cols, dtype=np.int32)


@pytest.mark.parametrize("n", [1, 2, 33, 300])
def test_csr_matches_brute_force_uniform(n):
    pos = synth.uniform_positions(n, seed=n)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    brp, bci = brute_csr(pos, 5.0)
    assert np.array_equal(rp, brp) and np.array_equal(ci, bci)


def test_csr_matches_brute_force_chains():
    pos, gp = synth.chain_replicas(3, 120, seed=5)
    rp, ci = oracle.neighbor_csr(pos, 10.0, gp)
    brp, bci = brute_csr(pos, 10.0, gp)
    assert np.array_equal(rp, brp) and np.array_equal(ci, bci)
    # no edge leaves its replica
    dst = np.repeat(np.arange(len(pos)), np.diff(rp))
    assert np.array_equal(dst // 120, ci // 120)


def test_csr_matches_brute_force_vectorised_1500():
    pos = synth.uniform_positions(1500, seed=11)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    p = pos.astype(np.float64)
    cols, row_ptr = [], [0]
    for i in range(len(p)):
        dx, dy, dz = p[:, 0] - p[i, 0], p[:, 1] - p[i, 1], p[:, 2] - p[i, 2]
        d2 = (dx * dx + dy * dy) + dz * dz
        js = np.nonzero(d2 < 25.0)[0]
        js = js[js != i]
        cols.extend(js.tolist())
        row_ptr.append(len(cols))
    assert np.array_equal(rp, np.array(row_ptr)) and np.array_equal(ci, np.array(cols))


def test_csr_sorted_symmetric_no_self():
    pos = synth.uniform_positions(2000, seed=3)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    n = len(pos)
    dst = np.repeat(np.arange(n), np.diff(rp))
    assert np.all(ci != dst)
    for i in range(n):
        row = ci[rp[i]:rp[i + 1]]
        assert np.all(np.diff(row) > 0)
    fwd = set(zip(dst.tolist(), ci.tolist()))
    assert all((j, i) in fwd for (i, j) in fwd)


def test_interior_degree_matches_density():
    # interior atoms of a uniform cube see rho * 4/3 pi r_c^3 = 52.36 neighbors on average
    pos = synth.uniform_positions(10_000, seed=0)
    rp, _ = oracle.neighbor_csr(pos, 5.0)
    L = synth.box_length(10_000)
    inner = np.all((pos > 5.0) & (pos < L - 5.0), axis=1)
    mean = np.diff(rp)[inner].mean()
    import json, os
    facts = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "workload_facts.json")))
    want = facts["interior_mean_degree_uniform_0.1_per_A3_rc5"]["value"]
    assert abs(want - 0.1 * 4.0 / 3.0 * math.pi * 125.0) < 1e-9
    assert abs(mean - want) < 1.5


def test_pair_exactly_at_cutoff_excluded():
    pos = np.array([[0, 0, 0], [5, 0, 0]], dtype=np.float32)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    assert rp.tolist() == [0, 0, 0] and len(ci) == 0
    pos[1, 0] = np.float32(4.9999)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    assert rp.tolist() == [0, 1, 2] and ci.tolist() == [1, 0]


def test_padded_list_keeps_nearest_k():
    pos = synth.uniform_positions(600, seed=4)
    K = 20
    nbr, mask = oracle.neighbor_padded(pos, 5.0, K)
    rp, ci = brute_csr(pos, 5.0)
    p = pos.astype(np.float64)
    for i in range(len(pos)):
        full = ci[rp[i]:rp[i + 1]]
        if len(full) <= K:
            want = full
        else:
            key = sorted(((float(((p[j, 0] - p[i, 0]) ** 2 + (p[j, 1] - p[i, 1]) ** 2)
                                 + (p[j, 2] - p[i, 2]) ** 2), int(j)) for j in full))
            want = np.sort(np.array([j for _, j in key[:K]]))
        cnt = int(mask[i].sum())
        assert cnt == len(want)
        assert np.array_equal(nbr[i, :cnt], want)
        assert np.all(nbr[i, cnt:] == -1) and np.all(mask[i, cnt:] == 0)


# ----------------------------------------------------------------------------- element functions
def test_rbf_closed_forms():
    mu = oracle.rbf_centres(50, 0.0, 5.0)
    assert mu[0] == 0.0 and abs(mu[-1] - 5.0) < 1e-15 and abs(mu[1] - 5.0 / 49) < 1e-15
    e = oracle.gaussian_rbf(mu, mu, 10.0)
    assert np.allclose(np.diag(e), 1.0, rtol=0, atol=0)
    d = np.array([1.234])
    assert abs(oracle.gaussian_rbf(d, mu, 10.0)[0, 7] - math.exp(-10.0 * (1.234 - mu[7]) ** 2)) < 1e-15
    h = 1e-6
    fd = (oracle.gaussian_rbf(d + h, mu, 10.0) - oracle.gaussian_rbf(d - h, mu, 10.0)) / (2 * h)
    assert np.allclose(oracle.gaussian_rbf_grad(d, mu, 10.0), fd, atol=1e-8)


def test_cosine_cutoff_closed_forms():
    rc = 5.0
    f = oracle.cosine_cutoff(np.array([0.0, 2.5, 5.0, 5.5, 100.0]), rc)
    assert f[0] == 1.0 and abs(f[1] - 0.5) < 1e-15
    assert f[2] == 0.0 and f[3] == 0.0 and f[4] == 0.0  # exactly zero at and beyond the cutoff
    g = oracle.cosine_cutoff_grad(np.array([0.0, 2.5, 5.0, 6.0]), rc)
    assert g[0] == 0.0 and abs(g[1] + math.pi / (2 * rc)) < 1e-15 and g[2] == 0.0 and g[3] == 0.0
    d = np.array([1.1, 3.3, 4.9])
    h = 1e-6
    fd = (oracle.cosine_cutoff(d + h, rc) - oracle.cosine_cutoff(d - h, rc)) / (2 * h)
    assert np.allclose(oracle.cosine_cutoff_grad(d, rc), fd, atol=1e-9)


def test_ssp_closed_forms():
    assert oracle.ssp(0.0) == 0.0
    assert abs(oracle.ssp_grad(0.0) - 0.5) < 1e-16
    for x in [-30.0, -3.0, -0.7, 0.2, 1.5, 4.0, 20.0]:
        assert abs(oracle.ssp(x) - math.log(0.5 * math.exp(x) + 0.5)) < 1e-14 * max(1, abs(x))
    assert abs(oracle.ssp(60.0) - (60.0 - math.log(2.0))) < 1e-12
    assert abs(oracle.ssp(-60.0) + math.log(2.0)) < 1e-12
    x = np.linspace(-6, 6, 25)
    fd = (oracle.ssp(x + 1e-6) - oracle.ssp(x - 1e-6)) / 2e-6
    assert np.allclose(oracle.ssp_grad(x), fd, atol=1e-8)


# ----------------------------------------------------------------------------- filter and cfconv
def test_filter_with_zero_first_layer_by_hand():
    model, w, wl = small_model()
    model.w["A1.0"][:] = 0.0
    d = 3.1
    c1, A2, c2 = w["c1.0"].astype(float), w["A2.0"].astype(float), w["c2.0"].astype(float)
    fc = 0.5 * (math.cos(math.pi * d / 5.0) + 1.0)
    F = wl.F
    want = []
    for f in range(F):
        acc = float(c2[f])
        for g in range(F):
            acc += math.log(0.5 * math.exp(float(c1[g])) + 0.5) * float(A2[g, f])
        want.append(fc * acc)
    got = oracle.filter_weights(model, 0, np.array([d]))[0]
    assert np.allclose(got, want, rtol=1e-13, atol=1e-14)


def test_two_atom_cfconv_by_hand():
    model, w, wl = small_model(F=4, R=5)
    pos = np.array([[0.1, 0.2, 0.3], [1.0, 2.0, 2.5]], dtype=np.float32)
    x = synth.node_features(2, 4, seed=9)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    m = oracle.cfconv(model, 0, pos, rp, ci, x)
    p = pos.astype(float)
    d = math.sqrt(sum((p[0, c] - p[1, c]) ** 2 for c in range(3)))
    mu = [5.0 * k / 4 for k in range(5)]
    e = [math.exp(-10.0 * (d - mu[k]) ** 2) for k in range(5)]
    A1, c1, A2, c2 = (w[k].astype(float) for k in ("A1.0", "c1.0", "A2.0", "c2.0"))
    h1 = [math.log(0.5 * math.exp(sum(e[k] * A1[k, g] for k in range(5)) + c1[g]) + 0.5)
          for g in range(4)]
    fc = 0.5 * (math.cos(math.pi * d / 5.0) + 1.0)
    W = [fc * (sum(h1[g] * A2[g, f] for g in range(4)) + c2[f]) for f in range(4)]
    assert np.allclose(m[0], [x[1, f] * W[f] for f in range(4)], rtol=1e-12, atol=1e-14)
    assert np.allclose(m[1], [x[0, f] * W[f] for f in range(4)], rtol=1e-12, atol=1e-14)


def test_cfconv_reduces_to_dense_spmm():
    # A1 = A2 = 0, c2 = 1  =>  W_ij = f_c(d_ij)  =>  m = A x with A_ij = f_c(d_ij) on neighbor pairs
    model, w, wl = small_model(F=8)
    model.w["A1.0"][:] = 0
    model.w["A2.0"][:] = 0
    model.w["c2.0"][:] = 1
    pos = synth.uniform_positions(150, seed=2)
    x = synth.node_features(150, 8, seed=1)
    rp, ci = brute_csr(pos, 5.0)
    A = np.zeros((150, 150))
    p = pos.astype(float)
    for i in range(150):
        for j in ci[rp[i]:rp[i + 1]]:
            d = math.sqrt(sum((p[i, c] - p[j, c]) ** 2 for c in range(3)))
            A[i, j] = 0.5 * (math.cos(math.pi * d / 5.0) + 1.0)
    m = oracle.cfconv(model, 0, pos, rp, ci, x)
    assert np.allclose(m, A @ x.astype(float), rtol=1e-12, atol=1e-12)


def test_pair_cfconv_two_atoms_by_hand():
    # one pair: the filter once, x_1 (.) W to row 0 and x_0 (.) W to row 1 (the hand formula above)
    model, w, wl = small_model(F=4, R=5)
    pos = np.array([[0.1, 0.2, 0.3], [1.0, 2.0, 2.5]], dtype=np.float32)
    x = synth.node_features(2, 4, seed=9)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    m = oracle.cfconv_pairs(model, 0, pos, rp, ci, x)
    p = pos.astype(float)
    d = math.sqrt(sum((p[0, c] - p[1, c]) ** 2 for c in range(3)))
    e = [math.exp(-10.0 * (d - 5.0 * k / 4) ** 2) for k in range(5)]
    A1, c1, A2, c2 = (w[k].astype(float) for k in ("A1.0", "c1.0", "A2.0", "c2.0"))
    h1 = [math.log(0.5 * math.exp(sum(e[k] * A1[k, g] for k in range(5)) + c1[g]) + 0.5)
          for g in range(4)]
    fc = 0.5 * (math.cos(math.pi * d / 5.0) + 1.0)
    W = [fc * (sum(h1[g] * A2[g, f] for g in range(4)) + c2[f]) for f in range(4)]
    assert np.allclose(m[0], [x[1, f] * W[f] for f in range(4)], rtol=1e-12, atol=1e-14)
    assert np.allclose(m[1], [x[0, f] * W[f] for f in range(4)], rtol=1e-12, atol=1e-14)


def test_pair_cfconv_reduces_to_symmetric_spmm():
    # W = f_c  =>  m = A x with A symmetric, A_ij = f_c(d_ij) on neighbor pairs
    model, w, wl = small_model(F=8)
    model.w["A1.0"][:] = 0
    model.w["A2.0"][:] = 0
    model.w["c2.0"][:] = 1
    pos = synth.uniform_positions(150, seed=2)
    x = synth.node_features(150, 8, seed=1)
    rp, ci = brute_csr(pos, 5.0)
    A = np.zeros((150, 150))
    p = pos.astype(float)
    for i in range(150):
        for j in ci[rp[i]:rp[i + 1]]:
            d = math.sqrt(sum((p[i, c] - p[j, c]) ** 2 for c in range(3)))
            A[i, j] = 0.5 * (math.cos(math.pi * d / 5.0) + 1.0)
    assert np.array_equal(A, A.T)
    m = oracle.cfconv_pairs(model, 0, pos, rp, ci, x)
    assert np.allclose(m, A @ x.astype(float), rtol=1e-12, atol=1e-12)


def test_pair_cfconv_evaluates_each_filter_once(monkeypatch):
    # the pair form calls the filter on E / 2 distances and gives the directed form's sums
    model, w, wl = small_model(F=8)
    pos = synth.uniform_positions(300, seed=6)
    x = synth.node_features(300, 8, seed=3)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    seen = []
    real = oracle.schnet.filter_weights

    def counting(model_, b, d, with_grad=False):
        seen.append(len(d))
        return real(model_, b, d, with_grad)

    monkeypatch.setattr(oracle.schnet, "filter_weights", counting)
    m_pair = oracle.cfconv_pairs(model, 0, pos, rp, ci, x)
    assert sum(seen) * 2 == len(ci) and len(ci) > 1000
    monkeypatch.setattr(oracle.schnet, "filter_weights", real)
    m_dir = oracle.cfconv(model, 0, pos, rp, ci, x)
    assert np.allclose(m_pair, m_dir, rtol=1e-12, atol=1e-12)


def test_undirected_pairs_need_a_symmetric_list():
    rp = np.array([0, 1, 1, 2])
    ci = np.array([1, 0])  # 1 -> 0 and 0 -> 2: the reverse of 0 -> 2 is missing
    with pytest.raises(ValueError):
        oracle.undirected_pairs(rp, ci)
    i, j = oracle.undirected_pairs(np.array([0, 2, 3, 4]), np.array([1, 2, 0, 0]))
    assert i.tolist() == [0, 0] and j.tolist() == [1, 2]


def test_cfconv_empty_rows_and_permutation():
    model, w, wl = small_model(F=8)
    pos = synth.uniform_positions(120, seed=5)
    pos[7] = [500.0, 500.0, 500.0]  # isolated atom -> empty row
    x = synth.node_features(120, 8, seed=2)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    m = oracle.cfconv(model, 0, pos, rp, ci, x)
    assert rp[8] == rp[7] and np.all(m[7] == 0.0)
    perm = np.random.default_rng(0).permutation(120)
    rp2, ci2 = oracle.neighbor_csr(pos[perm], 5.0)
    m2 = oracle.cfconv(model, 0, pos[perm], rp2, ci2, x[perm])
    assert np.allclose(m2, m[perm], rtol=1e-12, atol=1e-12)
    # sampled rows equal the same rows of the full computation
    rows = np.array([3, 7, 50, 119])
    assert np.array_equal(oracle.cfconv(model, 0, pos, rp, ci, x, rows=rows), m[rows])


# ----------------------------------------------------------------------------- energy and forces
@pytest.fixture(scope="module")
def fd_system():
    wl = synth.WORKLOADS["fd64"]
    w = synth.make_weights(wl)
    model = oracle.Model.from_workload(wl, w)
    pos = synth.uniform_positions(64, seed=0)
    types = synth.atom_types(64, wl.n_types)
    rp, ci = oracle.neighbor_csr(pos, wl.r_c)
    return model, pos, types, rp, ci


def test_forces_match_central_differences(fd_system):
    model, pos, types, rp, ci = fd_system
    E, F = oracle.energy_forces(model, pos, types, rp, ci)
    p0 = pos.astype(np.float64)
    h = 1e-3
    fd = np.zeros_like(p0)
    for a in range(len(p0)):
        for c in range(3):
            pp, pm = p0.copy(), p0.copy()
            pp[a, c] += h
            pm[a, c] -= h
            ep = oracle.energies(model, pp, types, rp, ci)[0]
            em = oracle.energies(model, pm, types, rp, ci)[0]
            fd[a, c] = -(ep - em) / (2 * h)
    rel = np.linalg.norm(fd - F) / np.linalg.norm(F)
    assert rel < 1e-5, rel


def test_force_forms_agree_and_momentum_zero(fd_system):
    model, pos, types, rp, ci = fd_system
    E1, F1 = oracle.energy_forces(model, pos, types, rp, ci, method="scatter")
    E2, F2 = oracle.energy_forces(model, pos, types, rp, ci, method="pair")
    assert np.array_equal(E1, E2)
    scale = np.abs(F1).max()
    assert np.max(np.abs(F1 - F2)) <= 1e-12 * scale
    assert np.max(np.abs(F1.sum(axis=0))) <= 1e-12 * scale * len(pos)
    torque = np.cross(pos.astype(float), F1).sum(axis=0)
    assert np.max(np.abs(torque)) <= 1e-11 * scale * len(pos) * 10


def test_rotation_translation_invariance(fd_system):
    model, pos, types, rp, ci = fd_system
    E, F = oracle.energy_forces(model, pos, types, rp, ci)
    rng = np.random.default_rng(42)
    Q, _ = np.linalg.qr(rng.normal(size=(3, 3)))
    if np.linalg.det(Q) < 0:
        Q[:, 0] = -Q[:, 0]
    assert abs(np.linalg.det(Q) - 1.0) < 1e-12
    t = rng.normal(size=3) * 10
    p2 = pos.astype(np.float64) @ Q.T + t
    rp2, ci2 = oracle.neighbor_csr(p2, 5.0)
    E2, F2 = oracle.energy_forces(model, p2, types, rp2, ci2)
    assert abs(E2[0] - E[0]) <= 1e-10 * abs(E[0])
    assert np.max(np.abs(F2 - F @ Q.T)) <= 1e-9 * np.abs(F).max()


def test_replica_additivity_and_isolation():
    model, w, wl = small_model(F=8, R=6, n_blocks=2, r_c=10.0)
    pos, gp = synth.chain_replicas(3, 60, seed=1)
    types = synth.atom_types(len(pos), wl.n_types)
    rp, ci = oracle.neighbor_csr(pos, 10.0, gp)
    E, F = oracle.energy_forces(model, pos, types, rp, ci, gp)
    for g in range(3):
        sl = slice(gp[g], gp[g + 1])
        rpg, cig = oracle.neighbor_csr(pos[sl], 10.0)
        Eg, Fg = oracle.energy_forces(model, pos[sl], types[sl], rpg, cig)
        assert abs(Eg[0] - E[g]) <= 1e-12 * max(1.0, abs(E[g]))
        assert np.allclose(Fg, F[sl], rtol=1e-11, atol=1e-12)


def test_exact_zero_at_cutoff():
    model, w, wl = small_model(F=8)
    types = np.array([0, 1], dtype=np.int32)
    pos = np.array([[0, 0, 0], [5, 0, 0]], dtype=np.float32)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    E, F = oracle.energy_forces(model, pos, types, rp, ci)
    assert np.all(F == 0.0)
    x = synth.node_features(2, 8)
    assert np.all(oracle.cfconv(model, 0, pos, rp, ci, x) == 0.0)
    # the same pair pushed just inside: small but non-zero force along x only
    pos[1, 0] = np.float32(5.0 - 1e-3)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    E2, F2 = oracle.energy_forces(model, pos, types, rp, ci)
    assert 0 < np.abs(F2[:, 0]).max() < 1e-3 and np.all(F2[:, 1:] == 0.0)
    assert abs(E2[0] - E[0]) < 1e-4


# ----------------------------------------------------------------------------- energy forward by hand
def _hand_ssp(v: float) -> float:
    return math.log(0.5 * math.exp(v) + 0.5)


def _hand_readout(w, x):
    """e = ssp(x B1 + d1) B2 + d2 with plain Python loops (x: list of F floats)."""
    B1, d1, B2, d2 = (np.asarray(w[k], dtype=float) for k in ("B1", "d1", "B2", "d2"))
    F, Fh = B1.shape
    e = float(d2[0])
    for g in range(Fh):
        a = float(d1[g]) + sum(x[f] * float(B1[f, g]) for f in range(F))
        e += _hand_ssp(a) * float(B2[g, 0])
    return e


def _hand_dense(W, b, x):
    W, b = np.asarray(W, dtype=float), np.asarray(b, dtype=float)
    return [float(b[o]) + sum(x[i] * float(W[i, o]) for i in range(len(x))) for o in range(W.shape[1])]


def test_isolated_atom_energy_by_hand():
    # no neighbor: m = 0 in every block, so x_B = emb[t] + sum_b b_out_b and
    # E = ssp((emb[t] + sum_b b_out_b) B1 + d1) B2 + d2 -- pins the embedding row, the residual
    # bias of every block and every readout term (a dropped b_out, d1, d2 or a wrong type row fails)
    model, w, wl = small_model(F=6, R=5, n_blocks=3, n_types=4)
    for t in range(4):
        pos = np.array([[1.0, 2.0, 3.0]], dtype=np.float32)
        types = np.array([t], dtype=np.int32)
        rp, ci = oracle.neighbor_csr(pos, 5.0)
        x = [float(v) for v in w["emb"][t]]
        for b in range(3):
            x = [x[f] + float(w[f"b_out.{b}"][f]) for f in range(6)]
        want = _hand_readout(w, x)
        got = oracle.energies(model, pos, types, rp, ci)[0]
        assert abs(got - want) <= 1e-12 * max(1.0, abs(want)), (t, got, want)
    # far-apart atoms: the energy is the sum of the isolated atoms' energies
    pos = np.array([[0, 0, 0], [50, 0, 0], [0, 50, 0], [0, 0, 50]], dtype=np.float32)
    types = np.array([3, 0, 2, 0], dtype=np.int32)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    singles = []
    for t in types:
        x = [float(v) for v in w["emb"][t]]
        for b in range(3):
            x = [x[f] + float(w[f"b_out.{b}"][f]) for f in range(6)]
        singles.append(_hand_readout(w, x))
    assert abs(oracle.energies(model, pos, types, rp, ci)[0] - sum(singles)) <= 1e-12 * 4


@pytest.mark.parametrize("n_blocks", [1, 2])
def test_two_atom_energy_by_hand(n_blocks):
    # every stage of the forward written out with math for a bound pair: embedding, per block
    # h = x W_in + b_in, m_i = h_j (.) W(d), x <- x + m W_out + b_out, then the readout of both atoms
    F, R = 4, 5
    model, w, wl = small_model(F=F, R=R, n_blocks=n_blocks, n_types=3)
    pos = np.array([[0.3, -0.2, 0.1], [2.1, 1.4, -1.9]], dtype=np.float32)
    types = np.array([2, 0], dtype=np.int32)
    rp, ci = oracle.neighbor_csr(pos, 5.0)
    assert ci.tolist() == [1, 0]
    p = pos.astype(float)
    d = math.sqrt(sum((p[0, c] - p[1, c]) ** 2 for c in range(3)))
    mu = [5.0 * k / (R - 1) for k in range(R)]
    e = [math.exp(-10.0 * (d - mu[k]) ** 2) for k in range(R)]
    fc = 0.5 * (math.cos(math.pi * d / 5.0) + 1.0)
    xs = [[float(v) for v in w["emb"][t]] for t in types]
    for b in range(n_blocks):
        A1, c1, A2, c2 = (np.asarray(w[f"{k}.{b}"], dtype=float) for k in ("A1", "c1", "A2", "c2"))
        h1 = [_hand_ssp(sum(e[k] * A1[k, g] for k in range(R)) + c1[g]) for g in range(F)]
        Wd = [fc * (sum(h1[g] * A2[g, f] for g in range(F)) + c2[f]) for f in range(F)]
        hs = [_hand_dense(w[f"W_in.{b}"], w[f"b_in.{b}"], x) for x in xs]
        ms = [[hs[1][f] * Wd[f] for f in range(F)], [hs[0][f] * Wd[f] for f in range(F)]]
        outs = [_hand_dense(w[f"W_out.{b}"], w[f"b_out.{b}"], m) for m in ms]
        xs = [[xs[a][f] + outs[a][f] for f in range(F)] for a in range(2)]
    want = _hand_readout(w, xs[0]) + _hand_readout(w, xs[1])
    got = oracle.energies(model, pos, types, rp, ci)[0]
    assert abs(got - want) <= 1e-12 * max(1.0, abs(want)), (got, want)
    # the same number from energy_forces (both force forms) and per-atom energies by hand
    E_s, _, e_atom = oracle.energy_forces(model, pos, types, rp, ci, return_atom_energy=True)
    assert abs(E_s[0] - want) <= 1e-12 * max(1.0, abs(want))
    assert abs(e_atom[0] - _hand_readout(w, xs[0])) <= 1e-12 * max(1.0, abs(e_atom[0]))


# ----------------------------------------------------------------------------- attention
def test_attention_uniform_weights_give_mean():
    model, w, wl = small_model(F=8, n_heads=2, head_dim=4)
    for k in ("Wq", "Wk", "P", "p"):
        model.w[k][:] = 0
    pos = synth.uniform_positions(80, seed=8)
    x = synth.node_features(80, 8, seed=4)
    nbr, mask = oracle.neighbor_padded(pos, 5.0, 16)
    out = oracle.attention(model, pos, nbr, mask, x)
    rp, ci = brute_csr(pos, 5.0)
    for i in range(80):
        cnt = int(mask[i].sum())
        if cnt == 0:
            assert np.all(out[i] == 0)
            continue
        js = nbr[i, :cnt]
        W = oracle.filter_weights(model, 0, np.linalg.norm(pos[i].astype(float) - pos[js], axis=1))
        assert np.allclose(out[i], (x[js] * W).mean(axis=0), rtol=1e-12, atol=1e-13)


def test_attention_two_neighbors_by_hand():
    model, w, wl = small_model(F=4, R=5, n_heads=2, head_dim=2)
    pos = np.array([[0, 0, 0], [1.5, 0.5, 0], [0, 2.5, 1.0], [40, 40, 40]], dtype=np.float32)
    x = synth.node_features(4, 4, seed=6)
    nbr = np.array([[1, 2, -1], [0, -1, -1], [0, -1, -1], [-1, -1, -1]], dtype=np.int32)
    mask = (nbr >= 0).astype(np.uint8)
    out = oracle.attention(model, pos, nbr, mask, x)
    W64 = {k: v.astype(float) for k, v in w.items()}
    p = pos.astype(float)
    xf = x.astype(float)
    q = [[sum(xf[0, a] * W64["Wq"][a, f] for a in range(4)) for f in range(4)]]
    kk = [[sum(xf[j, a] * W64["Wk"][a, f] for a in range(4)) for f in range(4)] for j in range(4)]
    mu = [5.0 * k / 4 for k in range(5)]
    logits, vals = [], []
    for j in (1, 2):
        d = math.sqrt(sum((p[0, c] - p[j, c]) ** 2 for c in range(3)))
        e = [math.exp(-10.0 * (d - mu[k]) ** 2) for k in range(5)]
        Wf = oracle.filter_weights(model, 0, np.array([d]))[0]
        vals.append([xf[j, f] * Wf[f] for f in range(4)])
        logits.append([sum(q[0][h * 2 + c] * kk[j][h * 2 + c] for c in range(2)) / math.sqrt(2)
                       + sum(e[k] * W64["P"][k, h] for k in range(5)) + W64["p"][h]
                       for h in range(2)])
    want = []
    for h in range(2):
        a = [math.exp(logits[0][h]), math.exp(logits[1][h])]
        s = a[0] + a[1]
        for c in range(2):
            f = h * 2 + c
            want.append((a[0] * vals[0][f] + a[1] * vals[1][f]) / s)
    assert np.allclose(out[0], want, rtol=1e-12, atol=1e-14)
    W1 = oracle.filter_weights(model, 0, np.array([np.linalg.norm(p[1] - p[0])]))[0]
    assert np.allclose(out[1], xf[0] * W1, rtol=1e-12)  # one valid neighbor: alpha = 1
    assert np.all(out[3] == 0.0)  # no valid neighbor: zero row


def test_attention_logit_shift_invariance():
    model, w, wl = small_model(F=8, n_heads=2, head_dim=4)
    pos = synth.uniform_positions(60, seed=3)
    x = synth.node_features(60, 8, seed=2)
    nbr, mask = oracle.neighbor_padded(pos, 5.0, 12)
    o1 = oracle.attention(model, pos, nbr, mask, x)
    model.w["p"] = model.w["p"] + 3.0
    o2 = oracle.attention(model, pos, nbr, mask, x)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-13)


@pytest.fixture(scope="module")
def attn_system():
    """24 atoms in a small box (up to 10 valid slots of 12 per row, some rows capped), F = 8."""
    model, w, wl = small_model(F=8, R=6, n_heads=2, head_dim=4)
    pos = (np.random.default_rng(21).uniform(0, 7.0, size=(24, 3))).astype(np.float64)
    x = synth.node_features(24, 8, seed=5).astype(np.float64)
    nbr, mask = oracle.neighbor_padded(pos.astype(np.float32), 5.0, 10)
    g = np.random.default_rng(22).normal(size=(24, 8))
    return model, pos, x, nbr, mask, g


def _loss(model, pos, x, nbr, mask, g):
    return float(np.sum(g * oracle.attention(model, pos, nbr, mask, x)))


def test_attention_vjp_matches_central_differences(attn_system):
    """The list is held fixed while an input moves by +-h (h = 1e-6): dL/dx and dL/dr against
    central differences of L = sum g . out, every entry."""
    model, pos, x, nbr, mask, g = attn_system
    assert 0 < mask.sum(axis=1).min() and mask.sum(axis=1).max() == 10  # some rows are capped
    gx, gpos = oracle.attention_vjp(model, pos, nbr, mask, x, g)
    h = 1e-6
    fdx = np.zeros_like(x)
    for a in range(x.shape[0]):
        for c in range(x.shape[1]):
            xp, xm = x.copy(), x.copy()
            xp[a, c] += h
            xm[a, c] -= h
            fdx[a, c] = (_loss(model, pos, xp, nbr, mask, g) - _loss(model, pos, xm, nbr, mask, g)) / (2 * h)
    fdp = np.zeros_like(pos)
    for a in range(pos.shape[0]):
        for c in range(3):
            pp, pm = pos.copy(), pos.copy()
            pp[a, c] += h
            pm[a, c] -= h
            fdp[a, c] = (_loss(model, pp, x, nbr, mask, g) - _loss(model, pm, x, nbr, mask, g)) / (2 * h)
    assert np.linalg.norm(gx - fdx) <= 1e-7 * np.linalg.norm(fdx)
    assert np.linalg.norm(gpos - fdp) <= 1e-7 * np.linalg.norm(fdp)


def test_attention_vjp_invariances_and_rows(attn_system):
    model, pos, x, nbr, mask, g = attn_system
    gx, gpos = oracle.attention_vjp(model, pos, nbr, mask, x, g)
    scale = np.abs(gpos).max()
    assert np.abs(gpos.sum(axis=0)).max() <= 1e-12 * scale * len(pos)  # translation invariance
    # the gradient at atom k needs only the rows that read k: k itself and the rows listing k
    k = 5
    rows = sorted({k} | {i for i in range(len(pos)) if np.any((nbr[i] == k) & (mask[i] != 0))})
    gx_k, gpos_k = oracle.attention_vjp(model, pos, nbr, mask, x, g, rows=rows)
    assert np.allclose(gx_k[k], gx[k], rtol=1e-12, atol=1e-14)
    assert np.allclose(gpos_k[k], gpos[k], rtol=1e-12, atol=1e-14)


def test_attention_vjp_single_neighbor_by_hand():
    """One valid slot per row: alpha = 1, so the logits carry no gradient and dL/dx_j is the sum of
    g_i (.) W(d_ij) over the rows i that list j."""
    model, w, wl = small_model(F=4, R=5, n_heads=2, head_dim=2)
    pos = np.array([[0, 0, 0], [1.5, 0.5, 0], [0, 2.5, 1.0]], dtype=np.float64)
    x = synth.node_features(3, 4, seed=6).astype(np.float64)
    nbr = np.array([[1, -1], [0, -1], [0, -1]], dtype=np.int32)
    mask = (nbr >= 0).astype(np.uint8)
    g = np.random.default_rng(3).normal(size=(3, 4))
    gx, gpos = oracle.attention_vjp(model, pos, nbr, mask, x, g)
    W10 = oracle.filter_weights(model, 0, np.array([np.linalg.norm(pos[1] - pos[0])]))[0]
    W20 = oracle.filter_weights(model, 0, np.array([np.linalg.norm(pos[2] - pos[0])]))[0]
    assert np.allclose(gx[0], g[1] * W10 + g[2] * W20, rtol=1e-12)
    assert np.allclose(gx[1], g[0] * W10, rtol=1e-12)
    assert np.allclose(gx[2], 0.0)


def test_solid_harmonics_match_library_real_sph_harm():
    """Unit vectors: S_lm = Y_lm, the real form of scipy's complex harmonics (Condon-Shortley
    phase): sqrt2 (-1)^m Re Y_l^m for m > 0, sqrt2 (-1)^m Im Y_l^|m| for m < 0; and S_lm is
    homogeneous of degree l."""
    import scipy.special as sp
    rng = np.random.default_rng(0)
    v = rng.normal(size=(200, 3))
    v /= np.linalg.norm(v, axis=1)[:, None]
    theta, phi = np.arccos(v[:, 2]), np.arctan2(v[:, 1], v[:, 0])
    S = oracle.solid_harmonics(v)
    col = 0
    for l in range(3):
        for m in range(-l, l + 1):
            Y = sp.sph_harm_y(l, abs(m), theta, phi)
            ref = Y.real if m == 0 else np.sqrt(2) * (-1) ** m * (Y.real if m > 0 else Y.imag)
            assert np.allclose(S[:, col], ref, rtol=0, atol=1e-13), (l, m)
            assert np.allclose(oracle.solid_harmonics(2.5 * v)[:, col], 2.5 ** l * S[:, col],
                               rtol=1e-13, atol=1e-14)
            col += 1


def test_equivariant_attention_scalar_part_and_rotation(attn_system):
    model, pos, x, nbr, mask, g = attn_system
    out = oracle.attention_equivariant(model, pos, nbr, mask, x)
    base = oracle.attention(model, pos, nbr, mask, x)
    assert np.allclose(out[:, 0, :], base / (2 * math.sqrt(math.pi)), rtol=1e-12, atol=1e-14)
    # rotate and translate the system: l = 1 rotates as a vector; each l block keeps its norm
    rng = np.random.default_rng(4)
    Q, _ = np.linalg.qr(rng.normal(size=(3, 3)))
    if np.linalg.det(Q) < 0:
        Q[:, 0] = -Q[:, 0]
    pos_r = pos @ Q.T + np.array([3.0, -1.0, 7.0])
    out_r = oracle.attention_equivariant(model, pos_r, nbr, mask, x)
    vec = out[:, [3, 1, 2], :]      # (x, y, z) from the l = 1 components (y, z, x)
    vec_r = out_r[:, [3, 1, 2], :]
    assert np.allclose(np.einsum("ab,nbf->naf", Q, vec), vec_r, rtol=1e-10, atol=1e-12)
    n2 = np.sum(out[:, 4:9, :] ** 2, axis=1)
    n2_r = np.sum(out_r[:, 4:9, :] ** 2, axis=1)
    assert np.allclose(n2, n2_r, rtol=1e-10, atol=1e-14)
    assert np.allclose(out[:, 0], out_r[:, 0], rtol=1e-10, atol=1e-14)


def test_equivariant_attention_node_centric_form(attn_system):
    """E2Former-V2 section 3.1 in its node-centric form: couple each source's value with the
    monomials of its own position, aggregate with the attention weights, then couple with the
    destination's position. Equals the per-edge definition."""
    model, pos, x, nbr, mask, g = attn_system
    out = oracle.attention_equivariant(model, pos, nbr, mask, x)
    w = model.w
    H, D = model.n_heads, model.head_dim
    n, K = nbr.shape
    q, k = x @ w["Wq"], x @ w["Wk"]
    mom = np.zeros((n, 10, x.shape[1]))
    for i in range(n):
        js = [int(nbr[i, s]) for s in range(K) if mask[i, s]]
        if not js:
            continue
        d = np.linalg.norm(pos[js] - pos[i], axis=1)
        e = oracle.gaussian_rbf(d, model.mu, model.gamma)
        l = (np.einsum("hd,jhd->jh", q[i].reshape(H, D), k[js].reshape(-1, H, D)) / np.sqrt(D)
             + e @ w["P"] + w["p"])
        a = np.exp(l - l.max(axis=0))
        a = np.repeat(a / a.sum(axis=0), D, axis=1)
        v = a * x[js] * oracle.filter_weights(model, 0, d)          # alpha v, source values
        X, Y, Z = pos[js, 0], pos[js, 1], pos[js, 2]                # source pre-coupling
        mono = np.stack([np.ones_like(X), X, Y, Z, X * X, X * Y, X * Z, Y * Y, Y * Z, Z * Z], 1)
        mom[i] = mono.T @ v
    node = oracle.moments_to_solid(mom, pos)                        # target coupling
    scale = np.abs(out).max()
    assert np.abs(node - out).max() <= 1e-10 * scale


# ----------------------------------------------------------------------------- molecular dynamics
def test_verlet_free_flight_is_exact():
    rng = np.random.default_rng(0)
    r0, v0 = rng.normal(size=(5, 3)), rng.normal(size=(5, 3))
    zero = lambda r: (np.zeros(1), np.zeros_like(r))  # noqa: E731
    r, v, f, e = oracle.velocity_verlet(zero, r0, v0, np.zeros((5, 3)), 0.1, 7)
    assert np.allclose(r, r0 + 0.7 * v0, rtol=0, atol=1e-12) and np.array_equal(v, v0)


def test_verlet_harmonic_closed_form():
    """F = -k x with per-atom masses. One velocity-Verlet step is the linear map
    x' = c x + h v,  v' = -h w^2 s x + c v  (c = 1 - h^2 w^2 / 2, s = 1 - h^2 w^2 / 4, w^2 = k / m),
    a rotation by theta = arccos(c) in the metric of the invariant v^2 + w^2 s x^2; so after n steps
    x_n = x0 cos(n theta) + h v0 sin(n theta) / sin(theta), and v_n likewise."""
    rng = np.random.default_rng(1)
    k, h, n = 2.0, 0.05, 1000
    im = np.array([1.0, 0.5, 2.0, 0.25])
    x0, v0 = rng.normal(size=(4, 3)), rng.normal(size=(4, 3))
    spring = lambda r: (np.array([0.5 * k * np.sum(r * r)]), -k * r)  # noqa: E731
    x, v, _, _ = oracle.velocity_verlet(spring, x0, v0, -k * x0, h, n, inv_mass=im)
    w2 = (k * im)[:, None]
    c, s = 1 - h * h * w2 / 2, 1 - h * h * w2 / 4
    th = np.arccos(c)
    xn = x0 * np.cos(n * th) + h * v0 * np.sin(n * th) / np.sin(th)
    vn = v0 * np.cos(n * th) - h * w2 * s * x0 * np.sin(n * th) / np.sin(th)
    assert np.allclose(x, xn, rtol=0, atol=1e-9) and np.allclose(v, vn, rtol=0, atol=1e-9)
    inv0 = v0 ** 2 + w2 * s * x0 ** 2
    assert np.allclose(v ** 2 + w2 * s * x ** 2, inv0, rtol=1e-10, atol=0)


def test_kinetic_energy_by_hand():
    v = np.array([[1.0, 2.0, 2.0], [0.0, 3.0, 4.0], [1.0, 0.0, 0.0]])
    im = np.array([0.5, 1.0, 0.25])
    # m |v|^2 / 2: 2 * 9 / 2 = 9; 1 * 25 / 2 = 12.5; 4 * 1 / 2 = 2
    assert np.allclose(oracle.kinetic_energy(v, im), [23.5])
    assert np.allclose(oracle.kinetic_energy(v, im, graph_ptr=[0, 2, 3]), [21.5, 2.0])
    assert np.allclose(oracle.kinetic_energy(v), [0.5 * (9 + 25 + 1)])


@pytest.fixture(scope="module")
def md_system(fd_system):
    """The 64-atom system with a neighbor list built with a 1 A skin (kept for the whole run)."""
    model, pos, types, _, _ = fd_system
    rp, ci = oracle.neighbor_csr(pos, model.r_c + 1.0)
    im = 1.0 / (1.0 + types.astype(np.float64))
    v0 = np.random.default_rng(7).normal(size=(len(pos), 3)) * np.sqrt(im)[:, None] * 0.05
    force = lambda r: oracle.energy_forces(model, r, types, rp, ci)  # noqa: E731
    return force, pos.astype(np.float64), v0, im


def test_verlet_schnet_time_reversible(md_system):
    force, r0, v0, im = md_system
    _, f0 = force(r0)
    r, v, f, _ = oracle.velocity_verlet(force, r0, v0, f0, 0.02, 8, im)
    assert np.abs(r - r0).max() > 1e-3
    rb, vb, _, _ = oracle.velocity_verlet(force, r, -v, f, 0.02, 8, im)
    assert np.abs(rb - r0).max() < 1e-10 and np.abs(vb + v0).max() < 1e-10


def test_verlet_schnet_energy_error_second_order(md_system):
    """Conservative forces: the total-energy error of the same trajectory shrinks 4x when dt
    halves (the scheme is second order), and the neighbor list with skin stays valid."""
    force, r0, v0, im = md_system
    e0, f0 = force(r0)
    etot0 = e0[0] + oracle.kinetic_energy(v0, im)[0]
    err = []
    for dt, n in ((0.02, 10), (0.01, 20)):
        r, v, f, worst = r0, v0, f0, 0.0
        for _ in range(n):
            r, v, f, e = oracle.velocity_verlet(force, r, v, f, dt, 1, im)
            worst = max(worst, abs(e[0] + oracle.kinetic_energy(v, im)[0] - etot0))
        assert np.abs(r - r0).max() < 0.5  # below skin / 2
        err.append(worst)
    assert err[0] > 1e-6 and 3.6 < err[0] / err[1] < 4.4, err
