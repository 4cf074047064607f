"""Equivariant attention values (mp_attn_eq_fwd) vs the fp64 oracle: element by element at sizes
spanning several slot batches, on sampled rows at the full attention workload, and the scalar
component against the scalar attention. Tolerances as the scalar attention: normwise 1e-5 with
fp32 features, 2e-2 with bf16 storage."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from atomistic_neighbor_list_b200 import synth
from helpers import TOL_BF16_FEAT, TOL_FP32, features_for, normwise, oracle_padded, oracle_weights

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("n,K,r_c,dtype", [(600, 20, 5.0, "fp32"), (1500, 64, 6.0, "fp32"),
                                           (1200, 48, 5.0, "bf16"), (300, 7, 8.5, "fp32")])
def test_attn_eq_matches_oracle(mp, n, K, r_c, dtype):
    wl = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=n, K=K, dtype=dtype, r_c=r_c)
    pos = synth.uniform_positions(n, seed=1)
    w = synth.make_weights(wl)
    nbr, mask = mp.neighbor_padded(dev(pos), r_c, K)
    onbr, omask = oracle_padded(pos, r_c, K, nbr, mask)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=1)
    x_t, x_ref = features_for(synth.node_features(n, wl.F, seed=4), dtype)
    out = ctx.attn_eq_fwd(dev(pos), nbr, mask, x_t.to(DEV))
    base = ctx.attn_fwd(dev(pos), nbr, mask, x_t.to(DEV))
    torch.cuda.synchronize()
    ctx.status_sync()
    model = oracle.Model.from_workload(wl, oracle_weights(w, dtype))
    ref = oracle.attention_equivariant(model, pos, onbr, omask, x_ref)
    got = out.float().cpu().numpy().astype(np.float64)
    tol = TOL_FP32 if dtype == "fp32" else TOL_BF16_FEAT
    for lo, hi in ((0, 1), (1, 4), (4, 9)):  # each l block against its own scale
        assert normwise(got[:, lo:hi], ref[:, lo:hi]) <= tol, (lo, hi)
    c0 = 1.0 / (2.0 * math.sqrt(math.pi))
    assert normwise(got[:, 0], c0 * base.float().cpu().numpy()) <= 2 * tol


def test_attn_eq_full_size_sampled(mp):
    wl = synth.WORKLOADS["cfg4"]
    n, K = wl.n_atoms, wl.K
    pos = synth.uniform_positions(n, seed=0)
    w = synth.make_weights(wl)
    nbr, mask = mp.neighbor_padded(dev(pos), wl.r_c, K)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=1)
    x_t, x_ref = features_for(synth.node_features(n, wl.F), wl.dtype)
    out = ctx.attn_eq_fwd(dev(pos), nbr, mask, x_t.to(DEV))
    torch.cuda.synchronize()
    ctx.status_sync()
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    onbr, omask = oracle_padded(pos, wl.r_c, K, nbr, mask)
    rows = np.random.default_rng(3).choice(n, 64, replace=False)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    ref = oracle.attention_equivariant(model, pos, onbr, omask, x_ref, rows=rows)
    for lo, hi in ((0, 1), (1, 4), (4, 9)):
        assert normwise(got[rows, lo:hi], ref[:, lo:hi]) <= TOL_BF16_FEAT, (lo, hi)


@pytest.mark.parametrize("n,K", [(2000, 128), (1500, 256)])
def test_attn_eq_tensor_core_path(mp, n, K):
    """bf16, 16 heads x 8, K a multiple of 128: the tensor-core kernel (one weighted-sum MMA per
    harmonic, p S_lm as bf16 operands); each l block within the bf16 feature bound."""
    wl = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=n, K=K)
    pos = synth.uniform_positions(n, seed=2)
    w = synth.make_weights(wl)
    nbr, mask = mp.neighbor_padded(dev(pos), wl.r_c, K)
    onbr, omask = oracle_padded(pos, wl.r_c, K, nbr, mask)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=1)
    x_t, x_ref = features_for(synth.node_features(n, wl.F, seed=5), "bf16")
    ctx.profile_begin()
    out = ctx.attn_eq_fwd(dev(pos), nbr, mask, x_t.to(DEV))
    prof = ctx.profile_end()
    ctx.status_sync()
    assert "attn_eq_tc" in prof and "attn_eq_simt" not in prof, prof
    model = oracle.Model.from_workload(wl, oracle_weights(w, "bf16"))
    ref = oracle.attention_equivariant(model, pos, onbr, omask, x_ref)
    got = out.float().cpu().numpy().astype(np.float64)
    errs = [normwise(got[:, lo:hi], ref[:, lo:hi]) for lo, hi in ((0, 1), (1, 4), (4, 9))]
    print("tc equivariant attention, per l block:", errs)
    assert max(errs) <= TOL_BF16_FEAT, errs


def test_attn_eq_tensor_core_empty_rows(mp):
    wl = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=1000, K=128)
    pos = synth.uniform_positions(1000, seed=6)
    w = synth.make_weights(wl)
    nbr, mask = mp.neighbor_padded(dev(pos), wl.r_c, 128)
    onbr, omask = oracle_padded(pos, wl.r_c, 128, nbr, mask)
    omask = omask.copy()
    omask[::4] = 0
    ctx = mp.Context.from_workload(wl, w, max_atoms=1000, max_edges=1)
    x_t, x_ref = features_for(synth.node_features(1000, wl.F, seed=7), "bf16")
    out = ctx.attn_eq_fwd(dev(pos), dev(onbr), dev(omask), x_t.to(DEV))
    torch.cuda.synchronize()
    ctx.status_sync()
    got = out.float().cpu().numpy()
    assert np.all(got[::4] == 0)  # no valid neighbor: zero rows
    model = oracle.Model.from_workload(wl, oracle_weights(w, "bf16"))
    ref = oracle.attention_equivariant(model, pos, onbr, omask, x_ref)
    for lo, hi in ((0, 1), (1, 4), (4, 9)):
        assert normwise(got[:, lo:hi], ref[:, lo:hi]) <= TOL_BF16_FEAT
