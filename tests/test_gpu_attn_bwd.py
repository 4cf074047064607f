"""Attention backward (dL/dx, dL/dr of L = sum g . out) through mp_attn_bwd vs the fp64 oracle's
reverse-mode formulas (pinned by central differences), on seeded inputs: element by element at
sizes spanning several batches and rows with capped lists, and on sampled atoms at the full
attention workload (32,768 atoms, K = 256), where the oracle needs only the rows that read an atom.

Tolerance: the CUDA-core kernels compute in fp32 from the stored inputs (bf16 features under a
bf16 context), so their bound is an fp32 one: normwise max|d| / max|ref| <= 1e-4. The gradients
sum O(K) terms per row and O(K) entries per source of mixed sign, so cancellation costs about
one decimal digit over the fp32 feature bound of 1e-5. The tensor-core passes take the filter's
operands in bf16 as the forward does, so the bf16 bounds apply to them (grad_x normwise 2e-2,
grad_pos relative RMS 1e-2). At the full size the check is per sampled atom: one atom's row
against its own maximum (grad_x) or norm (grad_pos), a denominator smaller than a whole tensor's
maximum, so the per-atom bound is twice the tensor bound."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from atomistic_neighbor_list_b200 import synth
from helpers import (TOL_BF16_FEAT, TOL_BF16_FORCE, features_for, normwise, oracle_padded,
                     oracle_weights, rel_rms)

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-4


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def case(mp, n, K, r_c, dtype, seed=0):
    wl = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=n, K=K, dtype=dtype, r_c=r_c)
    pos = synth.uniform_positions(n, seed=seed)
    w = synth.make_weights(wl)
    nbr, mask = mp.neighbor_padded(dev(pos), wl.r_c, K)
    onbr, omask = oracle_padded(pos, wl.r_c, K, nbr, mask)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=1)
    x_t, x_ref = features_for(synth.node_features(n, wl.F, seed=seed + 3), dtype)
    g = np.random.default_rng(seed + 11).normal(size=(n, wl.F)).astype(np.float32)
    model = oracle.Model.from_workload(wl, oracle_weights(w, dtype))
    return wl, pos, nbr, mask, onbr, omask, ctx, x_t, x_ref, g, model


@pytest.mark.parametrize("n,K,r_c,dtype", [(600, 20, 5.0, "fp32"), (1500, 64, 6.0, "fp32"),
                                           (1200, 48, 5.0, "bf16"), (300, 16, 8.5, "fp32")])
def test_attn_bwd_matches_oracle(mp, n, K, r_c, dtype):
    wl, pos, nbr, mask, onbr, omask, ctx, x_t, x_ref, g, model = case(mp, n, K, r_c, dtype)
    gx, gp = ctx.attn_bwd(dev(pos), nbr, mask, x_t.to(DEV), dev(g))
    torch.cuda.synchronize()
    ctx.status_sync()
    rgx, rgp = oracle.attention_vjp(model, pos, onbr, omask, x_ref, g.astype(np.float64))
    assert normwise(gx.cpu().numpy(), rgx) <= TOL
    assert normwise(gp.cpu().numpy(), rgp) <= TOL
    # translation invariance of L: the position gradients sum to zero
    s = gp.double().sum(dim=0).abs().max().item()
    assert s <= 1e-5 * gp.abs().sum().item()


@pytest.mark.parametrize("n,K", [(2000, 128), (1500, 256)])
def test_attn_bwd_tensor_core_passes(mp, n, K):
    """bf16, 16 heads x 8, K a multiple of 128: both passes run on the tensor cores (filter and
    its d-derivative from bf16 MMAs, the source-side sums as MMAs of bf16 messages), so the bound
    is the bf16 one: dL/dx normwise 2e-2 (features), dL/dr relative RMS 1e-2 (forces)."""
    wl, pos, nbr, mask, onbr, omask, ctx, x_t, x_ref, g, model = case(mp, n, K, 8.5, "bf16", 3)
    ctx.profile_begin()
    gx, gp = ctx.attn_bwd(dev(pos), nbr, mask, x_t.to(DEV), dev(g))
    prof = ctx.profile_end()
    ctx.status_sync()
    assert "attn_bwd_dst_tc" in prof and "attn_bwd_src_tc" in prof, prof
    assert "attn_bwd_dst" not in prof and "attn_bwd_src" not in prof, prof
    rgx, rgp = oracle.attention_vjp(model, pos, onbr, omask, x_ref, g.astype(np.float64))
    ex = normwise(gx.cpu().numpy(), rgx)
    ep = rel_rms(gp.cpu().numpy(), rgp)
    print(f"tc passes: grad_x normwise {ex:.2e}, grad_pos rel-rms {ep:.2e}")
    assert ex <= TOL_BF16_FEAT and ep <= TOL_BF16_FORCE, (ex, ep)


def test_attn_bwd_deterministic_and_empty_rows(mp):
    """Rows without valid slots contribute nothing; two runs give the same bits."""
    wl, pos, nbr, mask, onbr, omask, ctx, x_t, x_ref, g, model = case(mp, 400, 12, 5.0, "fp32", 2)
    omask = omask.copy()
    omask[::7] = 0  # every 7th row has no valid slot
    nbr, mask = dev(onbr), dev(omask)
    a = ctx.attn_bwd(dev(pos), nbr, mask, x_t.to(DEV), dev(g))
    b = ctx.attn_bwd(dev(pos), nbr, mask, x_t.to(DEV), dev(g))
    torch.cuda.synchronize()
    ctx.status_sync()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    rgx, rgp = oracle.attention_vjp(model, pos, onbr, omask, x_ref, g.astype(np.float64))
    assert normwise(a[0].cpu().numpy(), rgx) <= TOL
    assert normwise(a[1].cpu().numpy(), rgp) <= TOL


def test_attn_bwd_full_size_sampled(mp):
    """32,768 atoms, K = 256, bf16: sampled atoms against the oracle restricted to the rows that
    read them (the gradient at atom k depends on row k and the rows listing k only)."""
    wl = synth.WORKLOADS["cfg4"]
    n, K = wl.n_atoms, wl.K
    pos = synth.uniform_positions(n, seed=0)
    w = synth.make_weights(wl)
    nbr, mask = mp.neighbor_padded(dev(pos), wl.r_c, K)
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=1)
    x_t, x_ref = features_for(synth.node_features(n, wl.F), wl.dtype)
    g = np.random.default_rng(11).normal(size=(n, wl.F)).astype(np.float32)
    gx, gp = ctx.attn_bwd(dev(pos), nbr, mask, x_t.to(DEV), dev(g))
    torch.cuda.synchronize()
    ctx.status_sync()
    gx, gp = gx.cpu().numpy(), gp.cpu().numpy()
    assert np.all(np.isfinite(gx)) and np.all(np.isfinite(gp))
    assert np.abs(gp.astype(np.float64).sum(axis=0)).max() <= 1e-5 * np.abs(gp).sum()
    onbr, omask = oracle_padded(pos, wl.r_c, K, nbr, mask)
    model = oracle.Model.from_workload(wl, oracle_weights(w, wl.dtype))
    errs = []
    for k in (0, 12345, n // 2 + 77, n - 1):
        rows = sorted({k} | set(np.nonzero(np.any((onbr == k) & (omask != 0), axis=1))[0].tolist()))
        rgx, rgp = oracle.attention_vjp(model, pos, onbr, omask, x_ref, g.astype(np.float64),
                                        rows=rows)
        errs.append((np.abs(gx[k] - rgx[k]).max() / np.abs(rgx[k]).max(),
                     np.linalg.norm(gp[k] - rgp[k]) / np.linalg.norm(rgp[k])))
    print("sampled atoms (grad_x, grad_pos) relative errors", errs)
    # bf16 tensor-core passes: per-atom bounds at twice the bf16 feature / force bounds
    assert all(a <= 2 * TOL_BF16_FEAT and b <= 2 * TOL_BF16_FORCE for a, b in errs), errs


def test_attn_bwd_tensor_core_empty_rows_and_determinism(mp):
    """The tensor-core passes with rows that have no valid slot (their statistics are empty and
    no source sees them) give the oracle's gradients, and the same bits twice."""
    wl, pos, nbr, mask, onbr, omask, ctx, x_t, x_ref, g, model = case(mp, 1200, 128, 8.5, "bf16", 4)
    omask = omask.copy()
    omask[::5] = 0
    omask[1::7, 64:] = 0  # some rows keep only their first tile
    nbr, mask = dev(onbr), dev(omask)
    a = ctx.attn_bwd(dev(pos), nbr, mask, x_t.to(DEV), dev(g))
    b = ctx.attn_bwd(dev(pos), nbr, mask, x_t.to(DEV), dev(g))
    torch.cuda.synchronize()
    ctx.status_sync()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    rgx, rgp = oracle.attention_vjp(model, pos, onbr, omask, x_ref, g.astype(np.float64))
    assert normwise(a[0].cpu().numpy(), rgx) <= TOL_BF16_FEAT
    assert rel_rms(a[1].cpu().numpy(), rgp) <= TOL_BF16_FORCE
