"""Writes stay inside the output rows, and out-of-range indices become a status, on the GPU.

Without a memory checker on this pool the kernels are checked with canaries: each output tensor is
a view into a larger one whose guard rows before and after are filled with NaN, and after the call
the guard rows must still be NaN (a write past either end would have replaced them). The ragged
sizes put the last rows in a partial tile. An out-of-range column or neighbor index (one entry set
to N) is skipped by the kernels' own bounds checks and reported as MP_ERR_DEVICE_BOUNDS, with the
guard rows intact.
"""
import dataclasses

import numpy as np
import pytest
import torch

from atomistic_neighbor_list_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 8  # rows; 8 x 128 x 2 bytes keeps a bf16 view 16-byte aligned


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as _mp
    return _mp


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def guarded(n, f, dtype):
    big = torch.full((n + 2 * GUARD, f), float("nan"), dtype=dtype, device="cuda")
    return big, big[GUARD:GUARD + n]


def guards_intact(big):
    return bool(torch.isnan(big[:GUARD]).all() and torch.isnan(big[-GUARD:]).all())


def system(mp, n, key="cfg2", dtype="bf16", seed=3):
    wl = dataclasses.replace(synth.WORKLOADS[key], dtype=dtype)
    pos = synth.uniform_positions(n, seed=seed)  # the workloads' density, any n
    rp, ci = mp.neighbor_csr(dev(pos), wl.r_c)
    return wl, pos, rp, ci


@pytest.mark.parametrize("n", [1000, 1161])
def test_cfconv_outputs_stay_in_their_rows(mp, n):
    wl, pos, rp, ci = system(mp, n)
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=n, max_edges=ci.numel())
    x = dev(synth.node_features(n, wl.F)).to(torch.bfloat16)
    big, out = guarded(n, wl.F, torch.bfloat16)
    ctx.cfconv_fwd(0, dev(pos), rp, ci, x, out)
    ctx.pair_plan(rp, ci)
    big2, out2 = guarded(n, wl.F, torch.bfloat16)
    ctx.cfconv_fwd_pairs(0, dev(pos), x, out2)
    torch.cuda.synchronize()
    ctx.status_sync()
    assert guards_intact(big) and guards_intact(big2)
    assert not torch.isnan(out).any() and not torch.isnan(out2).any()


def test_fp32_cfconv_and_forces_stay_in_their_rows(mp):
    n = 777
    wl, pos, rp, ci = system(mp, n, key="cfg1", dtype="fp32")
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=n, max_edges=ci.numel())
    big, out = guarded(n, wl.F, torch.float32)
    ctx.cfconv_fwd(0, dev(pos), rp, ci, dev(synth.node_features(n, wl.F)), out)
    bigf, forces = guarded(n, 3, torch.float32)
    types = dev(synth.atom_types(n, wl.n_types))
    ctx.energy_forces(dev(pos), types, rp, ci, forces=forces)
    torch.cuda.synchronize()
    ctx.status_sync()
    assert guards_intact(big) and guards_intact(bigf)
    assert not torch.isnan(out).any() and not torch.isnan(forces).any()


def test_bf16_forces_and_attention_stay_in_their_rows(mp):
    n = 1161
    wl, pos, rp, ci = system(mp, n)
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=n, max_edges=ci.numel())
    bigf, forces = guarded(n, 3, torch.float32)
    ctx.energy_forces(dev(pos), dev(synth.atom_types(n, wl.n_types)), rp, ci, forces=forces)
    wl4 = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=n, K=128)
    nbr, mask = mp.neighbor_padded(dev(pos), wl4.r_c, wl4.K)
    ctx4 = mp.Context.from_workload(wl4, synth.make_weights(wl4), max_atoms=n, max_edges=1)
    big, out = guarded(n, wl4.F, torch.bfloat16)
    ctx4.attn_fwd(dev(pos), nbr, mask, dev(synth.node_features(n, wl4.F)).to(torch.bfloat16), out)
    torch.cuda.synchronize()
    ctx.status_sync()
    ctx4.status_sync()
    assert guards_intact(bigf) and guards_intact(big)
    assert not torch.isnan(forces).any() and not torch.isnan(out).any()


def test_out_of_range_column_is_reported_not_followed(mp):
    n = 1000
    wl, pos, rp, ci = system(mp, n)
    bad = ci.clone()
    bad[5] = n  # one column index past the last atom; the list is otherwise valid
    ctx = mp.Context.from_workload(wl, synth.make_weights(wl), max_atoms=n, max_edges=ci.numel())
    x = dev(synth.node_features(n, wl.F)).to(torch.bfloat16)
    big, out = guarded(n, wl.F, torch.bfloat16)
    ctx.cfconv_fwd(0, dev(pos), rp, bad, x, out)
    torch.cuda.synchronize()
    with pytest.raises(mp.MpError) as e:
        ctx.status_sync()
    assert e.value.name == "MP_ERR_DEVICE_BOUNDS"
    assert guards_intact(big) and not torch.isnan(out).any()
    bigf, forces = guarded(n, 3, torch.float32)
    ctx.energy_forces(dev(pos), dev(synth.atom_types(n, wl.n_types)), rp, bad, forces=forces)
    torch.cuda.synchronize()
    with pytest.raises(mp.MpError) as e:
        ctx.status_sync()
    assert e.value.name == "MP_ERR_DEVICE_BOUNDS"
    assert guards_intact(bigf)
    with pytest.raises(mp.MpError) as e:  # the pair plan checks the same indices
        ctx.pair_plan(rp, bad)
    assert e.value.name == "MP_ERR_DEVICE_BOUNDS"
    ctx.status_sync()  # the context goes on


def test_out_of_range_neighbor_is_reported_not_followed(mp):
    n = 600
    wl4 = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=n, K=128)
    pos = synth.uniform_positions(n, seed=5)
    nbr, mask = mp.neighbor_padded(dev(pos), wl4.r_c, wl4.K)
    bad = nbr.clone()
    bad[3, 0] = n
    mask2 = mask.clone()
    mask2[3, 0] = 1
    ctx = mp.Context.from_workload(wl4, synth.make_weights(wl4), max_atoms=n, max_edges=1)
    big, out = guarded(n, wl4.F, torch.bfloat16)
    ctx.attn_fwd(dev(pos), bad, mask2, dev(synth.node_features(n, wl4.F)).to(torch.bfloat16), out)
    torch.cuda.synchronize()
    with pytest.raises(mp.MpError) as e:
        ctx.status_sync()
    assert e.value.name == "MP_ERR_DEVICE_BOUNDS"
    assert guards_intact(big) and not torch.isnan(out).any()
