"""The allocation-free attention entry point gives what the regular one gives.

mp_attn_fwd_noalloc exists for callers that cannot call cudaMalloc: hosts (an MD engine's plugin
interface, a serving process with a fixed memory plan) that own all device memory through their own
pool and hand a library only pre-allocated buffers. It keeps its query/key scratch in a static device
array inside the library instead of a context workspace. This test calls it through the C-ABI and
compares it with mp_attn_fwd (same fp32 kernels) within the fp32 tolerance, on two calls in a row of
different sizes, so that the shared array's leftover contents from the first call cannot leak into
the second. The file is named to run last.
"""
import dataclasses

import numpy as np
import pytest
import torch

from atomistic_neighbor_list_b200 import synth
from helpers import TOL_FP32, normwise

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mp(cuda_ok):
    from atomistic_neighbor_list_b200 import mp as _mp
    return _mp


def _case(mp, n, K, seed):
    wl = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=n, K=K, dtype="fp32")
    pos = torch.from_numpy(synth.uniform_positions(n, seed=seed)).cuda()
    w = synth.make_weights(wl, seed=seed + 20)
    nbr, mask = mp.neighbor_padded(pos, wl.r_c, K)
    x = torch.from_numpy(synth.node_features(n, wl.F, seed=seed + 10)).cuda()
    ctx = mp.Context.from_workload(wl, w, max_atoms=n, max_edges=1)
    ref = ctx.attn_fwd(pos, nbr, mask, x)
    wdev = {k: torch.from_numpy(w[k]).cuda()
            for k in ("Wq", "Wk", "P", "p", "A1.0", "c1.0", "A2.0", "c2.0")}
    out = torch.full_like(x, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    mp.attn_fwd_noalloc(F=wl.F, n_rbf=wl.n_rbf, n_heads=wl.n_heads, head_dim=wl.head_dim,
                        r_c=wl.r_c, gamma=wl.gamma, weights=wdev, pos=pos, nbr=nbr, mask=mask,
                        x=x, out=out, status=status)
    torch.cuda.synchronize()
    ctx.close()
    return out.cpu().numpy(), ref.cpu().numpy(), int(status.item())


def test_noalloc_matches_attn_fwd_on_two_calls_in_a_row(mp):
    for n, K, seed in ((3000, 128, 1), (1200, 256, 2)):
        got, ref, status = _case(mp, n, K, seed)
        assert status == 0
        assert np.all(np.isfinite(got))
        assert normwise(got, ref) <= TOL_FP32


def test_noalloc_allocates_nothing_and_matches_the_oracle(mp):
    # a warm call with every buffer given leaves the device's free memory unchanged, and a small
    # case agrees with the fp64 oracle directly (not only through mp_attn_fwd)
    import oracle
    n, K = 400, 64
    wl = dataclasses.replace(synth.WORKLOADS["cfg4"], n_atoms=n, K=K, dtype="fp32")
    pos_h = synth.uniform_positions(n, seed=4)
    pos = torch.from_numpy(pos_h).cuda()
    w = synth.make_weights(wl, seed=24)
    nbr, mask = mp.neighbor_padded(pos, wl.r_c, K)
    x_h = synth.node_features(n, wl.F, seed=14)
    x = torch.from_numpy(x_h).cuda()
    wdev = {k: torch.from_numpy(w[k]).cuda()
            for k in ("Wq", "Wk", "P", "p", "A1.0", "c1.0", "A2.0", "c2.0")}
    out = torch.empty_like(x)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    kw = dict(F=wl.F, n_rbf=wl.n_rbf, n_heads=wl.n_heads, head_dim=wl.head_dim, r_c=wl.r_c,
              gamma=wl.gamma, weights=wdev, pos=pos, nbr=nbr, mask=mask, x=x, out=out,
              status=status)
    mp.attn_fwd_noalloc(**kw)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    mp.attn_fwd_noalloc(**kw)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0 and int(status.item()) == 0
    onbr, omask = oracle.neighbor_padded(pos_h, wl.r_c, K)
    assert np.array_equal(nbr.cpu().numpy(), onbr) and np.array_equal(mask.cpu().numpy(), omask)
    model = oracle.Model.from_workload(wl, w)
    ref = oracle.attention(model, pos_h, onbr, omask, x_h)
    assert normwise(out.cpu().numpy(), ref) <= TOL_FP32


def test_noalloc_rejects_more_than_its_scratch_holds(mp):
    n = mp.NOALLOC_MAX_NF // 128 + 1
    pos = torch.zeros((n, 3), dtype=torch.float32, device="cuda")
    nbr = torch.full((n, 4), -1, dtype=torch.int32, device="cuda")
    mask = torch.zeros((n, 4), dtype=torch.uint8, device="cuda")
    x = torch.zeros((n, 128), dtype=torch.float32, device="cuda")
    # full-size weights: the call must fail on its capacity check, never by reading past them
    shapes = {"Wq": (128, 128), "Wk": (128, 128), "P": (50, 16), "p": (16,), "A1.0": (50, 128),
              "c1.0": (128,), "A2.0": (128, 128), "c2.0": (128,)}
    w = {k: torch.zeros(s, dtype=torch.float32, device="cuda") for k, s in shapes.items()}
    with pytest.raises(mp.MpError) as e:
        mp.attn_fwd_noalloc(F=128, n_rbf=50, n_heads=16, head_dim=8, r_c=8.5, weights=w, pos=pos,
                            nbr=nbr, mask=mask, x=x)
    assert e.value.name == "MP_ERR_CAPACITY"
