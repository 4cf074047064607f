"""Shared test helpers: seeded inputs for both sides, oracle models, error metrics."""
from __future__ import annotations

import numpy as np

from atomistic_neighbor_list_b200 import synth

# Tolerances (stated for the workloads): fp32 path relative error <= 1e-5; bf16 path <= 2e-2 on
# features and <= 1e-2 relative RMS on forces. Feature error is normwise: max|d| / max|ref| per tensor.
TOL_FP32 = 1e-5
TOL_BF16_FEAT = 2e-2
TOL_BF16_FORCE = 1e-2


def normwise(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref)) / (scale if scale > 0 else 1.0))


def rel_rms(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (n if n > 0 else 1.0))


def oracle_weights(weights: dict, dtype: str) -> dict:
    """The weight values the library holds: bf16-rounded (ties to even) under bf16."""
    if dtype != "bf16":
        return dict(weights)
    return {k: synth.round_bf16(v) for k, v in weights.items()}


def features_for(x: np.ndarray, dtype: str):
    """(torch tensor for the CUDA path, float64 array of the same stored values for the oracle)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t, t.float().numpy().astype(np.float64)


def oracle_csr(pos, r_c: float, rp, ci, graph_ptr=None):
    """The oracle's own cutoff CSR for the same positions, checked bit for bit against the CUDA
    path's lists (rp, ci: torch tensors), which then serve the CUDA side only: every oracle input
    comes from the seeded generator and the oracle itself."""
    import oracle
    orp, oci = oracle.neighbor_csr(pos, r_c, graph_ptr)
    assert np.array_equal(rp.cpu().numpy(), orp) and np.array_equal(ci.cpu().numpy(), oci)
    return orp, oci


def oracle_padded(pos, r_c: float, K: int, nbr, mask):
    """The oracle's own capped neighbor list, checked bit for bit against the CUDA path's."""
    import oracle
    onbr, omask = oracle.neighbor_padded(pos, r_c, K)
    assert np.array_equal(mask.cpu().numpy(), omask) and np.array_equal(nbr.cpu().numpy(), onbr)
    return onbr, omask
