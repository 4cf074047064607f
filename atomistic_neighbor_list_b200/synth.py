"""Seeded synthetic inputs for the five workloads (positions, atom types, node features, weights).

This module is shared by the CUDA path's tests and bench and by the oracle's tests. It draws random
numbers and lays them out; it holds none of the message-passing arithmetic (no distances, no radial
basis, no filter, no neighbor search).

Workloads (sizes, densities and cutoffs are the ones the five synthetic configurations state):

* ``cfg1`` -- 512 atoms uniform in a cube at 0.1 atoms/A^3 (no periodic boundary), one SchNet
  cfconv, F=64, 50 Gaussian radial functions, cutoff 5 A, fp32.
* ``cfg2`` -- 10,000 atoms uniform at 0.1 atoms/A^3, 10 atom types, 3 interaction blocks, F=128,
  cutoff 5 A, bf16 storage with fp32 accumulation, energy and forces.
* ``cfg3`` -- 64 replicas x 1,000 beads; each replica a self-avoiding random-walk chain with 3.8 A
  steps and 0.3 A Gaussian jitter, cutoff 10 A, 64 radial functions, 2 blocks, F=128, bf16.
* ``cfg4`` -- 32,768 atoms uniform at 0.1 atoms/A^3, cutoff 8.5 A, neighbor list capped/padded to
  K=256, 16 heads x 8 channels, online-softmax attention aggregation, bf16.
* ``cfg5`` -- 100,000 atoms uniform at 0.1 atoms/A^3, cutoff 5 A, 3 blocks, F=128, bf16, energy and
  forces; plus a 64-atom system of the same architecture for finite-difference checks.

Seeds: positions ``default_rng(0)``, atom types ``default_rng(1)``, weights ``default_rng(2)``,
node features ``default_rng(3)`` (the 512-atom case states seed 0; the others reuse the scheme).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

DENSITY = 0.1  # atoms per cubic Angstrom


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str               # "cfconv" | "energy_forces" | "attention"
    n_atoms: int
    r_c: float
    n_rbf: int
    F: int
    dtype: str              # "fp32" | "bf16"
    n_blocks: int = 1
    n_types: int = 10
    gamma: float = 10.0
    n_heads: int = 16
    head_dim: int = 8
    K: int = 0              # padded neighbor count (attention only)
    replicas: int = 1       # disjoint graphs (chain replicas)
    geometry: str = "uniform"  # "uniform" | "chains"

    @property
    def mu_min(self) -> float:
        return 0.0

    @property
    def mu_max(self) -> float:
        # Centres span 0 .. r_c inclusive ("centres 0-5 A" for the 5 A cutoff).
        return float(self.r_c)


WORKLOADS = {
    "cfg1": Workload("cfg1_512_fp32_cfconv", "cfconv", 512, 5.0, 50, 64, "fp32"),
    "cfg2": Workload("cfg2_10k_bf16_3blk_energy_forces", "energy_forces", 10_000, 5.0, 50, 128,
                     "bf16", n_blocks=3),
    "cfg3": Workload("cfg3_64x1000_chains_bf16_2blk", "energy_forces", 64_000, 10.0, 64, 128,
                     "bf16", n_blocks=2, replicas=64, geometry="chains"),
    "cfg4": Workload("cfg4_32768_attention_K256_bf16", "attention", 32_768, 8.5, 50, 128, "bf16",
                     K=256),
    "cfg5": Workload("cfg5_100k_bf16_3blk_energy_forces", "energy_forces", 100_000, 5.0, 50, 128,
                     "bf16", n_blocks=3),
    # 64-atom system with the 100k-atom architecture, for finite-difference force checks.
    "fd64": Workload("fd64_cfg5_arch", "energy_forces", 64, 5.0, 50, 128, "bf16", n_blocks=3),
}


def scaled(w: Workload, n_atoms: int, **kw) -> Workload:
    """The same architecture on a different number of atoms (same density)."""
    return dataclasses.replace(w, n_atoms=n_atoms, **kw)


def box_length(n_atoms: int, density: float = DENSITY) -> float:
    return (n_atoms / density) ** (1.0 / 3.0)


def uniform_positions(n_atoms: int, seed: int = 0, density: float = DENSITY) -> np.ndarray:
    """Atoms uniform in a cube of side (n/density)^(1/3), no periodic boundary, float32 [n,3]."""
    L = box_length(n_atoms, density)
    return np.random.default_rng(seed).uniform(0.0, L, size=(n_atoms, 3)).astype(np.float32)


def chain_replicas(n_rep: int, beads: int, seed: int = 0, step: float = 3.8,
                   jitter: float = 0.3, max_tries: int = 100):
    """Self-avoiding random-walk chains, one per replica, generated in sequence from one stream.

    Each step is a uniform random unit vector times ``step``; a trial bead closer than ``step`` to any
    earlier non-adjacent bead is rejected (``max_tries`` trials, then the chain restarts); after the
    walk every coordinate gets N(0, jitter^2). Returns float32 positions [n_rep*beads, 3] and the int32
    ``graph_ptr`` [n_rep+1] of contiguous replica ranges. Replicas share one frame (they overlap in
    space); the neighbor search keeps edges inside a replica.
    """
    rng = np.random.default_rng(seed)
    out = np.empty((n_rep * beads, 3), dtype=np.float64)
    for r in range(n_rep):
        while True:
            chain = np.zeros((beads, 3))
            ok = True
            for i in range(1, beads):
                placed = False
                for _ in range(max_tries):
                    v = rng.normal(size=3)
                    v *= step / np.linalg.norm(v)
                    cand = chain[i - 1] + v
                    if i >= 2:
                        dd = chain[: i - 1] - cand
                        if np.min(np.einsum("ij,ij->i", dd, dd)) < step * step:
                            continue
                    chain[i] = cand
                    placed = True
                    break
                if not placed:
                    ok = False
                    break
            if ok:
                break
        chain += rng.normal(scale=jitter, size=chain.shape)
        out[r * beads:(r + 1) * beads] = chain
    graph_ptr = (np.arange(n_rep + 1) * beads).astype(np.int32)
    return out.astype(np.float32), graph_ptr


def positions_for(w: Workload, seed: int = 0):
    """Positions float32 [N,3] and graph_ptr int32 [G+1] for a workload."""
    if w.geometry == "chains":
        beads = w.n_atoms // w.replicas
        return chain_replicas(w.replicas, beads, seed=seed)
    pos = uniform_positions(w.n_atoms, seed=seed)
    return pos, np.array([0, w.n_atoms], dtype=np.int32)


def atom_types(n_atoms: int, n_types: int = 10, seed: int = 1) -> np.ndarray:
    return np.random.default_rng(seed).integers(0, n_types, size=n_atoms).astype(np.int32)


def node_features(n_atoms: int, F: int, seed: int = 3) -> np.ndarray:
    return np.random.default_rng(seed).normal(size=(n_atoms, F)).astype(np.float32)


def _dense(rng, fan_in: int, shape) -> np.ndarray:
    """N(0, 1/fan_in) -- weights and biases alike, so that a dropped bias is visible."""
    return (rng.normal(size=shape) / math.sqrt(fan_in)).astype(np.float32)


def make_weights(w: Workload, seed: int = 2) -> dict:
    """All weights as float32 row-major [in][out] arrays, drawn in a fixed order from one stream.

    Keys: ``emb`` [n_types,F]; per block b: ``A1.b`` [R,F], ``c1.b`` [F], ``A2.b`` [F,F], ``c2.b`` [F],
    ``W_in.b`` [F,F], ``b_in.b`` [F], ``W_out.b`` [F,F], ``b_out.b`` [F]; readout ``B1`` [F,F/2],
    ``d1`` [F/2], ``B2`` [F/2,1], ``d2`` [1]; attention ``Wq``, ``Wk`` [F,F], ``P`` [R,H], ``p`` [H].
    """
    rng = np.random.default_rng(seed)
    F, R, H = w.F, w.n_rbf, w.n_heads
    out = {"emb": rng.normal(size=(w.n_types, F)).astype(np.float32)}
    for b in range(max(w.n_blocks, 1)):
        out[f"A1.{b}"] = _dense(rng, R, (R, F))
        out[f"c1.{b}"] = _dense(rng, R, (F,))
        out[f"A2.{b}"] = _dense(rng, F, (F, F))
        out[f"c2.{b}"] = _dense(rng, F, (F,))
        out[f"W_in.{b}"] = _dense(rng, F, (F, F))
        out[f"b_in.{b}"] = _dense(rng, F, (F,))
        out[f"W_out.{b}"] = _dense(rng, F, (F, F))
        out[f"b_out.{b}"] = _dense(rng, F, (F,))
    Fh = F // 2
    out["B1"] = _dense(rng, F, (F, Fh))
    out["d1"] = _dense(rng, F, (Fh,))
    out["B2"] = _dense(rng, Fh, (Fh, 1))
    out["d2"] = _dense(rng, Fh, (1,))
    out["Wq"] = _dense(rng, F, (F, F))
    out["Wk"] = _dense(rng, F, (F, F))
    out["P"] = _dense(rng, R, (R, H))
    out["p"] = _dense(rng, R, (H,))
    return out


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned as float32.

    Used to hand both sides of a bf16 comparison the same stored values; it is a storage-format
    conversion, not a step of the method.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    nan = np.isnan(a)
    r = (rounded & 0xFFFFFFFF).astype(np.uint32).view(np.float32).copy()
    r[nan] = np.nan
    return r.reshape(a.shape)
