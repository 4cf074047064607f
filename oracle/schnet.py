"""SchNet-style continuous-filter convolution, energy and analytic forces in float64 (oracle).

Test infrastructure only (see the package docstring). Definitions, in the order the method applies
them (FlashSchNet page, technical summary section 1 lists the stages; sections 2.1-2.3 fuse them):

1. distance        d_ij = |r_i - r_j|                                 (2.1: computed once per edge)
2. Gaussian basis  e_k(d) = exp(-gamma (d - mu_k)^2),  mu_k = mu_min + k (mu_max - mu_min)/(R-1)
3. cosine envelope f_c(d) = (cos(pi d / r_c) + 1)/2 for d < r_c, else exactly 0
4. filter MLP      W(d) = f_c(d) * ( ssp(e(d) A1 + c1) A2 + c2 ),  ssp(x) = ln(e^x/2 + 1/2)
5. cfconv          m_i = sum_{j in N(i)} x_j (.) W(d_ij)              (2.2 gather/multiply, 2.3 reduce)
6. block           h = x W_in + b_in;  m = cfconv(h);  x <- x + m W_out + b_out
7. embedding       x0 = emb[type];  readout e_i = ssp(x_i B1 + d1) B2 + d2;  E_g = sum_{i in g} e_i
8. forces          F = -dE/dr by reverse-mode differentiation of 1-7 (Tessera page: forces are the
                   gradient of the energy; FlashSchNet 2.3: the backward groups edges by source).

Readings where the pages are silent: the Gaussian form with centres spanning 0..r_c inclusive and
gamma = 10 / A^2; the envelope multiplies the filter output (the only placement that makes a pair at
the cutoff contribute exactly zero despite the filter biases); ssp follows the first filter layer
only and both filter layers carry biases; the block's dense layers are linear with biases and no
activation; the readout is F -> F/2 -> 1 with ssp; coincident atoms (d = 0) contribute no force.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.sparse as sp
from scipy.special import expit

LN2 = math.log(2.0)
EDGE_CHUNK = 1 << 17  # edges per destination-row chunk (memory bound only)


# ----------------------------------------------------------------------------- element functions
def rbf_centres(R: int, mu_min: float, mu_max: float) -> np.ndarray:
    return mu_min + np.arange(R, dtype=np.float64) * ((mu_max - mu_min) / (R - 1))


def gaussian_rbf(d, mu, gamma):
    """e_k(d) = exp(-gamma (d - mu_k)^2), shape [E, R]."""
    d = np.asarray(d, dtype=np.float64)
    return np.exp(-gamma * (d[:, None] - mu[None, :]) ** 2)


def gaussian_rbf_grad(d, mu, gamma):
    """de_k/dd = -2 gamma (d - mu_k) e_k(d)."""
    d = np.asarray(d, dtype=np.float64)
    diff = d[:, None] - mu[None, :]
    return -2.0 * gamma * diff * np.exp(-gamma * diff ** 2)


def cosine_cutoff(d, r_c):
    d = np.asarray(d, dtype=np.float64)
    return np.where(d < r_c, 0.5 * (np.cos(np.pi * d / r_c) + 1.0), 0.0)


def cosine_cutoff_grad(d, r_c):
    d = np.asarray(d, dtype=np.float64)
    return np.where(d < r_c, -0.5 * (np.pi / r_c) * np.sin(np.pi * d / r_c), 0.0)


def ssp(x):
    """Shifted softplus ln(e^x/2 + 1/2) = ln(1 + e^x) - ln 2, evaluated stably."""
    return np.logaddexp(0.0, np.asarray(x, dtype=np.float64)) - LN2


def ssp_grad(x):
    """d ssp / dx = logistic sigmoid."""
    return expit(np.asarray(x, dtype=np.float64))


# ----------------------------------------------------------------------------- model container
class Model:
    """Weights (float64 copies) and hyper-parameters of one SchNet-style force field."""

    def __init__(self, weights: dict, n_blocks: int, r_c: float, n_rbf: int, gamma: float = 10.0,
                 mu_min: float = 0.0, mu_max: float | None = None, n_heads: int = 16,
                 head_dim: int = 8):
        self.w = {k: np.asarray(v, dtype=np.float64) for k, v in weights.items()}
        self.n_blocks = n_blocks
        self.r_c = float(np.float32(r_c))
        self.R = n_rbf
        self.gamma = float(np.float32(gamma))
        self.mu = rbf_centres(n_rbf, float(np.float32(mu_min)),
                              float(np.float32(self.r_c if mu_max is None else mu_max)))
        self.n_heads = n_heads
        self.head_dim = head_dim

    @classmethod
    def from_workload(cls, wl, weights):
        return cls(weights, wl.n_blocks, wl.r_c, wl.n_rbf, wl.gamma, wl.mu_min, wl.mu_max,
                   wl.n_heads, wl.head_dim)

    def filt(self, b: int):
        w = self.w
        return w[f"A1.{b}"], w[f"c1.{b}"], w[f"A2.{b}"], w[f"c2.{b}"]


def filter_weights(model: Model, b: int, d, with_grad: bool = False):
    """Filter W(d) [E,F] of block ``b`` and, if asked, dW/dd by the chain rule."""
    A1, c1, A2, c2 = model.filt(b)
    e = gaussian_rbf(d, model.mu, model.gamma)
    z1 = e @ A1 + c1
    u = ssp(z1) @ A2 + c2
    fc = cosine_cutoff(d, model.r_c)
    W = fc[:, None] * u
    if not with_grad:
        return W
    dz1 = gaussian_rbf_grad(d, model.mu, model.gamma) @ A1
    du = (ssp_grad(z1) * dz1) @ A2
    dW = cosine_cutoff_grad(d, model.r_c)[:, None] * u + fc[:, None] * du
    return W, dW


# ----------------------------------------------------------------------------- CSR helpers
def _row_chunks(row_ptr: np.ndarray, rows=None, max_edges: int = EDGE_CHUNK):
    """Yield arrays of destination rows whose edges together stay near ``max_edges``."""
    rp = np.asarray(row_ptr, dtype=np.int64)
    n = len(rp) - 1
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    start = 0
    while start < len(rows):
        stop = start + 1
        count = rp[rows[start] + 1] - rp[rows[start]]
        while stop < len(rows):
            c = rp[rows[stop] + 1] - rp[rows[stop]]
            if count + c > max_edges:
                break
            count += c
            stop += 1
        yield rows[start:stop]
        start = stop


def _edges(pos64, row_ptr, col_idx, rows):
    """Edges of ``rows`` in CSR order: local row, dst, src, r_dst - r_src, distance."""
    rp = np.asarray(row_ptr, dtype=np.int64)
    counts = rp[rows + 1] - rp[rows]
    total = int(counts.sum())
    first = np.repeat(rp[rows], counts)
    offset = np.arange(total) - np.repeat(np.cumsum(counts) - counts, counts)
    eid = first + offset
    local = np.repeat(np.arange(len(rows)), counts)
    dst = rows[local]
    src = np.asarray(col_idx, dtype=np.int64)[eid]
    vec = pos64[dst] - pos64[src]
    d = np.sqrt(np.sum(vec * vec, axis=1))
    return local, counts, dst, src, vec, d


def _segment_sum(vals: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """Sum consecutive runs of rows of ``vals`` (run lengths ``counts``); empty runs give 0."""
    out = np.zeros((len(counts),) + vals.shape[1:], dtype=np.float64)
    nz = counts > 0
    if vals.shape[0]:
        starts = (np.cumsum(counts) - counts)[nz]
        out[nz] = np.add.reduceat(vals, starts, axis=0)
    return out


def _scatter_rows(index: np.ndarray, vals: np.ndarray, n: int) -> np.ndarray:
    """out[index[e]] += vals[e] (a sparse row sum)."""
    m = sp.csr_matrix((np.ones(len(index)), (index, np.arange(len(index)))), shape=(n, len(index)))
    return np.asarray(m @ vals)


# ----------------------------------------------------------------------------- cfconv
def cfconv(model: Model, b: int, pos, row_ptr, col_idx, x, rows=None) -> np.ndarray:
    """m_i = sum_{j in N(i)} x_j (.) W(d_ij) for every row (or only ``rows``, in that order)."""
    pos64 = np.asarray(pos, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    n = len(row_ptr) - 1
    sel = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(sel), x.shape[1]), dtype=np.float64)
    pos_in_out = 0
    for chunk in _row_chunks(row_ptr, sel):
        local, counts, dst, src, vec, d = _edges(pos64, row_ptr, col_idx, chunk)
        W = filter_weights(model, b, d)
        out[pos_in_out:pos_in_out + len(chunk)] = _segment_sum(x[src] * W, counts)
        pos_in_out += len(chunk)
    return out


def undirected_pairs(row_ptr, col_idx):
    """The pairs {i, j} of a symmetric CSR once each, as (i, j) with i < j, in CSR order of i.

    Raises ValueError when an edge j -> i has no reverse edge i -> j (the pair form needs the
    symmetric list a cutoff graph has; FlashSchNet page, 2.3)."""
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx, dtype=np.int64)
    n = len(rp) - 1
    dst = np.repeat(np.arange(n), np.diff(rp))
    fwd = set(zip(dst.tolist(), ci.tolist()))
    if any((j, i) not in fwd for i, j in fwd):
        raise ValueError("the neighbor list is not symmetric")
    up = ci > dst
    return dst[up], ci[up]


def cfconv_pairs(model: Model, b: int, pos, row_ptr, col_idx, x) -> np.ndarray:
    """The cfconv evaluated over undirected pairs: the filter W(d_ij) = W(d_ji) once per pair
    {i, j}, then both messages from it, x_j (.) W to row i and x_i (.) W to row j.

    Same sum as ``cfconv`` (the filter depends on the pair's distance only), reached with half the
    filter evaluations (the symmetric list of FlashSchNet page 2.3; the pair-once evaluation is the
    halving the filter-MLP stage allows)."""
    pos64 = np.asarray(pos, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    n = len(row_ptr) - 1
    i, j = undirected_pairs(row_ptr, col_idx)
    vec = pos64[i] - pos64[j]
    d = np.sqrt(np.sum(vec * vec, axis=1))
    W = filter_weights(model, b, d)
    return _scatter_rows(i, x[j] * W, n) + _scatter_rows(j, x[i] * W, n)


# ----------------------------------------------------------------------------- energy / forces
def _forward(model: Model, pos, types, row_ptr, col_idx):
    w = model.w
    x = w["emb"][np.asarray(types, dtype=np.int64)]
    hs = []
    for b in range(model.n_blocks):
        h = x @ w[f"W_in.{b}"] + w[f"b_in.{b}"]
        m = cfconv(model, b, pos, row_ptr, col_idx, h)
        x = x + m @ w[f"W_out.{b}"] + w[f"b_out.{b}"]
        hs.append(h)
    a = x @ w["B1"] + w["d1"]
    e_atom = ssp(a) @ w["B2"][:, 0] + w["d2"][0]
    return e_atom, hs, a


def _per_graph(e_atom, graph_ptr, n):
    gp = np.asarray([0, n] if graph_ptr is None else graph_ptr, dtype=np.int64)
    return np.array([e_atom[gp[g]:gp[g + 1]].sum() for g in range(len(gp) - 1)])


def energies(model: Model, pos, types, row_ptr, col_idx, graph_ptr=None) -> np.ndarray:
    """Per-graph energies E_g (float64 [G])."""
    e_atom, _, _ = _forward(model, pos, types, row_ptr, col_idx)
    return _per_graph(e_atom, graph_ptr, len(types))


def energy_forces(model: Model, pos, types, row_ptr, col_idx, graph_ptr=None,
                  method: str = "scatter", return_atom_energy: bool = False):
    """Per-graph energies and forces F = -dE/dr (float64 [N,3]).

    ``method="scatter"``: plain reverse-mode backprop over directed edges -- each edge (dst i, src j)
    sends g_i (.) W_ij to grad_h[j] and dE/dd_ij (r_i - r_j)/d_ij to +grad_r[i] and -grad_r[j].

    ``method="pair"``: the destination-gathered form the fused backward uses on a symmetric CSR --
    grad_h[k] = sum_{j in N(k)} g_j (.) W_kj and grad_r[k] = sum_{j in N(k)} s_kj (r_k - r_j)/d_kj with
    s_kj = sum_f (g_k h_j + g_j h_k)_f dW_f/dd(d_kj). Both forms must agree.
    """
    w = model.w
    pos64 = np.asarray(pos, dtype=np.float64)
    n = len(types)
    e_atom, hs, a = _forward(model, pos64, types, row_ptr, col_idx)
    g_x = (ssp_grad(a) * w["B2"][:, 0]) @ w["B1"].T
    grad_r = np.zeros((n, 3))
    for b in reversed(range(model.n_blocks)):
        g_m = g_x @ w[f"W_out.{b}"].T
        h = hs[b]
        grad_h = np.zeros_like(h)
        for chunk in _row_chunks(row_ptr):
            local, counts, dst, src, vec, d = _edges(pos64, row_ptr, col_idx, chunk)
            W, dW = filter_weights(model, b, d, with_grad=True)
            safe = d > 0
            inv_d = np.where(safe, 1.0 / np.where(safe, d, 1.0), 0.0)
            if method == "scatter":
                grad_h += _scatter_rows(src, g_m[dst] * W, n)
                dEdd = np.sum(g_m[dst] * h[src] * dW, axis=1)
                gvec = (dEdd * inv_d)[:, None] * vec
                grad_r += _scatter_rows(dst, gvec, n) - _scatter_rows(src, gvec, n)
            elif method == "pair":
                grad_h[chunk] += _segment_sum(g_m[src] * W, counts)
                s = np.sum((g_m[dst] * h[src] + g_m[src] * h[dst]) * dW, axis=1)
                grad_r[chunk] += _segment_sum((s * inv_d)[:, None] * vec, counts)
            else:
                raise ValueError(method)
        g_x = g_x + grad_h @ w[f"W_in.{b}"].T
    E = _per_graph(e_atom, graph_ptr, n)
    if return_atom_energy:
        return E, -grad_r, e_atom
    return E, -grad_r
