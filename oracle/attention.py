"""Neighbor attention aggregation over a padded neighbor list, float64 (oracle; test infrastructure).

E2Former-V2 page, section 3.1: aggregation at the destination, m_i = sum_j alpha_ij . h_j, with the
weights computed on the fly; section 3.2: per destination atom, a softmax over its (masked, padded)
neighbors. The fused kernel computes the softmax online (running maximum and normaliser); this oracle
computes the same quantity the plain two-pass way (maximum, then exponentials and their sum).

Per destination i, head h (H heads of D channels, F = H*D), valid slots j of row i:

    q = x Wq,  k = x Wk                                   (no bias)
    l_ijh = q_ih . k_jh / sqrt(D) + sum_k e_k(d_ij) P_kh + p_h
    alpha_ijh = exp(l_ijh - max_j l_ijh) / sum_j exp(l_ijh - max_j l_ijh)
    out_i[hD:(h+1)D] = sum_j alpha_ijh (x_j (.) W(d_ij))[hD:(h+1)D]

with e(d) the Gaussian basis and W(d) the cosine-enveloped filter MLP of the cfconv (first block's
filter weights). Readings: only the validity mask enters the logits (the envelope acts through the
value); a row with no valid neighbor gives a zero output.
"""
from __future__ import annotations

import math

import numpy as np

from .schnet import Model, filter_weights, gaussian_rbf

ROW_CHUNK = 256


def attention(model: Model, pos, nbr, mask, x, rows=None) -> np.ndarray:
    w = model.w
    H, D = model.n_heads, model.head_dim
    pos64 = np.asarray(pos, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    nbr = np.asarray(nbr)
    mask = np.asarray(mask)
    n, K = nbr.shape
    F = x.shape[1]
    assert F == H * D
    sel = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    q = x[sel] @ w["Wq"]
    kx = x @ w["Wk"]
    out = np.zeros((len(sel), F))
    for c0 in range(0, len(sel), ROW_CHUNK):
        rws = sel[c0:c0 + ROW_CHUNK]
        nc = len(rws)
        valid = mask[rws] != 0
        jj = np.where(valid, nbr[rws], 0).astype(np.int64)
        vec = pos64[rws][:, None, :] - pos64[jj]
        d = np.sqrt(np.sum(vec * vec, axis=2)).ravel()
        e = gaussian_rbf(d, model.mu, model.gamma)
        W = filter_weights(model, 0, d).reshape(nc, K, F)
        v = (x[jj] * W).reshape(nc, K, H, D)
        qk = np.einsum("nhd,nkhd->nkh", q[c0:c0 + nc].reshape(nc, H, D), kx[jj].reshape(nc, K, H, D))
        logits = qk / math.sqrt(D) + (e @ w["P"]).reshape(nc, K, H) + w["p"][None, None, :]
        logits = np.where(valid[:, :, None], logits, -np.inf)
        has = valid.any(axis=1)
        mx = np.where(has[:, None], np.max(np.where(has[:, None, None], logits, 0.0), axis=1), 0.0)
        p = np.where(valid[:, :, None], np.exp(logits - mx[:, None, :]), 0.0)
        z = p.sum(axis=1)
        alpha = p / np.where(z > 0, z, 1.0)[:, None, :]
        out[c0:c0 + nc] = np.einsum("nkh,nkhd->nhd", alpha, v).reshape(nc, F)
    return out
