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

from .schnet import Model, filter_weights, gaussian_rbf, gaussian_rbf_grad

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


def attention_vjp(model: Model, pos, nbr, mask, x, g, rows=None):
    """Gradients of L = sum_{i in rows} g_i . out_i with respect to x and the positions (float64).

    Reverse-mode differentiation of ``attention`` (E2Former-V2 page, section 3.2: the backward of
    the fused kernel; Tessera page: forces are gradients with respect to the positions). With
    v_ij = x_j (.) W(d_ij), alpha the softmax over the valid slots of row i, per head h:

        dalpha_ijh = sum_{c in h} g_i[c] v_ij[c]
        dl_ijh     = alpha_ijh (dalpha_ijh - sum_j' alpha_ij'h dalpha_ij'h)
        dL/dq_i    = sum_j dl_ijh k_jh / sqrt(D),      dL/dk_j += dl_ijh q_ih / sqrt(D)
        dL/dx_j   += alpha_ijh g_i (.) W(d_ij)          (value path)
        dL/dd_ij   = sum_c alpha g_i[c] x_j[c] W'(d_ij)[c] + sum_h dl_ijh sum_k e_k'(d_ij) P_kh
        dL/dr_i   += dL/dd_ij (r_i - r_j) / d_ij,  dL/dr_j -= the same
        dL/dx      = dL/dq Wq^T + dL/dk Wk^T + the value path.

    A pair at d = 0 contributes no position gradient. Rows not in ``rows`` contribute nothing.
    Returns (grad_x [N,F], grad_pos [N,3]).
    """
    w = model.w
    H, D = model.n_heads, model.head_dim
    pos64 = np.asarray(pos, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    nbr = np.asarray(nbr)
    mask = np.asarray(mask)
    n, K = nbr.shape
    F = x.shape[1]
    sel = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    sq = math.sqrt(D)
    q = x @ w["Wq"]
    kx = x @ w["Wk"]
    gq = np.zeros((n, F))
    gk = np.zeros((n, F))
    gx = np.zeros((n, F))
    gpos = np.zeros((n, 3))
    for c0 in range(0, len(sel), ROW_CHUNK):
        rws = sel[c0:c0 + ROW_CHUNK]
        nc = len(rws)
        valid = mask[rws] != 0
        jj = np.where(valid, nbr[rws], 0).astype(np.int64)
        vec = pos64[rws][:, None, :] - pos64[jj]
        d = np.sqrt(np.sum(vec * vec, axis=2)).ravel()
        e = gaussian_rbf(d, model.mu, model.gamma)
        de = gaussian_rbf_grad(d, model.mu, model.gamma)
        W, dW = filter_weights(model, 0, d, with_grad=True)
        W = W.reshape(nc, K, F)
        dW = dW.reshape(nc, K, F)
        xj = x[jj]
        v = (xj * W).reshape(nc, K, H, D)
        qi = q[rws].reshape(nc, H, D)
        kj = kx[jj].reshape(nc, K, H, D)
        logits = (np.einsum("nhd,nkhd->nkh", qi, kj) / sq
                  + (e @ w["P"]).reshape(nc, K, H) + w["p"][None, None, :])
        logits = np.where(valid[:, :, None], logits, -np.inf)
        has = valid.any(axis=1)
        mx = np.where(has[:, None], np.max(np.where(has[:, None, None], logits, 0.0), axis=1), 0.0)
        p = np.where(valid[:, :, None], np.exp(logits - mx[:, None, :]), 0.0)
        z = p.sum(axis=1)
        alpha = p / np.where(z > 0, z, 1.0)[:, None, :]
        gi = g[rws].reshape(nc, H, D)
        dalpha = np.einsum("nhd,nkhd->nkh", gi, v)
        dl = alpha * (dalpha - np.sum(alpha * dalpha, axis=1)[:, None, :])
        # logits: q_i and k_j
        gq[rws] += (np.einsum("nkh,nkhd->nhd", dl, kj) / sq).reshape(nc, F)
        dk = (dl[:, :, :, None] * qi[:, None, :, :] / sq).reshape(nc * K, F)
        # value path
        gv = (alpha[:, :, :, None] * gi[:, None, :, :]).reshape(nc, K, F)
        dxj = (gv * W).reshape(nc * K, F)
        keep = valid.ravel()
        np.add.at(gk, jj.ravel()[keep], dk[keep])
        np.add.at(gx, jj.ravel()[keep], dxj[keep])
        # distance: the filter and the logit bias
        s = (np.sum(gv * xj * dW, axis=2)
             + np.einsum("nkh,nkh->nk", dl, (de @ w["P"]).reshape(nc, K, H))).ravel()
        s = np.where(keep, s, 0.0)
        safe = d > 0
        u = np.where(safe[:, None], vec.reshape(nc * K, 3) / np.where(safe, d, 1.0)[:, None], 0.0)
        su = s[:, None] * u
        np.add.at(gpos, np.repeat(rws, K), su)
        np.add.at(gpos, jj.ravel(), -su)
    gx += gq @ w["Wq"].T + gk @ w["Wk"].T
    return gx, gpos


# ----------------------------------------------------------------------------- equivariant values
SH_C0 = 0.5 / math.sqrt(math.pi)
SH_C1 = math.sqrt(3.0 / (4.0 * math.pi))
SH_C2 = 0.5 * math.sqrt(15.0 / math.pi)
SH_C20 = 0.25 * math.sqrt(5.0 / math.pi)
SH_C22 = 0.25 * math.sqrt(15.0 / math.pi)


def solid_harmonics(r) -> np.ndarray:
    """Regular solid harmonics S_lm(r) = |r|^l Y_lm(r/|r|) for l <= 2 (float64 [..., 9]).

    Y_lm: the real spherical harmonics orthonormal on the sphere, components in the order
    (0,0), (1,-1), (1,0), (1,1), (2,-2), (2,-1), (2,0), (2,1), (2,2): as polynomials of (x, y, z),
    c0; c1 y, c1 z, c1 x; c2 xy, c2 yz, c20 (2z^2 - x^2 - y^2), c2 xz, c22 (x^2 - y^2).
    """
    r = np.asarray(r, dtype=np.float64)
    x, y, z = r[..., 0], r[..., 1], r[..., 2]
    return np.stack([np.full_like(x, SH_C0), SH_C1 * y, SH_C1 * z, SH_C1 * x,
                     SH_C2 * x * y, SH_C2 * y * z, SH_C20 * (2 * z * z - x * x - y * y),
                     SH_C2 * x * z, SH_C22 * (x * x - y * y)], axis=-1)


def attention_equivariant(model: Model, pos, nbr, mask, x, rows=None) -> np.ndarray:
    """Attention with an equivariant value path, float64 [n_rows, 9, F].

    E2Former-V2 page, section 3.1: direction enters only through the value path -- each value is
    coupled with spherical harmonics of the geometry, the attention weights stay scalar. Reading:
    the value of slot j of row i is v_ij (x) S(r_j - r_i) with v_ij = x_j (.) W(d_ij) and S the
    regular solid harmonics up to l = 2 (``solid_harmonics``), so

        out_i[lm, c] = sum_j alpha_ij,h(c) v_ij[c] S_lm(r_j - r_i),

    with the same softmax weights alpha as ``attention``; out_i[(0,0)] = c0 * attention(...)_i.
    """
    H, D = model.n_heads, model.head_dim
    pos64 = np.asarray(pos, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    nbr = np.asarray(nbr)
    mask = np.asarray(mask)
    n, K = nbr.shape
    F = x.shape[1]
    w = model.w
    sel = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    q = x[sel] @ w["Wq"]
    kx = x @ w["Wk"]
    out = np.zeros((len(sel), 9, F))
    for c0 in range(0, len(sel), ROW_CHUNK):
        rws = sel[c0:c0 + ROW_CHUNK]
        nc = len(rws)
        valid = mask[rws] != 0
        jj = np.where(valid, nbr[rws], 0).astype(np.int64)
        rel = pos64[jj] - pos64[rws][:, None, :]          # r_j - r_i
        d = np.sqrt(np.sum(rel * rel, axis=2)).ravel()
        e = gaussian_rbf(d, model.mu, model.gamma)
        W = filter_weights(model, 0, d).reshape(nc, K, F)
        v = x[jj] * W                                     # [nc, K, F]
        qk = np.einsum("nhd,nkhd->nkh", q[c0:c0 + nc].reshape(nc, H, D),
                       kx[jj].reshape(nc, K, H, D))
        logits = qk / math.sqrt(D) + (e @ w["P"]).reshape(nc, K, H) + w["p"][None, None, :]
        logits = np.where(valid[:, :, None], logits, -np.inf)
        has = valid.any(axis=1)
        mx = np.where(has[:, None], np.max(np.where(has[:, None, None], logits, 0.0), axis=1), 0.0)
        p = np.where(valid[:, :, None], np.exp(logits - mx[:, None, :]), 0.0)
        z = p.sum(axis=1)
        alpha = p / np.where(z > 0, z, 1.0)[:, None, :]
        a_f = np.repeat(alpha, D, axis=2)                 # [nc, K, F]: head of each channel
        S = solid_harmonics(rel)                          # [nc, K, 9]
        out[c0:c0 + nc] = np.einsum("nkf,nkm->nmf", a_f * v, S)
    return out


def moments_to_solid(m, ri) -> np.ndarray:
    """Target coupling of the node-centric form: given the moments m[..., mu, F] of the values
    against the monomials (1, x, y, z, xx, xy, xz, yy, yz, zz) of the SOURCE positions, and the
    destination position ri [..., 3], return sum_j a_j S(r_j - r_i) [..., 9, F] by expanding each
    solid harmonic of (r_j - r_i) in monomials of r_j with coefficients from r_i."""
    m = np.asarray(m, dtype=np.float64)
    xi, yi, zi = (np.asarray(ri, dtype=np.float64)[..., k, None] for k in range(3))
    one, X, Y, Z, XX, XY, XZ, YY, YZ, ZZ = (m[..., k, :] for k in range(10))
    dX, dY, dZ = X - xi * one, Y - yi * one, Z - zi * one          # sums of a (x_j - x_i) ...
    dXX = XX - 2 * xi * X + xi * xi * one
    dYY = YY - 2 * yi * Y + yi * yi * one
    dZZ = ZZ - 2 * zi * Z + zi * zi * one
    dXY = XY - xi * Y - yi * X + xi * yi * one
    dYZ = YZ - yi * Z - zi * Y + yi * zi * one
    dXZ = XZ - xi * Z - zi * X + xi * zi * one
    return np.stack([SH_C0 * one, SH_C1 * dY, SH_C1 * dZ, SH_C1 * dX, SH_C2 * dXY, SH_C2 * dYZ,
                     SH_C20 * (2 * dZZ - dXX - dYY), SH_C2 * dXZ, SH_C22 * (dXX - dYY)], axis=-2)
