"""fp64 gradients of the projector (TEST INFRASTRUCTURE ONLY).

The trained part of the bridge is the projector alone: the tower and the language
model stay frozen ("DeepSeek-V4-Flash-Vision-BF16", first section: only the
40,119,040 projector parameters are trained). Given the gradient of the loss with
respect to the combined embedding buffer (d_out, one row per id), this module
returns the gradients of every projector parameter - LayerNorm gamma / beta, W1, b1,
W2, b2, and the learned newline / view-separator rows of the 2D tiling - and of the
input features, by the chain rule through the forward steps of `projector`:

    rows of an image at its placeholders  <- assembly of per-view rows (+ newline, sep)
    y = h W2^T + b2,  h = bf16(GELU(p)),  p = a W1^T + b1,  a = unshuffle(bf16(LN(x)))

Reading: the bf16 rounding points (a and h) pass gradients through unchanged
(straight-through), as mixed-precision training treats them. Only depth-2 MLPs.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
from scipy.special import erf as _erf

from . import projector as O


def gelu_grad(p: np.ndarray) -> np.ndarray:
    """d/dp of 0.5 p (1 + erf(p / sqrt 2)) = Phi(p) + p phi(p)."""
    p = np.asarray(p, np.float64)
    return 0.5 * (1.0 + _erf(p / math.sqrt(2.0))) + p * np.exp(-0.5 * p * p) / math.sqrt(2.0 * math.pi)


def layernorm_backward(dsrc: np.ndarray, xhat: np.ndarray, rstd: np.ndarray, gamma: np.ndarray) -> np.ndarray:
    """Input gradient of y = xhat * gamma + beta, xhat = (x - mean) * rstd over the last
    axis (biased variance): rstd * (g - mean(g) - xhat * mean(g * xhat)), g = dy * gamma."""
    g = dsrc * gamma
    return rstd * (g - g.mean(axis=1, keepdims=True) - xhat * (g * xhat).mean(axis=1, keepdims=True))


def _image_row_map(hp: int, wp: int, crop: Optional[tuple], n_views: int, gvp: str) -> np.ndarray:
    """For each assembled row of an image: the token index (view-major, row-major inside
    a view) it holds, -1 for a newline, -2 for the view separator."""
    if crop is None:
        return np.arange(hp * wp)
    tw, th = crop
    views = np.arange(n_views * hp * wp, dtype=np.float64).reshape(n_views, hp * wp, 1)
    rows = O.assemble_2d(views, hp, wp, tw, th, np.array([-1.0]), np.array([-2.0]), gvp)
    return rows[:, 0].astype(np.int64)


def backward(features: np.ndarray, grid_hw: np.ndarray, spatial_crop: Optional[np.ndarray], k: int, params: dict,
             ids: np.ndarray, image_token_id: int, d_out: np.ndarray, ln_eps: float = 1e-5,
             feat_is_bf16_bits: bool = True, quantise: bool = True, gvp: str = "head",
             skip_zero_rows: bool = False, magnitudes: bool = False) -> dict:
    """Gradients for the loss <d_out, forward(...)>; ``d_out`` is (n_ids, N2) or anything
    indexable by an array of row numbers. With ``skip_zero_rows`` the MLP is evaluated
    only for merged tokens whose output gradient row is nonzero: the others contribute
    exactly zero to every gradient (dY = 0 gives dP = 0, dA = 0 and a zero LayerNorm
    input gradient).

    With ``magnitudes`` the result also holds, under "mag", the same chain evaluated on
    absolute values: for every gradient entry the sum of the absolute values of the
    terms it is made of (|dY|^T |H| for dW2, |dP|^T |A| for dW1, and so on through the
    LayerNorm backward). A relative perturbation of at most e in each term moves the
    entry by at most e times this sum, which is how the GPU parity tests bound the
    effect of bf16 rounding."""
    grid_hw = np.asarray(grid_hw)
    x_all = O.bf16_bits_to_f64(features) if feat_is_bf16_bits else np.asarray(features, np.float64)
    W1, b1, W2, b2 = params["W1"], params["b1"], params["W2"], params["b2"]
    gamma, beta = params.get("gamma"), params.get("beta")
    has_ln = gamma is not None
    C = x_all.shape[1]
    g = {"W1": np.zeros_like(W1), "b1": np.zeros_like(b1), "W2": np.zeros_like(W2), "b2": np.zeros_like(b2),
         "features": np.zeros_like(x_all)}
    if has_ln:
        g["gamma"] = np.zeros(C)
        g["beta"] = np.zeros(C)
    if spatial_crop is not None:
        g["newline"] = np.zeros(W2.shape[0])
        g["sep"] = np.zeros(W2.shape[0])

    mag = {key: np.zeros_like(v) for key, v in g.items()} if magnitudes else None
    pos = O.placeholder_positions(ids, image_token_id)
    offs = np.concatenate([[0], np.cumsum(grid_hw[:, 0].astype(np.int64) * grid_hw[:, 1])])
    if spatial_crop is None:
        groups = [([v], None) for v in range(len(grid_hw))]
    else:
        groups, v = [], 0
        for tw, th in np.asarray(spatial_crop):
            n = 1 + int(tw) * int(th)
            groups.append((list(range(v, v + n)), (int(tw), int(th))))
            v += n
    if len(pos) != sum(O.image_rows(grid_hw, k, spatial_crop)):
        raise ValueError("placeholder count does not match the image rows")

    base = 0
    for views, crop in groups:
        h0, w0 = int(grid_hw[views[0], 0]), int(grid_hw[views[0], 1])
        hp, wp = O.merged_side(h0, k), O.merged_side(w0, k)
        row_map = _image_row_map(hp, wp, crop, len(views), gvp)
        d_rows = d_out[pos[base:base + len(row_map)]]
        base += len(row_map)
        if crop is not None:
            g["newline"] += d_rows[row_map == -1].sum(axis=0)
            g["sep"] += d_rows[row_map == -2].sum(axis=0)
            if magnitudes:
                mag["newline"] += np.abs(d_rows[row_map == -1]).sum(axis=0)
                mag["sep"] += np.abs(d_rows[row_map == -2]).sum(axis=0)
        tok_rows = np.full(len(views) * hp * wp, -1, np.int64)
        tok_rows[row_map[row_map >= 0]] = np.flatnonzero(row_map >= 0)
        for vi, v in enumerate(views):
            x = x_all[offs[v]:offs[v + 1]]
            # forward of the view, keeping what the backward needs
            if has_ln:
                mu = x.mean(axis=1, keepdims=True)
                var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
                rstd = 1.0 / np.sqrt(var + ln_eps)
                xhat = (x - mu) * rstd
                src = xhat * gamma + beta
            else:
                src = x
            if quantise:
                src = O.round_bf16(src)
            a = O.unshuffle(src.reshape(h0, w0, C), k)
            dy = d_rows[tok_rows[vi * hp * wp:(vi + 1) * hp * wp]]
            sel = np.flatnonzero(np.any(dy != 0, axis=1)) if skip_zero_rows else np.arange(hp * wp)
            a, dy = a[sel], dy[sel]
            p = a @ W1.T + b1
            hid = O.gelu(p)
            if quantise:
                hid = O.round_bf16(hid)
            # gradients
            g["b2"] += dy.sum(axis=0)
            g["W2"] += dy.T @ hid
            dp = (dy @ W2) * gelu_grad(p)
            g["b1"] += dp.sum(axis=0)
            g["W1"] += dp.T @ a
            da = np.zeros((hp * wp, W1.shape[1]))
            da[sel] = dp @ W1
            dsrc = O.fold(da, hp, wp, k, C)[:h0, :w0].reshape(h0 * w0, C)
            if has_ln:
                g["gamma"] += (dsrc * xhat).sum(axis=0)
                g["beta"] += dsrc.sum(axis=0)
                dx = layernorm_backward(dsrc, xhat, rstd, gamma)
            else:
                dx = dsrc
            g["features"][offs[v]:offs[v + 1]] = dx
            if magnitudes:
                # |dP| plus the absolute sum of its dot product, scaled far below bf16
                # precision: a cancelling dY . W2 still gets the room of its fp32 rounding
                m_dp = np.abs(dp) + 2.0 ** -16 * (np.abs(dy) @ np.abs(W2)) * np.abs(gelu_grad(p))
                mag["b2"] += np.abs(dy).sum(axis=0)
                mag["W2"] += np.abs(dy).T @ np.abs(hid)
                mag["b1"] += m_dp.sum(axis=0)
                mag["W1"] += m_dp.T @ np.abs(a)
                m_da = np.zeros((hp * wp, W1.shape[1]))
                m_da[sel] = m_dp @ np.abs(W1)
                m_src = O.fold(m_da, hp, wp, k, C)[:h0, :w0].reshape(h0 * w0, C)
                if has_ln:
                    ax = np.abs(xhat)
                    mag["gamma"] += (m_src * ax).sum(axis=0)
                    mag["beta"] += m_src.sum(axis=0)
                    m_g = m_src * np.abs(gamma)
                    m_dx = rstd * (m_g + m_g.mean(axis=1, keepdims=True)
                                   + ax * (m_g * ax).mean(axis=1, keepdims=True))
                else:
                    m_dx = m_src
                mag["features"][offs[v]:offs[v + 1]] = m_dx
    if magnitudes:
        g["mag"] = mag
    return g
