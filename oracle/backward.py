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

Reading: the bf16 rounding points (a and every hidden activation) pass gradients
through unchanged (straight-through), as mixed-precision training treats them. With
depth > 2 ("port DeepSeek-VL2", Projector step 3) the middle Linear(N1 -> N1) layers'
gradients come back under "mid", one [dW, db] pair per layer, in order.
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

    mids = [(np.asarray(Wm, np.float64), np.asarray(bm, np.float64)) for Wm, bm in (params.get("mid") or ())]
    layers = [(W1, b1)] + mids + [(W2, b2)]
    g["mid"] = [[np.zeros_like(Wm), np.zeros_like(bm)] for Wm, bm in mids]
    mag = {key: (np.zeros_like(v) if key != "mid" else [[np.zeros_like(a), np.zeros_like(b)] for a, b in v])
           for key, v in g.items()} if magnitudes else None

    def acc(store, li, which, value):
        """Add to layer li's weight (which = 0) or bias (which = 1) gradient."""
        if li == 0:
            store[("W1", "b1")[which]] += value
        elif li == len(layers) - 1:
            store[("W2", "b2")[which]] += value
        else:
            store["mid"][li - 1][which] += value

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
            # forward through Linear -> GELU -> [Linear -> GELU] x len(mids) -> Linear,
            # keeping each layer's input and pre-activation
            xs, ps = [a], []
            for W, b in layers[:-1]:
                p = xs[-1] @ W.T + b
                hid = O.gelu(p)
                ps.append(p)
                xs.append(O.round_bf16(hid) if quantise else hid)
            # backward, top layer first: dW_l = dP_l^T x_l, db_l = sum dP_l,
            # dP_(l-1) = (dP_l W_l) * GELU'(P_(l-1)); the first layer's input gradient is dA
            dp = dy
            m_dp = np.abs(dy)
            for li in range(len(layers) - 1, -1, -1):
                W = layers[li][0]
                acc(g, li, 0, dp.T @ xs[li])
                acc(g, li, 1, dp.sum(axis=0))
                if magnitudes:
                    acc(mag, li, 0, m_dp.T @ np.abs(xs[li]))
                    acc(mag, li, 1, m_dp.sum(axis=0))
                if li == 0:
                    break
                gp_ = gelu_grad(ps[li - 1])
                nxt = (dp @ W) * gp_
                if magnitudes:
                    if li == len(layers) - 1:
                        # dY is exact: |dP| plus its dot product's room for fp32 rounding
                        m_dp = np.abs(nxt) + 2.0 ** -16 * (np.abs(dp) @ np.abs(W)) * np.abs(gp_)
                    else:
                        # dP above was rounded: its error reaches here through the whole sum
                        m_dp = np.abs(nxt) + (m_dp @ np.abs(W)) * np.abs(gp_)
                dp = nxt
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


def backward_image_sampled(feats, hw, k: int, params: dict, crop: Optional[tuple], d_rows: np.ndarray,
                           units: np.ndarray, tokens: dict, ln_eps: float = 1e-5, gvp: str = "head") -> dict:
    """The share of one image in selected gradient entries, for a dense ``d_out``
    (depth 2, bf16 quantisation as in `backward`). Every entry is a sum over the image's
    merged tokens, so the batch value is the sum of the images' shares.

    ``feats[v]`` / ``hw[v]``: the image's views as in `projector.project_image`;
    ``d_rows``: d_out at the image's placeholder rows, in assembled order; ``units``: the
    hidden units j whose columns are sampled; ``tokens``: {view index in the image:
    merged-token indices} whose patches' feature gradients are wanted.

    Returns, each with its magnitude chain under "mag" (as in `backward`):
      "W2_cols" (N2, |units|) = dW2[:, units];  "b1_sel" = db1[units];
      "W1_rows" (|units|, K1) = dW1[units, :];  "b2" = db2 (all of it);
      "newline", "sep" (tiled images); "features": {(view, patch row): gradient row}.
    By linearity the hidden units are independent: column j of P = A W1^T + b1 needs only
    row j of W1, and dW2[:, j], db1[j], dW1[j, :] need only that column. The feature
    gradient of a token's patches needs that token's whole row of dP (all units); each
    patch belongs to exactly one token, so its gradient row is complete."""
    W1, b1, W2, b2 = params["W1"], params["b1"], params["W2"], params["b2"]
    gamma, beta = params.get("gamma"), params.get("beta")
    has_ln = gamma is not None
    C = np.asarray(feats[0]).shape[1]
    units = np.asarray(units, np.int64)
    h0, w0 = hw[0]
    hp, wp = O.merged_side(h0, k), O.merged_side(w0, k)
    row_map = _image_row_map(hp, wp, crop, len(feats), gvp)
    tok_rows = np.full(len(feats) * hp * wp, -1, np.int64)
    tok_rows[row_map[row_map >= 0]] = np.flatnonzero(row_map >= 0)
    out = {"W2_cols": np.zeros((W2.shape[0], len(units))), "b1_sel": np.zeros(len(units)),
           "W1_rows": np.zeros((len(units), W1.shape[1])), "b2": np.zeros(W2.shape[0]), "features": {}}
    mag = {"W2_cols": np.zeros_like(out["W2_cols"]), "b1_sel": np.zeros(len(units)),
           "W1_rows": np.zeros_like(out["W1_rows"]), "b2": np.zeros(W2.shape[0]), "features": {}}
    if crop is not None:
        out["newline"] = d_rows[row_map == -1].sum(axis=0)
        out["sep"] = d_rows[row_map == -2].sum(axis=0)
        mag["newline"] = np.abs(d_rows[row_map == -1]).sum(axis=0)
        mag["sep"] = np.abs(d_rows[row_map == -2]).sum(axis=0)
    for vi, x in enumerate(feats):
        x = np.asarray(x, np.float64)
        h, w = hw[vi]
        if has_ln:
            mu = x.mean(axis=1, keepdims=True)
            rstd = 1.0 / np.sqrt(((x - mu) ** 2).mean(axis=1, keepdims=True) + ln_eps)
            xhat = (x - mu) * rstd
            src = xhat * gamma + beta
        else:
            src = x
        a = O.unshuffle(O.round_bf16(src).reshape(h, w, C), k)
        dy = d_rows[tok_rows[vi * hp * wp:(vi + 1) * hp * wp]]
        out["b2"] += dy.sum(axis=0)
        mag["b2"] += np.abs(dy).sum(axis=0)
        # the sampled hidden units, every token
        p = a @ W1[units].T + b1[units]
        hid = O.round_bf16(O.gelu(p))
        gp_ = gelu_grad(p)
        dp = (dy @ W2[:, units]) * gp_
        m_dp = np.abs(dp) + 2.0 ** -16 * (np.abs(dy) @ np.abs(W2[:, units])) * np.abs(gp_)
        out["W2_cols"] += dy.T @ hid
        mag["W2_cols"] += np.abs(dy).T @ np.abs(hid)
        out["b1_sel"] += dp.sum(axis=0)
        mag["b1_sel"] += m_dp.sum(axis=0)
        out["W1_rows"] += dp.T @ a
        mag["W1_rows"] += m_dp.T @ np.abs(a)
        # the sampled tokens, every hidden unit: their patches' feature gradients
        for t in np.asarray(tokens.get(vi, ()), np.int64):
            pt = a[t] @ W1.T + b1
            gt = gelu_grad(pt)
            dpt = (dy[t] @ W2) * gt
            m_dpt = np.abs(dpt) + 2.0 ** -16 * (np.abs(dy[t]) @ np.abs(W2)) * np.abs(gt)
            da, m_da = dpt @ W1, m_dpt @ np.abs(W1)
            i, j = int(t) // wp, int(t) % wp
            for dyy in range(k):
                for dxx in range(k):
                    r, s = k * i + dyy, k * j + dxx
                    if r >= h or s >= w:
                        continue
                    cols = np.arange(C) * k * k + dyy * k + dxx          # channel-outer merge order
                    dsrc, m_src = da[cols], m_da[cols]
                    prow = r * w + s
                    if has_ln:
                        gg = dsrc * gamma
                        xr = xhat[prow]
                        dx = rstd[prow, 0] * (gg - gg.mean() - xr * (gg * xr).mean())
                        mg = m_src * np.abs(gamma)
                        ax = np.abs(xr)
                        m_dx = rstd[prow, 0] * (mg + mg.mean() + ax * (mg * ax).mean())
                    else:
                        dx, m_dx = dsrc, m_src
                    out["features"][(vi, prow)] = dx
                    mag["features"][(vi, prow)] = m_dx
    out["mag"] = mag
    return out
