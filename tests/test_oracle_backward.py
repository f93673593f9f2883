"""Pins of the fp64 backward oracle (oracle/backward.py).

The gradients are checked against central finite differences of the (separately
pinned) forward oracle: the loss is <d_out, forward(theta)>, so its derivative in
any parameter entry is the entry of the returned gradient. Finite differences
share no step with the chain rule written out in the backward, so a dropped term,
a wrong sign, a transposed operand or a misplaced row fails them.
"""
import math

import numpy as np
import pytest

from oracle import backward as B
from oracle import projector as O

IMG = 7


def _case(seed, grid_hw, crop, k, C, N1, N2, has_ln, n_text=9, depth=2):
    rng = np.random.default_rng(seed)
    grid_hw = np.asarray(grid_hw, np.int32)
    P = int((grid_hw[:, 0] * grid_hw[:, 1]).sum())
    feats = rng.normal(0.0, 1.0, (P, C)) * rng.uniform(0.5, 2.0, (P, 1)) + rng.normal(0.0, 0.5, (P, 1))
    K1 = k * k * C
    params = {
        "W1": rng.normal(0.0, 0.3, (N1, K1)), "b1": rng.normal(0.0, 0.3, N1),
        "W2": rng.normal(0.0, 0.3, (N2, N1)), "b2": rng.normal(0.0, 0.3, N2),
        "gamma": rng.uniform(0.5, 1.5, C) if has_ln else None,
        "beta": rng.normal(0.0, 0.2, C) if has_ln else None,
        "newline": rng.normal(0.0, 1.0, N2) if crop is not None else None,
        "sep": rng.normal(0.0, 1.0, N2) if crop is not None else None,
        "mid": [(rng.normal(0.0, 0.3, (N1, N1)), rng.normal(0.0, 0.3, N1)) for _ in range(depth - 2)],
    }
    rows = sum(O.image_rows(grid_hw, k, crop))
    ids = rng.integers(IMG + 1, IMG + 50, rows + n_text)      # text ids never equal the placeholder
    slots = np.sort(rng.choice(rows + n_text, rows, replace=False))
    ids[slots] = IMG
    d_out = rng.normal(0.0, 1.0, (len(ids), N2))
    embeds = rng.normal(0.0, 1.0, (len(ids), N2))
    return dict(features=feats, grid_hw=grid_hw, spatial_crop=crop, k=k, params=params, ids=ids,
                d_out=d_out, embeds=embeds)


CASES = {
    "untiled_ln_ragged": dict(seed=1, grid_hw=[[3, 5], [4, 4]], crop=None, k=2, C=4, N1=6, N2=5, has_ln=True),
    "untiled_k3_ln": dict(seed=2, grid_hw=[[4, 5]], crop=None, k=3, C=3, N1=5, N2=4, has_ln=True),
    "untiled_no_ln": dict(seed=3, grid_hw=[[2, 3], [1, 1]], crop=None, k=2, C=3, N1=4, N2=3, has_ln=False),
    "tiled_2x1": dict(seed=4, grid_hw=[[3, 3]] * 3, crop=np.array([[2, 1]]), k=2, C=3, N1=4, N2=3, has_ln=True),
    "tiled_two_images": dict(seed=5, grid_hw=[[2, 2]] * 3 + [[3, 2]] * 3, crop=np.array([[1, 2], [2, 1]]),
                             k=2, C=2, N1=3, N2=4, has_ln=False),
}


def _loss(c, params=None, features=None, quantise=False, gvp="head"):
    out = O.forward(c["features"] if features is None else features, c["grid_hw"], c["spatial_crop"], c["k"],
                    c["params"] if params is None else params, c["ids"], IMG, c["embeds"], 1e-5,
                    feat_is_bf16_bits=False, quantise=quantise, global_view_pos=gvp)
    return float((out * c["d_out"]).sum())


def _grads(c, quantise=False, gvp="head"):
    return B.backward(c["features"], c["grid_hw"], c["spatial_crop"], c["k"], c["params"], c["ids"], IMG,
                      c["d_out"], 1e-5, feat_is_bf16_bits=False, quantise=quantise, gvp=gvp)


def _fd(c, name, eps=1e-6, quantise=False, gvp="head"):
    """Central finite difference of the loss in every entry of parameter `name`
    (("mid", i, 0 | 1) names a middle layer's weight or bias)."""
    if isinstance(name, tuple):
        return _fd_mid(c, name[1], name[2], eps)
    if name == "features":
        base = c["features"]
    else:
        base = c["params"][name]
    g = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        vals = []
        for s in (+1.0, -1.0):
            t = base.copy()
            t[idx] += s * eps
            if name == "features":
                vals.append(_loss(c, features=t, quantise=quantise, gvp=gvp))
            else:
                p = dict(c["params"])
                p[name] = t
                vals.append(_loss(c, params=p, quantise=quantise, gvp=gvp))
        g[idx] = (vals[0] - vals[1]) / (2 * eps)
    return g


def _fd_mid(c, i, which, eps):
    base = c["params"]["mid"][i][which]
    g = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        vals = []
        for sgn in (+1.0, -1.0):
            t = base.copy()
            t[idx] += sgn * eps
            mids = [list(m) for m in c["params"]["mid"]]
            mids[i][which] = t
            p = dict(c["params"])
            p["mid"] = [tuple(m) for m in mids]
            vals.append(_loss(c, params=p))
        g[idx] = (vals[0] - vals[1]) / (2 * eps)
    return g


def _names(c):
    names = ["W1", "b1", "W2", "b2", "features"]
    if c["params"]["gamma"] is not None:
        names += ["gamma", "beta"]
    if c["spatial_crop"] is not None:
        names += ["newline", "sep"]
    return names


def test_gelu_grad_matches_finite_difference():
    x = np.linspace(-6.0, 6.0, 241)
    h = 1e-6
    fd = (O.gelu(x + h) - O.gelu(x - h)) / (2 * h)
    np.testing.assert_allclose(B.gelu_grad(x), fd, rtol=0, atol=1e-9)
    # closed forms: GELU'(0) = 1/2, GELU' -> 0 and 1 in the tails
    assert B.gelu_grad(np.array([0.0]))[0] == 0.5
    assert abs(B.gelu_grad(np.array([-12.0]))[0]) < 1e-20
    assert abs(B.gelu_grad(np.array([12.0]))[0] - 1.0) < 1e-20


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_finite_differences(name):
    spec = CASES[name]
    c = _case(**spec)
    g = _grads(c)
    for key in _names(c):
        fd = _fd(c, key)
        scale = max(1.0, float(np.abs(fd).max()))
        np.testing.assert_allclose(g[key], fd, rtol=0, atol=2e-6 * scale, err_msg=f"{name}: d{key}")


@pytest.mark.parametrize("name,depth", [("untiled_ln_ragged", 3), ("tiled_2x1", 4), ("untiled_k3_ln", 3)])
def test_deeper_mlp_backward_matches_finite_differences(name, depth):
    c = _case(**CASES[name], depth=depth)
    g = _grads(c)
    assert len(g["mid"]) == depth - 2
    keys = _names(c) + [("mid", i, w) for i in range(depth - 2) for w in (0, 1)]
    for key in keys:
        fd = _fd(c, key)
        got = g["mid"][key[1]][key[2]] if isinstance(key, tuple) else g[key]
        np.testing.assert_allclose(got, fd, rtol=0, atol=2e-6 * max(1.0, float(np.abs(fd).max())),
                                   err_msg=f"{name} depth {depth}: d{key}")


def test_deeper_mlp_magnitudes_bound_the_gradients():
    c = _case(**CASES["tiled_2x1"], depth=4)
    g = B.backward(c["features"], c["grid_hw"], c["spatial_crop"], c["k"], c["params"], c["ids"], IMG, c["d_out"],
                   1e-5, feat_is_bf16_bits=False, quantise=True, magnitudes=True)
    for key in _names(c):
        assert np.all(g["mag"][key] >= np.abs(g[key]) * (1 - 1e-12)), key
    for i in range(2):
        for w in (0, 1):
            assert np.all(g["mag"]["mid"][i][w] >= np.abs(g["mid"][i][w]) * (1 - 1e-12))


def test_backward_tail_global_view_matches_finite_differences():
    c = _case(**CASES["tiled_2x1"])
    g = _grads(c, gvp="tail")
    for key in ("W2", "newline", "sep", "features"):
        fd = _fd(c, key, gvp="tail")
        np.testing.assert_allclose(g[key], fd, rtol=0, atol=2e-6 * max(1.0, float(np.abs(fd).max())))


def test_quantised_backward_exact_in_the_affine_parameters():
    """With the bf16 rounding points on, the rows are still affine in W2, b2 and the
    newline / separator rows (the rounded hidden state does not depend on them), so a
    finite difference of any step is their exact gradient."""
    c = _case(**CASES["tiled_two_images"])
    g = _grads(c, quantise=True)
    for key in ("W2", "b2", "newline", "sep"):
        fd = _fd(c, key, eps=0.25, quantise=True)
        np.testing.assert_allclose(g[key], fd, rtol=0, atol=1e-9 * max(1.0, float(np.abs(fd).max())))


def test_quantised_backward_is_close_to_the_exact_one():
    """Straight-through rounding changes the gradients only by the bf16 rounding of the
    saved activations (relative 2^-8 per value)."""
    c = _case(**CASES["untiled_ln_ragged"])
    gq = _grads(c, quantise=True)
    g = _grads(c, quantise=False)
    for key in _names(c):
        scale = float(np.abs(g[key]).max())
        assert float(np.abs(gq[key] - g[key]).max()) <= 3e-2 * scale, key


def test_text_rows_carry_no_gradient():
    c = _case(**CASES["untiled_ln_ragged"])
    g0 = _grads(c)
    mask = c["ids"] != IMG
    c["d_out"][mask] += 100.0
    g1 = _grads(c)
    for key in _names(c):
        np.testing.assert_array_equal(g0[key], g1[key])


@pytest.mark.parametrize("name", ["untiled_ln_ragged", "tiled_two_images"])
def test_skipping_zero_gradient_rows_changes_nothing(name):
    """Tokens whose output gradient is zero contribute nothing, so evaluating only the
    others gives the same gradients."""
    c = _case(**CASES[name])
    rng = np.random.default_rng(11)
    keep = rng.random(len(c["ids"])) < 0.3
    c["d_out"][~keep] = 0.0
    full = _grads(c)
    part = B.backward(c["features"], c["grid_hw"], c["spatial_crop"], c["k"], c["params"], c["ids"], IMG,
                      c["d_out"], 1e-5, feat_is_bf16_bits=False, quantise=False, skip_zero_rows=True)
    for key in _names(c):
        np.testing.assert_allclose(part[key], full[key], rtol=0, atol=1e-12 * max(1.0, float(np.abs(full[key]).max())))


def _bf16(x):
    import torch
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().float().numpy().astype(np.float64)


def _emulated_rounding_grads(c):
    """dW1, db1, d_features, dgamma, dbeta under the GPU's rounding model: fp32 products
    and sums, GELU'(P) rounded to bf16, dP rounded to bf16 (A and H as the oracle's)."""
    f32 = lambda t: np.asarray(t, np.float32)
    prm, k = c["params"], c["k"]
    W1, b1, W2 = prm["W1"], prm["b1"], prm["W2"]
    gamma, beta = prm["gamma"], prm["beta"]
    x_all, hw = c["features"], c["grid_hw"]
    pos = O.placeholder_positions(c["ids"], IMG)
    offs = np.concatenate([[0], np.cumsum(hw[:, 0].astype(np.int64) * hw[:, 1])])
    out = {"W1": np.zeros_like(W1), "b1": np.zeros_like(b1), "features": np.zeros_like(x_all),
           "gamma": np.zeros_like(gamma), "beta": np.zeros_like(beta)}
    base = 0
    for v in range(len(hw)):
        h0, w0 = int(hw[v, 0]), int(hw[v, 1])
        hp, wp = O.merged_side(h0, k), O.merged_side(w0, k)
        x = x_all[offs[v]:offs[v + 1]]
        mu = x.mean(axis=1, keepdims=True)
        rstd = 1.0 / np.sqrt(((x - mu) ** 2).mean(axis=1, keepdims=True) + 1e-5)
        xhat = (x - mu) * rstd
        a = O.unshuffle(O.round_bf16(xhat * gamma + beta).reshape(h0, w0, -1), k)
        dy = c["d_out"][pos[base:base + hp * wp]]
        base += hp * wp
        p = (f32(a) @ f32(W1).T + f32(b1)).astype(np.float64)
        dp = _bf16((f32(dy) @ f32(W2)).astype(np.float64) * _bf16(B.gelu_grad(p)))
        out["W1"] += (f32(dp).T @ f32(a)).astype(np.float64)
        out["b1"] += f32(dp).sum(axis=0)
        da = (f32(dp) @ f32(W1)).astype(np.float64)
        dsrc = O.fold(da, hp, wp, k, x.shape[1])[:h0, :w0].reshape(h0 * w0, -1)
        out["gamma"] += (dsrc * xhat).sum(axis=0)
        out["beta"] += dsrc.sum(axis=0)
        out["features"][offs[v]:offs[v + 1]] = B.layernorm_backward(dsrc, xhat, rstd, gamma)
    return out


def test_magnitudes_bound_the_gradients_and_the_rounding_model():
    """The absolute-value chain is at least |gradient| everywhere, and the GPU's rounding
    model (bf16 GELU'(P) and dP) stays within 2^-7 of it."""
    c = _case(**CASES["untiled_ln_ragged"])
    c["params"]["W1"] = _bf16(c["params"]["W1"])
    c["params"]["W2"] = _bf16(c["params"]["W2"])
    c["d_out"] = _bf16(c["d_out"])
    g = B.backward(c["features"], c["grid_hw"], None, c["k"], c["params"], c["ids"], IMG, c["d_out"], 1e-5,
                   feat_is_bf16_bits=False, quantise=True, magnitudes=True)
    mag = g["mag"]
    for key in _names(c):
        assert np.all(mag[key] >= np.abs(g[key]) * (1 - 1e-12)), key
    emu = _emulated_rounding_grads(c)
    for key, val in emu.items():
        err = np.abs(val - g[key])
        assert np.all(err <= 2.0 ** -7 * mag[key]), key
        assert np.any(err > 2.0 ** -12 * mag[key]), key      # the model does round


def test_backward_rejects_count_mismatch():
    c = _case(**CASES["untiled_no_ln"])
    ids = c["ids"].copy()
    ids[np.flatnonzero(ids == IMG)[0]] = 1
    with pytest.raises(ValueError):
        B.backward(c["features"], c["grid_hw"], None, 2, c["params"], ids, IMG, c["d_out"], feat_is_bf16_bits=False)


# ------------------------------------------------------------------ planted mistakes
def test_pins_catch_a_wrong_gelu_derivative(monkeypatch):
    c = _case(**CASES["untiled_no_ln"])
    monkeypatch.setattr(B, "gelu_grad", lambda p: 0.5 * (1.0 + np.vectorize(math.erf)(p / math.sqrt(2.0))))
    g = _grads(c)
    fd = _fd(c, "W1")
    assert not np.allclose(g["W1"], fd, rtol=0, atol=2e-6 * max(1.0, float(np.abs(fd).max())))


def test_pins_catch_a_dropped_layernorm_term(monkeypatch):
    """LayerNorm's input gradient without the xhat * mean(g * xhat) projection term."""
    c = _case(**CASES["untiled_k3_ln"])
    monkeypatch.setattr(B, "layernorm_backward",
                        lambda d, xh, r, gm: r * (d * gm - (d * gm).mean(axis=1, keepdims=True)))
    g = _grads(c)
    fd = _fd(c, "features")
    assert not np.allclose(g["features"], fd, rtol=0, atol=2e-6 * max(1.0, float(np.abs(fd).max())))


def test_pins_catch_an_unflipped_fold(monkeypatch):
    """The input gradient folded back with the channels of each patch reversed."""
    c = _case(**CASES["untiled_ln_ragged"])
    real = O.fold
    monkeypatch.setattr(O, "fold", lambda a, hp, wp, k, C: real(a[:, ::-1].copy(), hp, wp, k, C))
    g = _grads(c)
    fd = _fd(c, "features")
    assert not np.allclose(g["features"], fd, rtol=0, atol=2e-6 * max(1.0, float(np.abs(fd).max())))


def test_pins_catch_a_swapped_view_order(monkeypatch):
    """Gradient rows read from the wrong view of a tiled image (global and first local
    swapped) fail the finite differences of W2."""
    c = _case(**CASES["tiled_2x1"])
    real = B._image_row_map

    def wrong(hp, wp, crop, n_views, gvp):
        m = real(hp, wp, crop, n_views, gvp).copy()
        n = hp * wp
        tok = m >= 0
        v = np.where(tok, m // n, -1)
        swap = np.where(v == 0, 1, np.where(v == 1, 0, v))
        m[tok] = swap[tok] * n + m[tok] % n
        return m

    monkeypatch.setattr(B, "_image_row_map", wrong)
    g = _grads(c)
    fd = _fd(c, "W2")
    assert not np.allclose(g["W2"], fd, rtol=0, atol=2e-6 * max(1.0, float(np.abs(fd).max())))


def _sampled_sum(c, units, tokens_of, gvp="head"):
    """backward_image_sampled summed over the images of case c (quantised, as the GPU)."""
    grid_hw, crop, k = c["grid_hw"], c["spatial_crop"], c["k"]
    offs = np.concatenate([[0], np.cumsum(grid_hw[:, 0].astype(np.int64) * grid_hw[:, 1])])
    pos = O.placeholder_positions(c["ids"], IMG)
    rows = O.image_rows(grid_hw, k, crop)
    per = [1] * len(grid_hw) if crop is None else [1 + int(a) * int(b) for a, b in crop]
    total, v0, r0 = None, 0, 0
    for img, n in enumerate(per):
        views = list(range(v0, v0 + n))
        feats = [c["features"][offs[v]:offs[v + 1]] for v in views]
        hw = [(int(grid_hw[v, 0]), int(grid_hw[v, 1])) for v in views]
        cr = None if crop is None else (int(crop[img, 0]), int(crop[img, 1]))
        d_rows = c["d_out"][pos[r0:r0 + rows[img]]]
        part = B.backward_image_sampled(feats, hw, k, c["params"], cr, d_rows, units, tokens_of(img, views), 1e-5,
                                        gvp)
        part["features"] = {(views[vi], prow): g for (vi, prow), g in part["features"].items()}
        part["mag"]["features"] = {(views[vi], prow): g for (vi, prow), g in part["mag"]["features"].items()}
        if total is None:
            total = part
        else:
            for d, s in ((total, part), (total["mag"], part["mag"])):
                for key, val in s.items():
                    if key == "mag":
                        continue
                    if key == "features":
                        d[key].update(val)
                    else:
                        d[key] = d[key] + val
        v0, r0 = v0 + n, r0 + rows[img]
    return total, offs


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("gvp", ["head", "tail"])
def test_sampled_backward_equals_the_whole_backward(name, gvp):
    """The per-image, per-unit restriction used for full-size checks gives exactly the
    entries of the whole backward (depth 2, quantised) and of its magnitude chain."""
    c = _case(**CASES[name])
    if c["spatial_crop"] is None and gvp == "tail":
        pytest.skip("untiled")
    full = B.backward(c["features"], c["grid_hw"], c["spatial_crop"], c["k"], c["params"], c["ids"], IMG,
                      c["d_out"], 1e-5, feat_is_bf16_bits=False, quantise=True, gvp=gvp, magnitudes=True)
    N1 = c["params"]["W1"].shape[0]
    units = np.array([0, N1 - 1, N1 // 2])
    k = c["k"]

    def tokens_of(img, views):
        out = {}
        for vi, v in enumerate(views):
            n = O.tokens_untiled(int(c["grid_hw"][v, 0]), int(c["grid_hw"][v, 1]), k)
            out[vi] = np.arange(n)                           # every token: every patch is checked
        return out

    got, offs = _sampled_sum(c, units, tokens_of, gvp)
    for src, ref in ((got, full), (got["mag"], full["mag"])):
        np.testing.assert_allclose(src["W2_cols"], ref["W2"][:, units], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(src["b1_sel"], ref["b1"][units], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(src["W1_rows"], ref["W1"][units], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(src["b2"], ref["b2"], rtol=1e-12, atol=1e-13)
        if c["spatial_crop"] is not None:
            np.testing.assert_allclose(src["newline"], ref["newline"], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(src["sep"], ref["sep"], rtol=1e-12, atol=1e-13)
        P = int(offs[-1])
        assert len(src["features"]) == P                     # every patch covered once
        for (v, prow), g in src["features"].items():
            np.testing.assert_allclose(g, ref["features"][offs[v] + prow], rtol=1e-11, atol=1e-13)
