"""GPU parity of vlproj_backward with the fp64 backward oracle (oracle/backward.py).

Tolerance, per gradient entry:  |gpu - oracle| <= e * mag,  where mag is the oracle's
absolute-value chain (for dW1[n, q] the sum over tokens of |dP[m, n]| |A[m, q]|, and
so on, see oracle/backward.py), so each term of an entry may be off by a relative e:
  * bf16 keeps 8 significant bits: rounding moves a value by at most 2^-8 of it, and a
    value that the GPU's fp32 arithmetic puts on the other side of a rounding boundary
    than the fp64 oracle does lands one ulp away, at most 2^-7 of it;
  * dW2 terms hold H (one such boundary): e = 2^-7;
  * dW1 terms hold dP, rounded twice (GELU'(P), then dP: (1 + 2^-8)^2 - 1 < 2^-7 + 2^-15),
    and A (one boundary, 2^-7): e = 2^-6; db1 carries dP's rounding only; with a
    LayerNorm, dA is rounded to bf16 too (2^-8 more), so d_features, dgamma and dbeta
    carry under 2^-7 + 2^-8 + 2^-15: all take the same e;
  * db2 and the newline / separator rows are fp32 sums of exact bf16 values: e = 2^-8.
An entry whose terms are all zero must come out exactly zero.
"""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
import workloads as W
from oracle import backward as B
from oracle import projector as O
from gpu_harness import DeviceInputs, custom, dev_bf16, make_case, make_projector, w1_for_gpu

pytestmark = pytest.mark.gpu

EPS_DP = 2.0 ** -6
EPS = {"W2": 2.0 ** -7, "b2": 2.0 ** -8, "newline": 2.0 ** -8, "sep": 2.0 ** -8}


def grad_shapes(case):
    wl = case.wl
    P = int((case.hw[:, 0].astype(np.int64) * case.hw[:, 1]).sum())
    shapes = {"W1": (wl.N1, wl.K1), "b1": (wl.N1,), "W2": (wl.N2, wl.N1), "b2": (wl.N2,), "features": (P, wl.C)}
    if wl.has_ln:
        shapes.update(gamma=(wl.C,), beta=(wl.C,))
    if wl.tiled:
        shapes.update(newline=(wl.N2,), sep=(wl.N2,))
    return shapes


def run_backward(case, proj, dev, d_out, names=None, check=True):
    """Gradients from the GPU as fp64 numpy arrays; outputs start as NaN so that an
    element the library fails to write shows up."""
    shapes = grad_shapes(case)
    names = list(shapes) if names is None else names
    grads = {n: torch.full(shapes[n], float("nan"), dtype=torch.float32, device="cuda") for n in names}
    rc = proj.backward(dev.feats, case.hw, case.crop, dev.ids, W.IMAGE_TOKEN_ID, d_out, grads,
                       n_images=case.wl.n_images, check=check)
    torch.cuda.synchronize()
    return rc, {n: t.double().cpu().numpy() for n, t in grads.items()}


def oracle_grads(case, d_out, skip_zero_rows=False):
    g = B.backward(case.feats, case.hw, case.crop, case.wl.k, O.params_f64(case.w), case.ids, W.IMAGE_TOKEN_ID,
                   d_out, case.wl.ln_eps, feat_is_bf16_bits=not case.wl.feat_fp32, quantise=True, gvp=case.gvp,
                   skip_zero_rows=skip_zero_rows, magnitudes=True)
    if case.k_order == vp.ORDER_POSITION_OUTER:
        kk, C = case.wl.k * case.wl.k, case.wl.C
        for d in (g, g["mag"]):
            d["W1"] = d["W1"].reshape(-1, C, kk).transpose(0, 2, 1).reshape(d["W1"].shape[0], -1)
    return g


def assert_grads_close(got, want, label=""):
    stats = {}
    for n, gv in got.items():
        wv, mag = want[n], want["mag"][n]
        assert gv.shape == wv.shape, n
        assert np.isfinite(gv).all(), f"{label} d{n}: unwritten or non-finite elements"
        err = np.abs(gv - wv)
        bound = EPS.get(n, EPS_DP) * mag
        assert np.all(err[mag == 0] == 0), f"{label} d{n}: nonzero where every term is zero"
        live = mag > 0
        ratio = float((err[live] / bound[live]).max()) if live.any() else 0.0
        stats[n] = ratio
        assert ratio <= 1.0, f"{label} d{n}: max err / bound = {ratio:.3f}"
    return stats


def dev_dout(case, seed=0):
    bits = W.grad_out(case.wl, len(case.ids), seed)
    return bits, dev_bf16(bits), O.bf16_bits_to_f64(bits)


SMALL = {
    "tiny": lambda: W.WORKLOADS["tiny"],
    "ragged_ln_bf16": lambda: custom("ragged_ln_bf16", 40, 2, 128, 256, 160, 3, 1, 900, has_ln=True),
    "k3_no_ln": lambda: custom("k3_no_ln", 41, 3, 64, 192, 128, 2, 2, 200),
    "tiled_2x1": lambda: custom("tiled_2x1", 42, 2, 64, 128, 128, 2, 2, 260, tiled=True, tw=2, th=1),
    "fp32_no_ln": lambda: custom("fp32_no_ln", 43, 2, 64, 128, 96, 2, 1, 300, feat_fp32=True),
    # regular grids (k | h, k | w), bf16, no LayerNorm, N2 not a multiple of 64: 5 images
    # of 320 tokens, a ragged last tile
    "regular_k3": lambda: custom("regular_k3", 44, 3, 64, 256, 160, 5, 5, 320),
}
GRIDS = {
    "ragged_ln_bf16": [[20, 30], [17, 9], [32, 32]],
    "k3_no_ln": [[10, 11], [7, 3]],
    "tiled_2x1": [[9, 9]] * 3 + [[7, 5]] * 3,
    "fp32_no_ln": [[15, 13], [4, 4]],
    "regular_k3": [[30, 96]] * 5,
}


@pytest.mark.parametrize("name", list(SMALL))
def test_backward_matches_oracle(name):
    wl = SMALL[name]()
    case = make_case(wl, GRIDS.get(name))
    proj = make_projector(case)
    dev = DeviceInputs(case)
    _, d_dev, d_f64 = dev_dout(case)
    rc, got = run_backward(case, proj, dev, d_dev)
    assert rc == vp.OK and proj.status() == vp.OK
    assert_grads_close(got, oracle_grads(case, d_f64), name)


@pytest.mark.parametrize("gvp", ["head", "tail"])
def test_backward_tiled_global_view_position(gvp):
    wl = SMALL["tiled_2x1"]()
    case = make_case(wl, GRIDS["tiled_2x1"], gvp=gvp)
    proj = make_projector(case)
    _, d_dev, d_f64 = dev_dout(case, seed=3)
    _, got = run_backward(case, proj, DeviceInputs(case), d_dev)
    assert_grads_close(got, oracle_grads(case, d_f64), gvp)


def test_backward_position_outer_weights():
    wl = SMALL["ragged_ln_bf16"]()
    case = make_case(wl, GRIDS["ragged_ln_bf16"], k_order=vp.ORDER_POSITION_OUTER)
    proj = make_projector(case)
    _, d_dev, d_f64 = dev_dout(case, seed=5)
    _, got = run_backward(case, proj, DeviceInputs(case), d_dev)
    assert_grads_close(got, oracle_grads(case, d_f64), "position-outer")


@pytest.mark.parametrize("name", ["ragged_ln_bf16", "regular_k3"])
def test_backward_is_deterministic_and_tile_shape_independent(name):
    wl = SMALL[name]()
    case = make_case(wl, GRIDS[name])
    proj = make_projector(case)
    dev = DeviceInputs(case)
    _, d_dev, _ = dev_dout(case)
    _, a = run_backward(case, proj, dev, d_dev)
    _, b = run_backward(case, proj, dev, d_dev)
    proj.set_tile_pairs(False)
    _, c = run_backward(case, proj, dev, d_dev)
    proj.set_tile_pairs(True)
    proj.set_tile_order(vp.TILE_ORDER_DYNAMIC)    # every GEMM from a counter: same tiles, same K order
    _, d = run_backward(case, proj, dev, d_dev)
    proj.set_tile_order(vp.TILE_ORDER_STATIC)
    _, e = run_backward(case, proj, dev, d_dev)
    for n in a:
        np.testing.assert_array_equal(a[n], b[n], err_msg=n)
        np.testing.assert_array_equal(a[n], c[n], err_msg=n)
        np.testing.assert_array_equal(a[n], d[n], err_msg=n)
        np.testing.assert_array_equal(a[n], e[n], err_msg=n)


@pytest.mark.parametrize("name", ["tiled_2x1", "ragged_ln_bf16"])
def test_backward_subset_of_outputs_matches_full_run(name):
    wl = SMALL[name]()
    case = make_case(wl, GRIDS[name])
    proj = make_projector(case)
    dev = DeviceInputs(case)
    _, d_dev, _ = dev_dout(case)
    _, full = run_backward(case, proj, dev, d_dev)
    for names in (["W2"], ["b1", "newline"], ["features"], ["gamma", "beta"], ["W1", "sep"], ["b2"], ["gamma"]):
        names = [n for n in names if n in full]
        if not names:
            continue
        _, part = run_backward(case, proj, dev, d_dev, names)
        for n in names:
            np.testing.assert_array_equal(part[n], full[n], err_msg=str(names))


def test_backward_count_mismatch_gives_zero_gradients():
    wl = SMALL["ragged_ln_bf16"]()
    case = make_case(wl, GRIDS["ragged_ln_bf16"])
    proj = make_projector(case)
    dev = DeviceInputs(case)
    ids = dev.ids.clone()
    ids[int(np.flatnonzero(case.ids == W.IMAGE_TOKEN_ID)[0])] = 5
    dev.ids = ids
    _, d_dev, _ = dev_dout(case)
    rc, got = run_backward(case, proj, dev, d_dev)
    assert rc == vp.OK
    assert proj.status() == vp.ERR_TOKEN_COUNT
    for n, v in got.items():
        assert not np.any(v), n


def test_backward_without_images_zeroes_outputs():
    wl = SMALL["tiled_2x1"]()
    case = make_case(wl, GRIDS["tiled_2x1"])
    proj = make_projector(case)
    dev = DeviceInputs(case)
    text = torch.randint(0, 1000, (64,), dtype=torch.int64, device="cuda")
    d = torch.ones((64, wl.N2), dtype=torch.bfloat16, device="cuda")
    grads = {n: torch.full(s, float("nan"), device="cuda") for n, s in grad_shapes(case).items() if n != "features"}
    proj.backward(None, None, None, text, W.IMAGE_TOKEN_ID, d, grads, n_images=0)
    assert proj.status() == vp.OK
    for n, t in grads.items():
        assert not bool(t.any()), n


def test_backward_rejects_bad_alignment():
    wl = SMALL["tiny"]()
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    _, d_dev, _ = dev_dout(case)
    g = torch.zeros(wl.N2 + 1, device="cuda")
    rc = proj.backward(dev.feats, case.hw, None, dev.ids, W.IMAGE_TOKEN_ID, d_dev, {"b2": g[1:]}, check=False)
    assert rc == vp.ERR_INVALID_ARG


def run_backward_mid(case, proj, dev, d_out, depth, want=("W1", "b1", "W2", "b2", "features"), mid=True):
    """Like run_backward, plus the middle layers' gradients (lists under "W_mid" / "b_mid")."""
    shapes = grad_shapes(case)
    wl = case.wl
    grads = {n: torch.full(shapes[n], float("nan"), dtype=torch.float32, device="cuda") for n in want if n in shapes}
    if mid:
        grads["W_mid"] = [torch.full((wl.N1, wl.N1), float("nan"), device="cuda") for _ in range(depth - 2)]
        grads["b_mid"] = [torch.full((wl.N1,), float("nan"), device="cuda") for _ in range(depth - 2)]
    proj.backward(dev.feats, case.hw, case.crop, dev.ids, W.IMAGE_TOKEN_ID, d_out, grads, n_images=wl.n_images)
    torch.cuda.synchronize()
    out = {n: t.double().cpu().numpy() for n, t in grads.items() if n not in ("W_mid", "b_mid")}
    if mid:
        out["mid"] = [[w.double().cpu().numpy(), b.double().cpu().numpy()]
                      for w, b in zip(grads["W_mid"], grads["b_mid"])]
    return out


def assert_frobenius_close(got, want, label, tol=1e-2):
    num = float(np.linalg.norm(got - want))
    den = float(np.linalg.norm(want))
    assert num <= tol * den + 1e-30, f"{label}: relative Frobenius error {num / max(den, 1e-30):.2e}"


@pytest.mark.parametrize("name,depth", [("ragged_ln_bf16", 3), ("tiled_2x1", 4)])
def test_backward_deeper_mlp_matches_oracle(name, depth):
    """depth > 2: every gradient, the middle layers' included, within the elementwise
    magnitude bound (which below the top layer carries the rounded dP of the layer
    above through the whole sum) and within 1 % relative Frobenius error."""
    wl = SMALL[name]()
    case = make_case(wl, GRIDS[name], depth=depth)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    _, d_dev, d_f64 = dev_dout(case)
    want_names = tuple(grad_shapes(case))
    got = run_backward_mid(case, proj, dev, d_dev, depth, want_names)
    assert proj.status() == vp.OK
    want = oracle_grads(case, d_f64)
    flat_got = {n: v for n, v in got.items() if n != "mid"}
    assert_grads_close(flat_got, want, f"{name} depth {depth}")
    for n, v in flat_got.items():
        assert_frobenius_close(v, want[n], f"d{n}")
    for i, (gw, gb) in enumerate(got["mid"]):
        for which, gv in ((0, gw), (1, gb)):
            wv, mag = want["mid"][i][which], want["mag"]["mid"][i][which]
            assert np.isfinite(gv).all()
            assert np.all(np.abs(gv - wv) <= EPS_DP * mag), f"mid {i} {which}"
            assert_frobenius_close(gv, wv, f"mid {i} {'W' if which == 0 else 'b'}")


def test_backward_deeper_mlp_partial_chain():
    """Asking only for a middle layer's gradients stops the dP chain there; the values
    equal those of the full run."""
    wl = SMALL["ragged_ln_bf16"]()
    case = make_case(wl, GRIDS["ragged_ln_bf16"], depth=4)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    _, d_dev, _ = dev_dout(case)
    full = run_backward_mid(case, proj, dev, d_dev, 4, tuple(grad_shapes(case)))
    part = run_backward_mid(case, proj, dev, d_dev, 4, ("W2",))
    np.testing.assert_array_equal(part["W2"], full["W2"])
    for i in range(2):
        for which in (0, 1):
            np.testing.assert_array_equal(part["mid"][i][which], full["mid"][i][which])


@pytest.mark.parametrize("name", ["moonvit", "vl2", "dsvit"])
def test_backward_full_size_sparse_gradient(name):
    """Full-size workload, d_out nonzero on 24 placeholder rows and 8 text rows: the
    oracle evaluates only the tokens with a nonzero output gradient (the others add
    exactly zero), the GPU runs the whole batch."""
    wl = W.WORKLOADS[name]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    rng = np.random.default_rng(7)
    ph = np.flatnonzero(case.ids == W.IMAGE_TOKEN_ID)
    tx = np.flatnonzero(case.ids != W.IMAGE_TOKEN_ID)
    rows = np.sort(np.concatenate([rng.choice(ph, 24, replace=False), rng.choice(tx, 8, replace=False)]))
    vals = W.grad_out_rows(wl, len(rows))
    d_dev = torch.zeros((len(case.ids), wl.N2), dtype=torch.bfloat16, device="cuda")
    d_dev[torch.from_numpy(rows).cuda()] = dev_bf16(vals)

    class Sparse:
        def __getitem__(self, idx):
            idx = np.asarray(idx)
            out = np.zeros((len(idx), wl.N2))
            hit = np.searchsorted(rows, idx)
            ok = (hit < len(rows)) & (rows[np.minimum(hit, len(rows) - 1)] == idx)
            out[ok] = O.bf16_bits_to_f64(vals[hit[ok]])
            return out

    rc, got = run_backward(case, proj, dev, d_dev)
    assert rc == vp.OK and proj.status() == vp.OK
    assert_grads_close(got, oracle_grads(case, Sparse(), skip_zero_rows=True), name)


@pytest.mark.parametrize("name", ["stress", "dsvit", "vl2", "moonvit"])
def test_backward_full_size_dense_gradient(name):
    """Full-size workload with d_out ~N(0, 1) on every id. Checked against the oracle's
    per-image shares of sampled entries (oracle/backward.py, backward_image_sampled):
    dW2 columns, db1 and dW1 rows of five hidden units (the first, the last and three
    seeded), all of db2 (and the newline / separator gradients when tiled), and the
    feature gradient of every patch of one seeded token per image. Every sampled entry
    is a sum over all merged tokens of the batch."""
    from concurrent.futures import ThreadPoolExecutor
    wl = W.WORKLOADS[name]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    n_ids = len(case.ids)
    bits = W.grad_out_blocks(wl, n_ids, seed=2)
    d_dev = dev_bf16(bits)
    shapes = grad_shapes(case)
    names = ["W1", "b1", "W2", "b2", "features"] + (["newline", "sep"] if wl.tiled else [])
    grads = {n: torch.full(shapes[n], float("nan"), dtype=torch.float32, device="cuda") for n in names}
    rc = proj.backward(dev.feats, case.hw, case.crop, dev.ids, W.IMAGE_TOKEN_ID, d_dev, grads, n_images=wl.n_images)
    assert rc == vp.OK and proj.status() == vp.OK
    del d_dev

    rng = np.random.default_rng(11)
    units = np.unique(np.concatenate([[0, wl.N1 - 1], rng.choice(wl.N1, 3, replace=False)]))
    per = wl.views_per_image
    hw = case.hw
    offs = np.concatenate([[0], np.cumsum(hw[:, 0].astype(np.int64) * hw[:, 1])])
    pos = O.placeholder_positions(case.ids, W.IMAGE_TOKEN_ID)
    rbase = np.concatenate([[0], np.cumsum(case.rows)])
    params = O.params_f64(case.w)
    picks = []
    for img in range(wl.n_images):
        vi = int(rng.integers(per))
        v = img * per + vi
        picks.append((vi, int(rng.integers(O.tokens_untiled(int(hw[v, 0]), int(hw[v, 1]), wl.k)))))

    def share(img):
        views = list(range(img * per, (img + 1) * per))
        feats = [O.bf16_bits_to_f64(case.feats[offs[v]:offs[v + 1]]) for v in views]
        vhw = [(int(hw[v, 0]), int(hw[v, 1])) for v in views]
        crop = None if case.crop is None else (int(case.crop[img, 0]), int(case.crop[img, 1]))
        d_rows = O.bf16_bits_to_f64(bits[pos[rbase[img]:rbase[img + 1]]])
        vi, t = picks[img]
        return B.backward_image_sampled(feats, vhw, wl.k, params, crop, d_rows, units, {vi: [t]}, wl.ln_eps, case.gvp)

    with ThreadPoolExecutor(8) as ex:
        parts = list(ex.map(share, range(wl.n_images)))
    want, mag = {}, {}
    for key in ("W2_cols", "b1_sel", "W1_rows", "b2") + (("newline", "sep") if wl.tiled else ()):
        want[key] = sum(pt[key] for pt in parts)
        mag[key] = sum(pt["mag"][key] for pt in parts)
    got = {"W2_cols": grads["W2"][:, torch.from_numpy(units).cuda()], "b1_sel": grads["b1"][torch.from_numpy(units).cuda()],
           "W1_rows": grads["W1"][torch.from_numpy(units).cuda()], "b2": grads["b2"]}
    if wl.tiled:
        got.update(newline=grads["newline"], sep=grads["sep"])
    eps = {"W2_cols": EPS["W2"], "b2": EPS["b2"], "newline": EPS["newline"], "sep": EPS["sep"]}
    worst = {}
    for key, g in got.items():
        g = g.double().cpu().numpy()
        assert np.isfinite(g).all(), key
        bound = eps.get(key, EPS_DP) * mag[key]
        err = np.abs(g - want[key])
        assert np.all(err[mag[key] == 0] == 0), key
        live = mag[key] > 0
        worst[key] = float((err[live] / bound[live]).max())
        assert worst[key] <= 1.0, f"{name} {key}: max err / bound {worst[key]:.3f}"
    # feature gradients of the sampled tokens' patches
    rows, want_f, mag_f = [], [], []
    for img, pt in enumerate(parts):
        for (vi, prow), g in pt["features"].items():
            rows.append(int(offs[img * per + vi]) + prow)
            want_f.append(g)
            mag_f.append(pt["mag"]["features"][(vi, prow)])
    gf = grads["features"][torch.tensor(rows, device="cuda")].double().cpu().numpy()
    want_f, mag_f = np.stack(want_f), np.stack(mag_f)
    assert np.isfinite(gf).all()
    err = np.abs(gf - want_f)
    assert np.all(err[mag_f == 0] == 0)
    live = mag_f > 0
    worst["features"] = float((err[live] / (EPS_DP * mag_f[live])).max())
    assert worst["features"] <= 1.0, f"{name} features: max err / bound {worst['features']:.3f}"
    print(name, worst)
