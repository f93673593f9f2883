"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each check uses a value the
pages print (tests/golden/, each with its citation), a library routine that
computes the same special case, a closed form, an invariant, or the scalar C
brute force (a separate formulation by direct index formulas).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import projector as O
from oracle import build_brute
from workloads import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def brute():
    return build_brute.load()


def _ptr(a):
    return a.ctypes.data


# ------------------------------------------------------------------ number formats
def test_round_bf16_matches_torch_fp32_to_bf16():
    """torch's fp32 -> bf16 cast is round-to-nearest-even; on fp32 inputs the oracle's
    direct fp64 -> bf16 rounding must agree bit for bit, ties included."""
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(20_000) * 1e-30).astype(np.float32),
        (rng.standard_normal(20_000) * 1e30).astype(np.float32),
    ])
    # exact ties: low 16 bits == 0x8000, both parities of the kept bit
    ties = (rng.integers(0x3F000000, 0x41000000, 4096, dtype=np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_matches_c_brute(brute):
    rng = np.random.default_rng(1)
    x = rng.standard_normal(5000) * np.exp(rng.uniform(-40, 40, 5000))
    got = O.round_bf16(x)
    ref = np.array([brute.brute_round_bf16(float(v)) for v in x])
    np.testing.assert_array_equal(got, ref)


def test_bf16_bits_decode():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x8000, 0x7F7F], np.uint16)
    want = [1.0, -1.0, 3.140625, 0.0, -0.0, 3.3895313892515355e38]
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), want)


# ------------------------------------------------------------------ elementwise maths
def test_gelu_matches_torch_exact_gelu():
    x = np.linspace(-8, 8, 10001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    np.testing.assert_allclose(O.gelu(x), ref, rtol=1e-14, atol=1e-15)
    assert O.gelu(np.array([0.0]))[0] == 0.0


def test_layernorm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((37, 1152)) * 3 + 0.5
    g = 1 + 0.1 * rng.standard_normal(1152)
    b = 0.02 * rng.standard_normal(1152)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (1152,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-5).numpy()
    np.testing.assert_allclose(O.layernorm(x, g, b, 1e-5), ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ space-to-depth
@pytest.mark.parametrize("case", _golden("unshuffle_hand.json")["cases"], ids=lambda c: c["name"])
def test_unshuffle_hand_examples(case):
    h, w, C, k = case["h"], case["w"], case["C"], case["k"]
    r, s, c = np.meshgrid(np.arange(h), np.arange(w), np.arange(C), indexing="ij")
    x = (100 * c + 10 * r + s).astype(np.float64)
    np.testing.assert_array_equal(O.unshuffle(x, k), np.array(case["tokens"], np.float64))


@pytest.mark.parametrize("h,w,C,k", [(4, 6, 3, 2), (9, 6, 5, 3), (24, 24, 64, 2), (96, 96, 2, 3), (5, 5, 2, 1)])
def test_unshuffle_matches_torch_pixel_unshuffle(h, w, C, k):
    """pixel_unshuffle on NCHW puts channel c, offset (dy, dx) at output channel
    c*k*k + dy*k + dx: the same order the page fixes."""
    x = np.random.default_rng(3).standard_normal((h, w, C))
    ref = torch.nn.functional.pixel_unshuffle(torch.from_numpy(x).permute(2, 0, 1)[None], k)
    ref = ref[0].permute(1, 2, 0).reshape(-1, C * k * k).numpy()
    np.testing.assert_array_equal(O.unshuffle(x, k), ref)


@pytest.mark.parametrize("h,w,k", [(27, 27, 2), (25, 31, 3), (1, 1, 2), (7, 2, 3)])
def test_unshuffle_odd_grid_is_padded_pixel_unshuffle(h, w, k):
    C = 3
    x = np.random.default_rng(4).standard_normal((h, w, C))
    hp, wp = O.merged_side(h, k), O.merged_side(w, k)
    xp = np.zeros((hp * k, wp * k, C))
    xp[:h, :w] = x
    ref = torch.nn.functional.pixel_unshuffle(torch.from_numpy(xp).permute(2, 0, 1)[None], k)
    ref = ref[0].permute(1, 2, 0).reshape(-1, C * k * k).numpy()
    np.testing.assert_array_equal(O.unshuffle(x, k), ref)


@pytest.mark.parametrize("h,w,k", [(96, 96, 3), (27, 27, 2), (24, 24, 2), (10, 14, 2)])
def test_unshuffle_is_a_bijection(h, w, k):
    """Space-to-depth loses nothing ("La voie visuelle", pixel-unshuffle section): the
    inverse restores the (padded) input bit for bit, and the pad is exactly zero."""
    C = 7
    x = np.random.default_rng(5).standard_normal((h, w, C))
    hp, wp = O.merged_side(h, k), O.merged_side(w, k)
    back = O.fold(O.unshuffle(x, k), hp, wp, k, C)
    np.testing.assert_array_equal(back[:h, :w], x)
    assert not back[h:].any() and not back[:, w:].any()


# ------------------------------------------------------------------ counts
def test_counts_printed_on_pages():
    g = _golden("counts.json")
    for c in g["untiled"]:
        assert c["image"] // c["patch"] == c["side"]
        assert O.tokens_untiled(c["side"], c["side"], c["k"]) == c["tokens"], c["cite"]
    for c in g["tiled_2d"]:
        side = c["image"] // c["patch"]
        hp = O.merged_side(side, c["k"])
        assert hp == c["hp"], c["cite"]
        assert O.tokens_tiled(hp, hp, c["tw"], c["th"]) == c["tokens"], c["cite"]


def test_counts_of_the_workloads():
    assert O.tokens_untiled(24, 24, 2) == 144            # tiny
    assert O.tokens_untiled(27, 27, 2) == 196            # 27 -> pad 28 -> 14 x 14
    assert O.tokens_tiled(14, 14, 2, 3) == 1429          # VL2 2x3 tiling (tw=2, th=3)
    assert O.tokens_tiled(14, 14, 3, 2) == 1415          # the other reading, for contrast
    hw = np.array([[27, 27]] * 7, np.int32)
    assert O.image_rows(hw, 2, np.array([[2, 3]], np.int32)) == [1429]


def test_param_count_pins_moonvit_projector_shape():
    g = _golden("params.json")
    assert O.projector_params(g["C"], g["k"], g["N1"], g["N2"], g["has_ln"]) == g["params"], g["cite"]
    # The alternatives do not reach the printed count.
    assert O.projector_params(1152, 2, 4608, 4096, False) != g["params"]
    assert 2 * 4608 + 4608 * 4608 + 4608 + 4608 * 4096 + 4096 != g["params"]   # post-merge LN(4608)
    wl = WORKLOADS["moonvit"]
    assert O.projector_params(wl.C, wl.k, wl.N1, wl.N2, wl.has_ln) == g["params"]


# ------------------------------------------------------------------ assembly
def _labels_assembled(hp, wp, tw, th, gvp="head"):
    """Run the oracle's assembly on label 'vectors' (object arrays of names)."""
    n_views = 1 + tw * th
    views = np.empty((n_views, hp * wp, 1), dtype=object)
    for v in range(n_views):
        for i in range(hp):
            for j in range(wp):
                views[v, i * wp + j, 0] = f"G{i}{j}" if v == 0 else f"L{v-1}_{i}{j}"
    nl = np.array(["NL"], dtype=object)
    sep = np.array(["SEP"], dtype=object)
    return list(O.assemble_2d(views, hp, wp, tw, th, nl, sep, gvp)[:, 0])


@pytest.mark.parametrize("case", _golden("assembly_hand.json")["cases"], ids=lambda c: str(c["rows"][:3]))
def test_assembly_hand_examples(case):
    got = _labels_assembled(case["hp"], case["wp"], case["tw"], case["th"], case.get("global_view_pos", "head"))
    assert got == case["rows"]
    assert len(got) == O.tokens_tiled(case["hp"], case["wp"], case["tw"], case["th"])


@pytest.mark.parametrize("hp,wp,tw,th", [(14, 14, 2, 3), (3, 5, 3, 2), (2, 2, 1, 1), (4, 3, 2, 2)])
def test_assembly_matches_c_index_formulas(brute, hp, wp, tw, th):
    n_views = 1 + tw * th
    D = 3
    views = np.zeros((n_views, hp * wp, D))
    for v in range(n_views):
        for i in range(hp):
            for j in range(wp):
                views[v, i * wp + j] = (v, i, j)
    rows = O.assemble_2d(views, hp, wp, tw, th, np.full(D, -1.0), np.full(D, -2.0))
    assert len(rows) == O.tokens_tiled(hp, wp, tw, th)
    seen = np.zeros(len(rows), bool)
    for v in range(n_views):
        for i in range(hp):
            for j in range(wp):
                r = brute.brute_row_of_token(1, v, i, j, hp, wp, tw)
                np.testing.assert_array_equal(rows[r], (v, i, j))
                seen[r] = True
    for n in range(hp + th * hp):
        r = brute.brute_row_of_newline(n, hp, wp, tw)
        assert (rows[r] == -1).all()
        seen[r] = True
    r = brute.brute_row_of_separator(hp, wp)
    assert (rows[r] == -2).all()
    seen[r] = True
    assert seen.all()


def test_scatter_in_order_and_count_check():
    ids = np.array([5, 7, 7, 1, 7, 2, 7], np.int64)
    emb = np.arange(7 * 2, dtype=np.float64).reshape(7, 2)
    rows = np.array([[10, 10], [20, 20], [30, 30], [40, 40]], np.float64)
    out = O.scatter(emb, ids, 7, rows)
    want = emb.copy()
    for r, p in zip(rows, [1, 2, 4, 6]):
        want[p] = r
    np.testing.assert_array_equal(out, want)
    with pytest.raises(ValueError):
        O.scatter(emb, ids, 7, rows[:3])


# ------------------------------------------------------------------ MLP vs brute force
def _tiny_case(h, w, C, k, N1, N2, has_ln, seed):
    rng = np.random.default_rng(seed)
    feat = rng.standard_normal((h * w, C))
    W1 = O.round_bf16(0.2 * rng.standard_normal((N1, k * k * C)))
    W2 = O.round_bf16(0.2 * rng.standard_normal((N2, N1)))
    b1 = 0.1 * rng.standard_normal(N1)
    b2 = 0.1 * rng.standard_normal(N2)
    gamma = 1 + 0.1 * rng.standard_normal(C) if has_ln else None
    beta = 0.1 * rng.standard_normal(C) if has_ln else None
    return feat, dict(W1=W1, b1=b1, W2=W2, b2=b2, gamma=gamma, beta=beta)


@pytest.mark.parametrize("h,w,C,k,has_ln,quantise", [
    (4, 4, 3, 2, True, True), (5, 3, 4, 2, False, True), (6, 6, 2, 3, True, True),
    (7, 5, 2, 3, False, False), (3, 3, 5, 1, True, True), (1, 1, 3, 2, True, True),
])
def test_mlp_matches_c_brute_force(brute, h, w, C, k, has_ln, quantise):
    N1, N2 = 9, 5
    feat, p = _tiny_case(h, w, C, k, N1, N2, has_ln, seed=h * 100 + w * 10 + C)
    got = O.project_image([feat], [(h, w)], k, p, None, 1e-5, quantise)
    hp, wp = O.merged_side(h, k), O.merged_side(w, k)
    assert got.shape == (hp * wp, N2)
    fe = np.ascontiguousarray(feat)
    W1, W2 = np.ascontiguousarray(p["W1"]), np.ascontiguousarray(p["W2"])
    g = np.ascontiguousarray(p["gamma"] if has_ln else np.zeros(C))
    b = np.ascontiguousarray(p["beta"] if has_ln else np.zeros(C))
    sa, sg, y = np.zeros(k * k * C), np.zeros(N1), np.zeros(N2)
    for i in range(hp):
        for j in range(wp):
            brute.brute_token_y(_ptr(fe), h, w, C, k, i, j, int(has_ln), _ptr(g), _ptr(b), 1e-5,
                                _ptr(W1), _ptr(p["b1"]), N1, _ptr(W2), _ptr(p["b2"]), N2,
                                int(quantise), _ptr(sa), _ptr(sg), _ptr(y))
            np.testing.assert_allclose(got[i * wp + j], y, rtol=1e-12, atol=1e-12)


def test_merged_operand_matches_c_brute_force(brute):
    h, w, C, k = 5, 7, 4, 2
    feat, p = _tiny_case(h, w, C, k, 3, 2, True, seed=9)
    a = O.merge_view(feat, h, w, k, (p["gamma"], p["beta"], 1e-5))
    hp, wp = O.merged_side(h, k), O.merged_side(w, k)
    fe = np.ascontiguousarray(feat)
    row = np.zeros(k * k * C)
    for i in range(hp):
        for j in range(wp):
            brute.brute_token_a(_ptr(fe), h, w, C, k, i, j, 1, _ptr(p["gamma"]), _ptr(p["beta"]),
                                1e-5, 1, _ptr(row))
            np.testing.assert_allclose(a[i * wp + j], row, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------ planted mistakes
def test_pins_catch_a_position_outer_unshuffle(monkeypatch):
    """A plausible slip (position-outer instead of channel-outer order) must fail the pins."""
    def wrong(y, k):
        h, w, C = y.shape
        hp, wp = O.merged_side(h, k), O.merged_side(w, k)
        pad = np.zeros((hp * k, wp * k, C))
        pad[:h, :w] = y
        return pad.reshape(hp, k, wp, k, C).transpose(0, 2, 1, 3, 4).reshape(hp * wp, -1)
    monkeypatch.setattr(O, "unshuffle", wrong)
    case = _golden("unshuffle_hand.json")["cases"][0]
    with pytest.raises(AssertionError):
        test_unshuffle_hand_examples(case)


def test_pins_catch_a_missing_local_transpose(monkeypatch):
    def wrong(views, hp, wp, tw, th, newline, sep, global_view_pos="head"):
        D = views.shape[-1]
        g = np.concatenate([views[0].reshape(hp, wp, D), np.broadcast_to(newline.reshape(1, 1, D), (hp, 1, D))], 1)
        loc = views[1:].reshape(th * hp, tw * wp, D)          # no (0, 2, 1, 3) transpose
        loc = np.concatenate([loc, np.broadcast_to(newline.reshape(1, 1, D), (th * hp, 1, D))], 1)
        return np.concatenate([g.reshape(-1, D), sep.reshape(1, D), loc.reshape(-1, D)], 0)
    monkeypatch.setattr(O, "assemble_2d", wrong)
    case = _golden("assembly_hand.json")["cases"][1]
    with pytest.raises(AssertionError):
        test_assembly_hand_examples(case)


def test_pins_catch_a_dropped_bias(brute, monkeypatch):
    real = O.mlp
    monkeypatch.setattr(O, "mlp", lambda a, W1, b1, W2, b2, q=True, mids=(): real(a, W1, 0 * b1, W2, b2, q, mids))
    with pytest.raises(AssertionError):
        test_mlp_matches_c_brute_force(brute, 4, 4, 3, 2, True, True)


# ------------------------------------------------------------------ whole path vs brute force
@pytest.mark.parametrize("tiled", [False, True])
def test_forward_matches_brute_composition(brute, tiled):
    """forward() = per-token brute-force rows placed at brute-force assembly indices,
    then written to the placeholder positions in order; text rows untouched."""
    k, C, N1, N2 = 2, 3, 6, 4
    rng = np.random.default_rng(11 + tiled)
    if tiled:
        tw, th = 2, 1
        hw = np.array([[5, 5]] * 3 + [[3, 4]] * 3, np.int32)     # two images, 3 views each
        crop = np.array([[tw, th], [tw, th]], np.int32)
    else:
        hw = np.array([[5, 3], [2, 2], [4, 6]], np.int32)
        crop = None
    feats = [rng.standard_normal((int(h) * int(w), C)) for h, w in hw]
    _, p = _tiny_case(1, 1, C, k, N1, N2, True, seed=3)
    p["newline"] = O.round_bf16(rng.standard_normal(N2))
    p["sep"] = O.round_bf16(rng.standard_normal(N2))
    rows = O.image_rows(hw, k, crop)
    ids = []
    for r in rows:
        ids += list(rng.integers(0, 50, 3)) + [999] * r
    ids = np.array(ids + [1, 2], np.int64)
    emb = rng.standard_normal((len(ids), N2))
    got = O.forward(np.concatenate(feats), hw, crop, k, p, ids, 999, emb, feat_is_bf16_bits=False)

    want = emb.copy()
    pos = [q for q in range(len(ids)) if ids[q] == 999]
    g, b = p["gamma"], p["beta"]
    sa, sg, y = np.zeros(k * k * C), np.zeros(N1), np.zeros(N2)
    base, v = 0, 0
    groups = [(1, None)] * len(hw) if crop is None else [(1 + tw * th, (tw, th)) for tw, th in crop]
    for n_views, cr in groups:
        for vv in range(n_views):
            h, w = int(hw[v + vv, 0]), int(hw[v + vv, 1])
            hp, wp = O.merged_side(h, k), O.merged_side(w, k)
            fe = np.ascontiguousarray(feats[v + vv])
            for i in range(hp):
                for j in range(wp):
                    brute.brute_token_y(_ptr(fe), h, w, C, k, i, j, 1, _ptr(g), _ptr(b), 1e-5,
                                        _ptr(p["W1"]), _ptr(p["b1"]), N1, _ptr(p["W2"]), _ptr(p["b2"]), N2,
                                        1, _ptr(sa), _ptr(sg), _ptr(y))
                    r = brute.brute_row_of_token(int(cr is not None), vv, i, j, hp, wp, cr[0] if cr else 1)
                    want[pos[base + r]] = y
        if cr is not None:
            for n in range(hp + cr[1] * hp):
                want[pos[base + brute.brute_row_of_newline(n, hp, wp, cr[0])]] = p["newline"]
            want[pos[base + brute.brute_row_of_separator(hp, wp)]] = p["sep"]
        base += O.tokens_tiled(hp, wp, *cr) if cr else hp * wp
        v += n_views
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ generator sanity
@pytest.mark.parametrize("name", list(WORKLOADS))
def test_generator_places_runs_in_order(name):
    import workloads as W
    wl = W.WORKLOADS[name]
    hw = W.grid_hw(wl)
    rows = O.image_rows(hw, wl.k, W.spatial_crop(wl))
    ids = W.input_ids(wl, rows)
    assert ids.shape == (wl.B * wl.S,)
    mask = ids == W.IMAGE_TOKEN_ID
    assert mask.sum() == sum(rows)
    assert not np.isin(ids[~mask], [W.IMAGE_TOKEN_ID]).any() and ids[~mask].max() < W.TEXT_VOCAB
    per_seq = wl.n_images // wl.B
    for b in range(wl.B):
        m = mask[b * wl.S:(b + 1) * wl.S]
        assert m.sum() == sum(rows[b * per_seq:(b + 1) * per_seq])
    if wl.fixed_hw is None:
        assert (hw % 2 == 0).all() and hw.min() >= 16 and hw.max() <= 96



@pytest.mark.parametrize("depth", [3, 4])
def test_deeper_mlp_matches_c_brute_force(brute, depth):
    """depth > 2: extra GELU + Linear(N1 -> N1) pairs in the middle ("port DeepSeek-VL2",
    Projector step 3), every hidden activation rounded to bf16; checked layer by layer
    against the scalar C dense layer."""
    h, w, C, k, N1, N2 = 4, 6, 3, 2, 7, 5
    feat, p = _tiny_case(h, w, C, k, N1, N2, True, seed=20 + depth)
    rng = np.random.default_rng(depth)
    p["mid"] = [(O.round_bf16(0.3 * rng.standard_normal((N1, N1))), 0.1 * rng.standard_normal(N1))
                for _ in range(depth - 2)]
    got = O.project_image([feat], [(h, w)], k, p, None, 1e-5, True)
    fe = np.ascontiguousarray(feat)
    a = np.zeros(k * k * C)
    for i in range(O.merged_side(h, k)):
        for j in range(O.merged_side(w, k)):
            brute.brute_token_a(_ptr(fe), h, w, C, k, i, j, 1, _ptr(p["gamma"]), _ptr(p["beta"]), 1e-5, 1, _ptr(a))
            x = np.zeros(N1)
            brute.brute_dense(_ptr(a), k * k * C, _ptr(np.ascontiguousarray(p["W1"])), _ptr(p["b1"]), N1, 1, 1,
                              _ptr(x))
            for Wm, bm in p["mid"]:
                y = np.zeros(N1)
                brute.brute_dense(_ptr(x), N1, _ptr(np.ascontiguousarray(Wm)), _ptr(bm), N1, 1, 1, _ptr(y))
                x = y
            out = np.zeros(N2)
            brute.brute_dense(_ptr(x), N1, _ptr(np.ascontiguousarray(p["W2"])), _ptr(p["b2"]), N2, 0, 0, _ptr(out))
            np.testing.assert_allclose(got[i * O.merged_side(w, k) + j], out, rtol=1e-12, atol=1e-12)


def test_param_count_with_depth():
    g = _golden("params.json")
    assert O.projector_params(g["C"], g["k"], g["N1"], g["N2"], g["has_ln"], depth=2) == g["params"]
    assert O.projector_params(64, 2, 128, 32, False, depth=4) == (256 * 128 + 128) + 2 * (128 * 128 + 128) + (128 * 32 + 32)
