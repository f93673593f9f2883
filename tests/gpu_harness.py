"""Shared plumbing of the GPU parity tests: build a seeded case, run the CUDA path
through the C ABI, and compare with the fp64 oracle.

Tolerance for projected rows (bf16 out, fp32 accumulation, bf16 hidden):
|gpu - oracle| <= 1e-2 + 1e-2 * |oracle| elementwise. Text rows, newline rows and
separator rows must be bit-exact; so must the placement of every row (a row at
the wrong placeholder fails the tolerance by orders of magnitude).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

import vision_language_projector_b200 as vp
import workloads as W
from oracle import projector as O

TOL_ABS = 1e-2
TOL_REL = 1e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_f32(a) -> Optional[torch.Tensor]:
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def custom(name: str, cfg_id: int, k: int, C: int, N1: int, N2: int, n_images: int, B: int, S: int, *,
           has_ln=False, feat_fp32=False, tiled=False, tw=0, th=0, bias_zero=False) -> W.Workload:
    return W.Workload(name, cfg_id, n_images, k, C, N1, N2, has_ln, feat_fp32, tiled, tw, th, B, S,
                      None, None, bias_zero)


@dataclasses.dataclass
class Case:
    wl: W.Workload
    hw: np.ndarray
    crop: Optional[np.ndarray]
    w: dict
    feats: np.ndarray
    rows: list
    ids: np.ndarray
    prefill: np.ndarray
    gvp: str = "head"
    k_order: int = vp.ORDER_CHANNEL_OUTER


def make_case(wl: W.Workload, hw: Optional[np.ndarray] = None, seed: int = 0, gvp: str = "head",
              k_order: int = vp.ORDER_CHANNEL_OUTER, depth: int = 2) -> Case:
    hw = W.grid_hw(wl, seed) if hw is None else np.asarray(hw, np.int32)
    crop = W.spatial_crop(wl)
    w = W.weights(wl, seed)
    w["mid"] = W.mid_weights(wl, depth, seed)
    feats = W.features(wl, hw, seed)
    rows = O.image_rows(hw, wl.k, crop)
    ids = W.input_ids(wl, rows, seed)
    prefill = W.prefill_embeds(wl, ids, W.embed_table(wl, seed))
    return Case(wl, hw, crop, w, feats, rows, ids, prefill, gvp, k_order)


def w1_for_gpu(case: Case) -> np.ndarray:
    """W1 bits in the column order the projector is told to expect."""
    W1 = case.w["W1"]
    if case.k_order == vp.ORDER_CHANNEL_OUTER:
        return W1
    kk, C = case.wl.k * case.wl.k, case.wl.C
    # position-outer column p*C + c holds the channel-outer column c*kk + p
    return W1.reshape(-1, C, kk).transpose(0, 2, 1).reshape(W1.shape[0], -1)


def make_projector(case: Case) -> vp.Projector:
    wl = case.wl
    w = case.w
    mids = w.get("mid") or []
    case._mid_dev = [(dev_bf16(Wm), dev_f32(bm)) for Wm, bm in mids]      # keep alive until create copied them
    return vp.Projector(
        wl.k, wl.C, wl.N1, wl.N2, dev_bf16(w1_for_gpu(case)), dev_bf16(w["W2"]), dev_f32(w["b1"]), dev_f32(w["b2"]),
        has_ln=wl.has_ln, ln_gamma=dev_f32(w["gamma"]), ln_beta=dev_f32(w["beta"]), ln_eps=wl.ln_eps,
        feat_dtype=vp.FEAT_F32 if wl.feat_fp32 else vp.FEAT_BF16,
        tile_tag=vp.TILE_2D if wl.tiled else vp.TILE_NONE,
        global_view_pos=vp.GLOBAL_TAIL if case.gvp == "tail" else vp.GLOBAL_HEAD, k_order=case.k_order,
        depth=2 + len(mids), W_mid=[a for a, _ in case._mid_dev] or None, b_mid=[b for _, b in case._mid_dev] or None)


class DeviceInputs:
    def __init__(self, case: Case):
        wl = case.wl
        self.feats = dev_f32(case.feats) if wl.feat_fp32 else dev_bf16(case.feats)
        self.ids = torch.from_numpy(case.ids).cuda()
        self.prefill = dev_bf16(case.prefill)
        self.newline = dev_bf16(case.w["newline"]) if wl.tiled else None
        self.sep = dev_bf16(case.w["sep"]) if wl.tiled else None


def run(case: Case, proj: vp.Projector, dev: DeviceInputs, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    if out is None:
        out = dev.prefill.clone()
    proj.forward(dev.feats, case.hw, case.crop, dev.ids, W.IMAGE_TOKEN_ID, out, dev.newline, dev.sep,
                 n_images=case.wl.n_images)
    return out


def oracle_params(case: Case) -> dict:
    return O.params_f64(case.w)


def view_groups(case: Case) -> list:
    per = case.wl.views_per_image
    return [list(range(i * per, (i + 1) * per)) for i in range(case.wl.n_images)]


def feats_f64(case: Case, view: int) -> np.ndarray:
    offs = np.concatenate([[0], np.cumsum(case.hw[:, 0].astype(np.int64) * case.hw[:, 1])])
    f = case.feats[offs[view]:offs[view + 1]]
    return f.astype(np.float64) if case.wl.feat_fp32 else O.bf16_bits_to_f64(f)


def oracle_image(case: Case, img: int, params: Optional[dict] = None) -> np.ndarray:
    params = oracle_params(case) if params is None else params
    views = view_groups(case)[img]
    feats = [feats_f64(case, v) for v in views]
    hw = [(int(case.hw[v, 0]), int(case.hw[v, 1])) for v in views]
    crop = None if case.crop is None else (int(case.crop[img, 0]), int(case.crop[img, 1]))
    return O.project_image(feats, hw, case.wl.k, params, crop, case.wl.ln_eps, True, case.gvp)


def special_mask(case: Case, img: int) -> np.ndarray:
    """True on the assembled rows of image img that are newline / separator rows."""
    n = case.rows[img]
    if case.crop is None:
        return np.zeros(n, bool)
    v0 = view_groups(case)[img][0]
    hp, wp = O.merged_side(case.hw[v0, 0], case.wl.k), O.merged_side(case.hw[v0, 1], case.wl.k)
    tw, th = int(case.crop[img, 0]), int(case.crop[img, 1])
    views = np.zeros((1 + tw * th, hp * wp, 1))
    m = O.assemble_2d(views, hp, wp, tw, th, np.ones(1), np.ones(1), case.gvp)[:, 0]
    return m == 1


def check(case: Case, out: torch.Tensor, dev: DeviceInputs, images: Optional[Sequence[int]] = None) -> dict:
    """Assert parity; return error statistics of the compared rows."""
    mask = dev.ids == W.IMAGE_TOKEN_ID
    assert int(mask.sum()) == sum(case.rows)
    # text rows untouched, bit for bit
    assert torch.equal(out[~mask].view(torch.int16), dev.prefill[~mask].view(torch.int16)), "text rows changed"
    # every placeholder row written (the prefill sentinel is NaN)
    assert bool(torch.isfinite(out[mask].float()).all()), "unwritten or non-finite placeholder rows"
    pos = np.flatnonzero(case.ids == W.IMAGE_TOKEN_ID)
    base = np.concatenate([[0], np.cumsum(case.rows)])
    images = range(case.wl.n_images) if images is None else images
    params = oracle_params(case)
    worst = 0.0
    max_abs = 0.0
    for img in images:
        want = oracle_image(case, img, params)
        p = torch.from_numpy(pos[base[img]:base[img + 1]]).cuda()
        got = out.index_select(0, p).double().cpu().numpy()
        err = np.abs(got - want)
        bound = TOL_ABS + TOL_REL * np.abs(want)
        ratio = float((err / bound).max()) if err.size else 0.0
        worst = max(worst, ratio)
        max_abs = max(max_abs, float(err.max()) if err.size else 0.0)
        assert ratio <= 1.0, f"image {img}: max err/bound {ratio:.3f} (max abs err {err.max():.3g})"
        sm = special_mask(case, img)
        if sm.any():
            np.testing.assert_array_equal(got[sm], want[sm])      # newline / separator rows exact
    return {"worst_err_over_bound": worst, "max_abs_err": max_abs}


def token_rows_in_image(case: Case, img: int) -> np.ndarray:
    """(views, h'*w') table: the assembled row, inside image img, of every merged token of
    each of its views. Built by running the oracle's own assembly on token labels."""
    views = view_groups(case)[img]
    v0 = views[0]
    hp, wp = O.merged_side(case.hw[v0, 0], case.wl.k), O.merged_side(case.hw[v0, 1], case.wl.k)
    if case.crop is None:
        return np.arange(hp * wp, dtype=np.int64)[None, :]
    tw, th = int(case.crop[img, 0]), int(case.crop[img, 1])
    n_tok = hp * wp
    labels = (np.arange(len(views) * n_tok, dtype=np.float64) + 1.0).reshape(len(views), n_tok, 1)
    col = O.assemble_2d(labels, hp, wp, tw, th, np.zeros(1), np.full(1, -1.0), case.gvp)[:, 0]
    table = np.full(len(views) * n_tok, -1, np.int64)
    rows = np.flatnonzero(col > 0)
    table[col[rows].astype(np.int64) - 1] = rows
    assert (table >= 0).all()
    return table.reshape(len(views), n_tok)


def token_a(case: Case, view: int, i: int, j: int) -> np.ndarray:
    """The merged operand of token (i, j) of `view`: the oracle's merge applied to the
    token's own k x k window of patches (cut at the grid's high end, where the merge pads
    with zeros). The LayerNorm is per patch, so the window gives the same values as the
    whole view."""
    k = case.wl.k
    h, w = int(case.hw[view, 0]), int(case.hw[view, 1])
    if not hasattr(case, "_patch0"):
        case._patch0 = np.concatenate([[0], np.cumsum(case.hw[:, 0].astype(np.int64) * case.hw[:, 1])])
    raw = case.feats[case._patch0[view]:case._patch0[view + 1]].reshape(h, w, -1)
    win = raw[k * i:min(h, k * i + k), k * j:min(w, k * j + k)]
    hs, ws = win.shape[0], win.shape[1]
    win = win.astype(np.float64) if case.wl.feat_fp32 else O.bf16_bits_to_f64(win)
    p = oracle_params(case) if not hasattr(case, "_params") else case._params
    ln = (p["gamma"], p["beta"], case.wl.ln_eps) if case.wl.has_ln else None
    a = O.merge_view(win.reshape(hs * ws, -1), hs, ws, k, ln)
    assert a.shape[0] == 1
    return a[0]


def sample_tokens(case: Case, per_image: int = 4, block: int = 128, seed: int = 0) -> list:
    """Seeded (view, token) picks: one token in every `block` consecutive merged tokens
    (views in order, so every GEMM M-tile holds one) plus `per_image` more in every image."""
    rng = np.random.default_rng(seed)
    k = case.wl.k
    n_tok = np.array([O.tokens_untiled(int(h), int(w), k) for h, w in case.hw], np.int64)
    start = np.concatenate([[0], np.cumsum(n_tok)])
    M = int(start[-1])
    picks = set()
    for b0 in range(0, M, block):
        m = int(rng.integers(b0, min(M, b0 + block)))
        v = int(np.searchsorted(start, m, side="right") - 1)
        picks.add((v, m - int(start[v])))
    for views in view_groups(case):
        tot = int(sum(n_tok[v] for v in views))
        for m in rng.choice(tot, size=min(per_image, tot), replace=False):
            m = int(m)
            for v in views:
                if m < n_tok[v]:
                    picks.add((v, m))
                    break
                m -= int(n_tok[v])
    return sorted(picks)


def check_tokens(case: Case, out: torch.Tensor, picks: Sequence[tuple]) -> dict:
    """Compare the placeholder row of every picked (view, token) with the oracle's row
    of that token: its merged operand from token_a, then the oracle's MLP. The row is
    located independently of the CUDA path: the image's assembled order from
    token_rows_in_image, and the oracle's placeholder positions."""
    params = oracle_params(case)
    case._params = params
    k = case.wl.k
    pos = O.placeholder_positions(case.ids, W.IMAGE_TOKEN_ID)
    base = np.concatenate([[0], np.cumsum(case.rows)])
    per = case.wl.views_per_image
    tables = {}
    A, dest = [], []
    for v, t in picks:
        img = v // per
        if img not in tables:
            tables[img] = token_rows_in_image(case, img)
        wp = O.merged_side(case.hw[v, 1], k)
        A.append(token_a(case, v, t // wp, t % wp))
        dest.append(int(pos[base[img] + tables[img][v - img * per, t]]))
    want = O.mlp(np.stack(A), params["W1"], params["b1"], params["W2"], params["b2"], True, params.get("mid") or ())
    got = out.index_select(0, torch.tensor(dest, dtype=torch.int64, device=out.device)).double().cpu().numpy()
    err = np.abs(got - want)
    ratio = err / (TOL_ABS + TOL_REL * np.abs(want))
    bad = np.argwhere(ratio > 1.0)
    assert bad.size == 0, (f"{len(np.unique(bad[:, 0]))} of {len(picks)} sampled tokens out of tolerance, first "
                           f"(view, token) {picks[int(bad[0, 0])]}: max err/bound {ratio.max():.3f}")
    return {"tokens": len(picks), "worst_err_over_bound": float(ratio.max()), "max_abs_err": float(err.max())}
