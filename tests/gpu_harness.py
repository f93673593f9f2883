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
