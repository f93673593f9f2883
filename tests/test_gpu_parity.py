"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Small cases compare every row and span several output tiles with ragged tails in
M and N; the five full-size workloads run in the benchmark's launch configuration
and compare every row of sampled images, every text row, and a seeded token in every
128-row M-block plus four in every image.
"""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
import workloads as W
from oracle import projector as O

from gpu_harness import (DeviceInputs, check, check_tokens, custom, dev_bf16, feats_f64, make_case, make_projector,
                         oracle_params, run, sample_tokens, view_groups, TOL_ABS, TOL_REL)

pytestmark = pytest.mark.gpu

SMALL = {
    # k=3, LayerNorm, odd grids, M = 199 (2 tiles, ragged), N1 = 320 (ragged 2nd tile), N2 = 96 < 128
    "ragged_k3_ln": (custom("ragged_k3_ln", 100, 3, 128, 320, 96, 4, 2, 160, has_ln=True),
                     [[25, 31], [9, 9], [3, 2], [30, 27]], "head", vp.ORDER_CHANNEL_OUTER),
    # k=1: no merge, 24x24 -> 576 tokens per image (the SigLIP 384/16 count)
    "k1_siglip": (custom("k1_siglip", 101, 1, 64, 128, 64, 2, 2, 700), [[24, 24], [24, 24]], "head",
                  vp.ORDER_CHANNEL_OUTER),
    # 2D tiling, odd 5x5 grids (pad to 6), 2x2 local tiles, global view first / last
    "tiled_head_odd": (custom("tiled_head_odd", 102, 2, 64, 192, 128, 3, 3, 80, tiled=True, tw=2, th=2),
                       [[5, 5]] * 15, "head", vp.ORDER_CHANNEL_OUTER),
    "tiled_tail_odd": (custom("tiled_tail_odd", 103, 2, 64, 192, 128, 3, 3, 80, tiled=True, tw=2, th=2),
                       [[5, 5]] * 15, "tail", vp.ORDER_CHANNEL_OUTER),
    # fp32 features without LayerNorm (converted to bf16 on the device)
    "fp32_noln": (custom("fp32_noln", 104, 2, 64, 256, 128, 2, 1, 200, feat_fp32=True), [[16, 12], [7, 9]],
                  "head", vp.ORDER_CHANNEL_OUTER),
    # W1 handed over in position-outer column order
    "position_outer": (custom("position_outer", 105, 2, 128, 256, 256, 3, 3, 300, has_ln=True),
                       [[20, 14], [13, 13], [2, 30]], "head", vp.ORDER_POSITION_OUTER),
    # a single 1x1 grid (one merged token, three pad neighbours)
    "one_patch": (custom("one_patch", 106, 2, 64, 64, 32, 1, 1, 10), [[1, 1]], "head", vp.ORDER_CHANNEL_OUTER),
    # many images, 8 sequences; M = 1536 (12 full tiles), N2 = 512 (two 256 tiles); regular grid (w' = 8)
    "many_images": (custom("many_images", 107, 2, 64, 256, 512, 32, 8, 256), [[12, 16]] * 32, "head",
                    vp.ORDER_CHANNEL_OUTER),
    # regular k = 3 grid with w' = 32: M = 800, a ragged last tile (the 5D box path)
    "regular_k3": (custom("regular_k3", 109, 3, 128, 256, 256, 5, 5, 256), [[15, 96]] * 5, "head",
                   vp.ORDER_CHANNEL_OUTER),
    # same-shape odd grids (TMA im2col) with N1 = 1024: 256 x 512 pair tiles, M = 588 (a
    # ragged third tile), two N-tiles
    "wide_im2col": (custom("wide_im2col", 120, 2, 64, 1024, 256, 3, 3, 200), [[27, 27]] * 3, "head",
                    vp.ORDER_CHANNEL_OUTER),
}


# (gather mode, 256 x 256 tiles on CTA pairs)
MODES = [(vp.GATHER_AUTO, True), (vp.GATHER_AUTO, False), (vp.GATHER_IM2COL, True), (vp.GATHER_IM2COL, False),
         (vp.GATHER_CPASYNC, True), (vp.GATHER_BOX, True), (vp.GATHER_BOX, False), (vp.GATHER_THREADS, True),
         (vp.GATHER_THREADS, False), (vp.GATHER_FUSED, True), (vp.GATHER_FUSED, False), (vp.GATHER_MERGED, True)]
MODE_IDS = ["auto-pairs", "auto-single", "im2col-pairs", "im2col-single", "cpasync", "box-pairs", "box-single",
            "threads-pairs", "threads-single", "fused-pairs", "fused-single", "merged-pairs"]


@pytest.mark.parametrize("mode", MODES, ids=MODE_IDS)
@pytest.mark.parametrize("name", list(SMALL))
def test_small_case_all_rows(name, mode):
    wl, hw, gvp, order = SMALL[name]
    case = make_case(wl, np.array(hw, np.int32), gvp=gvp, k_order=order)
    proj = make_projector(case)
    proj.set_gather_mode(mode[0])
    proj.set_tile_pairs(mode[1])
    dev = DeviceInputs(case)
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    check(case, out, dev)
    # a second call on the same handle gives the same bits
    out2 = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("mode", MODES, ids=MODE_IDS)
@pytest.mark.parametrize("name", ["ragged_k3_ln", "tiled_head_odd", "fp32_noln", "many_images", "regular_k3", "wide_im2col"])
def test_hidden_stage(name, mode):
    """Stage parity of H = bf16(GELU(A W1^T + b1)) for every merged token."""
    wl, hw, gvp, order = SMALL[name]
    case = make_case(wl, np.array(hw, np.int32), gvp=gvp, k_order=order)
    proj = make_projector(case)
    proj.set_gather_mode(mode[0])
    proj.set_tile_pairs(mode[1])
    dev = DeviceInputs(case)
    M = sum(O.tokens_untiled(h, w, wl.k) for h, w in case.hw)
    H = torch.empty((M, wl.N1), dtype=torch.bfloat16, device="cuda")
    proj.hidden(dev.feats, case.hw, H)
    assert proj.status() == vp.OK
    got = H.double().cpu().numpy()
    params = oracle_params(case)
    ln = (params["gamma"], params["beta"], wl.ln_eps) if wl.has_ln else None
    r = 0
    for v in range(len(case.hw)):
        h, w = int(case.hw[v, 0]), int(case.hw[v, 1])
        a = O.merge_view(feats_f64(case, v), h, w, wl.k, ln)
        want = O.hidden(a, params["W1"], params["b1"])
        g = got[r:r + len(want)]
        assert (np.abs(g - want) <= TOL_ABS + TOL_REL * np.abs(want)).all(), f"view {v}"
        if not wl.has_ln and not wl.feat_fp32:
            # A is then exact on both sides, so H is the oracle's bf16 value or a neighbour
            # of it: the fp32 pre-activation (summation error far below 2^-16 of the sum of
            # |terms|) and the fp32 GELU may round it the other way
            _, e = np.frexp(want)
            ulp = np.where(want != 0, np.ldexp(1.0, np.maximum(e, -125) - 8), 0.0)
            mag_p = np.abs(a) @ np.abs(params["W1"]).T + np.abs(params["b1"])
            bound = ulp + 2.0 ** -16 * mag_p + 1e-6
            assert (np.abs(g - want) <= bound).all(), f"view {v}: H more than one bf16 ulp away"
        r += len(want)


# image subsets compared against the oracle at full size (all text rows always checked)
SAMPLES = {"tiny": None, "moonvit": "extremes", "dsvit": [0, 7], "vl2": [0, 17, 31], "stress": [0, 131, 255]}


@pytest.mark.parametrize("name", list(SAMPLES))
def test_workload_full_size(name):
    wl = W.WORKLOADS[name]
    case = make_case(wl)
    images = SAMPLES[name]
    if images == "extremes":
        rows = np.array(case.rows)
        images = sorted({int(rows.argmin()), int(rows.argmax()), 5})
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    stats = check(case, out, dev, images)
    # on top of the whole images: a seeded token in every 128-row M-block (so every GEMM
    # tile, persistent-loop position and view is value-checked) and 4 more in every image
    tok = check_tokens(case, out, sample_tokens(case, per_image=4, block=128, seed=1))
    print(name, stats, tok)


def test_gemm_ragged_edges_are_exact_zero_pad():
    """An image whose odd grid needs padding must give the same rows as the same image
    with the pad written out as explicit zero patches (pad rows exactly 0)."""
    wl = custom("pad_equiv", 108, 3, 64, 128, 64, 1, 1, 64)
    case = make_case(wl, np.array([[7, 8]], np.int32))
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out = run(case, proj, dev)
    padded = np.zeros((9 * 9, wl.C), np.uint16)
    padded.reshape(9, 9, wl.C)[:7, :8] = case.feats.reshape(7, 8, wl.C)
    out2 = dev.prefill.clone()
    proj.forward(dev_bf16(padded), np.array([[9, 9]], np.int32), None, dev.ids, W.IMAGE_TOKEN_ID, out2)
    assert proj.status() == vp.OK
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_gather_modes_agree_bit_for_bit():
    """im2col and cp.async fetch the same operand bytes, so the outputs are identical."""
    wl = W.WORKLOADS["moonvit"]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    proj.set_gather_mode(vp.GATHER_IM2COL)
    out_a = run(case, proj, dev)
    proj.set_gather_mode(vp.GATHER_CPASYNC)
    out_b = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


def test_box_and_im2col_agree_bit_for_bit():
    wl = W.WORKLOADS["dsvit"]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    proj.set_gather_mode(vp.GATHER_BOX)
    out_a = run(case, proj, dev)
    proj.set_gather_mode(vp.GATHER_IM2COL)
    out_b = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


@pytest.mark.parametrize("mode", ["threads", "fused"])
@pytest.mark.parametrize("name", ["dsvit", "vl2"])
def test_thread_gather_and_fused_agree_bit_for_bit(name, mode):
    """The thread gather (cp.async by four extra warps, CTA pairs) and the fused producer
    warps fetch the same operand bytes as the TMA box / im2col modes AUTO picks."""
    wl = W.WORKLOADS[name]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out_a = run(case, proj, dev)
    proj.set_gather_mode(vp.GATHER_THREADS if mode == "threads" else vp.GATHER_FUSED)
    out_b = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


@pytest.mark.parametrize("name", ["dsvit", "vl2"])
def test_tile_pairs_agree_bit_for_bit(name):
    """256 x 256 tiles on CTA pairs and 128 x 256 tiles on single CTAs accumulate each
    output over the same K order, so they give identical bits."""
    wl = W.WORKLOADS[name]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out_a = run(case, proj, dev)
    proj.set_tile_pairs(False)
    out_b = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


def test_layernorm_paths_agree_bit_for_bit():
    """With a LayerNorm, AUTO writes the normalised features straight in merged-token
    order; the patch-order LayerNorm + gather path and the thread gather that normalises
    inside GEMM1 (from per-patch statistics) read the same values."""
    wl = W.WORKLOADS["moonvit"]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out_a = run(case, proj, dev)                     # AUTO
    proj.set_gather_mode(vp.GATHER_CPASYNC)
    out_b = run(case, proj, dev)
    proj.set_gather_mode(vp.GATHER_THREADS)
    out_c = run(case, proj, dev)
    proj.set_gather_mode(vp.GATHER_FUSED)
    out_d = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    assert torch.equal(out_a.view(torch.int16), out_c.view(torch.int16))
    assert torch.equal(out_a.view(torch.int16), out_d.view(torch.int16))



@pytest.mark.parametrize("pairs", [True, False], ids=["pairs", "single"])
@pytest.mark.parametrize("depth", [3, 4])
def test_deeper_mlp_all_rows(depth, pairs):
    """depth > 2: middle GELU + Linear(N1 -> N1) layers chained on the device."""
    wl = custom(f"depth{depth}", 150 + depth, 2, 128, 256, 256, 3, 3, 300, has_ln=(depth == 3))
    case = make_case(wl, np.array([[20, 14], [13, 13], [8, 30]], np.int32), depth=depth)
    proj = make_projector(case)
    proj.set_tile_pairs(pairs)
    dev = DeviceInputs(case)
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    check(case, out, dev)


@pytest.mark.parametrize("workload", ["dsvit", "vl2"])
def test_tile_order_does_not_change_the_bits(workload):
    """The dynamic tile order (units take the next tile from a counter), the static one
    and the automatic choice run the same tiles with the same K order. Forty more
    forwards in the dynamic order take the handle's 64 tile queues round more than once:
    each GEMM must leave its queue at zero."""
    wl = W.WORKLOADS[workload]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out_auto = run(case, proj, dev)
    proj.set_tile_order(vp.TILE_ORDER_STATIC)
    out_static = run(case, proj, dev)
    proj.set_tile_order(vp.TILE_ORDER_DYNAMIC)
    out_dyn = run(case, proj, dev)
    for _ in range(40):
        out_again = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_auto.view(torch.int16), out_static.view(torch.int16))
    assert torch.equal(out_auto.view(torch.int16), out_dyn.view(torch.int16))
    assert torch.equal(out_auto.view(torch.int16), out_again.view(torch.int16))


@pytest.mark.parametrize("budget", [1 << 20, 256 << 20])
def test_raster_budget_does_not_change_the_bits(budget):
    """The raster band width (how many N-blocks share the L2 at once) only reorders the
    output tiles; each output is accumulated over the same K order."""
    wl = W.WORKLOADS["dsvit"]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out_a = run(case, proj, dev)
    proj.set_raster_budget(budget)
    out_b = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
