"""The LayerNorm-merge kernels on a B200, for every width class the launch picks.

The classes are 2, 5 and 8 packed vectors per lane, and the two-pass form past
C = 2048, with bf16 and fp32 features. The cases include a ring with more slots than
the warp has items, and warps that walk more than 32 items (the source-row table is
reloaded). For each case: the hidden activations against the oracle, the whole
forward against the oracle, and bit for bit against each other: the default path (the
LayerNorm written already merged), the patch-order LayerNorm + cp.async gather path, and
the thread gather (bf16 features: statistics pass + LayerNorm applied inside GEMM1), and
the fused producer warps (LayerNorm-merge written inside GEMM1 ahead of its TMA loads).
"""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
from oracle import projector as O

from gpu_harness import (DeviceInputs, check, custom, feats_f64, make_case, make_projector, oracle_params, run,
                         TOL_ABS, TOL_REL)

pytestmark = pytest.mark.gpu

# name: (C, fp32 features, grids (h, w) of the views, sequence length)
CASES = {
    "c64_ring_longer_than_work": (64, False, [[3, 3]], 64),          # 16 ring slots, one item per warp
    "c1152_f32": (1152, True, [[9, 7], [4, 6], [11, 3]], 64),       # 5 vectors per lane
    "c1536_bf16": (1536, False, [[9, 7], [4, 6], [11, 3]], 64),     # 8 vectors per lane
    "c2048_f32": (2048, True, [[7, 7], [6, 4]], 64),
    "c2304_bf16_two_pass": (2304, False, [[7, 9], [5, 4]], 64),     # past the register forms
    "c2560_f32_two_pass": (2560, True, [[5, 5]], 64),
    "c64_long_walk": (64, False, [[120, 120]] * 10, 4096),          # about 40 items per warp
}


def _case(name):
    C, f32, hw, S = CASES[name]
    n = len(hw)
    cfg = 170 + list(CASES).index(name)
    wl = custom(f"ln_{name}", cfg, 2, C, 128, 64, n, n, S, has_ln=True, feat_fp32=f32)
    return make_case(wl, np.array(hw, np.int32))


@pytest.mark.parametrize("name", list(CASES))
def test_merged_layernorm_hidden_matches_oracle(name):
    case = _case(name)
    wl = case.wl
    proj = make_projector(case)
    dev = DeviceInputs(case)
    M = sum(O.tokens_untiled(h, w, wl.k) for h, w in case.hw)
    H = torch.empty((M, wl.N1), dtype=torch.bfloat16, device="cuda")
    proj.hidden(dev.feats, case.hw, H)
    assert proj.status() == vp.OK
    got = H.double().cpu().numpy()
    params = oracle_params(case)
    ln = (params["gamma"], params["beta"], wl.ln_eps)
    r = 0
    for v in range(len(case.hw)):
        h, w = int(case.hw[v, 0]), int(case.hw[v, 1])
        want = O.hidden(O.merge_view(feats_f64(case, v), h, w, wl.k, ln), params["W1"], params["b1"])
        g = got[r:r + len(want)]
        assert (np.abs(g - want) <= TOL_ABS + TOL_REL * np.abs(want)).all(), f"view {v}"
        r += len(want)
    assert r == M


@pytest.mark.parametrize("name", list(CASES))
def test_merged_and_patch_order_layernorm_agree_bit_for_bit(name):
    case = _case(name)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out_a = run(case, proj, dev)                     # AUTO: LayerNorm written already merged
    assert proj.status() == vp.OK
    check(case, out_a, dev)
    proj.set_gather_mode(vp.GATHER_CPASYNC)          # patch-order LayerNorm, GEMM1 gathers
    out_b = run(case, proj, dev)
    assert proj.status() == vp.OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    for mode in (vp.GATHER_THREADS, vp.GATHER_FUSED):  # thread gather, fused producers
        for pairs in (True, False):                      # CTA pairs and single CTAs
            proj.set_gather_mode(mode)
            proj.set_tile_pairs(pairs)
            out_c = run(case, proj, dev)
            assert proj.status() == vp.OK
            assert torch.equal(out_a.view(torch.int16), out_c.view(torch.int16)), f"mode={mode} pairs={pairs}"
