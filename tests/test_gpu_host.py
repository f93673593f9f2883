"""vlproj_project_host on a B200: features from page-locked host memory, the assembled
rows back to host memory, copies pipelined against the projection. Its rows must be
the bits vlproj_forward_ex writes to rows_out (which the parity tests tie to the
oracle), for any chunking."""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
import workloads as W

from gpu_harness import DeviceInputs, check, custom, make_case, make_projector

pytestmark = pytest.mark.gpu


def device_rows(case, proj, dev):
    R = sum(case.rows)
    rows = torch.empty((R, case.wl.N2), dtype=torch.bfloat16, device="cuda")
    out = dev.prefill.clone()
    proj.forward_ex(dev.feats, case.hw, case.crop, dev.ids, W.IMAGE_TOKEN_ID, out, dev.newline, dev.sep,
                    rows_out=rows, n_images=case.wl.n_images)
    assert proj.status() == vp.OK
    return rows.view(torch.int16).cpu(), out


def host_rows(case, proj, dev, chunks, extra=0):
    wl = case.wl
    R = sum(case.rows)
    feats = (torch.from_numpy(case.feats) if wl.feat_fp32 else torch.from_numpy(case.feats.view(np.int16))).pin_memory()
    rows = torch.full((R + extra, wl.N2), -1, dtype=torch.int16).pin_memory()
    proj.project_host(feats, case.hw, case.crop, rows, dev.newline, dev.sep, chunks=chunks, n_images=wl.n_images)
    torch.cuda.synchronize()
    assert proj.status() == vp.OK
    return rows


CASES = {
    "tiny": (lambda: W.WORKLOADS["tiny"], None, 2),
    "ragged_ln": (lambda: custom("host_ragged_ln", 150, 2, 128, 256, 96, 5, 5, 300, has_ln=True),
                  [[20, 30], [17, 9], [32, 32], [3, 5], [10, 10]], 2),
    "tiled_tail": (lambda: custom("host_tiled", 151, 2, 64, 128, 128, 3, 3, 200, tiled=True, tw=2, th=1),
                   [[9, 9]] * 3 + [[7, 5]] * 3 + [[6, 6]] * 3, 2),
    "k3_deep": (lambda: custom("host_k3", 152, 3, 64, 192, 128, 4, 4, 100), [[10, 11], [7, 3], [9, 9], [4, 4]], 3),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("chunks", [0, 1, 2, 3, 7])
def test_host_rows_equal_device_rows(name, chunks):
    make_wl, hw, depth = CASES[name]
    wl = make_wl()
    case = make_case(wl, hw, gvp="tail" if name == "tiled_tail" else "head", depth=depth)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    want, out = device_rows(case, proj, dev)
    got = host_rows(case, proj, dev, chunks, extra=2)
    assert torch.equal(got[:want.shape[0]], want)
    assert bool((got[want.shape[0]:] == -1).all())          # nothing past R is written
    if chunks == 0:
        check(case, out, dev)                                 # and those rows match the oracle


@pytest.mark.parametrize("name", ["moonvit", "vl2"])
def test_host_rows_full_size(name):
    wl = W.WORKLOADS[name]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    want, _ = device_rows(case, proj, dev)
    got = host_rows(case, proj, dev, 0)
    assert torch.equal(got, want)


def test_host_rejects_small_output_and_missing_buffers():
    wl = W.WORKLOADS["tiny"]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    feats = torch.from_numpy(case.feats).pin_memory()
    small = torch.empty((sum(case.rows) - 1, wl.N2), dtype=torch.int16)
    assert proj.project_host(feats, case.hw, None, small, check=False) == vp.ERR_INVALID_ARG
    assert proj.project_host(None, case.hw, None, small, check=False) == vp.ERR_INVALID_ARG
    assert proj.status() == vp.OK
