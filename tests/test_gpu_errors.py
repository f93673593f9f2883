"""Device-found errors and degenerate calls, on a B200. No test here faults, traps or
hangs the GPU: count mismatches are latched by the index kernel and make the
scatter write nothing; the timeout test shrinks the kernels' wait bound so their
bounded waits run out, after which the kernels drain and return."""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
import workloads as W

from gpu_harness import DeviceInputs, check, custom, make_case, make_projector, run

pytestmark = pytest.mark.gpu


def _case():
    wl = custom("err_case", 110, 2, 64, 128, 64, 2, 2, 64, has_ln=True)
    return make_case(wl, np.array([[8, 8], [6, 10]], np.int32))


def test_count_mismatch_writes_nothing():
    case = _case()
    proj = make_projector(case)
    dev = DeviceInputs(case)
    ids = dev.ids.clone()
    first_text = int(torch.nonzero(ids != W.IMAGE_TOKEN_ID)[0])
    ids[first_text] = W.IMAGE_TOKEN_ID                      # one placeholder too many
    out = dev.prefill.clone()
    proj.forward(dev.feats, case.hw, None, ids, W.IMAGE_TOKEN_ID, out)
    assert proj.status() == vp.ERR_TOKEN_COUNT
    assert torch.equal(out.view(torch.int16), dev.prefill.view(torch.int16))
    assert proj.status() == vp.OK                           # cleared once read
    ids2 = dev.ids.clone()
    ids2[int(torch.nonzero(ids2 == W.IMAGE_TOKEN_ID)[0])] = 7   # one too few
    proj.forward(dev.feats, case.hw, None, ids2, W.IMAGE_TOKEN_ID, out)
    assert proj.status() == vp.ERR_TOKEN_COUNT
    assert torch.equal(out.view(torch.int16), dev.prefill.view(torch.int16))
    # the handle still works afterwards
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    check(case, out, dev)


def test_text_only_is_a_noop():
    case = _case()
    proj = make_projector(case)
    ids = torch.randint(0, 1000, (500,), device="cuda", dtype=torch.int64)
    out = torch.randn(500, case.wl.N2, device="cuda").to(torch.bfloat16)
    ref = out.clone()
    proj.forward(None, None, None, ids, W.IMAGE_TOKEN_ID, out, n_images=0)
    assert proj.status() == vp.OK
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    ids[17] = W.IMAGE_TOKEN_ID                              # placeholders without images
    proj.forward(None, None, None, ids, W.IMAGE_TOKEN_ID, out, n_images=0)
    assert proj.status() == vp.ERR_TOKEN_COUNT
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_empty_ids_with_images_is_a_count_error():
    case = _case()
    proj = make_projector(case)
    dev = DeviceInputs(case)
    ids = torch.empty(0, dtype=torch.int64, device="cuda")
    out = torch.empty(0, case.wl.N2, dtype=torch.bfloat16, device="cuda")
    proj.forward(dev.feats, case.hw, None, ids, W.IMAGE_TOKEN_ID, out)
    assert proj.status() == vp.ERR_TOKEN_COUNT


def test_host_argument_errors():
    case = _case()
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out = dev.prefill.clone()
    with pytest.raises(vp.VlprojError) as e:
        proj.forward(dev.feats, np.array([[8, 0], [6, 10]], np.int32), None, dev.ids, W.IMAGE_TOKEN_ID, out)
    assert e.value.code == vp.ERR_INVALID_ARG
    with pytest.raises(vp.VlprojError):
        proj.forward(None, case.hw, None, dev.ids, W.IMAGE_TOKEN_ID, out)
    with pytest.raises(vp.VlprojError):       # misaligned output rows
        proj.forward(dev.feats, case.hw, None, dev.ids, W.IMAGE_TOKEN_ID, out.view(-1)[1:].view(torch.int16))
    assert torch.equal(out.view(torch.int16), dev.prefill.view(torch.int16))


def test_tiled_requires_newline_and_separator():
    wl = custom("err_tiled", 111, 2, 64, 64, 32, 1, 1, 64, tiled=True, tw=1, th=1)
    case = make_case(wl, np.array([[4, 4]] * 2, np.int32))
    proj = make_projector(case)
    dev = DeviceInputs(case)
    with pytest.raises(vp.VlprojError):
        proj.forward(dev.feats, case.hw, case.crop, dev.ids, W.IMAGE_TOKEN_ID, dev.prefill.clone(), None, None)


def test_bounded_wait_timeout_then_recovery():
    """With a 1 ns bound the GEMMs' first unsatisfied wait runs out: the kernels latch
    VLPROJ_ERR_TIMEOUT, drain their copies and MMAs, free TMEM and return. The
    context stays usable and the next call with the default bound is correct."""
    wl = custom("timeout_case", 112, 3, 1024, 512, 256, 4, 2, 400)
    case = make_case(wl, np.array([[30, 30]] * 4, np.int32))
    proj = make_projector(case)
    dev = DeviceInputs(case)
    proj.set_tile_order(vp.TILE_ORDER_DYNAMIC)
    proj.set_wait_limit(1)
    run(case, proj, dev)
    assert proj.status() == vp.ERR_TIMEOUT
    proj.set_wait_limit(0)
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    check(case, out, dev)
    # the timed-out GEMMs' tile counters were set back to zero: 33 more forwards (66
    # GEMMs) take every one of the handle's 64 counter pairs again
    for _ in range(33):
        out = run(case, proj, dev)
    assert proj.status() == vp.OK
    check(case, out, dev)


def test_wait_bound_runs_out_in_layernorm_merge():
    """The same with a LayerNorm: the LayerNorm-merge kernel's ring waits run out too; it
    latches VLPROJ_ERR_TIMEOUT, lets the copies already issued land, and returns."""
    wl = custom("timeout_ln", 113, 2, 1152, 256, 128, 4, 2, 800, has_ln=True)
    case = make_case(wl, np.array([[24, 24]] * 4, np.int32))
    proj = make_projector(case)
    dev = DeviceInputs(case)
    proj.set_wait_limit(1)
    run(case, proj, dev)
    assert proj.status() == vp.ERR_TIMEOUT
    proj.set_wait_limit(0)
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    check(case, out, dev)
