"""vlproj_forward_ex on a B200: the token-embedding lookup of the text rows and the
compact copy of the assembled rows, alongside the usual projection."""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
import workloads as W

from gpu_harness import DeviceInputs, check, custom, dev_bf16, make_case, make_projector

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["vl2", "moonvit", "tiny"])
def test_lookup_and_rows_out(name):
    wl = W.WORKLOADS[name]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    table = dev_bf16(W.embed_table(wl))                       # the table the prefill was gathered from
    out = torch.zeros_like(dev.prefill)
    R = sum(case.rows)
    rows_out = torch.full((R + 3, wl.N2), float("nan"), dtype=torch.bfloat16, device="cuda")
    proj.forward_ex(dev.feats, case.hw, case.crop, dev.ids, W.IMAGE_TOKEN_ID, out, dev.newline, dev.sep,
                    embed_table=table, rows_out=rows_out, n_images=wl.n_images)
    assert proj.status() == vp.OK
    # text rows equal the prefill (table[ids]) bit for bit; image rows match the oracle
    check(case, out, dev, images=[0, wl.n_images - 1] if wl.n_images > 1 else None)
    pos = torch.nonzero(dev.ids == W.IMAGE_TOKEN_ID).flatten()
    assert torch.equal(rows_out[:R].view(torch.int16), out.index_select(0, pos).view(torch.int16))
    assert torch.isnan(rows_out[R:].float()).all()


def test_forward_ex_without_extras_equals_forward():
    wl = W.WORKLOADS["dsvit"]
    case = make_case(wl)
    proj = make_projector(case)
    dev = DeviceInputs(case)
    a = dev.prefill.clone()
    proj.forward(dev.feats, case.hw, None, dev.ids, W.IMAGE_TOKEN_ID, a)
    b = dev.prefill.clone()
    proj.forward_ex(dev.feats, case.hw, None, dev.ids, W.IMAGE_TOKEN_ID, b)
    assert proj.status() == vp.OK
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_lookup_out_of_range_id_latches_and_zeroes():
    wl = custom("lookup_bad", 140, 2, 64, 64, 32, 1, 1, 50)
    case = make_case(wl, np.array([[4, 4]], np.int32))
    proj = make_projector(case)
    dev = DeviceInputs(case)
    ids = dev.ids.clone()
    bad = int(torch.nonzero(ids != W.IMAGE_TOKEN_ID)[0])
    ids[bad] = 5000                                            # vocab is 1000
    table = dev_bf16(W.embed_table(wl))
    out = torch.ones_like(dev.prefill)
    proj.forward_ex(dev.feats, case.hw, None, ids, W.IMAGE_TOKEN_ID, out, embed_table=table)
    assert proj.status() == vp.ERR_INVALID_ARG
    assert (out[bad].float() == 0).all()


def test_rows_out_too_small_is_rejected_before_launch():
    wl = custom("rows_small", 141, 2, 64, 64, 32, 1, 1, 50)
    case = make_case(wl, np.array([[4, 4]], np.int32))
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out = dev.prefill.clone()
    small = torch.zeros((sum(case.rows) - 1, wl.N2), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vp.VlprojError) as e:
        proj.forward_ex(dev.feats, case.hw, None, dev.ids, W.IMAGE_TOKEN_ID, out, rows_out=small)
    assert e.value.code == vp.ERR_INVALID_ARG
    assert torch.equal(out.view(torch.int16), dev.prefill.view(torch.int16))
