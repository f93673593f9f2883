"""Host-side checks of the C-ABI library that need no GPU.

* the library loads and exports every function ``include/vlproj.h`` declares;
* its closed-form placeholder counts agree with the oracle's on every workload
  and on edge grids;
* configuration errors the pages ask to be loud about are rejected before any
  device work.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import vision_language_projector_b200 as vp
import workloads as W
from oracle import projector as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "vlproj.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vlproj_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 9
    out = subprocess.run(["nm", "-D", "--defined-only", vp.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (vlproj_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(vp._lib, n)
    assert set(vp.EXPORTED) == set(names)


def test_library_is_built_for_sm100a():
    out = subprocess.run(["cuobjdump", "--list-elf", vp.LIB_PATH], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    assert "sm_100a" in out.stdout


def test_version_and_strerror():
    assert "sm_100a" in vp.version()
    for code in (0, -1, -2, -3, -4, -5):
        assert vp.strerror(code) and vp.strerror(code) != "unknown status"


def _cfg(wl):
    return vp.make_config(wl.k, wl.C, wl.N1, wl.N2, has_ln=wl.has_ln,
                          tile_tag=vp.TILE_2D if wl.tiled else vp.TILE_NONE)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_image_rows_match_oracle(name):
    wl = W.WORKLOADS[name]
    hw = W.grid_hw(wl)
    crop = W.spatial_crop(wl)
    got = vp.image_rows(_cfg(wl), hw, crop, wl.n_images)
    assert list(got) == O.image_rows(hw, wl.k, crop)


@pytest.mark.parametrize("k,hw", [(1, [[24, 24]]), (3, [[96, 96]]), (2, [[27, 27], [1, 1], [5, 96]]),
                                  (3, [[25, 31], [2, 2], [4, 1]])])
def test_image_rows_edge_grids(k, hw):
    cfg = vp.make_config(k, 64, 64, 32)
    hw = np.array(hw, np.int32)
    assert list(vp.image_rows(cfg, hw)) == O.image_rows(hw, k, None)


def test_image_rows_tiled_pages_examples():
    # 384/14 = 27 patches -> h' = 14; 384/16 = 24 -> h' = 12 ("port DeepSeek-VL2", Processor step 7)
    cfg = vp.make_config(2, 64, 64, 32, tile_tag=vp.TILE_2D)
    assert list(vp.image_rows(cfg, [[27, 27]] * 2, [[1, 1]])) == [421]
    assert list(vp.image_rows(cfg, [[27, 27]] * 3, [[2, 1]])) == [617]
    assert list(vp.image_rows(cfg, [[24, 24]] * 2, [[1, 1]])) == [313]
    tail = vp.make_config(2, 64, 64, 32, tile_tag=vp.TILE_2D, global_view_pos=vp.GLOBAL_TAIL)
    assert list(vp.image_rows(tail, [[27, 27]] * 3, [[2, 1]])) == [617]


def test_image_rows_rejects_bad_shapes():
    cfg = vp.make_config(2, 64, 64, 32, tile_tag=vp.TILE_2D)
    with pytest.raises(vp.VlprojError) as e:
        vp.image_rows(cfg, [[27, 27], [27, 26], [27, 27]], [[2, 1]])    # views of one image differ
    assert e.value.code == vp.ERR_INVALID_ARG
    with pytest.raises(vp.VlprojError):
        vp.image_rows(cfg, [[0, 5]] * 3, [[2, 1]])
    with pytest.raises(vp.VlprojError):
        vp.image_rows(cfg, [[4, 4]] * 3, [[0, 1]])


@pytest.mark.parametrize("kw,code", [
    (dict(depth=1), vp.ERR_UNSUPPORTED),
    (dict(depth=9), vp.ERR_UNSUPPORTED),
    (dict(tile_tag=vp.TILE_1D), vp.ERR_UNSUPPORTED),
    (dict(token_pooling=1), vp.ERR_UNSUPPORTED),
    (dict(k=4), vp.ERR_UNSUPPORTED),
    (dict(C=100), vp.ERR_INVALID_ARG),
    (dict(N1=100), vp.ERR_INVALID_ARG),
    (dict(N2=40), vp.ERR_INVALID_ARG),
    (dict(), vp.ERR_INVALID_ARG),           # weights missing
])
def test_create_rejects_before_device_work(kw, code):
    base = dict(k=2, C=64, N1=64, N2=32)
    base.update(kw)
    k, C, N1, N2 = base.pop("k"), base.pop("C"), base.pop("N1"), base.pop("N2")
    cfg = vp.make_config(k, C, N1, N2, **base)
    h = ctypes.c_void_p()
    assert vp._lib.vlproj_create(ctypes.byref(cfg), ctypes.byref(h)) == code
    assert not h.value


def test_create_rejects_deeper_mlp_without_middle_weights():
    cfg = vp.make_config(2, 64, 64, 32, depth=3, W1=16, W2=16)     # non-null stand-ins, never dereferenced
    h = ctypes.c_void_p()
    assert vp._lib.vlproj_create(ctypes.byref(cfg), ctypes.byref(h)) == vp.ERR_INVALID_ARG


def test_setters_reject_a_null_handle_and_bad_values():
    """Host-side argument checks of the tuning setters, no device work."""
    assert vp._lib.vlproj_set_tile_order(None, vp.TILE_ORDER_AUTO) == vp.ERR_INVALID_ARG
    assert vp._lib.vlproj_set_raster_budget(None, 0) == vp.ERR_INVALID_ARG
    assert vp._lib.vlproj_set_tile_pairs(None, 1) == vp.ERR_INVALID_ARG
    assert (vp.TILE_ORDER_STATIC, vp.TILE_ORDER_AUTO, vp.TILE_ORDER_DYNAMIC) == (0, 1, 2)
