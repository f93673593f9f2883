"""The Python binding's argument checks, on the CPU: the C ABI receives bare pointers and
cannot tell host from device memory or see a buffer's length, so the binding rejects,
before any library call, tensors in the wrong memory, of the wrong element size, not
contiguous or too small, and host arrays shorter than the image count implies. No
handle is created (that needs a GPU): the checks run first."""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp

K, C, N1, N2 = 2, 64, 128, 64


def _proj(**kw):
    p = vp.Projector.__new__(vp.Projector)
    p.cfg = vp.make_config(K, C, N1, N2, **kw)
    p._h = None
    return p


def _raises(fn, name):
    with pytest.raises(vp.VlprojError) as e:
        fn()
    assert e.value.code == vp.ERR_INVALID_ARG
    assert name in str(e.value)


HW = np.array([[4, 4], [3, 5]], np.int32)        # 16 + 15 patches, 4 + 6 merged tokens


def test_device_arguments_must_be_cuda_tensors():
    p = _proj()
    ids = torch.zeros(100, dtype=torch.int64)
    _raises(lambda: p.forward(torch.zeros(31, C, dtype=torch.bfloat16), HW, None, ids, 7, None), "features")
    _raises(lambda: p.forward(np.zeros((31, C), np.float32), HW, None, ids, 7, None), "features")
    _raises(lambda: p.forward(None, HW, None, ids, 7, None), "input_ids")


def test_check_false_returns_the_code():
    p = _proj()
    rc = p.forward(torch.zeros(31, C, dtype=torch.bfloat16), HW, None, None, 7, None, check=False)
    assert rc == vp.ERR_INVALID_ARG


def test_host_arrays_shorter_than_the_images_are_rejected():
    p = _proj()
    _raises(lambda: p.forward(None, HW, None, None, 7, None, n_images=3), "grid_hw")
    t = _proj(tile_tag=vp.TILE_2D)
    crop = np.array([[2, 1]], np.int32)                     # 3 views for one image, 2 rows given
    _raises(lambda: t.forward(None, HW, crop, None, 7, None, n_images=1), "grid_hw")
    _raises(lambda: t.forward(None, np.zeros((6, 2), np.int32), crop, None, 7, None, n_images=2), "spatial_crop")


def test_backward_middle_layer_lists_match_the_depth():
    p = _proj(depth=3)
    grads = {"W_mid": [], "b_mid": None}
    _raises(lambda: p.backward(None, None, None, None, 7, None, grads, n_images=0), "W_mid")


def test_backward_gradients_must_be_cuda_fp32():
    p = _proj()
    grads = {"b2": torch.zeros(N2)}
    _raises(lambda: p.backward(None, None, None, None, 7, None, grads, n_images=0), "b2")


def test_project_host_memory_kinds_and_sizes():
    p = _proj()
    feats = torch.zeros(31, C, dtype=torch.bfloat16)       # host features: accepted
    rows = torch.zeros(10, N2, dtype=torch.float32)        # wrong element size
    _raises(lambda: p.project_host(feats, HW, None, rows), "rows_out")
    short = torch.zeros(30, C, dtype=torch.bfloat16)       # 30 < 31 patches
    _raises(lambda: p.project_host(short, HW, None, torch.zeros(10, N2, dtype=torch.int16)), "features")
    strided = torch.zeros(31, 2 * C, dtype=torch.bfloat16)[:, ::2]
    _raises(lambda: p.project_host(strided, HW, None, torch.zeros(10, N2, dtype=torch.int16)), "features")
    narrow = np.zeros((10, N2 // 2), np.int16)            # rows narrower than N2
    _raises(lambda: p.project_host(feats, HW, None, narrow), "rows_out")


def test_fp32_features_need_four_byte_elements():
    p = _proj(feat_dtype=vp.FEAT_F32)
    _raises(lambda: p.project_host(torch.zeros(31, C, dtype=torch.bfloat16), HW, None,
                                   torch.zeros(10, N2, dtype=torch.int16)), "features")


class _FakeCuda:
    """Stands in for a CUDA tensor on this CPU-only machine: only what the binding's
    checks look at. Every check below fails before the library is called."""

    is_cuda = True
    device = "cuda:0"
    dtype = "fake"

    def __init__(self, numel: int, itemsize: int, contiguous: bool = True):
        self._n, self._size, self._contig = numel, itemsize, contiguous

    def numel(self):
        return self._n

    def element_size(self):
        return self._size

    def is_contiguous(self):
        return self._contig

    def data_ptr(self):
        return 0x1000


def test_noalloc_index_checks_its_tensors():
    ids, pos, cnt = _FakeCuda(100, 8), _FakeCuda(100, 4), _FakeCuda(1, 8)
    f = vp.placeholder_index_noalloc
    _raises(lambda: f(_FakeCuda(100, 4), 7, pos, cnt), "input_ids")                 # int32 ids
    _raises(lambda: f(ids, 7, _FakeCuda(100, 8), cnt), "positions")                 # int64 positions
    _raises(lambda: f(ids, 7, pos, _FakeCuda(1, 4)), "count")                       # int32 count
    _raises(lambda: f(ids, 7, pos, _FakeCuda(0, 8)), "count")                       # no room for the count
    _raises(lambda: f(ids, 7, pos, cnt, n_ids=101), "input_ids")                    # more ids than the tensor
    _raises(lambda: f(ids, 7, pos, cnt, max_positions=101), "positions")            # more room than the tensor
    _raises(lambda: f(_FakeCuda(100, 8, contiguous=False), 7, pos, cnt), "input_ids")
    _raises(lambda: f(torch.zeros(100, dtype=torch.int64), 7, pos, cnt), "input_ids")   # host memory
    _raises(lambda: f(ids, 7, pos, cnt, n_ids=-1), "n_ids")
