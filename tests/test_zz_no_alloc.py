"""The placeholder index that allocates nothing, against the forward pass's own.

`vlproj_placeholder_index_noalloc` is for callers that must not allocate device
memory when they call it (an allocation there would synchronise the device or break
a latency budget, or the caller has no allocator of its own). It keeps its only
scratch in a fixed array in the library's device memory.

Reference: `vlproj_forward` writes a projected, newline or separator row to exactly
the placeholder positions its own index step finds, so the rows it overwrote in a
sentinel-prefilled buffer are that step's output. Two calls in a row of the
no-allocation entry point must return those positions and their count exactly
(integer results: bit-exact).
"""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
import workloads as W

from gpu_harness import DeviceInputs, custom, make_case, make_projector, run

pytestmark = pytest.mark.gpu


def _forward_positions(case):
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    changed = (out.view(torch.int16) != dev.prefill.view(torch.int16)).any(dim=1)
    return dev.ids, torch.nonzero(changed).flatten().to(torch.int64).cpu().numpy()


def _noalloc_twice(ids, expect):
    n = ids.numel()
    for _ in range(2):
        positions = torch.full((max(n, 1),), -1, dtype=torch.int32, device="cuda")
        count = torch.full((1,), -1, dtype=torch.int64, device="cuda")
        rc = vp.placeholder_index_noalloc(ids, W.IMAGE_TOKEN_ID, positions, count)
        assert rc == vp.OK
        torch.cuda.synchronize()
        c = int(count.item())
        assert c == len(expect)
        np.testing.assert_array_equal(positions[:c].cpu().numpy().astype(np.int64), expect)
        assert (positions[c:].cpu().numpy() == -1).all()


@pytest.mark.parametrize("name", ["tiny", "dsvit", "vl2"])
def test_noalloc_index_matches_forward(name):
    case = make_case(W.WORKLOADS[name])
    ids, expect = _forward_positions(case)
    assert len(expect) == sum(case.rows)
    _noalloc_twice(ids, expect)


def test_noalloc_index_many_blocks_and_text_only():
    # 8 sequences of 3,000 ids: placeholder runs cross the 4096-id block boundaries
    wl = custom("noalloc_blocks", 130, 2, 64, 64, 32, 16, 8, 3000)
    case = make_case(wl, np.array([[20, 22]] * 16, np.int32))
    ids, expect = _forward_positions(case)
    _noalloc_twice(ids, expect)
    # no placeholders at all
    text = torch.randint(0, 1000, (10_000,), dtype=torch.int64, device="cuda")
    _noalloc_twice(text, np.zeros(0, np.int64))


def test_noalloc_index_rejects_more_than_its_limit():
    ids = torch.zeros(16, dtype=torch.int64, device="cuda")
    positions = torch.zeros(16, dtype=torch.int32, device="cuda")
    count = torch.zeros(1, dtype=torch.int64, device="cuda")
    rc = vp.placeholder_index_noalloc(ids, W.IMAGE_TOKEN_ID, positions, count, n_ids=vp.NOALLOC_MAX_IDS + 1)
    assert rc == vp.ERR_INVALID_ARG
