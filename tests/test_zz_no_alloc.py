"""The placeholder index that allocates nothing, against the oracle.

`vlproj_placeholder_index_noalloc` is for callers that must not allocate device
memory when they call it (an allocation there would synchronise the device or break
a latency budget, or the caller has no allocator of its own). It keeps its only
scratch in a fixed array in the library's device memory, shared by every call.

Expected values come from the oracle's `placeholder_positions` (the flat indices
holding the image id, in order: "port DeepSeek-VL2", end of Tile-sequence assembly).
Two calls in a row must return those positions and their count exactly (integer
results: bit-exact), and the second call must not see anything the first one left in
the shared array. One case also checks that the forward pass's own index step writes
its rows to the same positions.
"""
import numpy as np
import pytest
import torch

import vision_language_projector_b200 as vp
import workloads as W
from oracle import projector as O

from gpu_harness import DeviceInputs, make_case, make_projector, run

pytestmark = pytest.mark.gpu

CHUNK = 4096        # ids per block of the index kernels


def _noalloc_twice(ids_np: np.ndarray, token: int = W.IMAGE_TOKEN_ID, room=None):
    expect = O.placeholder_positions(ids_np, token)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, np.int64)).cuda()
    n = ids.numel()
    room = max(n, 1) if room is None else room
    for _ in range(2):
        positions = torch.full((room,), -1, dtype=torch.int32, device="cuda")
        count = torch.full((1,), -1, dtype=torch.int64, device="cuda")
        rc = vp.placeholder_index_noalloc(ids, token, positions, count)
        assert rc == vp.OK
        torch.cuda.synchronize()
        assert int(count.item()) == len(expect)
        got = positions.cpu().numpy().astype(np.int64)
        kept = min(len(expect), room)
        np.testing.assert_array_equal(got[:kept], expect[:kept])
        assert (got[kept:] == -1).all()
    return expect


@pytest.mark.parametrize("name", ["tiny", "dsvit", "vl2", "stress"])
def test_noalloc_index_matches_oracle_on_workloads(name):
    wl = W.WORKLOADS[name]
    hw = W.grid_hw(wl)
    rows = O.image_rows(hw, wl.k, W.spatial_crop(wl))
    ids = W.input_ids(wl, rows)
    expect = _noalloc_twice(ids)
    assert len(expect) == sum(rows)


def test_noalloc_index_edge_cases():
    rng = np.random.default_rng(7)
    tok = W.IMAGE_TOKEN_ID
    # every id a placeholder, over several blocks and a ragged last block
    _noalloc_twice(np.full(3 * CHUNK + 17, tok, np.int64))
    # no placeholders at all
    _noalloc_twice(rng.integers(0, 1000, 10_000))
    # placeholders on both sides of every block edge, and none exactly at one
    ids = rng.integers(0, 1000, 5 * CHUNK)
    for b in range(1, 5):
        ids[b * CHUNK - 3:b * CHUNK - 1] = tok          # ends one id before the edge
        ids[b * CHUNK + 1:b * CHUNK + 4] = tok          # starts one id after it
    _noalloc_twice(ids)
    # a run that covers whole blocks, starting and ending mid-block
    ids = rng.integers(0, 1000, 6 * CHUNK)
    ids[CHUNK // 2:4 * CHUNK + 100] = tok
    _noalloc_twice(ids)
    # a single id, and an empty input
    _noalloc_twice(np.array([tok], np.int64))
    _noalloc_twice(np.zeros(0, np.int64))
    # fewer slots than placeholders: the first ones are written, the count is the total
    ids = np.full(2 * CHUNK, tok, np.int64)
    _noalloc_twice(ids, room=1000)


def test_noalloc_index_after_a_larger_call():
    """A small call right after a large one must not read the large call's block
    counts left in the shared array."""
    rng = np.random.default_rng(11)
    big = rng.integers(0, 1000, 40 * CHUNK)
    big[rng.choice(big.size, 5000, replace=False)] = W.IMAGE_TOKEN_ID
    _noalloc_twice(big)
    small = rng.integers(0, 1000, CHUNK + 5)
    small[[0, 100, CHUNK - 1, CHUNK, CHUNK + 4]] = W.IMAGE_TOKEN_ID
    _noalloc_twice(small)


def test_noalloc_index_agrees_with_the_forward_pass():
    """The forward pass writes a row exactly at the positions its own index step finds;
    the rows it changed in a sentinel-prefilled buffer are those positions."""
    case = make_case(W.WORKLOADS["tiny"])
    proj = make_projector(case)
    dev = DeviceInputs(case)
    out = run(case, proj, dev)
    assert proj.status() == vp.OK
    changed = (out.view(torch.int16) != dev.prefill.view(torch.int16)).any(dim=1)
    written = torch.nonzero(changed).flatten().cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(written, _noalloc_twice(case.ids))


def test_noalloc_index_rejects_more_than_its_limit():
    ids = torch.zeros(16, dtype=torch.int64, device="cuda")
    positions = torch.zeros(16, dtype=torch.int32, device="cuda")
    count = torch.zeros(1, dtype=torch.int64, device="cuda")
    rc = vp.placeholder_index_noalloc(ids, W.IMAGE_TOKEN_ID, positions, count, n_ids=vp.NOALLOC_MAX_IDS + 1)
    assert rc == vp.ERR_INVALID_ARG
