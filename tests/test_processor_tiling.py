"""Processor tiling choices of the 2D tile scheme: the oracle against hand-worked
cases and the pages' counts, and the library's host function against the oracle."""
import json
import os

import numpy as np
import pytest

import vision_language_projector_b200 as vp
from oracle import processor as P

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "processor_hand.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["cases"], ids=lambda c: str(c["sizes"]))
def test_oracle_hand_worked(case):
    g = _golden()
    grids, counts = P.plan_images(case["sizes"], g["candidates"], g["image_size"], g["patch_size"], g["downsample"])
    assert [list(x) for x in grids] == case["grids"], case["work"]
    assert counts == case["counts"]


def test_oracle_counts_match_the_pages_examples():
    # 1x1 at patch 14 -> 421, 2x1 -> 617, patch 16 1x1 -> 313 ("port DeepSeek-VL2", Processor step 7)
    assert P.plan_images([[300, 300]], [[384, 384]], 384, 14, 2)[1] == [421]
    assert P.plan_images([[800, 400]], [[768, 384]], 384, 14, 2)[1] == [617]
    assert P.plan_images([[300, 300]], [[384, 384]], 384, 16, 2)[1] == [313]


def test_planted_tie_break_mistake_is_caught(monkeypatch):
    def wrong(w0, h0, candidates):      # keeps the LAST best candidate on ties of effective area
        best, be = None, -1
        for W, H in candidates:
            s = min(W / w0, H / h0)
            e = min(int(w0 * s) * int(h0 * s), w0 * h0)
            if e >= be:
                best, be = (W, H), e
        return best
    monkeypatch.setattr(P, "best_resolution", wrong)
    with pytest.raises(AssertionError):
        test_oracle_hand_worked(_golden()["cases"][0])


@pytest.mark.parametrize("case", _golden()["cases"], ids=lambda c: str(c["sizes"]))
def test_library_matches_golden(case):
    g = _golden()
    crop, rows, views = vp.plan_tiles(case["sizes"], g["candidates"], g["image_size"], g["patch_size"],
                                      g["downsample"])
    assert crop.tolist() == case["grids"]
    assert rows.tolist() == case["counts"]
    assert views == sum(1 + tw * th for tw, th in case["grids"])


def test_library_matches_oracle_on_random_requests():
    rng = np.random.default_rng(7)
    cands = [[384 * i, 384 * j] for i in range(1, 4) for j in range(1, 4) if i * j <= 6]
    for _ in range(2000):
        n = int(rng.integers(1, 4))
        sizes = rng.integers(16, 3000, size=(n, 2)).tolist()
        perm = rng.permutation(len(cands))
        cl = [cands[p] for p in perm[: int(rng.integers(1, len(cands) + 1))]]
        patch = int(rng.choice([14, 16]))
        grids, counts = P.plan_images(sizes, cl, 384, patch, 2)
        crop, rows, views = vp.plan_tiles(sizes, cl, 384, patch, 2)
        assert crop.tolist() == [list(x) for x in grids], (sizes, cl)
        assert rows.tolist() == counts


def test_library_rejects_bad_arguments():
    with pytest.raises(vp.VlprojError):
        vp.plan_tiles([[100, 100]], [[500, 384]], 384, 14, 2)     # candidate not a multiple of the tile
    with pytest.raises(vp.VlprojError):
        vp.plan_tiles([[0, 100]], [[384, 384]], 384, 14, 2)
