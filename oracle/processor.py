"""Processor tiling geometry of the 2D tile scheme (TEST INFRASTRUCTURE ONLY).

Restates "port DeepSeek-VL2", section Processor, steps 1, 2, 6 and 7: whether an
image is cropped, which candidate resolution it is fitted to (largest effective
area, ties to the least wasted area), its tile grid (tw, th) with the width count
first, and its placeholder count. Arithmetic in Python floats (IEEE double).
"""
from __future__ import annotations

import math
from typing import Sequence

from .projector import merged_side, tokens_tiled


def best_resolution(w0: int, h0: int, candidates: Sequence[Sequence[int]]) -> tuple:
    """Step 2: for each candidate (W, H): scale = min(W / w0, H / h0), effective =
    min(floor(w0 * scale) * floor(h0 * scale), w0 * h0), wasted = W * H - effective;
    keep the largest effective area, ties broken by the smallest waste (first wins)."""
    best, best_eff, best_waste = None, -1, None
    for W, H in candidates:
        scale = min(W / w0, H / h0)
        eff = min(math.floor(w0 * scale) * math.floor(h0 * scale), w0 * h0)
        waste = W * H - eff
        if eff > best_eff or (eff == best_eff and waste < best_waste):
            best, best_eff, best_waste = (W, H), eff, waste
    return best


def plan_images(sizes: Sequence[Sequence[int]], candidates: Sequence[Sequence[int]], image_size: int,
                patch_size: int, downsample: int) -> tuple:
    """Steps 1, 6, 7 for one request: returns ([(tw, th)], [placeholder count]).
    Cropping only when the request has at most 2 images; otherwise every grid is 1x1."""
    crop = len(sizes) <= 2
    hp = merged_side(image_size // patch_size, downsample)
    grids, counts = [], []
    for w0, h0 in sizes:
        W, H = best_resolution(w0, h0, candidates) if crop else (image_size, image_size)
        tw, th = W // image_size, H // image_size
        grids.append((tw, th))
        counts.append(tokens_tiled(hp, hp, tw, th))
    return grids, counts
