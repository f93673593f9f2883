"""Seeded synthetic inputs for the vision-to-language projector workloads.

This module is shared by the tests, the benchmark and the oracle checks. It
only draws random numbers and lays out buffers; it holds none of the
projector's arithmetic. Where a buffer's layout depends on the method (how
many placeholder tokens an image expands to), the caller passes that number
in, computed by whichever side is being exercised.

Every tensor is drawn from ``numpy.random.default_rng(SeedSequence([cfg_id,
tensor_id, index, seed]))``, so any single image can be regenerated on its
own. bf16 tensors are fp32 draws rounded to nearest-even and are returned as
their raw 16-bit patterns (``numpy.uint16``); fp32 tensors are returned as
``numpy.float32``.

Workloads (sizes and distributions from the five configurations of the
vision-language projector study):

* ``tiny``    one 24x24 grid of 64-channel fp32 patches, 2x2 merge, LayerNorm(64),
              MLP 256 -> 256 -> 128, zero biases, 200 token ids.
* ``moonvit`` MoonViT PatchMerger: 16 images, each side even in [16, 96],
              1152-channel bf16, LayerNorm(1152), 2x2 merge, MLP 4608 -> 4608 -> 4096,
              16 sequences of 8192 tokens, one image each.
* ``dsvit``   DeepSeek-ViT 3x3 path: 8 images of 96x96x1024 bf16, 3x3 merge,
              MLP 9216 -> 5120 -> 5120, 8 sequences of 4096 tokens.
* ``vl2``     DeepSeek-VL2 2D tiling: 32 images x (1 global + 2x3 local) views of
              27x27x1152 bf16, 2x2 merge (grid zero-padded to 28), MLP
              4608 -> 2560 -> 2560, newline and view-separator rows, 32 sequences
              of 2048 tokens.
* ``stress``  256 images of 96x96x1024 bf16, 3x3 merge, MLP 9216 -> 5120 -> 5120,
              8 sequences of 65,536 tokens holding 32 images each.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Sequence

import numpy as np

IMAGE_TOKEN_ID = 100015          # DeepSeek-VL2 / DeepSeek-VL config default
TEXT_VOCAB = 1000                # non-image ids are uniform in [0, TEXT_VOCAB)

# tensor ids inside the seed sequence
_T_FEAT, _T_W1, _T_B1, _T_W2, _T_B2, _T_GAMMA, _T_BETA = 1, 2, 3, 4, 5, 6, 7
_T_NEWLINE, _T_SEP, _T_GRID, _T_IDS, _T_TABLE = 8, 9, 10, 11, 12


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int
    n_images: int
    k: int                  # merge factor (k x k neighbourhood -> one token)
    C: int                  # vision feature width
    N1: int                 # MLP hidden width
    N2: int                 # output embedding width (n_embed)
    has_ln: bool
    feat_fp32: bool         # features are fp32 (else bf16)
    tiled: bool             # DeepSeek-VL2 "2D" tile tag: global + local views
    tw: int                 # local tiles across (width count first)
    th: int                 # local tiles down
    B: int                  # sequences
    S: int                  # tokens per sequence
    fixed_hw: Optional[tuple]      # (h, w) of every view, or None for seeded varlen
    varlen_range: Optional[tuple]  # (lo, hi) inclusive, even sides, when varlen
    bias_zero: bool
    ln_eps: float = 1e-5

    @property
    def K1(self) -> int:
        return self.k * self.k * self.C

    @property
    def views_per_image(self) -> int:
        return 1 + self.tw * self.th if self.tiled else 1

    @property
    def n_views(self) -> int:
        return self.n_images * self.views_per_image


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 2, 64, 256, 128, True, True, False, 0, 0,
                     1, 200, (24, 24), None, True),
    "moonvit": Workload("moonvit", 1, 16, 2, 1152, 4608, 4096, True, False, False, 0, 0,
                        16, 8192, None, (16, 96), False),
    "dsvit": Workload("dsvit", 2, 8, 3, 1024, 5120, 5120, False, False, False, 0, 0,
                      8, 4096, (96, 96), None, False),
    "vl2": Workload("vl2", 3, 32, 2, 1152, 2560, 2560, False, False, True, 2, 3,
                    32, 2048, (27, 27), None, False),
    "stress": Workload("stress", 4, 256, 3, 1024, 5120, 5120, False, False, False, 0, 0,
                       8, 65536, (96, 96), None, False),
}


def _rng(wl: Workload, tensor_id: int, index: int = 0, seed: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([wl.cfg_id, tensor_id, index, seed]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); return the bit patterns.

    Inputs here are finite draws, so the NaN/Inf cases of the rounding do not arise.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------- geometry
def grid_hw(wl: Workload, seed: int = 0) -> np.ndarray:
    """(n_views, 2) int32 patch-grid sides (h, w) of every view, views in order."""
    if wl.fixed_hw is not None:
        g = np.empty((wl.n_views, 2), np.int32)
        g[:, 0], g[:, 1] = wl.fixed_hw
        return g
    lo, hi = wl.varlen_range
    r = _rng(wl, _T_GRID, 0, seed)
    sides = 2 * r.integers(lo // 2, hi // 2 + 1, size=(wl.n_views, 2))
    return sides.astype(np.int32)


def spatial_crop(wl: Workload) -> Optional[np.ndarray]:
    """(n_images, 2) int32 (tw, th) per image for tiled workloads, else None."""
    if not wl.tiled:
        return None
    s = np.empty((wl.n_images, 2), np.int32)
    s[:, 0], s[:, 1] = wl.tw, wl.th
    return s


# --------------------------------------------------------------------------- tensors
def _normal_bits(r: np.random.Generator, shape, scale: float = 1.0, shift: float = 0.0) -> np.ndarray:
    x = r.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    if shift != 0.0:
        x += np.float32(shift)
    return f32_to_bf16_bits(x)


def view_features(wl: Workload, view: int, h: int, w: int, seed: int = 0) -> np.ndarray:
    """Features of one view, (h*w, C), rows row-major over (h, w)."""
    r = _rng(wl, _T_FEAT, view, seed)
    if wl.feat_fp32:
        return r.standard_normal((h * w, wl.C), dtype=np.float32)
    return _normal_bits(r, (h * w, wl.C))


def features(wl: Workload, hw: np.ndarray, seed: int = 0, views: Optional[Sequence[int]] = None,
             out: Optional[np.ndarray] = None, threads: int = 8) -> np.ndarray:
    """Packed channel-last features of the given views (default: all), views back to back."""
    views = list(range(len(hw))) if views is None else list(views)
    counts = [int(hw[v, 0]) * int(hw[v, 1]) for v in views]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    dt = np.float32 if wl.feat_fp32 else np.uint16
    if out is None:
        out = np.empty((int(offs[-1]), wl.C), dt)

    def fill(i):
        v = views[i]
        out[offs[i]:offs[i + 1]] = view_features(wl, v, int(hw[v, 0]), int(hw[v, 1]), seed)

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range(len(views))))
    return out


def weights(wl: Workload, seed: int = 0) -> dict:
    """Projector parameters. Linear weights are (out, in) bf16, input order c*k*k + dy*k + dx."""
    d = {
        "W1": _normal_bits(_rng(wl, _T_W1, 0, seed), (wl.N1, wl.K1), 0.02),
        "W2": _normal_bits(_rng(wl, _T_W2, 0, seed), (wl.N2, wl.N1), 0.02),
    }
    if wl.bias_zero:
        d["b1"] = np.zeros(wl.N1, np.float32)
        d["b2"] = np.zeros(wl.N2, np.float32)
    else:
        d["b1"] = (_rng(wl, _T_B1, 0, seed).standard_normal(wl.N1, dtype=np.float32) * np.float32(0.02))
        d["b2"] = (_rng(wl, _T_B2, 0, seed).standard_normal(wl.N2, dtype=np.float32) * np.float32(0.02))
    if wl.has_ln:
        d["gamma"] = np.float32(1.0) + _rng(wl, _T_GAMMA, 0, seed).standard_normal(wl.C, dtype=np.float32) * np.float32(0.1)
        d["beta"] = _rng(wl, _T_BETA, 0, seed).standard_normal(wl.C, dtype=np.float32) * np.float32(0.02)
    else:
        d["gamma"] = None
        d["beta"] = None
    if wl.tiled:
        d["newline"] = _normal_bits(_rng(wl, _T_NEWLINE, 0, seed), (wl.N2,), 0.02)
        d["sep"] = _normal_bits(_rng(wl, _T_SEP, 0, seed), (wl.N2,), 0.02)
    else:
        d["newline"] = None
        d["sep"] = None
    return d


_T_MID = 13


def mid_weights(wl: Workload, depth: int, seed: int = 0) -> list:
    """(depth - 2) middle layers (W bf16 bits (N1, N1) ~N(0, 0.02), b fp32 ~N(0, 0.02))."""
    out = []
    for i in range(depth - 2):
        r = _rng(wl, _T_MID, i, seed)
        out.append((_normal_bits(r, (wl.N1, wl.N1), 0.02),
                    r.standard_normal(wl.N1, dtype=np.float32) * np.float32(0.02)))
    return out


_T_DOUT = 14


def grad_out(wl: Workload, n_ids: int, seed: int = 0) -> np.ndarray:
    """(n_ids, N2) bf16 bits ~N(0, 1): a loss gradient with respect to the embedding buffer."""
    return _normal_bits(_rng(wl, _T_DOUT, 0, seed), (n_ids, wl.N2))


def grad_out_blocks(wl: Workload, n_ids: int, seed: int = 0, threads: int = 8, block: int = 4096) -> np.ndarray:
    """(n_ids, N2) bf16 bits ~N(0, 1), drawn in blocks of `block` rows from streams of
    their own (so large batches are generated in parallel): a dense loss gradient."""
    out = np.empty((n_ids, wl.N2), np.uint16)

    def fill(b):
        r0, r1 = b * block, min(n_ids, (b + 1) * block)
        out[r0:r1] = _normal_bits(_rng(wl, _T_DOUT, 16 + b, seed), (r1 - r0, wl.N2))

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range((n_ids + block - 1) // block)))
    return out


def grad_out_rows(wl: Workload, n_rows: int, seed: int = 0) -> np.ndarray:
    """(n_rows, N2) bf16 bits ~N(0, 1): the nonzero rows of a sparse loss gradient."""
    return _normal_bits(_rng(wl, _T_DOUT, 1, seed), (n_rows, wl.N2))


def input_ids(wl: Workload, rows_per_image: Sequence[int], seed: int = 0,
              image_token_id: int = IMAGE_TOKEN_ID) -> np.ndarray:
    """Flattened (B*S,) int64 ids: each sequence holds n_images/B images as placeholder runs.

    ``rows_per_image[i]`` is how many placeholder tokens image i expands to; the caller
    computes it. Runs of one sequence keep image order; the text tokens around them are
    split into gaps by a seeded uniform composition.
    """
    per_seq = wl.n_images // wl.B
    assert per_seq * wl.B == wl.n_images and len(rows_per_image) == wl.n_images
    r = _rng(wl, _T_IDS, 0, seed)
    ids = r.integers(0, TEXT_VOCAB, size=(wl.B, wl.S), dtype=np.int64)
    for b in range(wl.B):
        runs = [int(x) for x in rows_per_image[b * per_seq:(b + 1) * per_seq]]
        free = wl.S - sum(runs)
        if free < 0:
            raise ValueError(f"sequence {b}: {sum(runs)} placeholders exceed S={wl.S}")
        cuts = np.sort(r.integers(0, free + 1, size=len(runs)))
        gaps = np.diff(np.concatenate([[0], cuts]))
        p = 0
        for g, n in zip(gaps, runs):
            p += int(g)
            ids[b, p:p + n] = image_token_id
            p += n
    return ids.reshape(-1)


def embed_table(wl: Workload, seed: int = 0) -> np.ndarray:
    """(TEXT_VOCAB, N2) bf16 bits used to prefill the text rows of the embedding buffer."""
    return _normal_bits(_rng(wl, _T_TABLE, 0, seed), (TEXT_VOCAB, wl.N2), 0.02)


BF16_NAN_SENTINEL = np.uint16(0x7FC1)


def prefill_embeds(wl: Workload, ids: np.ndarray, table: np.ndarray,
                   image_token_id: int = IMAGE_TOKEN_ID) -> np.ndarray:
    """Text rows gathered from ``table`` by id; placeholder rows set to a NaN sentinel."""
    out = np.empty((ids.shape[0], wl.N2), np.uint16)
    mask = ids == image_token_id
    out[~mask] = table[ids[~mask] % TEXT_VOCAB]
    out[mask] = BF16_NAN_SENTINEL
    return out
