"""fp64 oracle of the vision-to-language bridge (TEST INFRASTRUCTURE ONLY).

Plain numpy restatement of what the projector path computes. Each function
cites the passage it follows. Page names:

* "port DeepSeek-VL2" - mlxcel issue #533, sections "Projector
  (downsample_mlp_gelu)", "Tile-sequence assembly (tile_tag "2D")", "Processor"
  (step 7, placeholder expansion) and "Safetensors weight keys".
* "DeepSeek-V4-Flash-Vision-BF16" - WebBrain model card, first section
  (MoonViT PatchMerger, 2x2 merge, 4608 -> 4096, 40,119,040 parameters).
* "La voie visuelle" - DeepSeek-V4.1-Flash notes, sections "Le pixel-unshuffle
  3x3" and "Le calcul" (96 x 96 -> 32 x 32 = 1,024 tokens).
* "DeepSeek-VL Hybrid" - KerasFormers docs, processor table (576 tokens per
  image) and config table (image_token_id 100015).

Readings where the pages are silent (each also listed in the design notes):
LayerNorm is pre-merge, per patch over C, biased variance, eps 1e-5; zero pad is
applied after the LayerNorm; GELU is the exact erf form; the bf16 quantisation
points are Q1 (the merged A operand) and Q2 (the GELU output H); the final Y is
returned unrounded in fp64.

Nothing in this module touches a GPU or the CUDA library.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np
from scipy.special import erf as _erf


# ----------------------------------------------------------------- number formats
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns: the high half of an IEEE fp32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value, ties to even (returned as fp64).

    bf16 keeps 8 significant bits and fp32's exponent range. For |x| in
    [2^(e-1), 2^e) the spacing of bf16 values is 2^(e-8); below the smallest
    normal (2^-126) the spacing stays 2^-133. ``np.rint`` rounds half to even.
    Values beyond the bf16 range do not occur here (|x| << 3e38).
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                       # x = m * 2^e, m in [0.5, 1)
    e = np.maximum(e, -125)                  # subnormal bf16 spacing 2^-133
    q = np.ldexp(np.ones_like(x), e - 8)
    return np.rint(x / q) * q


# ----------------------------------------------------------------- counts
def merged_side(n: int, k: int) -> int:
    """Tokens along one side after a k x k merge: the side is zero-padded at the high
    end to the next multiple of k, then divided ("port DeepSeek-VL2", Projector step 1,
    and the output note h' = ceil(floor(image_size / patch_size) / ds))."""
    return -(-int(n) // int(k))


def tokens_untiled(h: int, w: int, k: int) -> int:
    """Merged tokens of one view: h' * w' ("port DeepSeek-VL2", Projector step 2)."""
    return merged_side(h, k) * merged_side(w, k)


def tokens_tiled(hp: int, wp: int, tw: int, th: int) -> int:
    """Placeholder tokens of a 2D-tiled image: h'(w'+1) + 1 + (th h')(tw w' + 1)
    ("port DeepSeek-VL2", Processor step 7)."""
    return hp * (wp + 1) + 1 + (th * hp) * (tw * wp + 1)


def image_rows(grid_hw: np.ndarray, k: int, spatial_crop: Optional[np.ndarray]) -> list:
    """Assembled rows of each image, views in order (global view first when tiled)."""
    if spatial_crop is None:
        return [tokens_untiled(h, w, k) for h, w in np.asarray(grid_hw)]
    rows, v = [], 0
    for tw, th in np.asarray(spatial_crop):
        h, w = grid_hw[v]
        rows.append(tokens_tiled(merged_side(h, k), merged_side(w, k), int(tw), int(th)))
        v += 1 + int(tw) * int(th)
    return rows


def projector_params(C: int, k: int, N1: int, N2: int, has_ln: bool, depth: int = 2) -> int:
    """Parameters of [LayerNorm(C)] + Linear(k*k*C -> N1) + (depth-2) x Linear(N1 -> N1)
    + Linear(N1 -> N2), with biases ("DeepSeek-V4-Flash-Vision-BF16", first section:
    2x2 merge, 4608 -> 4096; "port DeepSeek-VL2", Projector step 3 for depth > 2)."""
    n = (2 * C if has_ln else 0)
    n += k * k * C * N1 + N1
    n += (depth - 2) * (N1 * N1 + N1)
    n += N1 * N2 + N2
    return n


# ----------------------------------------------------------------- steps
def layernorm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """Per-row LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * gamma + beta,
    with the biased (1/C) variance. Applied per patch, before the merge."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: 0.5 x (1 + erf(x / sqrt 2))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def unshuffle(y: np.ndarray, k: int) -> np.ndarray:
    """Space-to-depth of one view ("port DeepSeek-VL2", Projector steps 1-2).

    ``y`` is (h, w, C). It is zero-padded at the high end of both axes to multiples
    of k, cut into non-overlapping k x k blocks scanned row-major, and each block
    becomes one vector ordered channel-outermost: index c*k*k + dy*k + dx.
    Returns (h'*w', k*k*C), tokens row-major over (h', w').
    """
    h, w, C = y.shape
    hp, wp = merged_side(h, k), merged_side(w, k)
    pad = np.zeros((hp * k, wp * k, C), dtype=y.dtype)
    pad[:h, :w] = y
    blocks = pad.reshape(hp, k, wp, k, C)            # (i, dy, j, dx, c)
    return blocks.transpose(0, 2, 4, 1, 3).reshape(hp * wp, C * k * k)


def fold(a: np.ndarray, hp: int, wp: int, k: int, C: int) -> np.ndarray:
    """Inverse of ``unshuffle`` before cropping: (h'*w', C*k*k) -> (k*h', k*w', C)."""
    blocks = a.reshape(hp, wp, C, k, k).transpose(0, 3, 1, 4, 2)   # (i, dy, j, dx, c)
    return blocks.reshape(hp * k, wp * k, C)


def hidden(a: np.ndarray, W1: np.ndarray, b1: np.ndarray, quantise_hidden: bool = True) -> np.ndarray:
    """First Linear and GELU: GELU(a W1^T + b1), W1 stored (out, in) and used as-is
    ("port DeepSeek-VL2", Projector step 3; Safetensors weight keys: Linear weights
    are consumed as stored). Rounded to bf16 (Q2) unless disabled."""
    g = gelu(a @ W1.T + b1)
    return round_bf16(g) if quantise_hidden else g


def mlp(a: np.ndarray, W1: np.ndarray, b1: np.ndarray, W2: np.ndarray, b2: np.ndarray,
        quantise_hidden: bool = True, mids: Sequence[tuple] = ()) -> np.ndarray:
    """Linear -> GELU -> [Linear -> GELU] x len(mids) -> Linear ("port DeepSeek-VL2",
    Projector step 3: with depth > 2 the extra GELU + Linear pairs sit in the middle).
    Every hidden activation is rounded to bf16 (Q2) unless disabled."""
    h = hidden(a, W1, b1, quantise_hidden)
    for Wm, bm in mids:
        h = hidden(h, Wm, bm, quantise_hidden)
    return h @ W2.T + b2


def merge_view(feat: np.ndarray, h: int, w: int, k: int, ln: Optional[tuple]) -> np.ndarray:
    """One view's merged A operand: optional pre-merge LayerNorm per patch, bf16
    rounding (Q1), then ``unshuffle``. ``feat`` is (h*w, C) fp64, rows row-major over
    (h, w) ("port DeepSeek-VL2", Vision tower: flatten row-major over (gh, gw))."""
    x = np.asarray(feat, np.float64)
    if ln is not None:
        gamma, beta, eps = ln
        x = layernorm(x, gamma, beta, eps)
    x = round_bf16(x)
    return unshuffle(x.reshape(h, w, -1), k)


def assemble_2d(views: np.ndarray, hp: int, wp: int, tw: int, th: int,
                newline: np.ndarray, sep: np.ndarray, global_view_pos: str = "head") -> np.ndarray:
    """Tile-sequence assembly for tile tag "2D" ("port DeepSeek-VL2", Tile-sequence
    assembly). ``views`` is (1 + tw*th, h'*w', D), view 0 the global view, then the
    local tiles row-major. Returns the assembled (rows, D) block."""
    D = views.shape[-1]
    g = views[0].reshape(hp, wp, D)
    nl = np.broadcast_to(newline.reshape(1, 1, D), (hp, 1, D))
    g = np.concatenate([g, nl], axis=1).reshape(hp * (wp + 1), D)
    loc = views[1:].reshape(th, tw, hp, wp, D).transpose(0, 2, 1, 3, 4).reshape(th * hp, tw * wp, D)
    nl = np.broadcast_to(newline.reshape(1, 1, D), (th * hp, 1, D))
    loc = np.concatenate([loc, nl], axis=1).reshape((th * hp) * (tw * wp + 1), D)
    s = sep.reshape(1, D)
    if global_view_pos == "head":
        return np.concatenate([g, s, loc], axis=0)
    if global_view_pos == "tail":
        return np.concatenate([loc, s, g], axis=0)
    raise ValueError(global_view_pos)


def placeholder_positions(ids: np.ndarray, image_token_id: int) -> np.ndarray:
    """Flat indices holding the image placeholder, in order ("port DeepSeek-VL2",
    end of Tile-sequence assembly: the images_seq_mask positions)."""
    return np.flatnonzero(np.asarray(ids) == image_token_id)


def scatter(embeds: np.ndarray, ids: np.ndarray, image_token_id: int, rows: np.ndarray) -> np.ndarray:
    """Overwrite the placeholder rows of ``embeds`` with ``rows`` in order; every other
    row is left as it was. The placeholder count must equal the row count."""
    pos = placeholder_positions(ids, image_token_id)
    if len(pos) != len(rows):
        raise ValueError(f"{len(pos)} placeholders for {len(rows)} rows")
    out = np.array(embeds, dtype=np.float64, copy=True)
    out[pos] = rows
    return out


# ----------------------------------------------------------------- whole path
def project_image(feats: Sequence[np.ndarray], hw: Sequence[tuple], k: int, params: dict,
                  crop: Optional[tuple], ln_eps: float = 1e-5,
                  quantise: bool = True, global_view_pos: str = "head") -> np.ndarray:
    """Assembled rows of one image. ``feats[v]`` is view v's (h*w, C) features as fp64.
    ``params`` holds fp64 W1, b1, W2, b2 and optionally gamma, beta, newline, sep."""
    ln = None
    if params.get("gamma") is not None:
        ln = (params["gamma"], params["beta"], ln_eps)
    outs = []
    for f, (h, w) in zip(feats, hw):
        if quantise:
            a = merge_view(f, h, w, k, ln)
        else:
            x = np.asarray(f, np.float64)
            if ln is not None:
                x = layernorm(x, *ln)
            a = unshuffle(x.reshape(h, w, -1), k)
        outs.append(mlp(a, params["W1"], params["b1"], params["W2"], params["b2"], quantise,
                        params.get("mid") or ()))
    if crop is None:
        assert len(outs) == 1
        return outs[0]
    tw, th = crop
    hp, wp = merged_side(hw[0][0], k), merged_side(hw[0][1], k)
    return assemble_2d(np.stack(outs), hp, wp, tw, th, params["newline"], params["sep"], global_view_pos)


def forward(features: np.ndarray, grid_hw: np.ndarray, spatial_crop: Optional[np.ndarray],
            k: int, params: dict, ids: np.ndarray, image_token_id: int, embeds: np.ndarray,
            ln_eps: float = 1e-5, feat_is_bf16_bits: bool = True, quantise: bool = True,
            global_view_pos: str = "head") -> np.ndarray:
    """The whole bridge: per image, merge + MLP (+ assembly), then scatter into ``embeds``
    (fp64 array (n_ids, D)). Returns the new fp64 embedding buffer."""
    grid_hw = np.asarray(grid_hw)
    f64 = bf16_bits_to_f64(features) if feat_is_bf16_bits else np.asarray(features, np.float64)
    offs = np.concatenate([[0], np.cumsum(grid_hw[:, 0].astype(np.int64) * grid_hw[:, 1])])
    if spatial_crop is None:
        groups = [([v], None) for v in range(len(grid_hw))]
    else:
        groups, v = [], 0
        for tw, th in np.asarray(spatial_crop):
            n = 1 + int(tw) * int(th)
            groups.append((list(range(v, v + n)), (int(tw), int(th))))
            v += n
    rows = []
    for views, crop in groups:
        feats = [f64[offs[v]:offs[v + 1]] for v in views]
        hw = [(int(grid_hw[v, 0]), int(grid_hw[v, 1])) for v in views]
        rows.append(project_image(feats, hw, k, params, crop, ln_eps, quantise, global_view_pos))
    all_rows = np.concatenate(rows, axis=0) if rows else np.zeros((0, embeds.shape[1]))
    return scatter(embeds, ids, image_token_id, all_rows)


def params_f64(w: dict) -> dict:
    """fp64 copies of the generator's parameter dict (bf16 bit patterns -> exact values)."""
    out = {
        "W1": bf16_bits_to_f64(w["W1"]),
        "W2": bf16_bits_to_f64(w["W2"]),
        "b1": np.asarray(w["b1"], np.float64),
        "b2": np.asarray(w["b2"], np.float64),
    }
    for key in ("gamma", "beta"):
        out[key] = None if w.get(key) is None else np.asarray(w[key], np.float64)
    for key in ("newline", "sep"):
        out[key] = None if w.get(key) is None else bf16_bits_to_f64(w[key])
    out["mid"] = [(bf16_bits_to_f64(Wm), np.asarray(bm, np.float64)) for Wm, bm in (w.get("mid") or ())]
    return out
