"""Python binding of ``libvlproj.so``, the B200 vision-to-language projector.

Argument marshalling only: every step of the projector runs in the library's
CUDA kernels. Tensors are torch tensors (device memory and streams are the only
things torch provides here); their raw pointers are handed to the C ABI declared
in ``include/vlproj.h``. Importing this module without the built library raises
immediately; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvlproj.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TOKEN_COUNT, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
FEAT_BF16, FEAT_F32 = 0, 1
TILE_NONE, TILE_2D, TILE_1D = 0, 1, 2
GLOBAL_HEAD, GLOBAL_TAIL = 0, 1
ORDER_CHANNEL_OUTER, ORDER_POSITION_OUTER = 0, 1

EXPORTED = ("vlproj_create", "vlproj_forward", "vlproj_hidden", "vlproj_status", "vlproj_destroy",
            "vlproj_image_rows", "vlproj_set_wait_limit", "vlproj_strerror", "vlproj_version",
            "vlproj_profile_enable", "vlproj_profile_read", "vlproj_launch_count", "vlproj_set_gather_mode",
            "vlproj_set_tile_pairs", "vlproj_placeholder_index_noalloc", "vlproj_forward_ex",
            "vlproj_plan_tiles", "vlproj_backward", "vlproj_project_host", "vlproj_profile_stages")
NOALLOC_MAX_IDS = 64 * 1024 * 1024
GATHER_IM2COL, GATHER_CPASYNC, GATHER_AUTO, GATHER_BOX = 0, 1, 2, 3
NUM_STAGES = 15
STAGES = ("index", "geometry", "layernorm", "gemm1", "gemm2", "special_rows",
          "bwd_index", "bwd_merge", "bwd_gemm1", "bwd_dy", "bwd_dh", "bwd_dw2", "bwd_dw1", "bwd_da", "bwd_tail")
GRAD_NAMES = ("W1", "b1", "W2", "b2", "gamma", "beta", "newline", "sep", "features")


class VlprojError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


class ForwardArgs(ctypes.Structure):
    """Mirror of ``vlproj_forward_args``."""
    _fields_ = [
        ("features", ctypes.c_void_p), ("grid_hw", ctypes.c_void_p), ("spatial_crop", ctypes.c_void_p),
        ("n_images", ctypes.c_int32), ("input_ids", ctypes.c_void_p), ("n_ids", ctypes.c_int64),
        ("image_token_id", ctypes.c_int64), ("newline", ctypes.c_void_p), ("sep", ctypes.c_void_p),
        ("out_embeds", ctypes.c_void_p), ("embed_table", ctypes.c_void_p), ("vocab", ctypes.c_int64),
        ("rows_out", ctypes.c_void_p), ("rows_out_cap", ctypes.c_int64),
    ]


class BackwardArgs(ctypes.Structure):
    """Mirror of ``vlproj_backward_args``."""
    _fields_ = [
        ("features", ctypes.c_void_p), ("grid_hw", ctypes.c_void_p), ("spatial_crop", ctypes.c_void_p),
        ("n_images", ctypes.c_int32), ("input_ids", ctypes.c_void_p), ("n_ids", ctypes.c_int64),
        ("image_token_id", ctypes.c_int64), ("d_out", ctypes.c_void_p),
    ] + [("d_" + n, ctypes.c_void_p) for n in ("W1", "b1", "W2", "b2", "gamma", "beta", "newline", "sep",
                                                  "features")] + [("d_W_mid", ctypes.c_void_p),
                                                                  ("d_b_mid", ctypes.c_void_p)]


class HostArgs(ctypes.Structure):
    """Mirror of ``vlproj_host_args``."""
    _fields_ = [
        ("features", ctypes.c_void_p), ("grid_hw", ctypes.c_void_p), ("spatial_crop", ctypes.c_void_p),
        ("n_images", ctypes.c_int32), ("newline", ctypes.c_void_p), ("sep", ctypes.c_void_p),
        ("rows_out", ctypes.c_void_p), ("rows_out_cap", ctypes.c_int64), ("chunks", ctypes.c_int32),
    ]


class Config(ctypes.Structure):
    """Mirror of ``vlproj_config``."""
    _fields_ = [
        ("k", ctypes.c_int32), ("C", ctypes.c_int32), ("N1", ctypes.c_int32), ("N2", ctypes.c_int32),
        ("depth", ctypes.c_int32), ("has_ln", ctypes.c_int32), ("ln_eps", ctypes.c_float),
        ("feat_dtype", ctypes.c_int32), ("k_order", ctypes.c_int32), ("tile_tag", ctypes.c_int32),
        ("global_view_pos", ctypes.c_int32), ("token_pooling", ctypes.c_int32),
        ("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p),
        ("ln_gamma", ctypes.c_void_p), ("ln_beta", ctypes.c_void_p),
        ("W_mid", ctypes.c_void_p), ("b_mid", ctypes.c_void_p),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m vision_language_projector_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
    lib.vlproj_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(P)]
    lib.vlproj_create.restype = ctypes.c_int
    lib.vlproj_forward.argtypes = [P, P, P, P, I32, P, I64, I64, P, P, P, P]
    lib.vlproj_forward.restype = ctypes.c_int
    lib.vlproj_hidden.argtypes = [P, P, P, I32, P, P]
    lib.vlproj_hidden.restype = ctypes.c_int
    lib.vlproj_status.argtypes = [P, P]
    lib.vlproj_status.restype = ctypes.c_int
    lib.vlproj_destroy.argtypes = [P]
    lib.vlproj_destroy.restype = None
    lib.vlproj_image_rows.argtypes = [ctypes.POINTER(Config), P, P, I32, P]
    lib.vlproj_image_rows.restype = I64
    lib.vlproj_set_wait_limit.argtypes = [P, U64]
    lib.vlproj_set_wait_limit.restype = ctypes.c_int
    lib.vlproj_strerror.argtypes = [ctypes.c_int]
    lib.vlproj_strerror.restype = ctypes.c_char_p
    lib.vlproj_version.argtypes = []
    lib.vlproj_version.restype = ctypes.c_char_p
    lib.vlproj_profile_enable.argtypes = [P, ctypes.c_int]
    lib.vlproj_profile_enable.restype = ctypes.c_int
    lib.vlproj_profile_stages.argtypes = [P, ctypes.c_uint32]
    lib.vlproj_profile_stages.restype = ctypes.c_int
    lib.vlproj_profile_read.argtypes = [P, P, ctypes.c_int]
    lib.vlproj_profile_read.restype = ctypes.c_int
    lib.vlproj_launch_count.argtypes = [P]
    lib.vlproj_launch_count.restype = I64
    lib.vlproj_set_gather_mode.argtypes = [P, ctypes.c_int]
    lib.vlproj_set_gather_mode.restype = ctypes.c_int
    lib.vlproj_set_tile_pairs.argtypes = [P, ctypes.c_int]
    lib.vlproj_set_tile_pairs.restype = ctypes.c_int
    lib.vlproj_plan_tiles.argtypes = [P, I32, P, I32, I32, I32, I32, P, P]
    lib.vlproj_plan_tiles.restype = I64
    lib.vlproj_forward_ex.argtypes = [P, ctypes.POINTER(ForwardArgs), P]
    lib.vlproj_forward_ex.restype = ctypes.c_int
    lib.vlproj_project_host.argtypes = [P, ctypes.POINTER(HostArgs), P]
    lib.vlproj_project_host.restype = ctypes.c_int
    lib.vlproj_backward.argtypes = [P, ctypes.POINTER(BackwardArgs), P]
    lib.vlproj_backward.restype = ctypes.c_int
    lib.vlproj_placeholder_index_noalloc.argtypes = [P, I64, I64, P, I64, P, P]
    lib.vlproj_placeholder_index_noalloc.restype = ctypes.c_int
    return lib


_lib = _load()


def strerror(code: int) -> str:
    return _lib.vlproj_strerror(int(code)).decode()


def version() -> str:
    return _lib.vlproj_version().decode()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _host_i32(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def make_config(k: int, C: int, N1: int, N2: int, *, has_ln: bool = False, ln_eps: float = 1e-5,
                feat_dtype: int = FEAT_BF16, tile_tag: int = TILE_NONE, global_view_pos: int = GLOBAL_HEAD,
                k_order: int = ORDER_CHANNEL_OUTER, depth: int = 2, token_pooling: int = 0,
                W1=None, b1=None, W2=None, b2=None, ln_gamma=None, ln_beta=None, W_mid=None, b_mid=None) -> Config:
    cfg = Config(k, C, N1, N2, depth, int(has_ln), ln_eps, feat_dtype, k_order, tile_tag, global_view_pos,
                 token_pooling, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(ln_gamma), _ptr(ln_beta), None, None)
    # host arrays of device pointers for the middle layers; kept alive on the Config
    if W_mid is not None:
        cfg._w_mid = (ctypes.c_void_p * len(W_mid))(*[_ptr(t) for t in W_mid])
        cfg.W_mid = ctypes.cast(cfg._w_mid, ctypes.c_void_p)
    if b_mid is not None:
        cfg._b_mid = (ctypes.c_void_p * len(b_mid))(*[_ptr(t) for t in b_mid])
        cfg.b_mid = ctypes.cast(cfg._b_mid, ctypes.c_void_p)
    return cfg


def image_rows(cfg: Config, grid_hw, spatial_crop=None, n_images: Optional[int] = None) -> np.ndarray:
    """Closed-form placeholder count of every image (host only, no GPU needed)."""
    g = _host_i32(grid_hw)
    c = _host_i32(spatial_crop)
    if n_images is None:
        n_images = len(c) if c is not None else (0 if g is None else len(g))
    out = np.zeros(max(n_images, 1), np.int64)
    r = _lib.vlproj_image_rows(ctypes.byref(cfg), _ptr(g), _ptr(c), n_images, out.ctypes.data)
    if r < 0:
        raise VlprojError(int(r), "vlproj_image_rows")
    return out[:n_images]


def placeholder_index_noalloc(input_ids, image_token_id: int, positions, count, stream=None,
                              n_ids: Optional[int] = None, max_positions: Optional[int] = None) -> int:
    """Placeholder positions and count without any allocation (see vlproj.h): for callers
    that must not allocate device memory at the call. Returns the status code."""
    n = int(input_ids.numel()) if n_ids is None else int(n_ids)
    mp = int(positions.numel()) if max_positions is None else int(max_positions)
    return _lib.vlproj_placeholder_index_noalloc(_ptr(input_ids), n, int(image_token_id), _ptr(positions), mp,
                                                 _ptr(count), _stream_ptr(stream))


def plan_tiles(image_wh, candidates, image_size: int, patch_size: int, downsample: int):
    """Processor tiling (host only): ((n, 2) int32 (tw, th), (n,) int64 placeholder counts, views)."""
    wh = _host_i32(image_wh).reshape(-1, 2)
    cand = _host_i32(candidates).reshape(-1, 2)
    crop = np.zeros((max(len(wh), 1), 2), np.int32)
    rows = np.zeros(max(len(wh), 1), np.int64)
    v = _lib.vlproj_plan_tiles(wh.ctypes.data, len(wh), cand.ctypes.data, len(cand), image_size, patch_size,
                               downsample, crop.ctypes.data, rows.ctypes.data)
    if v < 0:
        raise VlprojError(int(v), "vlproj_plan_tiles")
    return crop[:len(wh)], rows[:len(wh)], int(v)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Projector:
    """Owns a ``vlproj_handle``. Weight tensors must be CUDA tensors on the current device:
    W1 bf16 (N1, k*k*C), W2 bf16 (N2, N1), biases / LayerNorm parameters fp32."""

    def __init__(self, k: int, C: int, N1: int, N2: int, W1, W2, b1=None, b2=None, *, has_ln: bool = False,
                 ln_gamma=None, ln_beta=None, ln_eps: float = 1e-5, feat_dtype: int = FEAT_BF16,
                 tile_tag: int = TILE_NONE, global_view_pos: int = GLOBAL_HEAD, k_order: int = ORDER_CHANNEL_OUTER,
                 depth: int = 2, token_pooling: int = 0, W_mid=None, b_mid=None):
        self.cfg = make_config(k, C, N1, N2, has_ln=has_ln, ln_eps=ln_eps, feat_dtype=feat_dtype,
                               tile_tag=tile_tag, global_view_pos=global_view_pos, k_order=k_order, depth=depth,
                               token_pooling=token_pooling, W1=W1, b1=b1, W2=W2, b2=b2, ln_gamma=ln_gamma,
                               ln_beta=ln_beta, W_mid=W_mid, b_mid=b_mid)
        h = ctypes.c_void_p()
        rc = _lib.vlproj_create(ctypes.byref(self.cfg), ctypes.byref(h))
        if rc != OK:
            raise VlprojError(rc, "vlproj_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            _lib.vlproj_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, features, grid_hw, spatial_crop, input_ids, image_token_id: int, out_embeds,
                newline=None, sep=None, stream=None, n_images: Optional[int] = None, check: bool = True) -> int:
        """Enqueue the bridge; raise on a host-detected error. Returns the status code."""
        g = _host_i32(grid_hw)
        c = _host_i32(spatial_crop)
        if n_images is None:
            n_images = len(c) if c is not None else (0 if g is None else len(g))
        n_ids = 0 if input_ids is None else int(input_ids.numel())
        rc = _lib.vlproj_forward(self._h, _ptr(features), _ptr(g), _ptr(c), n_images, _ptr(input_ids), n_ids,
                                 int(image_token_id), _ptr(newline), _ptr(sep), _ptr(out_embeds),
                                 _stream_ptr(stream))
        if check and rc != OK:
            raise VlprojError(rc, "vlproj_forward")
        return rc

    def forward_ex(self, features, grid_hw, spatial_crop, input_ids, image_token_id: int, out_embeds,
                   newline=None, sep=None, embed_table=None, rows_out=None, stream=None,
                   n_images: Optional[int] = None, check: bool = True) -> int:
        """vlproj_forward_ex: forward plus the optional token-embedding lookup (embed_table,
        (vocab, N2) bf16) and a compact copy of the assembled rows (rows_out, (>= R, N2))."""
        g = _host_i32(grid_hw)
        c = _host_i32(spatial_crop)
        if n_images is None:
            n_images = len(c) if c is not None else (0 if g is None else len(g))
        a = ForwardArgs(_ptr(features), _ptr(g), _ptr(c), n_images, _ptr(input_ids),
                        0 if input_ids is None else int(input_ids.numel()), int(image_token_id), _ptr(newline),
                        _ptr(sep), _ptr(out_embeds), _ptr(embed_table),
                        0 if embed_table is None else int(embed_table.shape[0]), _ptr(rows_out),
                        0 if rows_out is None else int(rows_out.shape[0]))
        rc = _lib.vlproj_forward_ex(self._h, ctypes.byref(a), _stream_ptr(stream))
        if check and rc != OK:
            raise VlprojError(rc, "vlproj_forward_ex")
        return rc

    def backward(self, features, grid_hw, spatial_crop, input_ids, image_token_id: int, d_out, grads: dict,
                 stream=None, n_images: Optional[int] = None, check: bool = True) -> int:
        """vlproj_backward: fp32 gradients into the tensors of ``grads`` (keys from
        GRAD_NAMES, plus "W_mid" / "b_mid": lists of depth - 2 tensors or None for the
        middle layers; a missing key is not computed) for the loss gradient ``d_out``
        ((n_ids, N2) bf16) of the batch given by the other arguments."""
        unknown = set(grads) - set(GRAD_NAMES) - {"W_mid", "b_mid"}
        if unknown:
            raise ValueError(f"unknown gradient names {sorted(unknown)}")
        mids = {}
        for key in ("W_mid", "b_mid"):
            if grads.get(key) is not None:
                arr = (ctypes.c_void_p * len(grads[key]))(*[_ptr(t) for t in grads[key]])
                mids[key] = arr
        g = _host_i32(grid_hw)
        c = _host_i32(spatial_crop)
        if n_images is None:
            n_images = len(c) if c is not None else (0 if g is None else len(g))
        a = BackwardArgs(_ptr(features), _ptr(g), _ptr(c), n_images, _ptr(input_ids),
                         0 if input_ids is None else int(input_ids.numel()), int(image_token_id), _ptr(d_out),
                         *[_ptr(grads.get(n)) for n in GRAD_NAMES],
                         *[ctypes.cast(mids[k], ctypes.c_void_p) if k in mids else None for k in ("W_mid", "b_mid")])
        rc = _lib.vlproj_backward(self._h, ctypes.byref(a), _stream_ptr(stream))
        if check and rc != OK:
            raise VlprojError(rc, "vlproj_backward")
        return rc

    def project_host(self, features, grid_hw, spatial_crop, rows_out, newline=None, sep=None, chunks: int = 0,
                     stream=None, n_images: Optional[int] = None, check: bool = True) -> int:
        """vlproj_project_host: features in HOST memory (page-locked for overlap), the
        assembled rows of every image written to ``rows_out`` (HOST, (>= R, N2) bf16),
        copies pipelined against the projection. Completes with ``stream``."""
        g = _host_i32(grid_hw)
        c = _host_i32(spatial_crop)
        if n_images is None:
            n_images = len(c) if c is not None else (0 if g is None else len(g))
        a = HostArgs(_ptr(features), _ptr(g), _ptr(c), n_images, _ptr(newline), _ptr(sep), _ptr(rows_out),
                     0 if rows_out is None else int(rows_out.shape[0]), int(chunks))
        rc = _lib.vlproj_project_host(self._h, ctypes.byref(a), _stream_ptr(stream))
        if check and rc != OK:
            raise VlprojError(rc, "vlproj_project_host")
        return rc

    def hidden(self, features, grid_hw, hidden, stream=None) -> None:
        g = _host_i32(grid_hw)
        rc = _lib.vlproj_hidden(self._h, _ptr(features), _ptr(g), 0 if g is None else len(g), _ptr(hidden),
                                _stream_ptr(stream))
        if rc != OK:
            raise VlprojError(rc, "vlproj_hidden")

    def status(self, stream=None) -> int:
        """Synchronise the stream and return (and clear) the latched device status."""
        return _lib.vlproj_status(self._h, _stream_ptr(stream))

    def profile(self, enable: bool = True) -> None:
        rc = _lib.vlproj_profile_enable(self._h, int(enable))
        if rc != OK:
            raise VlprojError(rc, "vlproj_profile_enable")

    def profile_stages(self, names=None) -> None:
        """Time only the named stages (STAGES names; None = all) while profiling."""
        mask = 0xFFFFFFFF if names is None else sum(1 << STAGES.index(n) for n in names)
        rc = _lib.vlproj_profile_stages(self._h, mask)
        if rc != OK:
            raise VlprojError(rc, "vlproj_profile_stages")

    def stage_ms(self) -> dict:
        """Per-stage device milliseconds of the most recent profiled call (synchronises)."""
        buf = (ctypes.c_float * NUM_STAGES)()
        rc = _lib.vlproj_profile_read(self._h, ctypes.cast(buf, ctypes.c_void_p), NUM_STAGES)
        if rc < 0:
            raise VlprojError(rc, "vlproj_profile_read")
        return {name: float(buf[i]) for i, name in enumerate(STAGES)}

    def launch_count(self) -> int:
        return int(_lib.vlproj_launch_count(self._h))

    def set_gather_mode(self, mode: int) -> None:
        rc = _lib.vlproj_set_gather_mode(self._h, int(mode))
        if rc != OK:
            raise VlprojError(rc, "vlproj_set_gather_mode")

    def set_tile_pairs(self, enable: bool) -> None:
        rc = _lib.vlproj_set_tile_pairs(self._h, int(enable))
        if rc != OK:
            raise VlprojError(rc, "vlproj_set_tile_pairs")

    def set_wait_limit(self, ns: int) -> None:
        rc = _lib.vlproj_set_wait_limit(self._h, int(ns))
        if rc != OK:
            raise VlprojError(rc, "vlproj_set_wait_limit")
