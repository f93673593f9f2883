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
            "vlproj_plan_tiles", "vlproj_backward", "vlproj_project_host", "vlproj_profile_stages",
            "vlproj_set_raster_budget", "vlproj_set_tile_order")
NOALLOC_MAX_IDS = 64 * 1024 * 1024
TILE_ORDER_STATIC, TILE_ORDER_AUTO, TILE_ORDER_DYNAMIC = 0, 1, 2
GATHER_IM2COL, GATHER_CPASYNC, GATHER_AUTO, GATHER_BOX, GATHER_THREADS, GATHER_FUSED, GATHER_MERGED = 0, 1, 2, 3, 4, 5, 6
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
    lib.vlproj_set_raster_budget.argtypes = [P, I64]
    lib.vlproj_set_raster_budget.restype = ctypes.c_int
    lib.vlproj_set_tile_order.argtypes = [P, I32]
    lib.vlproj_set_tile_order.restype = ctypes.c_int
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


def _arg_error(name: str, why: str) -> "VlprojError":
    return VlprojError(ERR_INVALID_ARG, f"{name}: {why}")


def _dev(t, name: str, itemsize: int, numel: int = 0) -> Optional[int]:
    """Device pointer of ``t`` after the checks only the binding can make (the C ABI gets
    bare pointers): a contiguous CUDA tensor whose elements are ``itemsize`` bytes, with at
    least ``numel`` of them. None and integer addresses pass through unchecked."""
    if t is None or isinstance(t, int):
        return t
    if isinstance(t, np.ndarray) or not hasattr(t, "is_cuda"):
        raise _arg_error(name, f"a CUDA tensor is required, got {type(t).__name__}")
    if not t.is_cuda:
        raise _arg_error(name, f"a CUDA tensor is required, got one on {t.device}")
    if not t.is_contiguous():
        raise _arg_error(name, "the tensor must be contiguous")
    if t.element_size() != itemsize:
        raise _arg_error(name, f"{t.dtype} has {t.element_size()}-byte elements, {itemsize} expected")
    if t.numel() < numel:
        raise _arg_error(name, f"{t.numel()} elements, at least {numel} needed")
    return t.data_ptr()


def _host(t, name: str, itemsize: int, numel: int = 0) -> Optional[int]:
    """Host address of ``t`` (a CPU tensor, page-locked for overlapped copies, or a numpy
    array) after the same checks."""
    if t is None or isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        if not t.flags["C_CONTIGUOUS"]:
            raise _arg_error(name, "the array must be C-contiguous")
        size, n, addr = t.itemsize, t.size, t.ctypes.data
    elif hasattr(t, "is_cuda"):
        if t.is_cuda:
            raise _arg_error(name, "host memory is required, got a CUDA tensor")
        if not t.is_contiguous():
            raise _arg_error(name, "the tensor must be contiguous")
        size, n, addr = t.element_size(), t.numel(), t.data_ptr()
    else:
        raise _arg_error(name, f"a host tensor or array is required, got {type(t).__name__}")
    if size != itemsize:
        raise _arg_error(name, f"{size}-byte elements, {itemsize} expected")
    if n < numel:
        raise _arg_error(name, f"{n} elements, at least {numel} needed")
    return addr


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
    that must not allocate device memory at the call. Returns the status code.

    Tensors are checked like every other entry point's (CUDA, contiguous, element size,
    enough elements for ``n_ids`` / ``max_positions``); integer addresses pass through
    unchecked, for callers that manage raw device memory themselves."""
    n = (0 if isinstance(input_ids, int) else int(input_ids.numel())) if n_ids is None else int(n_ids)
    mp = (0 if isinstance(positions, int) else int(positions.numel())) if max_positions is None else int(max_positions)
    if n < 0 or mp < 0:
        raise _arg_error("n_ids" if n < 0 else "max_positions", "must not be negative")
    # over the library's limit: the C ABI rejects it before touching any buffer
    pi = _ptr(input_ids) if n > NOALLOC_MAX_IDS else _dev(input_ids, "input_ids", 8, n)
    pp = _dev(positions, "positions", 4, mp)
    pc = _dev(count, "count", 8, 1)
    return _lib.vlproj_placeholder_index_noalloc(pi, n, int(image_token_id), pp, mp, pc, _stream_ptr(stream))


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

    # ---- argument checks the C ABI cannot make (it receives bare pointers)
    def _feat_size(self) -> int:
        return 4 if self.cfg.feat_dtype == FEAT_F32 else 2

    def _views(self, g, c, n_images: int) -> int:
        """grid_hw rows the library reads for n_images images; host arrays that are too
        short are rejected here (the library cannot see their length)."""
        if g is None or n_images <= 0:
            return 0
        nv = n_images
        if self.cfg.tile_tag == TILE_2D and c is not None:
            c2 = c.reshape(-1, 2)
            if len(c2) < n_images:
                raise _arg_error("spatial_crop", f"{len(c2)} rows for {n_images} images")
            nv = int(sum(1 + max(int(c2[i, 0]), 0) * max(int(c2[i, 1]), 0) for i in range(n_images)))
        rows = len(g.reshape(-1, 2))
        if rows < nv:
            raise _arg_error("grid_hw", f"{rows} rows, {nv} views")
        return nv

    def _extent(self, g, nv: int):
        """(patches, merged tokens) of the first nv views."""
        if g is None or nv <= 0:
            return 0, 0
        hw = np.maximum(g.reshape(-1, 2)[:nv].astype(np.int64), 0)
        k = self.cfg.k
        return int((hw[:, 0] * hw[:, 1]).sum()), int((((hw[:, 0] + k - 1) // k) * ((hw[:, 1] + k - 1) // k)).sum())

    @staticmethod
    def _fail(e: "VlprojError", check: bool) -> int:
        if check:
            raise e
        return e.code

    def forward(self, features, grid_hw, spatial_crop, input_ids, image_token_id: int, out_embeds,
                newline=None, sep=None, stream=None, n_images: Optional[int] = None, check: bool = True) -> int:
        """Enqueue the bridge; raise on a host-detected error. Returns the status code."""
        g = _host_i32(grid_hw)
        c = _host_i32(spatial_crop)
        if n_images is None:
            n_images = len(c) if c is not None else (0 if g is None else len(g))
        n_ids = 0 if input_ids is None else int(input_ids.numel())
        N2 = self.cfg.N2
        try:
            P, _ = self._extent(g, self._views(g, c, n_images))
            pf = _dev(features, "features", self._feat_size(), P * self.cfg.C)
            pi = _dev(input_ids, "input_ids", 8)
            pn, ps = _dev(newline, "newline", 2, N2), _dev(sep, "sep", 2, N2)
            po = _dev(out_embeds, "out_embeds", 2, n_ids * N2)
        except VlprojError as e:
            return self._fail(e, check)
        rc = _lib.vlproj_forward(self._h, pf, _ptr(g), _ptr(c), n_images, pi, n_ids, int(image_token_id), pn, ps,
                                 po, _stream_ptr(stream))
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
        n_ids = 0 if input_ids is None else int(input_ids.numel())
        vocab = 0 if embed_table is None else int(embed_table.shape[0])
        n_rows = 0 if rows_out is None else int(rows_out.shape[0])
        N2 = self.cfg.N2
        try:
            P, _ = self._extent(g, self._views(g, c, n_images))
            a = ForwardArgs(_dev(features, "features", self._feat_size(), P * self.cfg.C), _ptr(g), _ptr(c),
                            n_images, _dev(input_ids, "input_ids", 8), n_ids, int(image_token_id),
                            _dev(newline, "newline", 2, N2), _dev(sep, "sep", 2, N2),
                            _dev(out_embeds, "out_embeds", 2, n_ids * N2),
                            _dev(embed_table, "embed_table", 2, vocab * N2), vocab,
                            _dev(rows_out, "rows_out", 2, n_rows * N2), n_rows)
        except VlprojError as e:
            return self._fail(e, check)
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
        g = _host_i32(grid_hw)
        c = _host_i32(spatial_crop)
        if n_images is None:
            n_images = len(c) if c is not None else (0 if g is None else len(g))
        n_ids = 0 if input_ids is None else int(input_ids.numel())
        cfg = self.cfg
        K1 = cfg.k * cfg.k * cfg.C
        try:
            P, _ = self._extent(g, self._views(g, c, n_images))
            need = {"W1": cfg.N1 * K1, "b1": cfg.N1, "W2": cfg.N2 * cfg.N1, "b2": cfg.N2, "gamma": cfg.C,
                    "beta": cfg.C, "newline": cfg.N2, "sep": cfg.N2, "features": P * cfg.C}
            grad_ptrs = [_dev(grads.get(n), f"grads[{n!r}]", 4, need[n]) for n in GRAD_NAMES]
            mids = {}
            for key, numel in (("W_mid", cfg.N1 * cfg.N1), ("b_mid", cfg.N1)):
                if grads.get(key) is not None:
                    if len(grads[key]) != cfg.depth - 2:
                        raise _arg_error(f"grads[{key!r}]", f"{len(grads[key])} tensors, depth - 2 = "
                                                            f"{cfg.depth - 2} expected")
                    mids[key] = (ctypes.c_void_p * len(grads[key]))(
                        *[_dev(t, f"grads[{key!r}][{i}]", 4, numel) for i, t in enumerate(grads[key])])
            a = BackwardArgs(_dev(features, "features", self._feat_size(), P * cfg.C), _ptr(g), _ptr(c), n_images,
                             _dev(input_ids, "input_ids", 8), n_ids, int(image_token_id),
                             _dev(d_out, "d_out", 2, n_ids * cfg.N2), *grad_ptrs,
                             *[ctypes.cast(mids[k], ctypes.c_void_p) if k in mids else None
                               for k in ("W_mid", "b_mid")])
        except VlprojError as e:
            return self._fail(e, check)
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
        n_rows = 0 if rows_out is None else int(rows_out.shape[0])
        N2 = self.cfg.N2
        try:
            P, _ = self._extent(g, self._views(g, c, n_images))
            a = HostArgs(_host(features, "features", self._feat_size(), P * self.cfg.C), _ptr(g), _ptr(c), n_images,
                         _dev(newline, "newline", 2, N2), _dev(sep, "sep", 2, N2),
                         _host(rows_out, "rows_out", 2, n_rows * N2), n_rows, int(chunks))
        except VlprojError as e:
            return self._fail(e, check)
        rc = _lib.vlproj_project_host(self._h, ctypes.byref(a), _stream_ptr(stream))
        if check and rc != OK:
            raise VlprojError(rc, "vlproj_project_host")
        return rc

    def hidden(self, features, grid_hw, hidden, stream=None) -> None:
        g = _host_i32(grid_hw)
        nv = 0 if g is None else len(g.reshape(-1, 2))
        P, M = self._extent(g, nv)
        rc = _lib.vlproj_hidden(self._h, _dev(features, "features", self._feat_size(), P * self.cfg.C), _ptr(g), nv,
                                _dev(hidden, "hidden", 2, M * self.cfg.N1), _stream_ptr(stream))
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

    def set_raster_budget(self, nbytes: int) -> None:
        rc = _lib.vlproj_set_raster_budget(self._h, int(nbytes))
        if rc != OK:
            raise VlprojError(rc, "vlproj_set_raster_budget")

    def set_tile_order(self, order: int) -> None:
        """TILE_ORDER_STATIC, TILE_ORDER_AUTO (the default) or TILE_ORDER_DYNAMIC."""
        rc = _lib.vlproj_set_tile_order(self._h, int(order))
        if rc != OK:
            raise VlprojError(rc, "vlproj_set_tile_order")

    def set_wait_limit(self, ns: int) -> None:
        rc = _lib.vlproj_set_wait_limit(self._h, int(ns))
        if rc != OK:
            raise VlprojError(rc, "vlproj_set_wait_limit")
