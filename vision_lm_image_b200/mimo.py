"""Python binding of the C ABI in include/mimo.h (argument marshalling only).

Every step of the pixel path runs in the CUDA library ``libmimo_b200.so``;
this module only packs images into one buffer, allocates outputs with torch
on the caller's device and stream, and passes pointers and sizes. If the
library is missing, every call raises :class:`MimoLibraryMissing`: there is
no CPU fallback.

The user-level call mirrors ``MimoV2ImageProcessor.__call__`` (NeMo Automodel,
"mimo_v2_flash.processing"): images (HWC uint8, RGB or RGBA; one nesting level
is flattened) go in, ``pixel_values [total_patches, 1536]`` and
``image_grid_thw [n, 3]`` come out, plus the optional column-order
permutation (docs.rs "cortiq_engine::mimo_vision", column_permutation).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from typing import Iterable, Sequence

import numpy as np

from . import build as _build

OK = 0
F32, BF16 = 0, 1
ORDER_MERGE, ORDER_COLUMN = 0, 1
ROW_WIDTH = 1536
ALIGN = 16

STATUS_NAMES = {
    0: "MIMO_OK", 1: "MIMO_EINVAL", 2: "MIMO_EASPECT", 3: "MIMO_EDEGENERATE", 4: "MIMO_ECHANNELS",
    5: "MIMO_EUNSUPPORTED", 6: "MIMO_EALIGN", 7: "MIMO_ECAPACITY", 8: "MIMO_EOVERFLOW", 9: "MIMO_ECUDA",
    10: "MIMO_ERANGE", 11: "MIMO_ELIMIT",
}
EXPORTED = ("mimo_params_default", "mimo_smart_resize", "mimo_num_patches", "mimo_plan_batch",
            "mimo_preprocess_batch", "mimo_preprocess_batch_ex", "mimo_preprocess_units", "mimo_preprocess_batch_host",
            "mimo_preprocess_batch_host_noalloc", "mimo_expand_prompt_ids", "mimo_video_max_pixels",
            "mimo_smart_nframes", "mimo_sample_frames", "mimo_plan_video", "mimo_preprocess_video",
            "mimo_patch_embed", "mimo_patch_embed_stall_test", "mimo_preprocess_embed",
            "mimo_status_string", "mimo_version", "mimo_bounds_check_status")
NOALLOC_STAGING_BYTES = 64 << 20


class MimoLibraryMissing(RuntimeError):
    pass


class MimoError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        msg = _lib_status_string(status)
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}{(' (' + what + ')') if what else ''}")
        self.status = status


class MimoParams(ctypes.Structure):
    _fields_ = [
        ("patch_size", ctypes.c_int32),
        ("temporal_patch_size", ctypes.c_int32),
        ("merge_size", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("min_pixels", ctypes.c_int64),
        ("max_pixels", ctypes.c_int64),
        ("image_mean", ctypes.c_float * 3),
        ("image_std", ctypes.c_float * 3),
    ]


class MimoOutputs(ctypes.Structure):
    _fields_ = [
        ("out_dtype", ctypes.c_int32),
        ("row_order", ctypes.c_int32),
        ("d_out", ctypes.c_void_p),
        ("out_rows_capacity", ctypes.c_int64),
        ("d_column_perm", ctypes.c_void_p),
        ("d_positions", ctypes.c_void_p),
        ("d_window_index", ctypes.c_void_p),
    ]


_i32, _i64, _p, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return _build.LIB_PATH


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    """Argument and result types of every exported function."""
    L.mimo_params_default.argtypes = [ctypes.POINTER(MimoParams)]
    L.mimo_params_default.restype = None
    L.mimo_smart_resize.argtypes = [_i64, _i64, _i64, _i64, _i64, ctypes.POINTER(_i64), ctypes.POINTER(_i64)]
    L.mimo_smart_resize.restype = ctypes.c_int
    L.mimo_num_patches.argtypes = [_i64, _i64, ctypes.POINTER(MimoParams), ctypes.POINTER(_i64)]
    L.mimo_num_patches.restype = ctypes.c_int
    L.mimo_plan_batch.argtypes = [_i32, _p, _p, ctypes.POINTER(MimoParams), _p, _p]
    L.mimo_plan_batch.restype = ctypes.c_int
    L.mimo_preprocess_batch.argtypes = [ctypes.POINTER(MimoParams), _i32, _p, _sz, _p, _p, _p, _p, _i32,
                                        _p, _i64, _p, _p]
    L.mimo_preprocess_batch.restype = ctypes.c_int
    L.mimo_preprocess_batch_ex.argtypes = [ctypes.POINTER(MimoParams), _i32, _p, _sz, _p, _p, _p, _p,
                                           ctypes.POINTER(MimoOutputs), _p]
    L.mimo_preprocess_batch_ex.restype = ctypes.c_int
    L.mimo_preprocess_units.argtypes = [ctypes.POINTER(MimoParams), _i32, _p, _sz, _p, _p, _p, _p, _i64,
                                        _i64, ctypes.POINTER(MimoOutputs), _p]
    L.mimo_preprocess_units.restype = ctypes.c_int
    L.mimo_preprocess_batch_host.argtypes = [ctypes.POINTER(MimoParams), _i32, _p, _sz, _p, _p, _p, _p,
                                             _i32, _p, _i64, _p, _p, _sz, _p, _i64, _p, _p]
    L.mimo_preprocess_batch_host.restype = ctypes.c_int
    L.mimo_preprocess_batch_host_noalloc.argtypes = [ctypes.POINTER(MimoParams), _i32, _p, _sz, _p, _p, _p,
                                                     _p, _i32, _p, _i64, _p, _p]
    L.mimo_preprocess_batch_host_noalloc.restype = ctypes.c_int
    L.mimo_expand_prompt_ids.argtypes = [_p, _i64, _i32, _p, _i64, _p, _i64, ctypes.POINTER(_i64)]
    L.mimo_expand_prompt_ids.restype = ctypes.c_int
    L.mimo_video_max_pixels.argtypes = [_i64, _i64, ctypes.POINTER(MimoParams), ctypes.POINTER(_i64)]
    L.mimo_video_max_pixels.restype = ctypes.c_int
    L.mimo_smart_nframes.argtypes = [_i64, ctypes.c_double, ctypes.c_double, _i64, _i64,
                                     ctypes.POINTER(_i64)]
    L.mimo_smart_nframes.restype = ctypes.c_int
    L.mimo_sample_frames.argtypes = [_i64, _i64, ctypes.c_double, _p, _p, ctypes.POINTER(_i64)]
    L.mimo_sample_frames.restype = ctypes.c_int
    L.mimo_plan_video.argtypes = [_i32, _i32, _i32, _i64, ctypes.POINTER(MimoParams), _p,
                                  ctypes.POINTER(_i64)]
    L.mimo_plan_video.restype = ctypes.c_int
    L.mimo_preprocess_video.argtypes = [ctypes.POINTER(MimoParams), _i32, _p, _sz, _i64, _i32, _i32, _i32,
                                        _i64, ctypes.POINTER(MimoOutputs), _p]
    L.mimo_preprocess_video.restype = ctypes.c_int
    L.mimo_patch_embed.argtypes = [_p, _i64, _p, _i32, _p, _i32, _p, _p, _p]
    L.mimo_patch_embed.restype = ctypes.c_int
    L.mimo_patch_embed_stall_test.argtypes = [_p, _i64, _p, _i32, _p, _i32, _p, _p, _i32, ctypes.c_uint32, _p]
    L.mimo_patch_embed_stall_test.restype = ctypes.c_int
    L.mimo_preprocess_embed.argtypes = [ctypes.POINTER(MimoParams), _i32, _p, ctypes.c_size_t, _p, _p, _p, _p,
                                        _i32, _p, _i32, _p, _i32, _p, _i64, _p, ctypes.c_size_t, _p, _p]
    L.mimo_preprocess_embed.restype = ctypes.c_int
    L.mimo_status_string.argtypes = [ctypes.c_int]
    L.mimo_status_string.restype = ctypes.c_char_p
    L.mimo_version.argtypes = []
    L.mimo_version.restype = ctypes.c_int
    L.mimo_bounds_check_status.argtypes = [ctypes.POINTER(_i64), ctypes.POINTER(_i32)]
    L.mimo_bounds_check_status.restype = ctypes.c_int
    return L


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise MimoLibraryMissing(
                    f"{path} is missing: build it with `python -m vision_lm_image_b200.build` "
                    "(or __graft_entry__.build()); there is no fallback path")
            _lib = _declare(ctypes.CDLL(path))
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Runs the calls of this module inside the block through another build of the library (for example
    the bounds-checked debug build), then restores the default one."""
    global _lib
    other = _declare(ctypes.CDLL(path))
    with _lock:
        saved, _lib = _lib, other
    try:
        yield other
    finally:
        with _lock:
            _lib = saved


def bounds_check_status() -> tuple[int, int]:
    """(failed checks since the last query, kind of the first) of a bounds-checked build; clears both."""
    v, k = _i64(), _i32()
    _check(lib().mimo_bounds_check_status(ctypes.byref(v), ctypes.byref(k)), "bounds_check_status")
    return v.value, k.value


def _lib_status_string(status: int) -> str:
    try:
        return lib().mimo_status_string(status).decode()
    except MimoLibraryMissing:
        return "library missing"


def _check(status: int, what: str = ""):
    if status != OK:
        raise MimoError(status, what)


def _tensor(t, name: str, device=None, dtype=None, cols: int | None = None, host: bool = False):
    """Checks a tensor that goes to the library as a bare pointer.

    The library sees only the address and a count, so what it cannot see is
    checked here: dense layout, element type, the row width and the device
    (a CUDA tensor on ``device``, or a host tensor with ``host``). One
    combined test on the common path; the message is worked out on failure."""
    if (not t.is_contiguous() or (dtype is not None and t.dtype != dtype)
            or (cols is not None and (t.dim() != 2 or t.shape[1] != cols)) or t.is_cuda == host
            or (device is not None and t.get_device() != device.index)):
        _tensor_error(t, name, device, dtype, cols, host)


def _tensor_error(t, name, device, dtype, cols, host):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if cols is not None and (t.dim() != 2 or t.shape[1] != cols):
        raise ValueError(f"{name} must have shape [rows, {cols}], got {tuple(t.shape)}")
    if host:
        raise ValueError(f"{name} must be a host tensor, got {t.device}")
    raise ValueError(f"{name} must be a CUDA tensor on {device if device is not None else 'a CUDA device'}, "
                     f"got {t.device}")


_DTYPES = None  # (float32, bfloat16, int32, uint8), looked up once


def _dtypes():
    global _DTYPES
    if _DTYPES is None:
        import torch

        _DTYPES = (torch.float32, torch.bfloat16, torch.int32, torch.uint8)
    return _DTYPES


def _row_capacity(out, name: str, device=None, host: bool = False, perm=None, positions=None, window=None) -> int:
    """Rows the output tensors can hold: the pixel rows' count, lowered to what
    the permutation (1 per row), positions (2 per row) and window index (1 per
    4 rows) hold, so that the library's capacity check covers all of them."""
    f32, bf16, i32, _ = _DTYPES or _dtypes()
    if out.dtype is not f32 and out.dtype is not bf16:
        raise ValueError(f"unsupported output dtype {out.dtype}")
    _tensor(out, name, device, cols=ROW_WIDTH, host=host)
    cap = out.shape[0]
    if perm is not None:
        _tensor(perm, "perm", device, i32, host=host)
        cap = min(cap, perm.numel())
    if positions is not None:
        _tensor(positions, "positions", device, i32)
        cap = min(cap, positions.numel() // 2)
    if window is not None:
        _tensor(window, "window", device, i32)
        cap = min(cap, window.numel() * 4)
    return cap


def _packed_buffer(packed: "PackedBatch", device=None, host: bool = False):
    """The packed images' buffer, checked as a uint8 tensor on ``device`` (or the host)."""
    buf = packed.buffer
    _tensor(buf, "packed.buffer", device, (_DTYPES or _dtypes())[3], host=host)
    return buf


# ----------------------------------------------------------------- knobs
def make_params(mean=None, std=None, min_pixels: int | None = None, max_pixels: int | None = None,
                patch_size: int = 16, temporal_patch_size: int = 2, merge_size: int = 2) -> MimoParams:
    p = MimoParams()
    lib().mimo_params_default(ctypes.byref(p))
    p.patch_size, p.temporal_patch_size, p.merge_size = patch_size, temporal_patch_size, merge_size
    if min_pixels is not None:
        p.min_pixels = int(min_pixels)
    if max_pixels is not None:
        p.max_pixels = int(max_pixels)
    if mean is not None:
        for c in range(3):
            p.image_mean[c] = float(mean[c])
    if std is not None:
        for c in range(3):
            p.image_std[c] = float(std[c])
    return p


# ----------------------------------------------------------------- host-only geometry
def smart_resize(height: int, width: int, factor: int = 32, min_pixels: int = 8192,
                 max_pixels: int = 8388608) -> tuple[int, int]:
    oh, ow = _i64(), _i64()
    _check(lib().mimo_smart_resize(height, width, factor, min_pixels, max_pixels, ctypes.byref(oh),
                                   ctypes.byref(ow)), f"smart_resize({height}, {width})")
    return oh.value, ow.value


def smart_resize_status(height: int, width: int, factor: int = 32, min_pixels: int = 8192,
                        max_pixels: int = 8388608) -> int:
    oh, ow = _i64(), _i64()
    return lib().mimo_smart_resize(height, width, factor, min_pixels, max_pixels, ctypes.byref(oh), ctypes.byref(ow))


def get_number_of_image_patches(height: int, width: int, params: MimoParams | None = None) -> int:
    p = params if params is not None else make_params()
    out = _i64()
    _check(lib().mimo_num_patches(height, width, ctypes.byref(p), ctypes.byref(out)))
    return out.value


def plan_batch(heights: Sequence[int], widths: Sequence[int], params: MimoParams | None = None):
    """(grid_thw int64 [n, 3], row_offsets int64 [n + 1])."""
    p = params if params is not None else make_params()
    n = len(heights)
    h = np.ascontiguousarray(heights, dtype=np.int32)
    w = np.ascontiguousarray(widths, dtype=np.int32)
    grid = np.zeros((n, 3), np.int64)
    offs = np.zeros(n + 1, np.int64)
    _check(lib().mimo_plan_batch(n, h.ctypes.data, w.ctypes.data, ctypes.byref(p), grid.ctypes.data,
                                 offs.ctypes.data), "plan_batch")
    return grid, offs


def media_tokens(height: int, width: int, params: MimoParams | None = None) -> int:
    """Vision tokens of one image: patches after smart_resize over the merge_size**2 reduction."""
    p = params if params is not None else make_params()
    return get_number_of_image_patches(height, width, p) // (p.merge_size * p.merge_size)


def expand_prompt_ids(ids, pad_id: int, counts) -> np.ndarray:
    """Replaces the k-th ``pad_id`` in ``ids`` by ``counts[k]`` copies (int32 result)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int64)
    cap = int(ids.size + max(int(counts.sum()) if counts.size else 0, 0))
    out = np.empty(max(cap, 1), np.int32)
    n = _i64()
    _check(lib().mimo_expand_prompt_ids(ids.ctypes.data, ids.size, pad_id, counts.ctypes.data, counts.size,
                                        out.ctypes.data, cap, ctypes.byref(n)), "expand_prompt_ids")
    return out[:n.value]


# ----------------------------------------------------------------- packing
def _flatten_one_level(images):
    flat = []
    for item in images:
        if isinstance(item, (list, tuple)):
            flat.extend(item)
        else:
            flat.append(item)
    return flat


def packed_layout(shapes: Iterable[tuple[int, int, int]]):
    """Byte offsets (16-byte aligned) of HWC images packed back to back, and the total size."""
    offsets, pos = [], 0
    for (h, w, c) in shapes:
        offsets.append(pos)
        pos += h * w * c
        pos = (pos + ALIGN - 1) // ALIGN * ALIGN
    return np.asarray(offsets, np.int64), max(pos, ALIGN)


class PackedBatch:
    """Images packed into one uint8 buffer (host or device) with their sizes."""

    def __init__(self, buffer, offsets, heights, widths, channels):
        self.buffer = buffer  # torch uint8 tensor
        self.offsets = np.ascontiguousarray(offsets, np.int64)
        self.heights = np.ascontiguousarray(heights, np.int32)
        self.widths = np.ascontiguousarray(widths, np.int32)
        self.channels = np.ascontiguousarray(channels, np.int32)
        # host addresses of the four arrays, looked up once (they are passed on every call)
        self.ptrs = (self.offsets.ctypes.data, self.heights.ctypes.data, self.widths.ctypes.data,
                     self.channels.ctypes.data)

    @property
    def n(self) -> int:
        return int(self.heights.shape[0])

    def to(self, device, non_blocking: bool = False) -> "PackedBatch":
        return PackedBatch(self.buffer.to(device, non_blocking=non_blocking), self.offsets, self.heights,
                           self.widths, self.channels)


def pack_images(images, device="cpu", pin_memory: bool = False) -> PackedBatch:
    import torch

    imgs = _flatten_one_level(images)
    shapes = []
    for im in imgs:
        if im.ndim != 3:
            raise ValueError("images must be HWC uint8 arrays")
        shapes.append(tuple(int(s) for s in im.shape))
    offsets, total = packed_layout(shapes)
    dev = torch.device(device)
    buf = torch.empty(total, dtype=torch.uint8, device=dev,
                      pin_memory=(pin_memory and dev.type == "cpu"))
    for im, off, (h, w, c) in zip(imgs, offsets.tolist(), shapes):
        t = im if isinstance(im, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(im, dtype=np.uint8))
        if t.dtype != torch.uint8:
            raise ValueError("images must be uint8")
        buf[off:off + h * w * c].copy_(t.reshape(-1), non_blocking=True)
    return PackedBatch(buf, offsets, [s[0] for s in shapes], [s[1] for s in shapes], [s[2] for s in shapes])


# ----------------------------------------------------------------- device path
def _on_stream(stream):
    """Context that makes ``stream`` (when given) torch's current stream, so that the packing
    copies and allocations of a high-level call are ordered with its library call."""
    import torch

    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _stream_handle(stream, device):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def preprocess_batch(params: MimoParams, packed: PackedBatch, out, perm=None, stream=None) -> None:
    """Raw ABI call on device buffers (``packed.buffer``, ``out`` and ``perm`` on the same CUDA device)."""
    buf = _packed_buffer(packed)
    cap = _row_capacity(out, "out", buf.device, perm=perm)
    st = lib().mimo_preprocess_batch(
        ctypes.byref(params), packed.n, ctypes.c_void_p(buf.data_ptr()), buf.numel(),
        *packed.ptrs, _dtype_code(out.dtype), ctypes.c_void_p(out.data_ptr()),
        cap, ctypes.c_void_p(perm.data_ptr() if perm is not None else 0),
        _stream_handle(stream, buf.device))
    _check(st, "preprocess_batch")


def _dtype_code(dtype) -> int:
    import torch

    if dtype == torch.float32:
        return F32
    if dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported output dtype {dtype}")


def preprocess_batch_ex(params: MimoParams, packed: PackedBatch, out, perm=None, positions=None, window=None,
                        order: str = "merge", stream=None) -> None:
    """Raw ABI call of mimo_preprocess_batch_ex: row order and the optional index tables (device tensors)."""
    buf = _packed_buffer(packed)
    o = MimoOutputs()
    o.out_dtype = _dtype_code(out.dtype)
    o.row_order = {"merge": ORDER_MERGE, "column": ORDER_COLUMN}[order]
    o.d_out = out.data_ptr()
    o.out_rows_capacity = _row_capacity(out, "out", buf.device, perm=perm, positions=positions, window=window)
    o.d_column_perm = perm.data_ptr() if perm is not None else None
    o.d_positions = positions.data_ptr() if positions is not None else None
    o.d_window_index = window.data_ptr() if window is not None else None
    st = lib().mimo_preprocess_batch_ex(
        ctypes.byref(params), packed.n, ctypes.c_void_p(buf.data_ptr()), buf.numel(),
        *packed.ptrs, ctypes.byref(o), _stream_handle(stream, buf.device))
    _check(st, "preprocess_batch_ex")


def preprocess_units(params: MimoParams, packed: PackedBatch, first_unit: int, unit_count: int, out, perm=None,
                     positions=None, window=None, stream=None) -> None:
    """Raw ABI call of mimo_preprocess_units: merge units [first_unit, first_unit + unit_count) of the batch.

    ``out`` (and ``positions``) hold the window's rows only, merge order; ``perm`` [total_rows] and
    ``window`` [total_rows / 4] are batch-global and receive the window's entries."""
    buf = _packed_buffer(packed)
    _, offs = plan_batch(packed.heights, packed.widths, params)
    total = int(offs[-1])
    f32, bf16, i32, _ = _DTYPES or _dtypes()
    if perm is not None:
        _tensor(perm, "perm", buf.device, i32)
        if perm.numel() < total:
            raise ValueError(f"perm holds {perm.numel()} entries; the batch has {total} rows")
    if window is not None:
        _tensor(window, "window", buf.device, i32)
        if window.numel() < total // 4:
            raise ValueError(f"window holds {window.numel()} entries; the batch has {total // 4} merge units")
    o = MimoOutputs()
    o.out_dtype = _dtype_code(out.dtype)
    o.row_order = ORDER_MERGE
    o.d_out = out.data_ptr()
    o.out_rows_capacity = _row_capacity(out, "out", buf.device, positions=positions)
    o.d_column_perm = perm.data_ptr() if perm is not None else None
    o.d_positions = positions.data_ptr() if positions is not None else None
    o.d_window_index = window.data_ptr() if window is not None else None
    st = lib().mimo_preprocess_units(
        ctypes.byref(params), packed.n, ctypes.c_void_p(buf.data_ptr()), buf.numel(), *packed.ptrs,
        int(first_unit), int(unit_count), ctypes.byref(o), _stream_handle(stream, buf.device))
    _check(st, "preprocess_units")


def preprocess(images, mean=None, std=None, min_pixels: int | None = None, max_pixels: int | None = None,
               dtype=None, column_perm: bool = False, device="cuda", stream=None, order: str = "merge",
               positions: bool = False, window_index: bool = False):
    """The processor call on the GPU: returns (pixel_values, image_grid_thw, perm | None).

    ``images``: HWC uint8 numpy arrays or torch tensors (CPU or CUDA), RGB or
    RGBA, or a list of such lists (unpacked by one level). ``pixel_values`` is a
    CUDA tensor [total_patches, 1536] (float32 by default, bfloat16 on
    request); ``image_grid_thw`` a CPU int64 tensor [n, 3]. ``order="column"``
    emits the rows in column order. With ``positions`` or ``window_index`` the
    result gains two more entries: the int32 [rows, 2] rotary positions of the
    emitted rows and the int32 [rows / 4] window index (None when not asked).
    """
    import torch

    dtype = torch.float32 if dtype is None else dtype
    dev = torch.device(device)
    if dev.type != "cuda":
        raise ValueError("the MiMo preprocessing library runs on CUDA devices only")
    params = make_params(mean, std, min_pixels, max_pixels)
    with _on_stream(stream):
        packed = pack_images(images, device=dev)
        grid, offs = plan_batch(packed.heights, packed.widths, params)
        total = int(offs[-1])
        out = torch.empty((total, ROW_WIDTH), dtype=dtype, device=dev)
        perm = torch.empty(total, dtype=torch.int32, device=dev) if column_perm else None
        pos = torch.empty((total, 2), dtype=torch.int32, device=dev) if positions else None
        win = torch.empty(total // 4, dtype=torch.int32, device=dev) if window_index else None
        preprocess_batch_ex(params, packed, out, perm, pos, win, order, stream)
    if positions or window_index:
        return out, torch.from_numpy(grid), perm, pos, win
    return out, torch.from_numpy(grid), perm


# ----------------------------------------------------------------- video
def video_max_pixels(n_sampled: int, total_max_pixels: int, params: MimoParams | None = None) -> int:
    p = params if params is not None else make_params()
    out = _i64()
    _check(lib().mimo_video_max_pixels(n_sampled, total_max_pixels, ctypes.byref(p), ctypes.byref(out)))
    return out.value


def smart_nframes(total: int, fps_src: float, fps: float, min_frames: int, max_frames: int) -> int:
    out = _i64()
    _check(lib().mimo_smart_nframes(total, fps_src, fps, min_frames, max_frames, ctypes.byref(out)), "smart_nframes")
    return out.value


def sample_frames(total: int, n: int, fps_src: float):
    """(frame indices int64, timestamps float32 seconds)."""
    idx = np.empty(max(n, 1), np.int64)
    ts = np.empty(max(n, 1), np.float32)
    k = _i64()
    _check(lib().mimo_sample_frames(total, n, fps_src, idx.ctypes.data, ts.ctypes.data, ctypes.byref(k)),
           "sample_frames")
    return idx[:k.value], ts[:k.value]


def plan_video(n_frames: int, height: int, width: int, total_max_pixels: int = 0, params: MimoParams | None = None):
    """(grid_thw int64 [3], rows)."""
    p = params if params is not None else make_params()
    g = np.zeros(3, np.int64)
    rows = _i64()
    _check(lib().mimo_plan_video(n_frames, height, width, total_max_pixels, ctypes.byref(p), g.ctypes.data,
                                 ctypes.byref(rows)), "plan_video")
    return g, rows.value


def preprocess_video_raw(params: MimoParams, d_frames, n_frames: int, frame_stride: int, height: int, width: int,
                         channels: int, out, total_max_pixels: int = 0, perm=None, positions=None, window=None,
                         order: str = "merge", stream=None) -> None:
    """Raw ABI call of mimo_preprocess_video on frames already in device memory (uint8 tensor)."""
    import torch

    _tensor(d_frames, "d_frames", dtype=torch.uint8)
    o = MimoOutputs()
    o.out_dtype = _dtype_code(out.dtype)
    o.row_order = {"merge": ORDER_MERGE, "column": ORDER_COLUMN}[order]
    o.d_out = out.data_ptr()
    o.out_rows_capacity = _row_capacity(out, "out", d_frames.device, perm=perm, positions=positions, window=window)
    o.d_column_perm = perm.data_ptr() if perm is not None else None
    o.d_positions = positions.data_ptr() if positions is not None else None
    o.d_window_index = window.data_ptr() if window is not None else None
    _check(lib().mimo_preprocess_video(ctypes.byref(params), n_frames, ctypes.c_void_p(d_frames.data_ptr()),
                                       d_frames.numel(), frame_stride, height, width, channels, total_max_pixels,
                                       ctypes.byref(o), _stream_handle(stream, d_frames.device)), "preprocess_video")


def preprocess_video(frames, mean=None, std=None, min_pixels: int | None = None, max_pixels: int | None = None,
                     total_max_pixels: int = 0, dtype=None, column_perm: bool = False, device="cuda", stream=None,
                     order: str = "merge", positions: bool = False, window_index: bool = False):
    """One video (frames [n, H, W, C] uint8, numpy or torch) through the GPU path.

    Returns (pixel_values, video_grid_thw [1, 3], perm | None) and, with
    ``positions`` / ``window_index``, the two tables as well.
    """
    import torch

    dtype = torch.float32 if dtype is None else dtype
    dev = torch.device(device)
    if dev.type != "cuda":
        raise ValueError("the MiMo preprocessing library runs on CUDA devices only")
    params = make_params(mean, std, min_pixels, max_pixels)
    t = frames if isinstance(frames, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(frames, dtype=np.uint8))
    if t.ndim != 4 or t.dtype != torch.uint8:
        raise ValueError("frames must be a uint8 array [n, H, W, C]")
    n, H, W, C = (int(v) for v in t.shape)
    frame_bytes = H * W * C
    stride = (frame_bytes + ALIGN - 1) // ALIGN * ALIGN
    with _on_stream(stream):
        buf = torch.zeros(n * stride, dtype=torch.uint8, device=dev)
        buf.view(n, stride)[:, :frame_bytes].copy_(t.reshape(n, frame_bytes), non_blocking=True)
        grid, rows = plan_video(n, H, W, total_max_pixels, params)
        out = torch.empty((rows, ROW_WIDTH), dtype=dtype, device=dev)
        perm = torch.empty(rows, dtype=torch.int32, device=dev) if column_perm else None
        pos = torch.empty((rows, 2), dtype=torch.int32, device=dev) if positions else None
        win = torch.empty(rows // 4, dtype=torch.int32, device=dev) if window_index else None
        preprocess_video_raw(params, buf, n, stride, H, W, C, out, total_max_pixels, perm, pos, win, order, stream)
    g = torch.from_numpy(grid.reshape(1, 3))
    if positions or window_index:
        return out, g, perm, pos, win
    return out, g, perm


# ----------------------------------------------------------------- patch embedding (tensor cores)
class PatchEmbedError(RuntimeError):
    pass


def patch_embed(rows, weight, bias=None, out_dtype=None, out=None, error=None, stream=None, check: bool = True):
    """out [M, embed_dim] = rows [M, 1536] (bf16, CUDA) @ weight [embed_dim, 1536]^T (bf16) (+ bias fp32).

    ``error`` is an optional int32 CUDA tensor of one element that receives the
    kernel's status word; with ``check`` the call synchronises and raises if it
    is nonzero.
    """
    import torch

    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    _tensor(rows, "rows", dtype=torch.bfloat16, cols=ROW_WIDTH)
    dev = rows.device
    _tensor(weight, "weight", dev, torch.bfloat16, cols=ROW_WIDTH)
    M = rows.shape[0]
    N = weight.shape[0]
    if bias is not None:
        _tensor(bias, "bias", dev, torch.float32)
        if bias.numel() != N:
            raise ValueError(f"bias must hold {N} values, got {bias.numel()}")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    _tensor(out, "out", dev, cols=N)
    if int(out.shape[0]) != M:
        raise ValueError(f"out must have {M} rows, got {out.shape[0]}")
    if error is None:
        error = torch.zeros(1, dtype=torch.int32, device=dev)
    _tensor(error, "error", dev, torch.int32)
    _check(lib().mimo_patch_embed(ctypes.c_void_p(rows.data_ptr()), M, ctypes.c_void_p(weight.data_ptr()), N,
                                  ctypes.c_void_p(bias.data_ptr() if bias is not None else 0), _dtype_code(out.dtype),
                                  ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(error.data_ptr()),
                                  _stream_handle(stream, rows.device)), "patch_embed")
    if check:
        torch.cuda.current_stream(rows.device).synchronize() if stream is None else stream.synchronize()
        code = int(error.item())
        if code != 0:
            raise PatchEmbedError(f"patch_embed kernel stopped waiting on its pipeline (code {code})")
    return out


def preprocess_embed(images, weight, bias=None, mean=None, std=None, min_pixels: int | None = None,
                     max_pixels: int | None = None, out_dtype=None, order: str = "merge",
                     scratch_bytes: int = 192 << 20, scratch=None, device="cuda", stream=None, check: bool = True,
                     out=None, error=None):
    """Pixel path + patch embedding chunk by chunk: returns (embeddings [rows, embed_dim], image_grid_thw).

    ``out`` ([rows, embed_dim]) and ``error`` (one int32) may be passed in to be reused across calls."""
    import torch

    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    dev = torch.device(device)
    if dev.type != "cuda":
        raise ValueError("the MiMo preprocessing library runs on CUDA devices only")
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    _tensor(weight, "weight", dev, torch.bfloat16, cols=ROW_WIDTH)
    N = weight.shape[0]
    if bias is not None:
        _tensor(bias, "bias", dev, torch.float32)
        if bias.numel() != N:
            raise ValueError(f"bias must hold {N} values, got {bias.numel()}")
    params = make_params(mean, std, min_pixels, max_pixels)
    with _on_stream(stream):
        packed = pack_images(images, device=dev) if not isinstance(images, PackedBatch) else images
        _packed_buffer(packed, dev)
        grid, offs = plan_batch(packed.heights, packed.widths, params)
        total = int(offs[-1])
        if out is None:
            out = torch.empty((total, N), dtype=out_dtype, device=dev)
        _tensor(out, "out", dev, cols=N)
        if int(out.shape[0]) < total:
            raise ValueError(f"out must hold {total} rows, got {out.shape[0]}")
        out_dtype = out.dtype
        if scratch is None:
            scratch = torch.empty(scratch_bytes, dtype=torch.uint8, device=dev)
        _tensor(scratch, "scratch", dev, torch.uint8)
        err = torch.zeros(1, dtype=torch.int32, device=dev) if error is None else error
        _tensor(err, "error", dev, torch.int32)
        order_code = {"merge": ORDER_MERGE, "column": ORDER_COLUMN}[order]
        st = lib().mimo_preprocess_embed(
            ctypes.byref(params), packed.n, ctypes.c_void_p(packed.buffer.data_ptr()), packed.buffer.numel(),
            *packed.ptrs, order_code, ctypes.c_void_p(weight.data_ptr()), N,
            ctypes.c_void_p(bias.data_ptr() if bias is not None else 0), _dtype_code(out_dtype),
            ctypes.c_void_p(out.data_ptr()), int(out.shape[0]), ctypes.c_void_p(scratch.data_ptr()), scratch.numel(),
            ctypes.c_void_p(err.data_ptr()), _stream_handle(stream, dev))
        _check(st, "preprocess_embed")
    if check:
        (torch.cuda.current_stream(dev) if stream is None else stream).synchronize()
        code = int(err.item())
        if code != 0:
            raise PatchEmbedError(f"patch_embed kernel stopped waiting on its pipeline (code {code})")
    return out, torch.from_numpy(grid)


# ----------------------------------------------------------------- host-to-host path
def preprocess_batch_host(params: MimoParams, packed_host: PackedBatch, out_host, perm_host, src_stage,
                          out_stage, perm_stage=None, stream=None) -> None:
    """Raw ABI call of mimo_preprocess_batch_host: host input and output buffers (pinned for full
    bandwidth), caller-provided device staging buffers. Returns when ``out_host`` is filled."""
    import torch

    buf = _packed_buffer(packed_host, host=True)
    cap = _row_capacity(out_host, "out_host", host=True, perm=perm_host)
    _tensor(src_stage, "src_stage", dtype=torch.uint8)
    if out_stage.dtype != out_host.dtype:
        raise ValueError("out_stage and out_host must have the same dtype")
    # the permutation is staged only when it is asked for
    stage_cap = _row_capacity(out_stage, "out_stage", src_stage.device,
                              perm=perm_stage if perm_host is not None else None)
    st = lib().mimo_preprocess_batch_host(
        ctypes.byref(params), packed_host.n, ctypes.c_void_p(buf.data_ptr()), buf.numel(),
        packed_host.offsets.ctypes.data, packed_host.heights.ctypes.data, packed_host.widths.ctypes.data,
        packed_host.channels.ctypes.data, _dtype_code(out_host.dtype), ctypes.c_void_p(out_host.data_ptr()),
        cap, ctypes.c_void_p(perm_host.data_ptr() if perm_host is not None else 0),
        ctypes.c_void_p(src_stage.data_ptr()), src_stage.numel(), ctypes.c_void_p(out_stage.data_ptr()),
        stage_cap, ctypes.c_void_p(perm_stage.data_ptr() if perm_stage is not None else 0),
        _stream_handle(stream, src_stage.device))
    _check(st, "preprocess_batch_host")


def preprocess_batch_host_noalloc(params: MimoParams, packed_host: PackedBatch, out_host, perm_host=None,
                                  stream=None) -> None:
    """Host images in, host rows out, staged through the library's fixed device area: for callers that
    cannot allocate device memory. Runs on the current CUDA device; returns when ``out_host`` is filled."""
    import torch

    buf = _packed_buffer(packed_host, host=True)
    cap = _row_capacity(out_host, "out_host", host=True, perm=perm_host)
    st = lib().mimo_preprocess_batch_host_noalloc(
        ctypes.byref(params), packed_host.n, ctypes.c_void_p(buf.data_ptr()), buf.numel(),
        packed_host.offsets.ctypes.data, packed_host.heights.ctypes.data, packed_host.widths.ctypes.data,
        packed_host.channels.ctypes.data, _dtype_code(out_host.dtype), ctypes.c_void_p(out_host.data_ptr()),
        cap, ctypes.c_void_p(perm_host.data_ptr() if perm_host is not None else 0),
        _stream_handle(stream, torch.device("cuda", torch.cuda.current_device())))
    _check(st, "preprocess_batch_host_noalloc")
