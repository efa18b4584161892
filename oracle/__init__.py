"""TEST INFRASTRUCTURE ONLY: the CPU oracle of the MiMo-V2 pixel path.

A plain, slow restatement of what the path computes (``oracle.c``, fp64),
plus the batch assembly of ``MimoV2ImageProcessor.__call__`` (NeMo Automodel,
"mimo_v2_flash.processing", class MimoV2ImageProcessor: a list of
per-sample lists is unpacked by one level, the images' patch rows are
stacked in order, and ``image_grid_thw`` is ``[n, 3]``).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library
(``vision_lm_image_b200``) never imports, links or runs it, and this package
imports nothing from the product.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lib_override = None  # another build of oracle.c, set by load_build()
_lock = threading.Lock()

OK, EINVAL, EASPECT, EDEGENERATE, ECAPACITY, ENOMEM = range(6)

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_build(path: str | None) -> None:
    """Test hook: later calls run the oracle compiled at ``path`` (None: the
    default build of oracle.c). The mutation check of the pins uses it to run
    copies of oracle.c with planted mistakes; the arithmetic here is unchanged."""
    global _lib, _lib_override
    with _lock:
        _lib = None
        _lib_override = path


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = _lib_override if _lib_override is not None else build()
            L = ctypes.CDLL(path)
            L.oracle_smart_resize.argtypes = [_i64, _i64, _i64, _i64, _i64,
                                              ctypes.POINTER(_i64), ctypes.POINTER(_i64)]
            L.oracle_smart_resize.restype = ctypes.c_int
            L.oracle_flatten_on_white.argtypes = [ctypes.c_uint8, ctypes.c_uint8]
            L.oracle_flatten_on_white.restype = ctypes.c_uint8
            L.oracle_to_rgb.argtypes = [_p, _i64, _i64, _i32, _p]
            L.oracle_to_rgb.restype = ctypes.c_int
            L.oracle_load_planes.argtypes = [_p, _i64, _i64, _p]
            L.oracle_load_planes.restype = None
            L.oracle_resize_plane.argtypes = [_p, _i64, _i64, _p, _i64, _i64]
            L.oracle_resize_plane.restype = None
            L.oracle_normalize_planes.argtypes = [_p, _i64, _p, _p]
            L.oracle_normalize_planes.restype = None
            L.oracle_patchify.argtypes = [_p, _i64, _i64, _i32, _i32, _i32, _p]
            L.oracle_patchify.restype = None
            L.oracle_image_rows.argtypes = [_i64, _i64, _i32, _i32, _i64, _i64]
            L.oracle_image_rows.restype = _i64
            L.oracle_preprocess_image.argtypes = [_p, _i64, _i64, _i32, _i32, _i32, _i32, _i64, _i64,
                                                  _p, _p, _p, _i64, _p]
            L.oracle_preprocess_image.restype = ctypes.c_int
            L.oracle_patch_value.argtypes = [_p, _i64, _i64, _i32, _i64, _i64, _i32, _i32, _i32,
                                             _p, _p, _i64, _i64, ctypes.POINTER(ctypes.c_float)]
            L.oracle_patch_value.restype = ctypes.c_int
            L.oracle_column_permutation.argtypes = [_i64, _i64, _i64, _i32, _i64, _p]
            L.oracle_column_permutation.restype = None
            L.oracle_patchify_column.argtypes = [_p, _i64, _i64, _i32, _i32, _i32, _p]
            L.oracle_patchify_column.restype = None
            L.oracle_rotary_positions.argtypes = [_i64, _i64, _i64, _i32, _i32, _p]
            L.oracle_rotary_positions.restype = None
            L.oracle_window_index.argtypes = [_i64, _i64, _i64, _i32, _i64, _p]
            L.oracle_window_index.restype = None
            L.oracle_expand_prompt_ids.argtypes = [_p, _i64, _i32, _p, _i64, _p, _i64]
            L.oracle_expand_prompt_ids.restype = _i64
            L.oracle_video_max_pixels.argtypes = [_i64, _i64, _i32, _i64, _i64]
            L.oracle_video_max_pixels.restype = _i64
            L.oracle_smart_nframes.argtypes = [_i64, ctypes.c_double, ctypes.c_double, _i64, _i64, ctypes.POINTER(_i64)]
            L.oracle_smart_nframes.restype = ctypes.c_int
            L.oracle_sample_frames.argtypes = [_i64, _i64, ctypes.c_double, _p, _p]
            L.oracle_sample_frames.restype = _i64
            L.oracle_preprocess_video.argtypes = [_p, _i64, _i64, _i64, _i64, _i32, _i32, _i32, _i32, _i64, _i64,
                                                  _i64, _p, _p, _p, _i64, _p]
            L.oracle_preprocess_video.restype = ctypes.c_int
            L.oracle_patch_embed.argtypes = [_p, _i64, _i64, _p, _i64, _p, _p]
            L.oracle_patch_embed.restype = None
            _lib = L
    return _lib


class OracleError(ValueError):
    def __init__(self, status: int, what: str = ""):
        names = {EINVAL: "invalid argument", EASPECT: "aspect ratio above 200",
                 EDEGENERATE: "degenerate shrink", ECAPACITY: "capacity", ENOMEM: "out of memory"}
        super().__init__(f"oracle status {status} ({names.get(status, '?')}) {what}")
        self.status = status


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ---------------------------------------------------------------- geometry
def smart_resize(height: int, width: int, factor: int = 32,
                 min_pixels: int = 8192, max_pixels: int = 8388608) -> tuple[int, int]:
    oh, ow = _i64(), _i64()
    st = lib().oracle_smart_resize(height, width, factor, min_pixels, max_pixels,
                                   ctypes.byref(oh), ctypes.byref(ow))
    if st != OK:
        raise OracleError(st, f"smart_resize({height}, {width})")
    return oh.value, ow.value


def smart_resize_status(height, width, factor=32, min_pixels=8192, max_pixels=8388608) -> int:
    oh, ow = _i64(), _i64()
    return lib().oracle_smart_resize(height, width, factor, min_pixels, max_pixels,
                                     ctypes.byref(oh), ctypes.byref(ow))


def get_number_of_image_patches(height, width, patch=16, merge=2, min_pixels=8192, max_pixels=8388608) -> int:
    """Patches before the merge**2 reduction: grid_h * grid_w of the resized image."""
    r = lib().oracle_image_rows(height, width, patch, merge, min_pixels, max_pixels)
    if r < 0:
        raise OracleError(-r)
    return int(r)


# ---------------------------------------------------------------- steps
def flatten_on_white(c: int, a: int) -> int:
    return int(lib().oracle_flatten_on_white(c, a))


def to_rgb(img: np.ndarray) -> np.ndarray:
    img = np.ascontiguousarray(img, dtype=np.uint8)
    H, W, C = img.shape
    out = np.empty((H, W, 3), np.uint8)
    st = lib().oracle_to_rgb(_ptr(img), H, W, C, _ptr(out))
    if st != OK:
        raise OracleError(st)
    return out


def load_planes(rgb: np.ndarray) -> np.ndarray:
    rgb = np.ascontiguousarray(rgb, dtype=np.uint8)
    H, W, _ = rgb.shape
    out = np.empty((3, H, W), np.float64)
    lib().oracle_load_planes(_ptr(rgb), H, W, _ptr(out))
    return out


def resize_plane(plane: np.ndarray, out_h: int, out_w: int) -> np.ndarray:
    plane = np.ascontiguousarray(plane, dtype=np.float64)
    H, W = plane.shape
    out = np.empty((out_h, out_w), np.float64)
    lib().oracle_resize_plane(_ptr(plane), H, W, _ptr(out), out_h, out_w)
    return out


def normalize_planes(planes: np.ndarray, mean, std) -> np.ndarray:
    planes = np.array(planes, dtype=np.float64, copy=True, order="C")
    m = np.ascontiguousarray(mean, dtype=np.float64)
    s = np.ascontiguousarray(std, dtype=np.float64)
    lib().oracle_normalize_planes(_ptr(planes), planes.shape[1] * planes.shape[2], _ptr(m), _ptr(s))
    return planes


def patchify(planes: np.ndarray, patch=16, temporal=2, merge=2) -> np.ndarray:
    planes = np.ascontiguousarray(planes, dtype=np.float64)
    _, Hr, Wr = planes.shape
    rows = (Hr // patch) * (Wr // patch)
    out = np.empty((rows, 3 * temporal * patch * patch), np.float32)
    lib().oracle_patchify(_ptr(planes), Hr, Wr, patch, temporal, merge, _ptr(out))
    return out


def patchify_column(planes: np.ndarray, patch=16, temporal=2, merge=2) -> np.ndarray:
    planes = np.ascontiguousarray(planes, dtype=np.float64)
    _, Hr, Wr = planes.shape
    rows = (Hr // patch) * (Wr // patch)
    out = np.empty((rows, 3 * temporal * patch * patch), np.float32)
    lib().oracle_patchify_column(_ptr(planes), Hr, Wr, patch, temporal, merge, _ptr(out))
    return out


def rotary_positions(grid_h: int, grid_w: int, merge: int = 2, column_order: bool = False,
                     grid_t: int = 1) -> np.ndarray:
    """[rows, 2] int32 (patch row, patch column) of every emitted row."""
    out = np.empty((grid_t * grid_h * grid_w, 2), np.int32)
    lib().oracle_rotary_positions(grid_t, grid_h, grid_w, merge, int(column_order), _ptr(out))
    return out


def window_index(grid_h: int, grid_w: int, merge: int = 2, unit0: int = 0, grid_t: int = 1) -> np.ndarray:
    """[units] int32: merge-order unit index of each unit in column-major order."""
    out = np.empty(grid_t * (grid_h // merge) * (grid_w // merge), np.int32)
    lib().oracle_window_index(grid_t, grid_h, grid_w, merge, unit0, _ptr(out))
    return out


def column_permutation(grid_h: int, grid_w: int, merge: int = 2, row0: int = 0, grid_t: int = 1) -> np.ndarray:
    out = np.empty(grid_t * grid_h * grid_w, np.int32)
    lib().oracle_column_permutation(grid_t, grid_h, grid_w, merge, row0, _ptr(out))
    return out


# ---------------------------------------------------------------- whole path
def preprocess_image(img: np.ndarray, mean, std, min_pixels=8192, max_pixels=8388608,
                     patch=16, temporal=2, merge=2):
    """One image through the whole path. Returns (rows fp32 [R, 3*T*p*p], grid_thw (1, gh, gw))."""
    img = np.ascontiguousarray(img, dtype=np.uint8)
    H, W, C = img.shape
    rows = lib().oracle_image_rows(H, W, patch, merge, min_pixels, max_pixels)
    if rows < 0:
        raise OracleError(-rows, f"image {H}x{W}")
    out = np.empty((rows, 3 * temporal * patch * patch), np.float32)
    m = np.ascontiguousarray(mean, dtype=np.float64)
    s = np.ascontiguousarray(std, dtype=np.float64)
    g = np.zeros(3, np.int64)
    st = lib().oracle_preprocess_image(_ptr(img), H, W, C, patch, temporal, merge, min_pixels, max_pixels,
                                       _ptr(m), _ptr(s), _ptr(out), rows, _ptr(g))
    if st != OK:
        raise OracleError(st, f"image {H}x{W}x{C}")
    return out, tuple(int(v) for v in g)


def patch_value(img: np.ndarray, resized_hw, row: int, col: int, mean, std,
                patch=16, temporal=2, merge=2) -> float:
    """One output element (row, col) of one image, from the definition."""
    img = np.ascontiguousarray(img, dtype=np.uint8)
    H, W, C = img.shape
    m = np.ascontiguousarray(mean, dtype=np.float64)
    s = np.ascontiguousarray(std, dtype=np.float64)
    v = ctypes.c_float()
    st = lib().oracle_patch_value(_ptr(img), H, W, C, resized_hw[0], resized_hw[1], patch, temporal, merge,
                                  _ptr(m), _ptr(s), row, col, ctypes.byref(v))
    if st != OK:
        raise OracleError(st)
    return float(v.value)


def preprocess_image_column(img: np.ndarray, mean, std, min_pixels=8192, max_pixels=8388608,
                            patch=16, temporal=2, merge=2):
    """One image through the path with rows emitted in column order (units by block column)."""
    img = np.ascontiguousarray(img, dtype=np.uint8)
    H, W, _ = img.shape
    Hr, Wr = smart_resize(H, W, patch * merge, min_pixels, max_pixels)
    planes = load_planes(to_rgb(img))
    resized = np.stack([resize_plane(planes[c], Hr, Wr) for c in range(3)])
    rows = patchify_column(normalize_planes(resized, mean, std), patch, temporal, merge)
    return rows, (1, Hr // patch, Wr // patch)


def expand_prompt_ids(ids, pad_id: int, counts) -> np.ndarray:
    """Expands the k-th ``pad_id`` of ``ids`` into ``counts[k]`` copies."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int64)
    cap = int(ids.size + max(int(counts.sum()), 0))
    out = np.empty(max(cap, 1), np.int32)
    n = lib().oracle_expand_prompt_ids(_ptr(ids), ids.size, pad_id, _ptr(counts), counts.size, _ptr(out), cap)
    if n < 0:
        raise OracleError(EINVAL, "placeholder count does not match the items")
    return out[:n]


# ---------------------------------------------------------------- video
def video_max_pixels(n_sampled: int, total_max: int, temporal: int = 2, min_pixels: int = 8192,
                     max_pixels: int = 8388608) -> int:
    return int(lib().oracle_video_max_pixels(n_sampled, total_max, temporal, min_pixels, max_pixels))


def smart_nframes(total: int, fps_src: float, fps: float, min_frames: int, max_frames: int) -> int:
    out = _i64()
    st = lib().oracle_smart_nframes(total, fps_src, fps, min_frames, max_frames, ctypes.byref(out))
    if st != OK:
        raise OracleError(st, "smart_nframes")
    return out.value


def sample_frames(total: int, n: int, fps_src: float):
    idx = np.empty(max(n, 1), np.int64)
    ts = np.empty(max(n, 1), np.float32)
    k = lib().oracle_sample_frames(total, n, fps_src, _ptr(idx), _ptr(ts))
    if k < 0:
        raise OracleError(EINVAL, "sample_frames")
    return idx[:k], ts[:k]


def preprocess_video(frames, mean, std, min_pixels=8192, max_pixels=8388608, total_max_pixels=0,
                     patch=16, temporal=2, merge=2):
    """Frames [n, H, W, C] uint8 -> (rows fp32, grid_thw (t, h, w))."""
    frames = np.ascontiguousarray(frames, dtype=np.uint8)
    n, H, W, C = frames.shape
    budget = video_max_pixels(n, total_max_pixels, temporal, min_pixels, max_pixels) if total_max_pixels > 0 \
        else max_pixels
    Hr, Wr = smart_resize(H, W, patch * merge, min_pixels, budget)
    gt = (n + 1) // 2
    rows = gt * (Hr // patch) * (Wr // patch)
    out = np.empty((rows, 3 * temporal * patch * patch), np.float32)
    m = np.ascontiguousarray(mean, dtype=np.float64)
    s = np.ascontiguousarray(std, dtype=np.float64)
    g = np.zeros(3, np.int64)
    st = lib().oracle_preprocess_video(_ptr(frames), n, H * W * C, H, W, C, patch, temporal, merge, min_pixels,
                                       max_pixels, total_max_pixels, _ptr(m), _ptr(s), _ptr(out), rows, _ptr(g))
    if st != OK:
        raise OracleError(st, "preprocess_video")
    return out, tuple(int(v) for v in g)


def patch_embed(rows: np.ndarray, weight: np.ndarray, bias=None) -> np.ndarray:
    """fp64 [M, N] = rows [M, K] @ weight[N, K]^T (+ bias), inputs taken as given (float32 values)."""
    rows = np.ascontiguousarray(rows, dtype=np.float32)
    weight = np.ascontiguousarray(weight, dtype=np.float32)
    M, K = rows.shape
    N = weight.shape[0]
    out = np.empty((M, N), np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    lib().oracle_patch_embed(_ptr(rows), M, K, _ptr(weight), N, _ptr(b) if b is not None else None, _ptr(out))
    return out


def _flatten_one_level(images):
    flat = []
    for item in images:
        if isinstance(item, (list, tuple)):
            flat.extend(item)
        else:
            flat.append(item)
    return flat


def preprocess(images, mean, std, min_pixels=8192, max_pixels=8388608, column_perm=False,
               patch=16, temporal=2, merge=2, threads: int = 1, order: str = "merge",
               positions: bool = False, window: bool = False):
    """The batch call: returns (pixel_values fp32 [sum rows, 1536], image_grid_thw int64 [n, 3], perm|None).

    ``threads`` > 1 runs independent images on a thread pool (ctypes drops the
    GIL inside the C code); the arithmetic is unchanged.
    """
    imgs = _flatten_one_level(images)
    one = preprocess_image if order == "merge" else preprocess_image_column
    if threads > 1 and len(imgs) > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            res = list(ex.map(lambda im: one(im, mean, std, min_pixels, max_pixels, patch, temporal, merge), imgs))
    else:
        res = [one(im, mean, std, min_pixels, max_pixels, patch, temporal, merge) for im in imgs]
    cols = 3 * temporal * patch * patch
    pv = np.concatenate([r[0] for r in res], axis=0) if res else np.zeros((0, cols), np.float32)
    grid = np.array([r[1] for r in res], dtype=np.int64).reshape(-1, 3)
    perm = None
    if column_perm:
        parts, row0 = [], 0
        for (_, gh, gw) in grid.tolist():
            parts.append(column_permutation(gh, gw, merge, row0))
            row0 += gh * gw
        perm = np.concatenate(parts) if parts else np.zeros(0, np.int32)
    if not (positions or window):
        return pv, grid, perm
    pos_parts, win_parts, unit0 = [], [], 0
    for (_, gh, gw) in grid.tolist():
        pos_parts.append(rotary_positions(gh, gw, merge, column_order=(order == "column")))
        win_parts.append(window_index(gh, gw, merge, unit0))
        unit0 += (gh // merge) * (gw // merge)
    pos = np.concatenate(pos_parts) if pos_parts else np.zeros((0, 2), np.int32)
    win = np.concatenate(win_parts) if win_parts else np.zeros(0, np.int32)
    return pv, grid, perm, pos, win


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest, ties to even), returned as the bf16 bit pattern (uint16)."""
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = 0x7FFF + ((bits >> 16) & 1)
    return ((bits + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
