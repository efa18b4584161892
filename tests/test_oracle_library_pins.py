"""Pins of the oracle against the MiMo-V2 processor and vision tower installed as a library (CPU only).

The processing page (NeMo Automodel "mimo_v2_flash.processing", function smart_resize and the module
docstring) defines the path as the sglang MiMoProcessor semantics. The image ships vLLM's MiMo-V2 Omni
processor and model, an implementation of that processor lineage. Its functions are called here as
library routines (their source is not copied):

- ``_smart_resize``: every sub-factor shape with a short side under 32 and a long side up to 4000, both
  orientations, at the default bounds, and random shapes under random bounds. This pins the reading the
  pages leave open: in the upscale branch the scaled long side is truncated to an integer. The page's
  rejection of a degenerate shrink stays: the library returns a zero side there, the oracle an error.
- ``_transform_single`` + ``MiMoVLProcessor._flatten_visual``: the whole image path (resize, 0..255
  ImageNet normalisation, T = 2 duplication, (c, tt, py, px) rows in merge-block order) on random RGB
  images, including sub-factor and downscaled shapes.
- ``_to_rgb``: RGBA flattened onto white (PIL paste with the alpha mask).
- ``MiMoVLProcessor.process_video``: the video budget, the padding of an odd frame count and the frame
  pairing of the temporal patches.
- ``MiMoVisionTransformer.get_window_index_1d(col=True)``: the window index.
- ``MiMoVisionTransformer.rot_pos_emb`` (with a rotary table that returns its own index) and
  ``apply_index``: the rotary positions in merge order and in column order.

The library computes the resize in fp32 (torch's fp32 source coordinate, about 6e-8 relative error),
the oracle in fp64; on random 0..255 pixels that moves a normalised value by up to about
255 * 6e-8 * size / 57 (1e-4 at the sizes used here; 8e-5 observed), so the value bound is 5e-4, far
below what a wrong tap, weight, statistic or index would cause. Geometry, ordering and the tables are
compared exactly.
"""
import functools
import types

import numpy as np
import pytest
import torch

import oracle

vproc = pytest.importorskip("vllm.transformers_utils.processors.mimo_v2_omni")
try:
    from vllm.model_executor.models.mimo_v2_omni import MiMoVisionTransformer
except Exception:  # pragma: no cover
    MiMoVisionTransformer = None

IMAGENET_MEAN = (0.485, 0.456, 0.406)
IMAGENET_STD = (0.229, 0.224, 0.225)
VALUE_ATOL = 5e-4


def _lib_resize(h, w, mn=8192, mx=8388608):
    return tuple(int(v) for v in vproc._smart_resize(h, w, 32, mn, mx))


def test_smart_resize_sub_factor_exhaustive():
    for short in range(1, 32):
        for long in range(short, 4001):
            for h, w in ((short, long), (long, short)):
                assert oracle.smart_resize(h, w) == _lib_resize(h, w), (h, w)


def test_smart_resize_random_bounds():
    rng = np.random.Generator(np.random.PCG64(23))
    for _ in range(6000):
        short = int(rng.integers(1, 32))
        long = int(np.exp(rng.uniform(0.0, np.log(200000))))
        h, w = (short, long) if rng.integers(2) else (long, short)
        mn = int(rng.choice([0, 3136, 8192, 50_000]))
        mx = int(rng.choice([200_000, 1003520, 8388608, 1 << 40]))
        lib_hw = _lib_resize(h, w, mn, mx)
        st = oracle.smart_resize_status(h, w, 32, mn, mx)
        if min(lib_hw) == 0:
            # the page rejects a degenerate shrink where the library returns a zero side
            assert st == oracle.EDEGENERATE, (h, w, mn, mx)
        else:
            assert st == oracle.OK and oracle.smart_resize(h, w, 32, mn, mx) == lib_hw, (h, w, mn, mx)


def test_smart_resize_large_shapes_and_aspect_guard():
    rng = np.random.Generator(np.random.PCG64(29))
    for _ in range(3000):
        h, w = (int(v) for v in np.exp(rng.uniform(np.log(32), np.log(30000), size=2)))
        if max(h, w) / min(h, w) > 200:
            assert oracle.smart_resize_status(h, w) == oracle.EASPECT
            with pytest.raises(ValueError):
                vproc._smart_resize(h, w, 32, 8192, 8388608)
            continue
        assert oracle.smart_resize(h, w) == _lib_resize(h, w), (h, w)


def _stub_processor():
    s = types.SimpleNamespace(patch_size=16, merge_size=2, temporal_patch_size=2, temporal_compression_ratio=1,
                              device=None)
    s._flatten_visual = functools.partial(vproc.MiMoVLProcessor._flatten_visual, s)
    return s


@pytest.mark.parametrize("hw", [(64, 48), (37, 91), (16, 192), (7, 8), (13, 41), (31, 3984 // 8), (250, 333),
                                (480, 96), (97, 515)])
def test_image_path_matches_library(hw):
    h, w = hw
    rng = np.random.Generator(np.random.PCG64(h * 1000 + w))
    img = rng.integers(0, 256, size=(h, w, 3), dtype=np.uint8)
    rows, grid = oracle.preprocess_image(img, IMAGENET_MEAN, IMAGENET_STD)
    chw = torch.from_numpy(img).permute(2, 0, 1).contiguous()
    planes, w_bar, h_bar = vproc._transform_single(chw, factor=32, min_px=8192, max_px=8388608)
    lib_rows, thw = _stub_processor()._flatten_visual(planes, "image")
    assert tuple(int(v) for v in thw) == grid
    assert (h_bar, w_bar) == (grid[1] * 16, grid[2] * 16)
    assert lib_rows.shape == rows.shape
    np.testing.assert_allclose(rows, lib_rows.numpy(), rtol=0, atol=VALUE_ATOL)


def test_flatten_on_white_matches_library():
    from PIL import Image
    rng = np.random.Generator(np.random.PCG64(31))
    rgba = rng.integers(0, 256, size=(64, 80, 4), dtype=np.uint8)
    rgba[:, :, 3].flat[::3] = 0
    rgba[:, :, 3].flat[1::3] = 255
    lib = np.asarray(vproc._to_rgb(Image.fromarray(rgba, "RGBA")))
    assert np.array_equal(oracle.to_rgb(rgba), lib)


@pytest.mark.parametrize("n,hw,total_max", [(4, (96, 128), 0), (5, (80, 50), 0), (3, (480, 640), 400_000),
                                            (6, (20, 300), 0)])
def test_video_path_matches_library(n, hw, total_max):
    h, w = hw
    rng = np.random.Generator(np.random.PCG64(n * 7 + h))
    frames = rng.integers(0, 256, size=(n, h, w, 3), dtype=np.uint8)
    max_px = 8388608
    rows, grid = oracle.preprocess_video(frames, IMAGENET_MEAN, IMAGENET_STD, 8192, max_px, total_max)
    s = _stub_processor()
    kw = {"min_pixels": 8192, "max_pixels": max_px, "total_max_pixels": total_max if total_max else 1 << 62,
          "num_frames": n}
    s._resolve_vid_kw = lambda _vid: dict(kw)
    tchw = torch.from_numpy(frames).permute(0, 3, 1, 2).contiguous()
    stamps = torch.arange(n, dtype=torch.float64) * 0.5
    vid = vproc.VideoInput(video=(tchw, stamps))
    lib_rows, thw, _, _ = vproc.MiMoVLProcessor.process_video(s, vid)
    assert tuple(int(v) for v in thw) == grid
    assert lib_rows.shape == rows.shape
    np.testing.assert_allclose(rows, lib_rows.numpy(), rtol=0, atol=VALUE_ATOL)


GRIDS = [(1, 2, 2), (1, 4, 6), (1, 6, 4), (1, 68, 120), (2, 8, 10), (3, 2, 24), (1, 24, 2)]


def _tower_stub():
    s = types.SimpleNamespace(spatial_merge_size=2, spatial_merge_unit=4)
    # a rotary table whose row p holds p itself: cos[pos_ids] returns the positions
    s.rotary_pos_emb = types.SimpleNamespace(
        get_cos_sin=lambda n: (torch.arange(n).unsqueeze(1), torch.arange(n).unsqueeze(1)))
    return s


@pytest.mark.skipif(MiMoVisionTransformer is None, reason="vLLM MiMo-V2 model not importable")
def test_window_index_matches_library():
    grid = torch.tensor(GRIDS, dtype=torch.int64)
    lib = MiMoVisionTransformer.get_window_index_1d(_tower_stub(), grid, col=True).numpy()
    parts, unit0 = [], 0
    for t, gh, gw in GRIDS:
        parts.append(oracle.window_index(gh, gw, 2, unit0, grid_t=t))
        unit0 += t * (gh // 2) * (gw // 2)
    assert np.array_equal(np.concatenate(parts), lib)


@pytest.mark.skipif(MiMoVisionTransformer is None, reason="vLLM MiMo-V2 model not importable")
def test_rotary_positions_match_library_in_both_orders():
    stub = _tower_stub()
    grid = torch.tensor(GRIDS, dtype=torch.int64)
    cos, _ = MiMoVisionTransformer.rot_pos_emb(stub, grid)
    merge = np.concatenate([oracle.rotary_positions(gh, gw, 2, grid_t=t) for t, gh, gw in GRIDS])
    assert np.array_equal(cos.numpy(), merge)
    # column order: the tower reorders whole merge units by the window index
    win = MiMoVisionTransformer.get_window_index_1d(stub, grid, col=True)
    col = MiMoVisionTransformer.apply_index(stub, cos, win).numpy()
    want = np.concatenate([oracle.rotary_positions(gh, gw, 2, column_order=True, grid_t=t) for t, gh, gw in GRIDS])
    assert np.array_equal(col, want)
