"""Pins for the oracle's pixel steps.

- _to_rgb (NeMo Automodel 'mimo_v2_flash.processing', function _to_rgb: RGBA flattened onto white):
  exhaustive over all (c, a) against PIL's own compositing onto an opaque white image.
- resize (class MimoV2ImageProcessor: F.interpolate(mode="bilinear", align_corners=False); docs.rs
  'cortiq_engine::mimo_vision', resize_bilinear): against torch's F.interpolate on fp64 planes, plus
  hand-worked weights, identity and constant cases.
- normalisation (module docstring: mean/std on the 0..255 scale): constant-image closed form.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

try:
    from PIL import Image
except Exception:  # pragma: no cover
    Image = None


@pytest.mark.skipif(Image is None, reason="PIL not installed")
def test_flatten_exhaustive_vs_pil():
    c = np.tile(np.arange(256, dtype=np.uint8), 256)
    a = np.repeat(np.arange(256, dtype=np.uint8), 256)
    rgba = np.stack([c, c, c, a], axis=-1).reshape(256, 256, 4)
    img = Image.fromarray(rgba, "RGBA")
    white = Image.new("RGBA", img.size, (255, 255, 255, 255))
    composite = np.asarray(Image.alpha_composite(white, img).convert("RGB"))
    pasted = Image.new("RGB", img.size, (255, 255, 255))
    pasted.paste(img, mask=img.split()[3])
    pasted = np.asarray(pasted)
    ours = oracle.to_rgb(rgba)
    assert np.array_equal(ours, composite)
    assert np.array_equal(ours, pasted)


def test_flatten_special_cases():
    for c in range(256):
        assert oracle.flatten_on_white(c, 0) == 255      # fully transparent -> white
        assert oracle.flatten_on_white(c, 255) == c      # opaque -> unchanged


def test_rgb_passthrough():
    rng = np.random.Generator(np.random.PCG64(1))
    img = rng.integers(0, 256, size=(7, 5, 3), dtype=np.uint8)
    assert np.array_equal(oracle.to_rgb(img), img)


def _torch_resize(plane, oh, ow):
    t = torch.from_numpy(np.ascontiguousarray(plane, dtype=np.float64))[None, None]
    return F.interpolate(t, size=(oh, ow), mode="bilinear", align_corners=False, antialias=False)[0, 0].numpy()


@pytest.mark.parametrize("seed", range(6))
def test_resize_matches_torch_interpolate_fp64(seed):
    rng = np.random.Generator(np.random.PCG64(100 + seed))
    for _ in range(25):
        h, w = (int(v) for v in rng.integers(1, 70, size=2))
        oh, ow = (int(v) for v in rng.integers(1, 140, size=2))
        plane = rng.integers(0, 256, size=(h, w)).astype(np.float64)
        ours = oracle.resize_plane(plane, oh, ow)
        ref = _torch_resize(plane, oh, ow)
        np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-9)


def test_resize_config_shapes_match_torch():
    rng = np.random.Generator(np.random.PCG64(5))
    for (h, w, oh, ow) in [(64, 48, 128, 96), (16, 192, 32, 384), (31, 31, 96, 96), (20, 300, 32, 480),
                           (300, 213, 288, 224), (1080, 64, 1088, 64)]:
        plane = rng.integers(0, 256, size=(h, w)).astype(np.float64)
        np.testing.assert_allclose(oracle.resize_plane(plane, oh, ow), _torch_resize(plane, oh, ow), atol=1e-9)


def test_resize_hand_worked_2x():
    # 1x2 -> 2x4: source x for d = 0..3 is -0.25 (clamped to 0), 0.25, 0.75, 1.25 (taps clamped at the edge)
    a, b = 10.0, 50.0
    out = oracle.resize_plane(np.array([[a, b]]), 2, 4)
    want = np.array([a, 0.75 * a + 0.25 * b, 0.25 * a + 0.75 * b, b])
    assert np.allclose(out, np.stack([want, want]), atol=1e-12)


def test_resize_hand_worked_odd_downscale():
    # 1x5 -> 1x2: scale 2.5; x = 0.75 and 3.25 -> taps (0,1; 0.75) and (3,4; 0.25)
    row = np.array([[0.0, 100.0, 20.0, 40.0, 80.0]])
    out = oracle.resize_plane(row, 1, 2)
    assert np.allclose(out, [[0.25 * 0 + 0.75 * 100, 0.75 * 40 + 0.25 * 80]], atol=1e-12)


def test_resize_identity_exact():
    rng = np.random.Generator(np.random.PCG64(9))
    plane = rng.integers(0, 256, size=(37, 53)).astype(np.float64)
    assert np.array_equal(oracle.resize_plane(plane, 37, 53), plane)


def test_resize_constant():
    for v in (0.0, 1.0, 117.0, 255.0):
        out = oracle.resize_plane(np.full((13, 29), v), 41, 7)
        assert np.allclose(out, v, atol=1e-12, rtol=0)


def test_normalize_closed_form():
    mean, std = (0.485, 0.456, 0.406), (0.229, 0.224, 0.225)
    planes = np.stack([np.full((2, 3), 0.0), np.full((2, 3), 128.0), np.full((2, 3), 255.0)])
    out = oracle.normalize_planes(planes, mean, std)
    assert np.allclose(out[0], (0 - 255 * 0.485) / (255 * 0.229), atol=1e-14)
    assert np.allclose(out[1], (128 - 255 * 0.456) / (255 * 0.224), atol=1e-14)
    assert np.allclose(out[2], (255 - 255 * 0.406) / (255 * 0.225), atol=1e-14)
