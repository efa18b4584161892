"""Pins for the oracle's smart_resize (NeMo Automodel 'mimo_v2_flash.processing', function smart_resize
and module docstring; docs.rs 'cortiq_engine::mimo_vision', function smart_resize).

- closed forms derived by hand from the page's rules (tests/golden/geometry_closed_forms.json);
- for a short side >= factor the page says the algorithm is HF's: compared, bit for bit, with the
  installed transformers Qwen2-VL smart_resize (a library call; its source is not copied);
- the worked contrast of the module docstring: 16x192 differs from HF's per-side clamp.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")

try:
    from transformers.models.qwen2_vl.image_processing_qwen2_vl import smart_resize as hf_smart_resize
except Exception:  # pragma: no cover
    hf_smart_resize = None


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_closed_forms():
    g = _load("geometry_closed_forms.json")
    for case in g["cases"]:
        h, w = case["hw"]
        assert oracle.smart_resize(h, w, g["factor"], g["min_pixels"], g["max_pixels"]) == tuple(case["out"]), case


def test_error_cases():
    g = _load("geometry_closed_forms.json")
    want = {"aspect": oracle.EASPECT, "degenerate": oracle.EDEGENERATE, "invalid": oracle.EINVAL}
    for case in g["errors"]:
        h, w = case["hw"]
        assert oracle.smart_resize_status(h, w, g["factor"], g["min_pixels"], g["max_pixels"]) == want[case["status"]], case


@pytest.mark.skipif(hf_smart_resize is None, reason="transformers not installed")
def test_worked_contrast_16x192():
    # module docstring: below the factor MiMo upscales first while HF clamps each side
    assert oracle.smart_resize(16, 192) == (32, 384)
    assert hf_smart_resize(16, 192, factor=32, min_pixels=8192, max_pixels=8388608) != (32, 384)


@pytest.mark.skipif(hf_smart_resize is None, reason="transformers not installed")
def test_matches_hf_exhaustive_small():
    # every short side >= 32 up to 260, both orientations, default bounds
    for h in range(32, 261):
        for w in range(32, 261, 3):
            assert oracle.smart_resize(h, w) == tuple(hf_smart_resize(h, w, 32, 8192, 8388608)), (h, w)


@pytest.mark.skipif(hf_smart_resize is None, reason="transformers not installed")
@pytest.mark.parametrize("bounds", [(8192, 8388608), (50_000, 200_000), (3136, 1003520), (0, 1 << 40)])
def test_matches_hf_random(bounds):
    mn, mx = bounds
    rng = np.random.Generator(np.random.PCG64(7))
    n = 0
    while n < 4000:
        h = int(np.exp(rng.uniform(np.log(32), np.log(40000))))
        w = int(np.exp(rng.uniform(np.log(32), np.log(40000))))
        if max(h, w) / min(h, w) > 200:
            assert oracle.smart_resize_status(h, w, 32, mn, mx) == oracle.EASPECT
            with pytest.raises(ValueError):
                hf_smart_resize(h, w, 32, mn, mx)
            continue
        hf = tuple(hf_smart_resize(h, w, 32, mn, mx))
        if min(hf) == 32 and oracle.smart_resize_status(h, w, 32, mn, mx) == oracle.EDEGENERATE:
            # HF clamps a zero side to the factor; the MiMo variant rejects it instead
            n += 1
            continue
        assert oracle.smart_resize(h, w, 32, mn, mx) == hf, (h, w, mn, mx)
        n += 1


@pytest.mark.skipif(hf_smart_resize is None, reason="transformers not installed")
def test_other_factor_matches_hf():
    # factor 28 (Qwen2-VL's own) exercises inexact h/factor divisions
    rng = np.random.Generator(np.random.PCG64(11))
    for _ in range(3000):
        h, w = (int(v) for v in rng.integers(28, 5000, size=2))
        if max(h, w) / min(h, w) > 200:
            continue
        assert oracle.smart_resize(h, w, 28, 3136, 1003520) == tuple(hf_smart_resize(h, w, 28, 3136, 1003520))


def test_outputs_are_factor_multiples_and_bounded():
    rng = np.random.Generator(np.random.PCG64(3))
    for _ in range(3000):
        h, w = (int(v) for v in rng.integers(1, 9000, size=2))
        st = oracle.smart_resize_status(h, w)
        if st != oracle.OK:
            continue
        oh, ow = oracle.smart_resize(h, w)
        assert oh % 32 == 0 and ow % 32 == 0 and oh >= 32 and ow >= 32
        assert oh * ow <= 8388608


def test_token_count_is_patches_over_four():
    # get_number_of_image_patches returns grid_h*grid_w before the merge**2 reduction
    for h, w in [(64, 48), (480, 640), (16, 192), (4096, 4096), (1080, 1920), (333, 777)]:
        oh, ow = oracle.smart_resize(h, w)
        n = oracle.get_number_of_image_patches(h, w)
        assert n == (oh // 16) * (ow // 16)
        assert n % 4 == 0
        tokens = n // 4
        assert tokens == (oh // 32) * (ow // 32)
