"""Pins for the oracle's whole path, row layout and column permutation.

The patch layout comes from docs.rs 'cortiq_engine::mimo_vision' (conventions list). There are
T = 2 identical frames. A row holds its values in (c, tt, py, px) order, and rows follow the
merge-block order (t, block row, block col, mh, mw). column_permutation visits merge units by
(t, block col, block row), keeps each unit's m*m rows adjacent, and maps perm[dst] = src. Here that layout is re-expressed independently with torch reshape/permute
on planes produced by PIL compositing and torch's F.interpolate (the routines the NeMo Automodel
'mimo_v2_flash.processing' page names), and compared with the oracle's loop nest.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

try:
    from PIL import Image
except Exception:  # pragma: no cover
    Image = None

P, T, M = 16, 2, 2


def _pil_rgb(img):
    if img.shape[2] == 3:
        return img
    im = Image.fromarray(img, "RGBA")
    white = Image.new("RGBA", im.size, (255, 255, 255, 255))
    return np.asarray(Image.alpha_composite(white, im).convert("RGB"))


def reference_rows(img, mean, std, oh, ow):
    rgb = _pil_rgb(img)
    planes = torch.from_numpy(rgb.astype(np.float64)).permute(2, 0, 1).contiguous()
    r = F.interpolate(planes[None], size=(oh, ow), mode="bilinear", align_corners=False, antialias=False)[0]
    m = torch.tensor(mean, dtype=torch.float64)[:, None, None]
    s = torch.tensor(std, dtype=torch.float64)[:, None, None]
    r = (r - 255 * m) / (255 * s)
    frames = r[None].expand(T, 3, oh, ow)  # (tt, c, y, x)
    gh, gw = oh // P, ow // P
    x = frames.reshape(T, 3, gh // M, M, P, gw // M, M, P)  # tt c bh mh py bw mw px
    x = x.permute(2, 5, 3, 6, 1, 0, 4, 7)  # bh bw mh mw c tt py px
    return x.reshape(gh * gw, 3 * T * P * P).float().numpy()


needs_pil = pytest.mark.skipif(Image is None, reason="PIL not installed")


@needs_pil
@pytest.mark.parametrize("seed", range(4))
def test_whole_path_matches_independent_formulation(seed):
    imgs = workloads.random_small_batch(200 + seed, 6, max_side=150)
    for img in imgs:
        mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
        rows, g = oracle.preprocess_image(img, mean, std)
        oh, ow = g[1] * P, g[2] * P
        assert (oh, ow) == oracle.smart_resize(img.shape[0], img.shape[1])
        np.testing.assert_allclose(rows, reference_rows(img, mean, std, oh, ow), rtol=0, atol=1e-6)


@needs_pil
def test_whole_path_c1_and_clip_stats():
    w = workloads.workload("c1")
    img = w["images"][0]
    rows, g = oracle.preprocess_image(img, workloads.CLIP_MEAN, workloads.CLIP_STD)
    assert g == (1, 8, 6) and rows.shape == (48, 1536)
    np.testing.assert_allclose(rows, reference_rows(img, workloads.CLIP_MEAN, workloads.CLIP_STD, 128, 96), atol=1e-6)


def test_constant_image_maps_to_constant():
    mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
    img = np.empty((50, 70, 3), np.uint8)
    img[..., 0], img[..., 1], img[..., 2] = 12, 200, 255
    rows, _ = oracle.preprocess_image(img, mean, std)
    per_c = rows.reshape(rows.shape[0], 3, T * P * P)
    for c, v in enumerate((12, 200, 255)):
        assert np.allclose(per_c[:, c], (v - 255 * mean[c]) / (255 * std[c]), atol=1e-6)


def test_transparent_pixels_become_white():
    mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
    rng = np.random.Generator(np.random.PCG64(4))
    img = rng.integers(0, 256, size=(96, 128, 4), dtype=np.uint8)
    img[..., 3] = 0
    rows, _ = oracle.preprocess_image(img, mean, std)
    per_c = rows.reshape(rows.shape[0], 3, T * P * P)
    for c in range(3):
        assert np.allclose(per_c[:, c], (1 - mean[c]) / std[c], atol=1e-6)


def test_identity_resize_reproduces_pixels():
    # 96x128 is already a multiple of 32 inside the pixel bounds: no resampling at all
    mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
    rng = np.random.Generator(np.random.PCG64(8))
    img = rng.integers(0, 256, size=(96, 128, 3), dtype=np.uint8)
    planes = oracle.load_planes(img)
    resized = np.stack([oracle.resize_plane(planes[c], 96, 128) for c in range(3)])
    assert np.array_equal(resized, planes)
    rows, g = oracle.preprocess_image(img, mean, std)
    assert g == (1, 6, 8)
    # pixel (y, x) of channel c lands in row of merge unit (y//32, x//32), sub-patch ((y//16)%2, (x//16)%2)
    for (y, x, c) in [(0, 0, 0), (17, 33, 1), (95, 127, 2), (50, 64, 0)]:
        unit = (y // 32) * (128 // 32) + x // 32
        row = unit * 4 + ((y // 16) % 2) * 2 + (x // 16) % 2
        for tt in range(T):
            col = ((c * T + tt) * P + y % 16) * P + x % 16
            assert rows[row, col] == np.float32((img[y, x, c] - 255 * mean[c]) / (255 * std[c]))


def test_temporal_copies_identical():
    img = workloads.random_small_batch(31, 1, max_side=120)[0]
    rows, _ = oracle.preprocess_image(img, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    r = rows.reshape(rows.shape[0], 3, T, P * P)
    assert np.array_equal(r[:, :, 0], r[:, :, 1])


def test_patch_value_samples_match_full_output():
    rng = np.random.Generator(np.random.PCG64(12))
    for img in workloads.random_small_batch(40, 5, max_side=200):
        rows, g = oracle.preprocess_image(img, workloads.CLIP_MEAN, workloads.CLIP_STD)
        hw = (g[1] * P, g[2] * P)
        for _ in range(200):
            r, c = int(rng.integers(0, rows.shape[0])), int(rng.integers(0, 1536))
            v = oracle.patch_value(img, hw, r, c, workloads.CLIP_MEAN, workloads.CLIP_STD)
            assert v == rows[r, c], (r, c)


def test_batch_assembly_flattens_one_level():
    imgs = workloads.random_small_batch(50, 4, max_side=90)
    flat, g_flat, _ = oracle.preprocess(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    nested, g_nested, _ = oracle.preprocess([[imgs[0]], [imgs[1], imgs[2]], imgs[3]],
                                            workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    assert np.array_equal(flat, nested) and np.array_equal(g_flat, g_nested)
    assert g_flat.shape == (4, 3) and (g_flat[:, 0] == 1).all()
    assert flat.shape == (int((g_flat[:, 1] * g_flat[:, 2]).sum()), 1536)
    row0 = 0
    for img, (_, gh, gw) in zip(imgs, g_flat.tolist()):
        one, _ = oracle.preprocess_image(img, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
        assert np.array_equal(flat[row0:row0 + gh * gw], one)
        row0 += gh * gw


def test_column_permutation_hand_worked():
    # grid 4x6 patches -> 2x3 merge units; units listed by (block col, block row): 0, 3, 1, 4, 2, 5
    perm = oracle.column_permutation(4, 6)
    want = np.concatenate([np.arange(4) + 4 * u for u in (0, 3, 1, 4, 2, 5)])
    assert np.array_equal(perm, want)


def test_column_permutation_properties():
    rng = np.random.Generator(np.random.PCG64(2))
    for _ in range(50):
        gh, gw = 2 * int(rng.integers(1, 40)), 2 * int(rng.integers(1, 40))
        row0 = 4 * int(rng.integers(0, 1000))
        perm = oracle.column_permutation(gh, gw, 2, row0)
        n = gh * gw
        assert np.array_equal(np.sort(perm), np.arange(row0, row0 + n))          # bijection on the image's rows
        units = (perm - row0).reshape(-1, 4)
        assert (units % 4 == np.arange(4)).all() and (np.diff(units, axis=1) == 1).all()  # whole units
        # unit order = transpose of the (block row, block col) grid
        want = np.arange(n // 4).reshape(gh // 2, gw // 2).T.reshape(-1)
        assert np.array_equal(units[:, 0] // 4, want)


def test_batch_permutation_is_batch_global():
    imgs = workloads.random_small_batch(60, 3, max_side=100)
    pv, g, perm = oracle.preprocess(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, column_perm=True)
    assert perm.shape == (pv.shape[0],)
    assert np.array_equal(np.sort(perm), np.arange(pv.shape[0]))
    row0 = 0
    for (_, gh, gw) in g.tolist():
        seg = perm[row0:row0 + gh * gw]
        assert seg.min() == row0 and seg.max() == row0 + gh * gw - 1
        row0 += gh * gw


def test_bf16_rounding_helper():
    x = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e-3], np.float32)
    b = oracle.bf16_bits_to_f32(oracle.round_to_bf16(x))
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(b, ref)
