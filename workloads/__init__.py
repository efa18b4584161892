"""Seeded synthetic inputs for the MiMo-V2 pixel path.

This module only draws images (packed interleaved HWC uint8 arrays) and holds
the two sets of normalisation statistics; it contains none of the path's
arithmetic. Both the CUDA library's tests/benchmark and the CPU oracle consume
what it returns, and it imports neither of them.

Workloads (all drawn with numpy ``Generator(PCG64(seed))``):

``c1``  one RGB 64x48 image, i.i.d. uniform 0..255 (upscaled to the min_pixels
        grid); ImageNet statistics.
``c2``  16 RGBA 480x640 images; RGB uniform 0..255; alpha per pixel is 0, 255
        or uniform 0..255 with probability 1/3 each; ImageNet statistics.
``c3``  64 RGB images with H, W i.i.d. uniform in [224, 2048] (a pair with
        aspect above 8:1 is redrawn), plus four sub-factor images 16x192,
        20x300, 31x31 and 192x16; CLIP statistics.
``c4``  one RGB 4096x4096 image: smooth gradients (R along x, G along y, B
        along the diagonal) plus per-channel uniform noise in [-32, 32],
        clipped to 0..255; ImageNet statistics.
``c5``  256 images 1080x1920, even indices RGB and odd indices RGBA (alpha as in
        c2), uniform 0..255; ImageNet statistics.
``v1``  one video clip: 64 RGB frames 1080x1920, uniform 0..255, no overall
        pixel budget (each frame pair becomes one temporal patch); ImageNet
        statistics.
"""
from __future__ import annotations

import numpy as np

# MimoV2ImageProcessor constructor defaults (ImageNet statistics).
IMAGENET_MEAN = (0.485, 0.456, 0.406)
IMAGENET_STD = (0.229, 0.224, 0.225)
# Public OpenAI-CLIP preprocessing statistics (the MiMo-V2.5 family's).
CLIP_MEAN = (0.48145466, 0.4578275, 0.40821073)
CLIP_STD = (0.26862954, 0.26130258, 0.27577711)

SEED_BASE = 1000
SUB_FACTOR_SHAPES = ((16, 192), (20, 300), (31, 31), (192, 16))


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def uniform_image(rng: np.random.Generator, h: int, w: int, c: int) -> np.ndarray:
    return rng.integers(0, 256, size=(h, w, c), dtype=np.uint8)


def rgba_image(rng: np.random.Generator, h: int, w: int) -> np.ndarray:
    """RGB uniform; alpha is 0, 255 or uniform with probability 1/3 each."""
    img = rng.integers(0, 256, size=(h, w, 4), dtype=np.uint8)
    kind = rng.integers(0, 3, size=(h, w), dtype=np.uint8)
    alpha = img[:, :, 3]
    alpha[kind == 0] = 0
    alpha[kind == 1] = 255
    return img


def gradient_noise_image(rng: np.random.Generator, h: int, w: int) -> np.ndarray:
    y = np.arange(h, dtype=np.int64)[:, None]
    x = np.arange(w, dtype=np.int64)[None, :]
    base = np.empty((h, w, 3), np.int64)
    base[:, :, 0] = (255 * x) // max(w - 1, 1)
    base[:, :, 1] = (255 * y) // max(h - 1, 1)
    base[:, :, 2] = (255 * (x + y)) // max(w + h - 2, 1)
    noise = rng.integers(-32, 33, size=(h, w, 3), dtype=np.int64)
    return np.clip(base + noise, 0, 255).astype(np.uint8)


def random_sizes(rng: np.random.Generator, n: int, lo: int = 224, hi: int = 2048, max_aspect: float = 8.0):
    sizes = []
    while len(sizes) < n:
        h, w = (int(v) for v in rng.integers(lo, hi + 1, size=2))
        if max(h, w) / min(h, w) > max_aspect:
            continue
        sizes.append((h, w))
    return sizes


def video_workload(name: str, seed_offset: int = 0, n_frames: int | None = None):
    """Returns dict(frames=[n, H, W, C] uint8, mean, std, total_max_pixels, description)."""
    if name != "v1":
        raise KeyError(name)
    rng = rng_for(SEED_BASE + 10 + seed_offset)
    n = 64 if n_frames is None else n_frames
    frames = rng.integers(0, 256, size=(n, 1080, 1920, 3), dtype=np.uint8)
    return dict(frames=frames, mean=IMAGENET_MEAN, std=IMAGENET_STD, total_max_pixels=0, dtype="f32",
                description=f"{n} x RGB 1080x1920 video frames -> {(n + 1) // 2} temporal patches of 1088x1920")


def workload(name: str, seed_offset: int = 0, n_images: int | None = None):
    """Returns dict(images=[HWC uint8], mean, std, dtype, column_perm, description)."""
    idx = {"c1": 0, "c2": 1, "c3": 2, "c4": 3, "c5": 4}[name]
    rng = rng_for(SEED_BASE + idx + seed_offset)
    if name == "c1":
        images = [uniform_image(rng, 64, 48, 3)]
        return dict(images=images, mean=IMAGENET_MEAN, std=IMAGENET_STD, dtype="f32", column_perm=False,
                    description="1 x RGB 64x48 -> 128x96, fp32")
    if name == "c2":
        n = 16 if n_images is None else n_images
        images = [rgba_image(rng, 480, 640) for _ in range(n)]
        return dict(images=images, mean=IMAGENET_MEAN, std=IMAGENET_STD, dtype="f32", column_perm=False,
                    description=f"{n} x RGBA 480x640 (identity resize), fp32")
    if name == "c3":
        n = 64 if n_images is None else n_images
        images = [uniform_image(rng, h, w, 3) for (h, w) in random_sizes(rng, n)]
        images += [uniform_image(rng, h, w, 3) for (h, w) in SUB_FACTOR_SHAPES]
        return dict(images=images, mean=CLIP_MEAN, std=CLIP_STD, dtype="f32", column_perm=False,
                    description=f"{n} x RGB U[224,2048]^2 + 4 sub-factor, CLIP, fp32")
    if name == "c4":
        images = [gradient_noise_image(rng, 4096, 4096)]
        return dict(images=images, mean=IMAGENET_MEAN, std=IMAGENET_STD, dtype="f32", column_perm=False,
                    description="1 x RGB 4096x4096 gradient+noise -> 2880x2880, fp32")
    if name == "c5":
        n = 256 if n_images is None else n_images
        images = [uniform_image(rng, 1080, 1920, 3) if i % 2 == 0 else rgba_image(rng, 1080, 1920)
                  for i in range(n)]
        return dict(images=images, mean=IMAGENET_MEAN, std=IMAGENET_STD, dtype="f32", column_perm=True,
                    description=f"{n} x 1080x1920 half RGB / half RGBA -> 1088x1920, column perm")
    raise KeyError(name)


def random_small_batch(seed: int, n: int, max_side: int = 300, min_side: int = 1, rgba_fraction: float = 0.5,
                       sub_factor: bool = True):
    """Mixed small images for parity sweeps: sides in [min_side, max_side], C in {3, 4}.

    With ``sub_factor`` some images get a side below 32 to exercise the upscale
    branch. Shapes whose geometry is rejected (aspect above 200) are redrawn.
    """
    rng = rng_for(seed)
    images = []
    while len(images) < n:
        if sub_factor and rng.random() < 0.3:
            h = int(rng.integers(min_side, 32))
            w = int(rng.integers(min_side, max_side + 1))
            if rng.random() < 0.5:
                h, w = w, h
        else:
            h = int(rng.integers(max(min_side, 32), max_side + 1))
            w = int(rng.integers(max(min_side, 32), max_side + 1))
        if min(h, w) >= 32 and max(h, w) / min(h, w) > 200:
            continue
        if rng.random() < rgba_fraction:
            images.append(rgba_image(rng, h, w))
        else:
            images.append(uniform_image(rng, h, w, 3))
    return images
