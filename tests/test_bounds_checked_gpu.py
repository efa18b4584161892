"""The pixel kernels of the bounds-checked debug build (-DMIMO_BOUNDS_CHECK) on the parity sweeps.

compute-sanitizer is not available on the GPU pool these tests run on, so the library carries its own
check: in the debug build every global load and store of the three pixel kernels, and their shared-memory
tile and staging indices, are checked against the extents the host validated (the image and the caller's
source buffer, the output rows, the permutation / position / window tables). A failed check skips the
access and counts it; it never traps. These tests run the small-batch sweeps, the kept-width (unstaged
kernel) batches, shrunk batches (warp-staged kernel), images ending exactly at the end of the source
buffer, a video, merge-unit windows and every table through the debug build, and require zero failed
checks and outputs bit-identical to the release build.
"""
import numpy as np
import pytest
import torch

import workloads
from _shrunk import shrunk_batch
from vision_lm_image_b200 import build, mimo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def checked():
    build.build()
    return build.build_checked()


def _all_outputs(images, mean, std, dtype, order="merge", **kw):
    pv, grid, perm, pos, win = mimo.preprocess(images, mean, std, dtype=dtype, column_perm=True, order=order,
                                               positions=True, window_index=True, **kw)
    torch.cuda.synchronize()
    return pv, perm, pos, win


def _compare(images, mean, std, dtype, checked, order="merge", **kw):
    ref = _all_outputs(images, mean, std, dtype, order, **kw)
    with mimo.use_library(checked):
        assert mimo.bounds_check_status() == (0, 0)  # a fresh query starts clean
        got = _all_outputs(images, mean, std, dtype, order, **kw)
        status = mimo.bounds_check_status()
    assert status == (0, 0), f"{status[0]} failed bounds checks, first of kind {status[1]}"
    for a, b in zip(ref, got):
        assert torch.equal(a, b)


def test_release_build_reports_no_checks():
    build.build()
    with pytest.raises(mimo.MimoError) as e:
        mimo.bounds_check_status()
    assert e.value.status == 5  # MIMO_EUNSUPPORTED


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_small_batches_pass_every_check(checked, seed, dtype):
    imgs = workloads.random_small_batch(1300 + seed, 20, max_side=300, min_side=1)
    _compare(imgs, workloads.CLIP_MEAN, workloads.CLIP_STD, dtype, checked, order="column" if seed == 1 else "merge")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_kept_width_and_strong_downscale_pass_every_check(checked, dtype):
    rng = workloads.rng_for(1310)
    imgs = [workloads.rgba_image(rng, 200, 64), workloads.uniform_image(rng, 130, 96, 3),
            workloads.uniform_image(rng, 96, 352, 3), workloads.rgba_image(rng, 64, 160)]
    _compare(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, dtype, checked)
    # gathered taps (scale > 2) under a small max_pixels
    big = [workloads.uniform_image(rng, 1500, 1100, 3), workloads.rgba_image(rng, 900, 2100)]
    ref = mimo.preprocess(big, max_pixels=150_000, dtype=dtype, column_perm=True)
    with mimo.use_library(checked):
        got = mimo.preprocess(big, max_pixels=150_000, dtype=dtype, column_perm=True)
        torch.cuda.synchronize()
        assert mimo.bounds_check_status() == (0, 0)
    assert torch.equal(ref[0], got[0]) and torch.equal(ref[2], got[2])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shrunk_batches_pass_every_check(checked, dtype):
    # every height shrunk by 1.25 to 1.9 (warp-staged kernel), RGB and RGBA, both row orders
    imgs = shrunk_batch(1340, 8, 40_000)
    for order in ("merge", "column"):
        _compare(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, dtype, checked, order=order,
                 max_pixels=40_000)


@pytest.mark.parametrize("kept", [False, True])
def test_image_ending_at_the_buffer_end_passes_every_check(checked, kept):
    # the last image's final byte is the last byte of the source buffer: staged copies of 16-byte chunks
    # and 12/16-byte quads must stop there (kept: the unstaged kernel; else the staged kernel, then the
    # same batch shrunk by max_pixels for the warp-staged kernel)
    rng = workloads.rng_for(1320)
    shape = (64, 96) if kept else (61, 95)
    imgs = [workloads.uniform_image(rng, 40, 50, 3), workloads.uniform_image(rng, *shape, 3)]
    _buffer_end_case(imgs, shape, mimo.make_params(), checked)
    if not kept:
        big = (411, 397)
        imgs = [workloads.uniform_image(rng, 300, 350, 3), workloads.uniform_image(rng, *big, 3)]
        _buffer_end_case(imgs, big, mimo.make_params(max_pixels=60_000), checked)


def _buffer_end_case(imgs, shape, params, checked):
    host = mimo.pack_images(imgs, device="cpu")
    end = int(host.offsets[-1]) + shape[0] * shape[1] * 3
    packed = mimo.pack_images(imgs, device="cuda")
    packed.buffer = packed.buffer[:end]  # no padding after the last image
    _, offs = mimo.plan_batch(host.heights, host.widths, params)
    total = int(offs[-1])
    outs = []
    for lib_path in (None, checked):
        out = torch.empty((total, 1536), dtype=torch.float32, device="cuda")
        perm = torch.empty(total, dtype=torch.int32, device="cuda")
        if lib_path is None:
            mimo.preprocess_batch_ex(params, packed, out, perm)
        else:
            with mimo.use_library(lib_path):
                mimo.preprocess_batch_ex(params, packed, out, perm)
                torch.cuda.synchronize()
                assert mimo.bounds_check_status() == (0, 0)
        outs.append((out, perm))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_kept_width_video_passes_every_check(checked, dtype):
    # width 128 kept, height 100 -> 96 resized: the unstaged kernel in either dtype; each clip's last
    # frame ends at the end of its frame buffer
    rng = workloads.rng_for(1332)
    for frames in (np.stack([workloads.rgba_image(rng, 100, 128) for _ in range(5)]),
                   np.stack([workloads.uniform_image(rng, 100, 128, 3) for _ in range(4)])):
        ref = mimo.preprocess_video(frames, dtype=dtype)
        with mimo.use_library(checked):
            got = mimo.preprocess_video(frames, dtype=dtype)
            torch.cuda.synchronize()
            assert mimo.bounds_check_status() == (0, 0)
        assert torch.equal(ref[0], got[0])


def test_video_and_unit_windows_pass_every_check(checked):
    rng = workloads.rng_for(1330)
    frames = np.stack([workloads.rgba_image(rng, 70, 90) for _ in range(5)])
    ref = mimo.preprocess_video(frames, dtype=torch.float32)
    with mimo.use_library(checked):
        got = mimo.preprocess_video(frames, dtype=torch.float32)
        torch.cuda.synchronize()
        assert mimo.bounds_check_status() == (0, 0)
    assert torch.equal(ref[0], got[0])
    # merge-unit windows that start and end inside images
    imgs = workloads.random_small_batch(1331, 6, max_side=200, min_side=20)
    params = mimo.make_params()
    packed = mimo.pack_images(imgs, device="cuda")
    _, offs = mimo.plan_batch(packed.heights, packed.widths, params)
    total = int(offs[-1])
    units = total // 4
    with mimo.use_library(checked):
        perm = torch.empty(total, dtype=torch.int32, device="cuda")
        win = torch.empty(units, dtype=torch.int32, device="cuda")
        for first, count in ((0, units // 3), (units // 3, units - units // 3)):
            out = torch.empty((4 * count, 1536), dtype=torch.bfloat16, device="cuda")
            pos = torch.empty((4 * count, 2), dtype=torch.int32, device="cuda")
            mimo.preprocess_units(params, packed, first, count, out, perm, pos, win)
        torch.cuda.synchronize()
        assert mimo.bounds_check_status() == (0, 0)
