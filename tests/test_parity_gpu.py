"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle, element by element.

Bars (from the method's definition and the arithmetic of both sides):
- geometry, image_grid_thw, row offsets and the column permutation: bit-exact;
- fp32 patch values: |gpu - oracle| <= 1e-4 in normalised units;
- bf16 patch values: within one bf16 ulp of the oracle value rounded to bf16, with the ulp taken no
  smaller than 2**-19 (below |v| ~ 2**-12 the fp32 rounding noise of the GPU arithmetic, ~1e-6, is
  larger than a bf16 ulp and may move the rounding by more than one step).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from _shrunk import shrunk_batch
from vision_lm_image_b200 import build, mimo

pytestmark = pytest.mark.gpu

FP32_ATOL = 1e-4
BF16_ULP_FLOOR = 2.0 ** -19


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    oracle.build()


def gpu_run(images, mean, std, dtype=torch.float32, column_perm=False, min_pixels=None, max_pixels=None):
    pv, grid, perm = mimo.preprocess(images, mean, std, min_pixels=min_pixels, max_pixels=max_pixels,
                                     dtype=dtype, column_perm=column_perm)
    torch.cuda.synchronize()
    return pv, grid.numpy(), perm


def assert_fp32_close(gpu: np.ndarray, ref: np.ndarray, what=""):
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), what
    err = np.abs(gpu.astype(np.float64) - ref.astype(np.float64))
    worst = float(err.max()) if err.size else 0.0
    assert worst <= FP32_ATOL, f"{what}: max |gpu - oracle| = {worst:.3e}"
    return worst


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v.astype(np.float64))
    e = np.floor(np.log2(np.maximum(a, 1e-30)))
    return np.maximum(2.0 ** (e - 7), BF16_ULP_FLOOR)


def assert_bf16_close(gpu_bf16: torch.Tensor, ref_f32: np.ndarray, what=""):
    g = gpu_bf16.float().cpu().numpy().astype(np.float64)
    r = oracle.bf16_bits_to_f32(oracle.round_to_bf16(ref_f32)).astype(np.float64)
    assert g.shape == r.shape
    bad = np.abs(g - r) > bf16_ulp(r)
    assert not bad.any(), f"{what}: {int(bad.sum())} values beyond 1 bf16 ulp"


def check_against_oracle(images, mean, std, threads=8, min_pixels=8192, max_pixels=8388608, perm=True):
    pv, grid, gperm = gpu_run(images, mean, std, column_perm=perm, min_pixels=min_pixels, max_pixels=max_pixels)
    ref, rgrid, rperm = oracle.preprocess(images, mean, std, min_pixels=min_pixels, max_pixels=max_pixels,
                                          column_perm=perm, threads=threads)
    assert np.array_equal(grid, rgrid)
    worst = assert_fp32_close(pv.cpu().numpy(), ref)
    if perm:
        assert np.array_equal(gperm.cpu().numpy(), rperm)
    return worst


# ---------------------------------------------------------------- the five workloads
def test_c1_single_upscaled_image():
    w = workloads.workload("c1")
    check_against_oracle(w["images"], w["mean"], w["std"])


def test_c2_rgba_identity_batch():
    w = workloads.workload("c2")
    check_against_oracle(w["images"], w["mean"], w["std"])


def test_c3_mixed_sizes_clip():
    w = workloads.workload("c3")
    check_against_oracle(w["images"], w["mean"], w["std"], threads=16)


def test_c4_max_pixels_downscale():
    w = workloads.workload("c4")
    check_against_oracle(w["images"], w["mean"], w["std"], perm=False)


def test_c5_full_size_sampled():
    """Full 256-image batch in the launch the benchmark times: exact permutation, two whole images
    against the oracle, random samples across all images, both temporal copies identical."""
    w = workloads.workload("c5")
    imgs = w["images"]
    pv, grid, perm = gpu_run(imgs, w["mean"], w["std"], column_perm=True)
    assert pv.shape == (256 * 8160, 1536)
    assert (grid == np.array([1, 68, 120])).all()
    # permutation: bit-exact for the whole batch
    rperm = np.concatenate([oracle.column_permutation(68, 120, 2, 8160 * i) for i in range(256)])
    assert np.array_equal(perm.cpu().numpy(), rperm)
    # both frames identical everywhere
    v = pv.view(-1, 3, 2, 256)
    assert torch.equal(v[:, :, 0], v[:, :, 1])
    # two whole images: one RGB (index 2), one RGBA (index 255)
    for i in (2, 255):
        ref, g = oracle.preprocess_image(imgs[i], w["mean"], w["std"])
        assert_fp32_close(pv[8160 * i:8160 * (i + 1)].cpu().numpy(), ref, f"image {i}")
    # samples across the whole batch
    rng = np.random.Generator(np.random.PCG64(55))
    n = 3000
    img_idx = rng.integers(0, 256, n)
    rows = rng.integers(0, 8160, n)
    cols = rng.integers(0, 1536, n)
    flat = (torch.from_numpy(img_idx * 8160 + rows) * 1536 + torch.from_numpy(cols)).cuda()
    got = pv.view(-1).index_select(0, flat).cpu().numpy()
    want = np.array([oracle.patch_value(imgs[i], (1088, 1920), int(r), int(c), w["mean"], w["std"])
                     for i, r, c in zip(img_idx, rows, cols)], np.float32)
    assert_fp32_close(got, want, "samples")


def test_c5_full_size_bf16_sampled():
    """The bf16 launch of the full batch (as `bench.py --dtype bf16` times it): sampled values within one
    bf16 ulp of the oracle, the permutation bit-exact, both frames identical."""
    w = workloads.workload("c5")
    imgs = w["images"]
    pv, grid, perm = gpu_run(imgs, w["mean"], w["std"], dtype=torch.bfloat16, column_perm=True)
    assert pv.shape == (256 * 8160, 1536) and pv.dtype == torch.bfloat16
    rperm = np.concatenate([oracle.column_permutation(68, 120, 2, 8160 * i) for i in range(256)])
    assert np.array_equal(perm.cpu().numpy(), rperm)
    v = pv.view(-1, 3, 2, 256)
    assert torch.equal(v[:, :, 0], v[:, :, 1])
    rng = np.random.Generator(np.random.PCG64(56))
    n = 3000
    img_idx = rng.integers(0, 256, n)
    rows = rng.integers(0, 8160, n)
    cols = rng.integers(0, 1536, n)
    flat = (torch.from_numpy(img_idx * 8160 + rows) * 1536 + torch.from_numpy(cols)).cuda()
    got = pv.view(-1).index_select(0, flat)
    want = np.array([oracle.patch_value(imgs[i], (1088, 1920), int(r), int(c), w["mean"], w["std"])
                     for i, r, c in zip(img_idx, rows, cols)], np.float32)
    assert_bf16_close(got, want, "bf16 samples")


def test_c5_bf16_subset():
    w = workloads.workload("c5", n_images=6)
    pv, grid, perm = gpu_run(w["images"], w["mean"], w["std"], dtype=torch.bfloat16, column_perm=True)
    ref, rgrid, rperm = oracle.preprocess(w["images"], w["mean"], w["std"], column_perm=True, threads=6)
    assert np.array_equal(grid, rgrid) and np.array_equal(perm.cpu().numpy(), rperm)
    assert_bf16_close(pv, ref, "c5 bf16")


def test_c3_bf16():
    w = workloads.workload("c3", n_images=12)
    pv, _, _ = gpu_run(w["images"], w["mean"], w["std"], dtype=torch.bfloat16)
    ref, _, _ = oracle.preprocess(w["images"], w["mean"], w["std"], threads=8)
    assert_bf16_close(pv, ref, "c3 bf16")


# ---------------------------------------------------------------- sweeps and edge cases
@pytest.mark.parametrize("seed", range(5))
def test_random_small_batches(seed):
    imgs = workloads.random_small_batch(900 + seed, 24, max_side=300, min_side=1)
    check_against_oracle(imgs, workloads.CLIP_MEAN, workloads.CLIP_STD)


def test_flatten_exhaustive_identity_image():
    # every (c, a) pair once: 256x256 RGBA is a multiple of 32 inside the bounds -> identity resize
    c = np.tile(np.arange(256, dtype=np.uint8), 256).reshape(256, 256)
    a = np.repeat(np.arange(256, dtype=np.uint8), 256).reshape(256, 256)
    img = np.stack([c, 255 - c, c // 2 + 7, a], axis=-1)
    check_against_oracle([img], workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)


def test_gathered_taps_strong_downscale():
    # a per-call max_pixels override makes the shrink factor > 2, so the kernel gathers taps
    rng = workloads.rng_for(5)
    imgs = [workloads.uniform_image(rng, 2000, 2000, 3), workloads.rgba_image(rng, 1500, 3000),
            workloads.uniform_image(rng, 3000, 700, 3)]
    check_against_oracle(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, max_pixels=200_000)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shrunk_batch_warp_staged_matches_oracle(dtype):
    # every row, the permutation and the index tables, in both row orders, against the oracle
    imgs = shrunk_batch(71, 9, 40_000)
    mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
    for order in ("merge", "column"):
        pv, grid, perm, pos, win = mimo.preprocess(imgs, mean, std, dtype=dtype, column_perm=True, order=order,
                                                   positions=True, window_index=True, max_pixels=40_000)
        torch.cuda.synchronize()
        ref, rgrid, rperm, rpos, rwin = oracle.preprocess(imgs, mean, std, column_perm=True, order=order,
                                                          positions=True, window=True, threads=8,
                                                          max_pixels=40_000)
        assert np.array_equal(grid.numpy(), rgrid)
        assert np.array_equal(perm.cpu().numpy(), rperm)
        assert np.array_equal(pos.cpu().numpy(), rpos)
        assert np.array_equal(win.cpu().numpy(), rwin)
        if dtype == torch.float32:
            assert_fp32_close(pv.cpu().numpy(), ref, order)
        else:
            assert_bf16_close(pv, ref, order)


def test_shrink_of_exactly_the_warp_staged_threshold():
    # c2's RGBA images under a 200,000-pixel budget: 480x640 -> 384x512, a shrink of exactly 1.25 on both
    # axes (4 H = 5 H', the dispatch's equality case), compositing onto white on the warp-staged kernel
    w = workloads.workload("c2")
    assert oracle.smart_resize(480, 640, max_pixels=200_000) == (384, 512)
    check_against_oracle(w["images"], w["mean"], w["std"], max_pixels=200_000)


def test_shrunk_batch_in_the_large_parameter_block():
    # more than 32 images: the launch carries the 512-image parameter block (the other instantiation)
    imgs = shrunk_batch(73, 40, 40_000, lo=250, hi=420)
    check_against_oracle(imgs, workloads.CLIP_MEAN, workloads.CLIP_STD, max_pixels=40_000)


@pytest.mark.parametrize("c", [3, 4])
def test_shrunk_image_ending_at_the_buffer_end(c):
    # a shrunk image (warp-staged kernel) whose last row ends exactly at the end of the declared buffer:
    # its 16-byte staging copies are cut there (zero-filled) and nothing past it is read
    h, w, mp = 411, 397, 60_000
    hr, wr = oracle.smart_resize(h, w, max_pixels=mp)
    assert 4 * h >= 5 * hr and 10 * h <= 19 * hr and 10 * w <= 19 * wr
    rng = workloads.rng_for(912)
    img = workloads.rgba_image(rng, h, w) if c == 4 else workloads.uniform_image(rng, h, w, 3)
    nbytes = h * w * c
    dev_buf = torch.zeros(nbytes + 4096, dtype=torch.uint8, device="cuda")
    dev_buf[:nbytes] = torch.from_numpy(img.reshape(-1)).cuda()
    dev_buf[nbytes:] = 255  # bytes beyond the declared end: never used
    params = mimo.make_params(max_pixels=mp)
    rows = (hr // 16) * (wr // 16)
    out = torch.empty((rows, 1536), dtype=torch.float32, device="cuda")
    offs = np.zeros(1, np.int64)
    hh, ww, cc = (np.array([v], np.int32) for v in (h, w, c))
    st = mimo.lib().mimo_preprocess_batch(ctypes.byref(params), 1, ctypes.c_void_p(dev_buf.data_ptr()), nbytes,
                                          offs.ctypes.data, hh.ctypes.data, ww.ctypes.data, cc.ctypes.data, 0,
                                          ctypes.c_void_p(out.data_ptr()), rows, None, None)
    assert st == 0
    torch.cuda.synchronize()
    ref, _ = oracle.preprocess_image(img, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, max_pixels=mp)
    assert_fp32_close(out.cpu().numpy(), ref, "buffer end")


def test_extreme_shapes():
    rng = workloads.rng_for(6)
    imgs = [workloads.uniform_image(rng, 1, 1, 3), workloads.rgba_image(rng, 1, 200),
            workloads.uniform_image(rng, 32, 6400, 3), workloads.rgba_image(rng, 6400, 32),
            workloads.uniform_image(rng, 31, 33, 3), workloads.uniform_image(rng, 33, 4001, 3)]
    check_against_oracle(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)


def test_sub_factor_shapes_with_truncated_long_side():
    # sub-factor shapes whose upscaled long side is not an integer: the truncating reading of smart_resize
    # gives other grids here than keeping the fraction would (e.g. 7x8 -> 96x96, not 96x128)
    rng = workloads.rng_for(8)
    shapes = [(7, 8), (13, 41), (7, 22), (31, 3984), (3984, 31), (13, 15), (17, 77), (21, 95), (8, 7), (41, 13),
              (31, 140), (5, 1234)]
    imgs = [workloads.uniform_image(rng, h, w, 3) if i % 2 == 0 else workloads.rgba_image(rng, h, w)
            for i, (h, w) in enumerate(shapes)]
    check_against_oracle(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    pv, grid, _ = gpu_run(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, dtype=torch.bfloat16)
    ref, rgrid, _ = oracle.preprocess(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    assert np.array_equal(grid, rgrid)
    assert [tuple(g) for g in grid[:2].tolist()] == [(1, 6, 6), (1, 4, 10)]
    assert_bf16_close(pv, ref, "sub-factor bf16")


def test_more_images_than_one_launch():
    # more than 512 images: the host cuts the batch into several launches
    rng = workloads.rng_for(7)
    imgs = [workloads.uniform_image(rng, int(rng.integers(20, 70)), int(rng.integers(20, 70)), 3 + i % 2)
            for i in range(1100)]
    check_against_oracle(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)


def test_coverage_sentinels():
    """Every row and permutation entry of the batch is written; nothing past the batch is."""
    imgs = workloads.random_small_batch(13, 9, max_side=250)
    params = mimo.make_params(workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    packed = mimo.pack_images(imgs, device="cuda")
    grid, offs = mimo.plan_batch(packed.heights, packed.widths, params)
    total = int(offs[-1])
    for dtype in (torch.float32, torch.bfloat16):
        out = torch.full((total + 37, 1536), float("nan"), dtype=dtype, device="cuda")
        perm = torch.full((total + 37,), -7, dtype=torch.int32, device="cuda")
        mimo.preprocess_batch(params, packed, out, perm)
        torch.cuda.synchronize()
        assert not torch.isnan(out[:total]).any()
        assert torch.isnan(out[total:]).all()
        assert (perm[total:] == -7).all()
        assert torch.equal(torch.sort(perm[:total]).values, torch.arange(total, device="cuda", dtype=torch.int32))


def test_empty_batch():
    pv, grid, perm = mimo.preprocess([], workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, column_perm=True)
    assert pv.shape == (0, 1536) and grid.shape == (0, 3) and perm.shape == (0,)


def test_nested_input_flattens_one_level():
    imgs = workloads.random_small_batch(14, 3, max_side=120)
    a, ga, _ = gpu_run(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    b, gb, _ = gpu_run([[imgs[0]], [imgs[1], imgs[2]]], workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    assert torch.equal(a, b) and np.array_equal(ga, gb)


def test_device_resident_inputs_and_streams():
    imgs = workloads.random_small_batch(15, 5, max_side=200)
    ref, _, _ = gpu_run(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dev_imgs = [torch.from_numpy(im).cuda() for im in imgs]
        out, _, _ = mimo.preprocess(dev_imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    s.synchronize()
    assert torch.equal(out, ref)


def test_host_buffer_entry_point_matches_device_path():
    w = workloads.workload("c5", n_images=5)
    params = mimo.make_params(w["mean"], w["std"])
    for dtype in (torch.float32, torch.bfloat16):
        ref, _, rperm = gpu_run(w["images"], w["mean"], w["std"], dtype=dtype, column_perm=True)
        host = mimo.pack_images(w["images"], device="cpu", pin_memory=True)
        _, offs = mimo.plan_batch(host.heights, host.widths, params)
        total = int(offs[-1])
        out_h = torch.empty((total, 1536), dtype=dtype, pin_memory=True)
        perm_h = torch.empty(total, dtype=torch.int32, pin_memory=True)
        src_d = torch.empty_like(host.buffer, device="cuda")
        out_d = torch.empty((total, 1536), dtype=dtype, device="cuda")
        perm_d = torch.empty(total, dtype=torch.int32, device="cuda")
        mimo.preprocess_batch_host(params, host, out_h, perm_h, src_d, out_d, perm_d)
        assert torch.equal(out_h, ref.cpu()) and torch.equal(perm_h, rperm.cpu())


def test_host_buffer_entry_point_chunks_of_several_images():
    # 60 images of mixed sizes: the host call's chunks grow from about 1/64 of the rows to an eighth,
    # several images each, so uploads, launches and downloads of different chunks interleave
    imgs = workloads.random_small_batch(29, 60, max_side=400)
    params = mimo.make_params(workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    ref, _, rperm = gpu_run(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD, column_perm=True)
    host = mimo.pack_images(imgs, device="cpu", pin_memory=True)
    _, offs = mimo.plan_batch(host.heights, host.widths, params)
    total = int(offs[-1])
    out_h = torch.full((total, 1536), float("nan"), pin_memory=True)
    perm_h = torch.full((total,), -1, dtype=torch.int32, pin_memory=True)
    src_d = torch.empty_like(host.buffer, device="cuda")
    out_d = torch.empty((total, 1536), device="cuda")
    perm_d = torch.empty(total, dtype=torch.int32, device="cuda")
    mimo.preprocess_batch_host(params, host, out_h, perm_h, src_d, out_d, perm_d)
    assert torch.equal(out_h, ref.cpu()) and torch.equal(perm_h, rperm.cpu())


def test_device_validation_errors():
    imgs = workloads.random_small_batch(16, 2, max_side=100)
    params = mimo.make_params()
    packed = mimo.pack_images(imgs, device="cuda")
    _, offs = mimo.plan_batch(packed.heights, packed.widths, params)
    total = int(offs[-1])
    out = torch.empty((total, 1536), device="cuda")
    with pytest.raises(mimo.MimoError) as e:
        mimo.preprocess_batch(params, packed, out[: total - 1])
    assert e.value.status == 7
    bad = mimo.PackedBatch(packed.buffer[: packed.buffer.numel() - 16], packed.offsets, packed.heights,
                           packed.widths, packed.channels)
    with pytest.raises(mimo.MimoError) as e:
        mimo.preprocess_batch(params, bad, out)
    assert e.value.status == 10
    wide = torch.empty((total + 1) * 1536 + 1, device="cuda")
    shifted = wide[1:1 + total * 1536].view(total, 1536)  # starts 4 bytes past a 16-byte boundary
    with pytest.raises(mimo.MimoError) as e:
        mimo.preprocess_batch(params, packed, shifted)
    assert e.value.status == 6


# ---------------------------------------------------------------- row order and index tables
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_column_order_and_tables_match_oracle(dtype):
    imgs = workloads.random_small_batch(301, 12, max_side=280, min_side=1)
    mean, std = workloads.CLIP_MEAN, workloads.CLIP_STD
    for order in ("merge", "column"):
        pv, grid, perm, pos, win = mimo.preprocess(imgs, mean, std, dtype=dtype, column_perm=True, order=order,
                                                   positions=True, window_index=True)
        torch.cuda.synchronize()
        ref, rgrid, rperm, rpos, rwin = oracle.preprocess(imgs, mean, std, column_perm=True, order=order,
                                                          positions=True, window=True, threads=8)
        assert np.array_equal(grid.numpy(), rgrid)
        assert np.array_equal(perm.cpu().numpy(), rperm)
        assert np.array_equal(pos.cpu().numpy(), rpos)
        assert np.array_equal(win.cpu().numpy(), rwin)
        if dtype == torch.float32:
            assert_fp32_close(pv.cpu().numpy(), ref, order)
        else:
            assert_bf16_close(pv, ref, order)


def _kept_width_batch(shapes, seed):
    rng = workloads.rng_for(seed)
    imgs = [workloads.rgba_image(rng, h, w) if c == 4 else workloads.uniform_image(rng, h, w, 3) for h, w, c in shapes]
    for h, w, _ in shapes:
        assert oracle.smart_resize(h, w)[1] == w  # every width kept: the unstaged kernel takes the launch
    return imgs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_kept_width_launches_match_oracle(dtype):
    # bf16 takes the unstaged kernel for any heights; fp32 only when every height is kept as well
    shapes = [(1079, 1920, 4), (1088, 640, 3), (97, 352, 4), (64, 160, 3), (720, 1280, 3), (1000, 96, 4)]
    if dtype == torch.float32:
        shapes = [(1088, 640, 3), (64, 160, 4), (704, 1280, 3), (96, 352, 4)]
    imgs = _kept_width_batch(shapes, 909)
    mean, std = workloads.CLIP_MEAN, workloads.CLIP_STD
    for order in ("merge", "column"):
        pv, grid, perm, pos, win = mimo.preprocess(imgs, mean, std, dtype=dtype, column_perm=True, order=order,
                                                   positions=True, window_index=True)
        torch.cuda.synchronize()
        ref, rgrid, rperm, rpos, rwin = oracle.preprocess(imgs, mean, std, column_perm=True, order=order,
                                                          positions=True, window=True, threads=8)
        assert np.array_equal(grid.numpy(), rgrid)
        assert np.array_equal(perm.cpu().numpy(), rperm)
        assert np.array_equal(pos.cpu().numpy(), rpos)
        assert np.array_equal(win.cpu().numpy(), rwin)
        if dtype == torch.float32:
            assert_fp32_close(pv.cpu().numpy(), ref, order)
        else:
            assert_bf16_close(pv, ref, order)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_kept_width_image_ending_at_the_buffer_end(dtype):
    # an RGB image whose last row ends exactly at the end of the buffer the caller declares: the
    # unstaged kernel's 16-byte word loads past it must read nothing there
    h, w = 96, 352
    img = _kept_width_batch([(h, w, 3)], 910)[0]
    nbytes = h * w * 3
    dev_buf = torch.zeros(nbytes + 4096, dtype=torch.uint8, device="cuda")
    dev_buf[:nbytes] = torch.from_numpy(img.reshape(-1)).cuda()
    dev_buf[nbytes:] = 255  # bytes beyond the declared end: never used
    params = mimo.make_params()
    rows = (h // 16) * (w // 16)
    out = torch.empty((rows, 1536), dtype=dtype, device="cuda")
    offs = np.zeros(1, np.int64)
    hh, ww, cc = (np.array([v], np.int32) for v in (h, w, 3))
    st = mimo.lib().mimo_preprocess_batch(ctypes.byref(params), 1, ctypes.c_void_p(dev_buf.data_ptr()), nbytes,
                                          offs.ctypes.data, hh.ctypes.data, ww.ctypes.data, cc.ctypes.data,
                                          1 if dtype == torch.bfloat16 else 0, ctypes.c_void_p(out.data_ptr()), rows,
                                          None, None)
    assert st == 0
    torch.cuda.synchronize()
    ref, _ = oracle.preprocess_image(img, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    if dtype == torch.float32:
        assert_fp32_close(out.cpu().numpy(), ref, "buffer end")
    else:
        assert_bf16_close(out, ref, "buffer end")


def test_column_order_is_a_row_gather_full_c5():
    w = workloads.workload("c5", n_images=8)
    a, _, perm = gpu_run(w["images"], w["mean"], w["std"], column_perm=True)
    b, _, _ = mimo.preprocess(w["images"], w["mean"], w["std"], order="column")
    torch.cuda.synchronize()
    assert torch.equal(b, a[perm.long()])


# ---------------------------------------------------------------- video frames
@pytest.mark.parametrize("n,shape,c", [(2, (48, 80), 3), (5, (31, 200), 4), (8, (120, 90), 3), (1, (64, 64), 4)])
def test_video_matches_oracle(n, shape, c):
    rng = workloads.rng_for(500 + n)
    frames = np.stack([workloads.uniform_image(rng, shape[0], shape[1], 3) if c == 3
                       else workloads.rgba_image(rng, shape[0], shape[1]) for _ in range(n)])
    mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
    ref, g = oracle.preprocess_video(frames, mean, std)
    for order in ("merge", "column"):
        pv, grid, perm, pos, win = mimo.preprocess_video(frames, mean, std, column_perm=True, order=order,
                                                         positions=True, window_index=True)
        torch.cuda.synchronize()
        assert tuple(grid[0].tolist()) == g
        gt, gh, gw = g
        rperm = np.concatenate([oracle.column_permutation(gh, gw, 2, 0, gt)])
        assert np.array_equal(perm.cpu().numpy(), rperm)
        assert np.array_equal(win.cpu().numpy(), oracle.window_index(gh, gw, 2, 0, gt))
        assert np.array_equal(pos.cpu().numpy(), oracle.rotary_positions(gh, gw, 2, order == "column", gt))
        want = ref if order == "merge" else ref[rperm]
        assert_fp32_close(pv.cpu().numpy(), want, f"video {order}")


@pytest.mark.parametrize("dtype,shape", [(torch.bfloat16, (100, 128)), (torch.float32, (96, 128)),
                                         (torch.float32, (100, 128)), (torch.bfloat16, (1080, 1920)),
                                         (torch.float32, (1080, 1920))])
@pytest.mark.parametrize("n,c", [(3, 3), (4, 4)])
def test_video_with_kept_width_matches_oracle(dtype, shape, n, c):
    # frames whose width is kept go to the unstaged kernel, in either dtype and whether or not the
    # height is resized: halves pick frame 2t + tt, an odd count repeats its last frame
    assert oracle.smart_resize(*shape)[1] == shape[1]
    rng = workloads.rng_for(700 + n + shape[0])
    frames = np.stack([workloads.uniform_image(rng, shape[0], shape[1], 3) if c == 3
                       else workloads.rgba_image(rng, shape[0], shape[1]) for _ in range(n)])
    mean, std = workloads.CLIP_MEAN, workloads.CLIP_STD
    ref, g = oracle.preprocess_video(frames, mean, std)
    gt, gh, gw = g
    for order in ("merge", "column"):
        pv, grid, perm, pos, win = mimo.preprocess_video(frames, mean, std, dtype=dtype, column_perm=True,
                                                         order=order, positions=True, window_index=True)
        torch.cuda.synchronize()
        assert tuple(grid[0].tolist()) == g
        rperm = oracle.column_permutation(gh, gw, 2, 0, gt)
        assert np.array_equal(perm.cpu().numpy(), rperm)
        assert np.array_equal(win.cpu().numpy(), oracle.window_index(gh, gw, 2, 0, gt))
        assert np.array_equal(pos.cpu().numpy(), oracle.rotary_positions(gh, gw, 2, order == "column", gt))
        want = ref if order == "merge" else ref[rperm]
        if dtype == torch.float32:
            assert_fp32_close(pv.cpu().numpy(), want, f"video {order}")
        else:
            assert_bf16_close(pv, want, f"video {order}")


def test_video_budget_and_bf16_full_hd():
    rng = workloads.rng_for(600)
    frames = np.stack([workloads.uniform_image(rng, 1080, 1920, 3) for _ in range(6)])
    mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
    total_max = 6 * 600_000
    ref, g = oracle.preprocess_video(frames, mean, std, total_max_pixels=total_max)
    pv, grid, _ = mimo.preprocess_video(frames, mean, std, total_max_pixels=total_max)
    torch.cuda.synchronize()
    assert tuple(grid[0].tolist()) == g
    assert_fp32_close(pv.cpu().numpy(), ref, "video fp32")
    pvb, _, _ = mimo.preprocess_video(frames, mean, std, total_max_pixels=total_max, dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert_bf16_close(pvb, ref, "video bf16")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_full_clip_in_the_benchmarked_launch(dtype):
    """The 64-frame 1080p clip through the raw call and buffer layout `bench.py --workload v1` times.
    With no video budget every temporal patch has the clip's geometry, so temporal patch t equals the
    oracle's clip of frames 2t and 2t+1: three whole temporal patches are compared."""
    w = workloads.video_workload("v1")
    frames = w["frames"]
    n, H, W, C = frames.shape
    params = mimo.make_params(w["mean"], w["std"])
    stride = (H * W * C + 15) // 16 * 16
    d_frames = torch.zeros(n * stride, dtype=torch.uint8, device="cuda")
    d_frames.view(n, stride)[:, :H * W * C].copy_(torch.from_numpy(frames.reshape(n, -1)))
    grid, rows = mimo.plan_video(n, H, W, w["total_max_pixels"], params)
    assert tuple(int(x) for x in grid) == (32, 68, 120) and rows == 32 * 8160
    out = torch.empty((rows, 1536), dtype=dtype, device="cuda")
    mimo.preprocess_video_raw(params, d_frames, n, stride, H, W, C, out, w["total_max_pixels"])
    torch.cuda.synchronize()
    for t in (0, 17, 31):
        ref, g = oracle.preprocess_video(frames[2 * t:2 * t + 2], w["mean"], w["std"])
        assert g == (1, 68, 120)
        got = out[8160 * t:8160 * (t + 1)]
        if dtype == torch.float32:
            assert_fp32_close(got.cpu().numpy(), ref, f"temporal patch {t}")
        else:
            assert_bf16_close(got, ref, f"temporal patch {t}")


def test_video_of_equal_frames_equals_the_image_path():
    img = workloads.random_small_batch(601, 1, max_side=300)[0]
    a, _, _ = gpu_run([img], workloads.CLIP_MEAN, workloads.CLIP_STD)
    b, g, _ = mimo.preprocess_video(np.stack([img, img]), workloads.CLIP_MEAN, workloads.CLIP_STD)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ---------------------------------------------------------------- patch embedding on the tensor cores
def _embed_ref(rows_bf16: torch.Tensor, w_bf16: torch.Tensor, bias):
    a = rows_bf16.float().cpu().numpy()
    w = w_bf16.float().cpu().numpy()
    ref = oracle.patch_embed(a, w, None if bias is None else bias.cpu().numpy())
    scale = np.abs(a.astype(np.float64)) @ np.abs(w.astype(np.float64)).T  # sum_k |a_k w_k|
    return ref, scale


def _assert_embed_close(got: torch.Tensor, ref, scale, what):
    g = got.float().cpu().numpy().astype(np.float64)
    tol = 1e-5 * scale + 1e-6 + (2.0 ** -8 * np.abs(ref) if got.dtype == torch.bfloat16 else 0.0)
    bad = np.abs(g - ref) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} beyond tolerance, worst {np.abs(g - ref).max():.3e}"


@pytest.mark.parametrize("M,N", [(1, 256), (128, 256), (129, 1280), (1000, 1280), (4113, 512)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_patch_embed_matches_oracle(M, N, out_dtype):
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N)
    rows = torch.randn((M, 1536), generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn((N, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
    bias = torch.randn(N, generator=g).cuda() if M % 2 else None
    out = mimo.patch_embed(rows, w, bias, out_dtype=out_dtype)
    ref, scale = _embed_ref(rows, w, bias)
    _assert_embed_close(out, ref, scale, f"M={M} N={N}")


def test_preprocess_then_patch_embed_chain():
    imgs = workloads.random_small_batch(700, 10, max_side=300, min_side=1)
    mean, std = workloads.CLIP_MEAN, workloads.CLIP_STD
    pv, grid, _ = mimo.preprocess(imgs, mean, std, dtype=torch.bfloat16)
    g = torch.Generator(device="cpu").manual_seed(1)
    w = (torch.randn((1280, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
    out = mimo.patch_embed(pv, w)
    # oracle chain: fp64 rows rounded to bf16 (the tower consumes bf16 rows), then the fp64 contraction
    ref_rows, _, _ = oracle.preprocess(imgs, mean, std, threads=8)
    a = oracle.bf16_bits_to_f32(oracle.round_to_bf16(ref_rows))
    ref = oracle.patch_embed(a, w.float().cpu().numpy())
    scale = np.abs(a.astype(np.float64)) @ np.abs(w.float().cpu().numpy().astype(np.float64)).T
    # the GPU's bf16 rows may differ from the oracle's by one bf16 ulp: allow that through the weights
    tol_rows = 2.0 ** -8 * scale
    g_out = out.float().cpu().numpy().astype(np.float64)
    tol = tol_rows + 1e-5 * scale + 2.0 ** -8 * np.abs(ref) + 1e-6
    assert (np.abs(g_out - ref) <= tol).all(), np.abs(g_out - ref).max()


def test_patch_embed_full_bench_size_sampled():
    # the launch `bench.py --workload pe` times: 2,088,960 rows, embed_dim 1280, ~551 tiles per CTA pair,
    # so every stage and accumulator phase bit wraps hundreds of times; sampled rows against the oracle
    M, N = 256 * 8160, 1280
    g = torch.Generator(device="cuda").manual_seed(11)
    rows = torch.randn((M, 1536), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((N, 1536), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    bias = torch.randn(N, generator=g, device="cuda")
    out = mimo.patch_embed(rows, w, bias)
    rng = np.random.Generator(np.random.PCG64(12))
    pick = np.unique(np.concatenate([[0, 255, 256, M - 256, M - 1], rng.integers(0, M, 120)]))
    idx = torch.from_numpy(pick).cuda()
    ref, scale = _embed_ref(rows.index_select(0, idx), w, bias)
    _assert_embed_close(out.index_select(0, idx), ref, scale, "full-size sample")
    del rows, out


@pytest.mark.parametrize("order", ["merge", "column"])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_preprocess_embed_equals_two_step(order, out_dtype):
    # chunked pixel path + GEMM through a small scratch (several runs) == the two calls on the whole batch
    imgs = workloads.random_small_batch(701, 12, max_side=400, min_side=1)
    mean, std = workloads.CLIP_MEAN, workloads.CLIP_STD
    g = torch.Generator(device="cpu").manual_seed(2)
    w = (torch.randn((512, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
    bias = torch.randn(512, generator=g).cuda()
    rows, grid, _ = mimo.preprocess(imgs, mean, std, dtype=torch.bfloat16, order=order)
    ref = mimo.patch_embed(rows, w, bias, out_dtype=out_dtype)
    biggest = int((grid[:, 1] * grid[:, 2]).max())
    emb, grid2 = mimo.preprocess_embed(imgs, w, bias, mean, std, out_dtype=out_dtype, order=order,
                                       scratch_bytes=2 * (biggest + 300) * 3072)
    assert torch.equal(grid, grid2)
    assert torch.equal(emb.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32),
                       ref.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32))


def test_preprocess_embed_shrunk_batch_equals_two_step():
    # images the warp-staged kernel takes, through the chained call (its bf16 rows stored L2 evict-last)
    imgs = shrunk_batch(74, 7, 40_000)
    mean, std = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
    g = torch.Generator(device="cpu").manual_seed(8)
    w = (torch.randn((512, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
    bias = torch.randn(512, generator=g).cuda()
    rows, grid, _ = mimo.preprocess(imgs, mean, std, dtype=torch.bfloat16, max_pixels=40_000)
    ref = mimo.patch_embed(rows, w, bias)
    biggest = int((grid[:, 1] * grid[:, 2]).max())
    emb, grid2 = mimo.preprocess_embed(imgs, w, bias, mean, std, max_pixels=40_000,
                                       scratch_bytes=2 * (biggest + 100) * 3072)
    assert torch.equal(grid, grid2)
    assert torch.equal(emb.view(torch.int16), ref.view(torch.int16))


def test_preprocess_embed_one_image_runs_equal_two_step():
    # 1080p images (8,160 rows: 160 GEMM tiles, a ragged last wave on the CTA pairs) through a scratch whose
    # halves hold exactly one image: five runs alternate over the two halves and their two library streams,
    # so consecutive GEMMs overlap; bit for bit the two calls on the whole batch
    w5 = workloads.workload("c5", n_images=5)
    g = torch.Generator(device="cpu").manual_seed(6)
    w = (torch.randn((1280, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
    bias = torch.randn(1280, generator=g).cuda()
    rows, grid, _ = mimo.preprocess(w5["images"], w5["mean"], w5["std"], dtype=torch.bfloat16)
    ref = mimo.patch_embed(rows, w, bias)
    for _ in range(2):  # the second call reuses the library's streams and events
        emb, grid2 = mimo.preprocess_embed(w5["images"], w, bias, w5["mean"], w5["std"],
                                           scratch_bytes=2 * 8160 * 3072)
        assert torch.equal(grid, grid2)
        assert torch.equal(emb.view(torch.int16), ref.view(torch.int16))


def test_preprocess_embed_c5_sample_against_oracle():
    # full-size geometry (1080x1920 -> 8160 rows each, RGB and RGBA), default scratch; sampled rows vs the oracle chain
    w5 = workloads.workload("c5", n_images=4)
    g = torch.Generator(device="cpu").manual_seed(4)
    w = (torch.randn((1280, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
    emb, grid = mimo.preprocess_embed(w5["images"], w, None, w5["mean"], w5["std"])
    rng = np.random.Generator(np.random.PCG64(9))
    wt = w.float().cpu().numpy()
    for i in (0, 3):
        rows = oracle.preprocess_image(w5["images"][i], w5["mean"], w5["std"])[0]
        pick = rng.choice(rows.shape[0], 64, replace=False)
        a = oracle.bf16_bits_to_f32(oracle.round_to_bf16(rows[pick]))
        ref = oracle.patch_embed(a, wt)
        scale = np.abs(a.astype(np.float64)) @ np.abs(wt.astype(np.float64)).T
        got = emb[i * 8160 + pick].float().cpu().numpy().astype(np.float64)
        tol = 2.0 ** -8 * scale + 1e-5 * scale + 2.0 ** -8 * np.abs(ref) + 1e-6
        assert (np.abs(got - ref) <= tol).all(), np.abs(got - ref).max()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_calls_replay_from_a_cuda_graph(dtype):
    # the launches a call makes can be captured once and replayed (planning runs at capture); replays on
    # new pixels in the same buffers equal fresh calls, for the staged and the unstaged kernel
    for seed, shapes in ((31, [(1079, 1920, 4), (1088, 640, 3)]), (32, [(300, 200, 3), (47, 512, 4)])):
        rng = workloads.rng_for(seed)
        make = lambda: [workloads.rgba_image(rng, h, w) if c == 4 else workloads.uniform_image(rng, h, w, 3)
                        for h, w, c in shapes]
        params = mimo.make_params(workloads.CLIP_MEAN, workloads.CLIP_STD)
        packed = mimo.pack_images(make(), device="cuda")
        grid, offs = mimo.plan_batch(packed.heights, packed.widths, params)
        total = int(offs[-1])
        out = torch.empty((total, 1536), dtype=dtype, device="cuda")
        perm = torch.empty(total, dtype=torch.int32, device="cuda")
        g = torch.Generator(device="cpu").manual_seed(seed)
        w = (torch.randn((256, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
        emb = torch.empty((total, 256), dtype=torch.bfloat16, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        rows_bf16 = out if dtype == torch.bfloat16 else None
        mimo.preprocess_batch_ex(params, packed, out, perm)  # warm-up outside the capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            mimo.preprocess_batch_ex(params, packed, out, perm)
            if rows_bf16 is not None:
                mimo.patch_embed(rows_bf16, w, None, out=emb, error=err, check=False)
        # new pixels into the same device buffer, then replay
        fresh = mimo.pack_images(make(), device="cpu")
        packed.buffer.copy_(fresh.buffer)
        graph.replay()
        torch.cuda.synchronize()
        imgs = [np.ascontiguousarray(x) for x in _unpack(fresh)]
        want_rows, _, want_perm = mimo.preprocess(imgs, workloads.CLIP_MEAN, workloads.CLIP_STD, dtype=dtype,
                                                  column_perm=True)
        assert torch.equal(perm, want_perm)
        assert torch.equal(out.view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                           want_rows.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))
        if rows_bf16 is not None:
            assert int(err.item()) == 0
            assert torch.equal(emb.view(torch.int16), mimo.patch_embed(want_rows, w).view(torch.int16))
        del graph


def _unpack(packed):
    """The HWC images of a host PackedBatch."""
    buf = packed.buffer.numpy()
    return [buf[o:o + h * w * c].reshape(h, w, c)
            for o, h, w, c in zip(packed.offsets, packed.heights, packed.widths, packed.channels)]


# ---------------------------------------------------------------- merge-unit windows (multi-device split)
def _full_and_windows(images, mean, std, dtype, windows):
    """One mimo_preprocess_batch_ex call over the batch, and the same batch as unit windows."""
    params = mimo.make_params(mean, std)
    packed = mimo.pack_images(images, device="cuda")
    _, offs = mimo.plan_batch(packed.heights, packed.widths, params)
    total = int(offs[-1])
    ref = torch.empty((total, 1536), dtype=dtype, device="cuda")
    rperm = torch.empty(total, dtype=torch.int32, device="cuda")
    rpos = torch.empty((total, 2), dtype=torch.int32, device="cuda")
    rwin = torch.empty(total // 4, dtype=torch.int32, device="cuda")
    mimo.preprocess_batch_ex(params, packed, ref, rperm, rpos, rwin)
    perm = torch.full((total,), -1, dtype=torch.int32, device="cuda")
    win = torch.full((total // 4,), -1, dtype=torch.int32, device="cuda")
    parts, pos_parts = [], []
    for first, count in windows:
        out = torch.full((4 * count, 1536), float("nan"), dtype=dtype, device="cuda")
        pos = torch.full((4 * count, 2), -1, dtype=torch.int32, device="cuda")
        mimo.preprocess_units(params, packed, first, count, out, perm, pos, win)
        parts.append(out)
        pos_parts.append(pos)
    torch.cuda.synchronize()
    return (ref, rperm, rpos, rwin), (torch.cat(parts), perm, torch.cat(pos_parts), win), total


@pytest.mark.parametrize("split", ["halves", "ragged"])
def test_unit_windows_reproduce_one_large_image(split):
    # c4: one 4096x4096 image (8100 merge units) cut by merge-block ranges, warp-staged kernel
    w = workloads.workload("c4")
    windows = [(0, 4050), (4050, 4050)] if split == "halves" else [(0, 1), (1, 89), (90, 3911), (4001, 4099)]
    (ref, rperm, rpos, rwin), (got, perm, pos, win), total = _full_and_windows(
        w["images"], w["mean"], w["std"], torch.float32, windows)
    assert total == 32400
    assert torch.equal(got, ref)
    assert torch.equal(perm, rperm) and torch.equal(pos, rpos) and torch.equal(win, rwin)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_unit_windows_random_batches_both_kernels(dtype):
    rng = np.random.Generator(np.random.PCG64(61))
    # resized batch (staged kernel) and a kept-width batch (unstaged kernel in bf16)
    batches = [workloads.random_small_batch(62, 11, max_side=300, min_side=1), _kept_width_batch(
        [(96, 128, 3), (200, 64, 4), (130, 96, 3), (64, 160, 4)], 63)]
    for images in batches:
        params = mimo.make_params(workloads.CLIP_MEAN, workloads.CLIP_STD)
        hs = [im.shape[0] for im in images]
        ws = [im.shape[1] for im in images]
        units = int(mimo.plan_batch(hs, ws, params)[1][-1]) // 4
        cuts = sorted(set(int(c) for c in rng.integers(1, units, size=4)))
        bounds = [0] + cuts + [units]
        windows = [(bounds[k], bounds[k + 1] - bounds[k]) for k in range(len(bounds) - 1)]
        (ref, rperm, rpos, rwin), (got, perm, pos, win), _ = _full_and_windows(
            images, workloads.CLIP_MEAN, workloads.CLIP_STD, dtype, windows)
        assert torch.equal(got, ref)
        assert torch.equal(perm, rperm) and torch.equal(pos, rpos) and torch.equal(win, rwin)
    # the last batch's rows against the oracle too (one bf16 ulp / 1e-4)
    oref, _, operm = oracle.preprocess(images, workloads.CLIP_MEAN, workloads.CLIP_STD, column_perm=True)
    assert np.array_equal(perm.cpu().numpy(), operm)
    if dtype == torch.float32:
        assert_fp32_close(got.cpu().numpy(), oref, "windows")
    else:
        assert_bf16_close(got, oref, "windows")


def test_unit_windows_errors():
    w = workloads.workload("c1")
    params = mimo.make_params(w["mean"], w["std"])
    packed = mimo.pack_images(w["images"], device="cuda")
    out = torch.empty((48, 1536), dtype=torch.float32, device="cuda")
    with pytest.raises(mimo.MimoError) as e:   # the image has 12 units
        mimo.preprocess_units(params, packed, 10, 3, out)
    assert e.value.status == 10
    with pytest.raises(mimo.MimoError) as e:   # 8 rows of room for 3 units
        mimo.preprocess_units(params, packed, 0, 3, out[:8])
    assert e.value.status == 7
    o = mimo.MimoOutputs()
    o.out_dtype, o.row_order, o.d_out, o.out_rows_capacity = mimo.F32, mimo.ORDER_COLUMN, out.data_ptr(), 48
    buf = packed.buffer
    st = mimo.lib().mimo_preprocess_units(ctypes.byref(params), packed.n, ctypes.c_void_p(buf.data_ptr()), buf.numel(),
                                          *packed.ptrs, 0, 12, ctypes.byref(o), None)
    assert st == 5  # column order is not offered for windows
    mimo.preprocess_units(params, packed, 3, 0, out)  # an empty window launches nothing


# ---------------------------------------------------------------- failure path of the tensor-core kernel
def test_patch_embed_wait_runs_out_and_the_next_launch_is_correct():
    """The operand loader stops after 3 of the 24 K blocks and every wait gives up after 2^14 polling
    rounds: the kernel must return with a nonzero status word (operands or accumulator never came), not
    hang; a normal launch right after must be correct, so the failed launch gave its tensor memory back."""
    M, N = 1024, 512
    g = torch.Generator(device="cpu").manual_seed(91)
    rows = torch.randn((M, 1536), generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn((N, 1536), generator=g) * 0.02).to(torch.bfloat16).cuda()
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    st = mimo.lib().mimo_patch_embed_stall_test(
        ctypes.c_void_p(rows.data_ptr()), M, ctypes.c_void_p(w.data_ptr()), N, None, mimo.BF16,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(err.data_ptr()), 3, 1 << 14,
        ctypes.c_void_p(stream.cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert int(err.item()) in (1, 3), int(err.item())
    # bad hook arguments are rejected on the host
    for stop, rounds in ((-1, 100), (25, 100), (3, 0)):
        assert mimo.lib().mimo_patch_embed_stall_test(
            ctypes.c_void_p(rows.data_ptr()), M, ctypes.c_void_p(w.data_ptr()), N, None, mimo.BF16,
            ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(err.data_ptr()), stop, rounds, None) == 1
    # the next normal launches on the same device are complete and correct
    for out_dtype in (torch.bfloat16, torch.float32):
        emb = mimo.patch_embed(rows, w, out_dtype=out_dtype)
        ref, scale = _embed_ref(rows, w, None)
        _assert_embed_close(emb, ref, scale, "after a stalled launch")
