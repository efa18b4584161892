"""The no-allocation host entry point, checked against the host entry point with caller staging.

mimo_preprocess_batch_host_noalloc serves callers that cannot allocate device memory, such as code
running while another framework owns the device allocator. It stages images and rows through a
fixed device array compiled into the library instead of caller-provided buffers. These tests call
it through the C ABI and compare its rows and permutation with those of
mimo_preprocess_batch_host, within the fp32 parity tolerance (1e-4; equality is expected, because
both run the same kernel). There are two calls in a row: the second, smaller batch finds the first
call's bytes still in the shared array, and its rows are also checked against the CPU oracle (1e-4 for
fp32, one bf16 ulp of the rounded oracle value for bf16) and its permutation bit for bit. The file
sorts last so that a run stopping at the first failure has already run every other test; it also
passes when run alone.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from vision_lm_image_b200 import build, mimo

pytestmark = pytest.mark.gpu

FP32_ATOL = 1e-4
BF16_ULP_FLOOR = 2.0 ** -19  # the GPU parity tests' floor on the bf16 ulp


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    oracle.build()


def _assert_matches_oracle(images, mean, std, got_out, got_perm, dtype):
    ref, _, rperm = oracle.preprocess(images, mean, std, column_perm=True, threads=8)
    assert np.array_equal(got_perm.numpy(), rperm)
    if dtype == torch.float32:
        assert float(np.abs(got_out.numpy().astype(np.float64) - ref).max()) <= FP32_ATOL
    else:
        r = oracle.bf16_bits_to_f32(oracle.round_to_bf16(ref)).astype(np.float64)
        a = np.abs(r)
        ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(a, 1e-30))) - 7), BF16_ULP_FLOOR)
        assert (np.abs(got_out.float().numpy().astype(np.float64) - r) <= ulp).all()


def _host_batch(images):
    return mimo.pack_images(images, device="cpu", pin_memory=True)


def _reference(params, host, dtype, total):
    """mimo_preprocess_batch_host with caller-provided device staging buffers."""
    out_h = torch.empty((total, 1536), dtype=dtype, pin_memory=True)
    perm_h = torch.empty(total, dtype=torch.int32, pin_memory=True)
    src_d = torch.empty_like(host.buffer, device="cuda")
    out_d = torch.empty((total, 1536), dtype=dtype, device="cuda")
    perm_d = torch.empty(total, dtype=torch.int32, device="cuda")
    mimo.preprocess_batch_host(params, host, out_h, perm_h, src_d, out_d, perm_d)
    return out_h, perm_h


def _noalloc(params, host, dtype, total):
    """The entry point under test, called through the C ABI."""
    out_h = torch.full((total, 1536), float("nan"), dtype=dtype, pin_memory=True)
    perm_h = torch.full((total,), -1, dtype=torch.int32, pin_memory=True)
    buf = host.buffer
    st = mimo.lib().mimo_preprocess_batch_host_noalloc(
        ctypes.byref(params), host.n, ctypes.c_void_p(buf.data_ptr()), buf.numel(), host.offsets.ctypes.data,
        host.heights.ctypes.data, host.widths.ctypes.data, host.channels.ctypes.data,
        mimo.F32 if dtype == torch.float32 else mimo.BF16, ctypes.c_void_p(out_h.data_ptr()), total,
        ctypes.c_void_p(perm_h.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, mimo.lib().mimo_status_string(st)
    return out_h, perm_h


def _batches():
    # first call: three c5-sized images (one staging chunk each) plus small mixed ones;
    # second call: a smaller batch, so stale bytes of the first remain in the array
    big = workloads.workload("c5", n_images=3)
    first = big["images"] + workloads.random_small_batch(71, 9, max_side=400, min_side=1)
    second = workloads.random_small_batch(72, 7, max_side=250, min_side=1)
    return [(first, big["mean"], big["std"]), (second, workloads.CLIP_MEAN, workloads.CLIP_STD)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_host_entry_point_twice(dtype):
    for k, (images, mean, std) in enumerate(_batches()):
        params = mimo.make_params(mean, std)
        host = _host_batch(images)
        _, offs = mimo.plan_batch(host.heights, host.widths, params)
        total = int(offs[-1])
        ref_out, ref_perm = _reference(params, host, dtype, total)
        got_out, got_perm = _noalloc(params, host, dtype, total)
        assert torch.equal(got_perm, ref_perm)
        diff = (got_out.float() - ref_out.float()).abs().max().item()
        assert diff <= FP32_ATOL, diff
        if k == 1:
            _assert_matches_oracle(images, mean, std, got_out, got_perm, dtype)


def test_noalloc_rejects_an_image_beyond_the_staging_size():
    # 4096x4096 RGB resizes to 2880x2880: ~199 MB of fp32 rows, more than the fixed area
    img = workloads.gradient_noise_image(workloads.rng_for(3), 4096, 4096)
    params = mimo.make_params()
    host = _host_batch([img])
    _, offs = mimo.plan_batch(host.heights, host.widths, params)
    total = int(offs[-1])
    out_h = torch.empty((total, 1536), dtype=torch.float32)
    with pytest.raises(mimo.MimoError) as e:
        mimo.preprocess_batch_host_noalloc(params, host, out_h)
    assert e.value.status == 11
    assert mimo.NOALLOC_STAGING_BYTES == 64 << 20
