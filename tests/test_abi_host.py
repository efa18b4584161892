"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

- the library loads and exports every function include/mimo.h declares;
- the library's own smart_resize / plan agree bit for bit with the oracle's;
- argument validation returns the documented status before any device work.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import workloads
from vision_lm_image_b200 import build, mimo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(mimo_[a-z_0-9]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert {"mimo_smart_resize", "mimo_preprocess_batch", "mimo_plan_batch"} <= names
    L = ctypes.CDLL(mimo.library_path())
    for name in sorted(names):
        assert hasattr(L, name), name
    assert set(mimo.EXPORTED) == names


def header_enum_values():
    text = open(os.path.join(ROOT, "include", "mimo.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return {k: int(v) for k, v in re.findall(r"\b(MIMO_[A-Z0-9_]+)\s*=\s*(\d+)", text)}


def test_version_and_status_strings():
    L = mimo.lib()
    assert L.mimo_version() >= 10000
    statuses = {k: v for k, v in header_enum_values().items() if k == "MIMO_OK" or k.startswith("MIMO_E")}
    for s in statuses.values():
        assert L.mimo_status_string(s) and L.mimo_status_string(s) != b"unknown status"
    assert L.mimo_status_string(max(statuses.values()) + 1) == b"unknown status"


def test_binding_constants_match_the_header():
    enums = header_enum_values()
    assert {v: k for k, v in enums.items() if k == "MIMO_OK" or k.startswith("MIMO_E")} == mimo.STATUS_NAMES
    assert (enums["MIMO_F32"], enums["MIMO_BF16"]) == (mimo.F32, mimo.BF16)
    assert (enums["MIMO_ORDER_MERGE"], enums["MIMO_ORDER_COLUMN"]) == (mimo.ORDER_MERGE, mimo.ORDER_COLUMN)
    text = open(os.path.join(ROOT, "include", "mimo.h")).read()
    m = re.search(r"#define MIMO_NOALLOC_STAGING_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == mimo.NOALLOC_STAGING_BYTES


def test_ctypes_structs_match_the_c_layout(tmp_path):
    """The binding's ctypes mirrors of mimo_params and mimo_outputs have the C compiler's sizes and offsets."""
    structs = {"mimo_params": mimo.MimoParams, "mimo_outputs": mimo.MimoOutputs}
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "mimo.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'    printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'    printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["    return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    import subprocess

    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = {}
    for line in subprocess.check_output([str(exe)], text=True).splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for cname, cls in structs.items():
        assert got[(cname, "sizeof")] == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert got[(cname, field)] == getattr(cls, field).offset, (cname, field)


def test_defaults_match_processor_constructor():
    p = mimo.make_params()
    assert (p.patch_size, p.temporal_patch_size, p.merge_size) == (16, 2, 2)
    assert (p.min_pixels, p.max_pixels) == (8192, 8388608)
    assert np.allclose(list(p.image_mean), workloads.IMAGENET_MEAN)
    assert np.allclose(list(p.image_std), workloads.IMAGENET_STD)


def test_smart_resize_matches_oracle_exhaustive():
    for h in range(1, 200):
        for w in range(1, 200, 7):
            assert mimo.smart_resize_status(h, w) == oracle.smart_resize_status(h, w)
            if oracle.smart_resize_status(h, w) == oracle.OK:
                assert mimo.smart_resize(h, w) == oracle.smart_resize(h, w), (h, w)


@pytest.mark.parametrize("bounds", [(8192, 8388608), (50_000, 200_000), (0, 1 << 40), (8192, 30_000)])
def test_smart_resize_matches_oracle_random(bounds):
    mn, mx = bounds
    rng = np.random.Generator(np.random.PCG64(21))
    for _ in range(5000):
        h = int(np.exp(rng.uniform(0, np.log(60000))))
        w = int(np.exp(rng.uniform(0, np.log(60000))))
        for factor in (32, 28):
            so = oracle.smart_resize_status(h, w, factor, mn, mx)
            assert mimo.smart_resize_status(h, w, factor, mn, mx) == so, (h, w, factor)
            if so == oracle.OK:
                assert mimo.smart_resize(h, w, factor, mn, mx) == oracle.smart_resize(h, w, factor, mn, mx)


def test_plan_batch_matches_oracle():
    imgs = workloads.random_small_batch(77, 40, max_side=400)
    H = [im.shape[0] for im in imgs]
    W = [im.shape[1] for im in imgs]
    grid, offs = mimo.plan_batch(H, W)
    assert offs[0] == 0
    for i, (h, w) in enumerate(zip(H, W)):
        oh, ow = oracle.smart_resize(h, w)
        assert tuple(grid[i]) == (1, oh // 16, ow // 16)
        assert offs[i + 1] - offs[i] == oracle.get_number_of_image_patches(h, w)
    assert mimo.get_number_of_image_patches(1080, 1920) == 8160


def test_plan_batch_errors():
    with pytest.raises(mimo.MimoError) as e:
        mimo.plan_batch([32], [6401])
    assert e.value.status == 2
    with pytest.raises(mimo.MimoError) as e:
        mimo.plan_batch([16], [300000])
    assert e.value.status == 3
    with pytest.raises(mimo.MimoError) as e:
        mimo.plan_batch([0], [5])
    assert e.value.status == 1
    with pytest.raises(mimo.MimoError) as e:
        mimo.plan_batch([64], [64], mimo.make_params(patch_size=14))
    assert e.value.status == 5
    g, o = mimo.plan_batch([], [])
    assert g.shape == (0, 3) and list(o) == [0]
    # a sub-factor sliver upscaled past 2^30 columns (only reachable with a huge max_pixels)
    big = mimo.make_params(max_pixels=1 << 36)
    assert oracle.smart_resize(16, (1 << 29) + 1000, 32, 8192, 1 << 36)[1] >= 1 << 30
    with pytest.raises(mimo.MimoError) as e:
        mimo.plan_batch([16], [(1 << 29) + 1000], big)
    assert e.value.status == 8
    assert mimo.plan_batch([16], [(1 << 28)], big)[0][0, 2] == (1 << 29) // 16


# Validation-only calls: every call below must fail before launching. They are
# run only where no GPU is present, so a validation bug cannot send a bogus
# pointer to a real device.
no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(), reason="host-validation test uses fake device pointers")

FAKE = 1 << 20  # 16-byte aligned, never dereferenced


def _call(p=None, n=1, src=FAKE, src_bytes=1 << 30, offsets=(0,), H=(64,), W=(48,), C=(3,), dtype=0,
          out=FAKE, cap=1 << 20, perm=0):
    p = p or mimo.make_params()
    offs = np.asarray(offsets, np.int64)
    h = np.asarray(H, np.int32)
    w = np.asarray(W, np.int32)
    c = np.asarray(C, np.int32)
    return mimo.lib().mimo_preprocess_batch(ctypes.byref(p), n, ctypes.c_void_p(src), src_bytes, offs.ctypes.data,
                                            h.ctypes.data, w.ctypes.data, c.ctypes.data, dtype,
                                            ctypes.c_void_p(out), cap, ctypes.c_void_p(perm), None)


@no_gpu_only
def test_validation_statuses():
    assert _call(n=0) == 0                                  # empty batch: nothing to do
    assert _call(C=(2,)) == 4                               # channels
    assert _call(offsets=(8,)) == 6                         # misaligned offset
    assert _call(src=FAKE + 4) == 6                         # misaligned base
    assert _call(out=FAKE + 8) == 6                         # misaligned output
    assert _call(perm=FAKE + 4) == 6                        # misaligned permutation
    assert _call(cap=47) == 7                               # 64x48 -> 48 rows
    assert _call(src_bytes=64 * 48 * 3 - 1) == 10           # image past the end of the buffer
    assert _call(offsets=(16,), src_bytes=64 * 48 * 3) == 10
    assert _call(H=(32,), W=(6401,)) == 2                   # aspect
    assert _call(H=(16,), W=(300000,)) == 3                 # degenerate shrink
    assert _call(dtype=7) == 1                              # dtype
    assert _call(n=-1) == 1
    assert _call(out=0) == 1
    p = mimo.make_params(std=(0.2, 0.0, 0.2))
    assert _call(p=p) == 5                                  # std must be > 0
    p = mimo.make_params(merge_size=1)
    assert _call(p=p) == 5


def test_expand_prompt_ids_matches_oracle():
    rng = np.random.Generator(np.random.PCG64(41))
    PAD = 99
    for _ in range(200):
        n_items = int(rng.integers(0, 6))
        sizes = [(int(rng.integers(1, 3000)), int(rng.integers(1, 3000))) for _ in range(n_items)]
        sizes = [(h, w) for h, w in sizes if oracle.smart_resize_status(h, w) == oracle.OK]
        counts = [mimo.media_tokens(h, w) for h, w in sizes]
        assert counts == [oracle.get_number_of_image_patches(h, w) // 4 for h, w in sizes]
        text = rng.integers(0, 50, size=int(rng.integers(0, 20))).tolist()
        ids = text[:]
        for _ in counts:
            ids.insert(int(rng.integers(0, len(ids) + 1)), PAD)
        assert np.array_equal(mimo.expand_prompt_ids(ids, PAD, counts), oracle.expand_prompt_ids(ids, PAD, counts))


def test_expand_prompt_ids_errors():
    with pytest.raises(mimo.MimoError) as e:
        mimo.expand_prompt_ids([1, 7, 7], 7, [3])
    assert e.value.status == 1
    with pytest.raises(mimo.MimoError) as e:
        mimo.expand_prompt_ids([7], 7, [-1])
    assert e.value.status == 1
    ids = np.array([7], np.int32)
    counts = np.array([5], np.int64)
    out = np.empty(3, np.int32)
    n = ctypes.c_int64()
    st = mimo.lib().mimo_expand_prompt_ids(ids.ctypes.data, 1, 7, counts.ctypes.data, 1, out.ctypes.data, 3,
                                           ctypes.byref(n))
    assert st == 7


def test_video_host_formulas_match_oracle():
    rng = np.random.Generator(np.random.PCG64(43))
    p = mimo.make_params()
    for _ in range(300):
        n = int(rng.integers(1, 2000))
        total_max = int(rng.integers(1, 10**9))
        assert mimo.video_max_pixels(n, total_max, p) == oracle.video_max_pixels(n, total_max, 2, 8192, 8388608)
        total = int(rng.integers(1, 50000))
        fps_src = float(rng.uniform(1, 120))
        fps = float(rng.uniform(0.1, 8))
        mn = int(rng.integers(0, 8))
        mx = mn + int(rng.integers(0, 1000))
        try:
            want = oracle.smart_nframes(total, fps_src, fps, mn, mx)
        except oracle.OracleError:
            with pytest.raises(mimo.MimoError):
                mimo.smart_nframes(total, fps_src, fps, mn, mx)
            continue
        assert mimo.smart_nframes(total, fps_src, fps, mn, mx) == want
        k = int(rng.integers(1, 800))
        i1, t1 = mimo.sample_frames(total, k, fps_src)
        i2, t2 = oracle.sample_frames(total, k, fps_src)
        assert np.array_equal(i1, i2) and np.array_equal(t1, t2)
    assert mimo.video_max_pixels(7, 0, p) == 8388608  # no overall budget


def test_plan_video_matches_oracle_geometry():
    rng = np.random.Generator(np.random.PCG64(44))
    for _ in range(300):
        n = int(rng.integers(1, 64))
        h, w = (int(v) for v in rng.integers(1, 3000, size=2))
        total_max = int(rng.choice([0, int(rng.integers(100_000, 10**8))]))
        budget = oracle.video_max_pixels(n, total_max, 2, 8192, 8388608) if total_max else 8388608
        if oracle.smart_resize_status(h, w, 32, 8192, budget) != oracle.OK:
            with pytest.raises(mimo.MimoError):
                mimo.plan_video(n, h, w, total_max)
            continue
        hr, wr = oracle.smart_resize(h, w, 32, 8192, budget)
        g, rows = mimo.plan_video(n, h, w, total_max)
        assert tuple(g) == ((n + 1) // 2, hr // 16, wr // 16) and rows == g[0] * g[1] * g[2]


@no_gpu_only
def test_patch_embed_validation_statuses():
    L = mimo.lib()
    P = ctypes.c_void_p

    def call(rows=128, w=FAKE, n=256, bias=0, dt=0, out=FAKE, err=FAKE, a=FAKE):
        return L.mimo_patch_embed(P(a), rows, P(w), n, P(bias), dt, P(out), P(err), None)

    assert call(rows=0) == 0
    assert call(rows=-1) == 1
    assert call(n=100) == 1 and call(n=0) == 1
    assert call(dt=7) == 1
    assert call(a=0) == 1 and call(err=0) == 1
    assert call(a=FAKE + 8) == 6 and call(out=FAKE + 2) == 6 and call(bias=FAKE + 4) == 6 and call(err=FAKE + 2) == 6
    assert call(rows=1 << 31) == 8


@no_gpu_only
def test_preprocess_embed_validation_statuses():
    L = mimo.lib()
    P = ctypes.c_void_p
    p = mimo.make_params()
    offs = np.zeros(1, np.int64)
    h = np.array([1080], np.int32)
    w = np.array([1920], np.int32)
    c = np.array([3], np.int32)

    def call(order=0, n_embed=1280, scratch_bytes=1 << 30, cap=8160, weight=FAKE, scratch=FAKE, err=FAKE):
        return L.mimo_preprocess_embed(ctypes.byref(p), 1, P(FAKE), 1080 * 1920 * 3, offs.ctypes.data,
                                       h.ctypes.data, w.ctypes.data, c.ctypes.data, order, P(weight), n_embed,
                                       P(0), 1, P(FAKE), cap, P(scratch), scratch_bytes, P(err), None)

    assert call(order=5) == 1
    assert call(n_embed=1000) == 1
    assert call(cap=8159) == 7
    assert call(weight=0) == 1 and call(scratch=0) == 1
    assert call(scratch=FAKE + 8) == 6
    assert call(scratch_bytes=2 * 8160 * 3072 - 2) == 7   # half the scratch must hold one image's rows


def test_binding_checks_tensors_before_the_library_sees_them():
    """The library gets bare pointers and one row count: the binding rejects tensors whose width, layout,
    element type or device the library could not check, and folds the table sizes into that count."""
    imgs = workloads.random_small_batch(7, 3, max_side=90)
    params = mimo.make_params()
    host = mimo.pack_images(imgs, device="cpu")
    _, offs = mimo.plan_batch(host.heights, host.widths, params)
    total = int(offs[-1])
    with pytest.raises(ValueError, match="shape"):
        mimo.preprocess_batch_host_noalloc(params, host, torch.empty((total, 768)))
    with pytest.raises(ValueError, match="contiguous"):
        mimo.preprocess_batch_host_noalloc(params, host, torch.empty((1536, total)).t())
    with pytest.raises(ValueError, match="dtype"):
        mimo.preprocess_batch_host_noalloc(params, host, torch.empty((total, 1536), dtype=torch.float16))
    with pytest.raises(ValueError, match="int32"):
        mimo.preprocess_batch_host_noalloc(params, host, torch.empty((total, 1536)),
                                           torch.empty(total, dtype=torch.int64))
    # a table shorter than the rows lowers the row count the library is given (MIMO_ECAPACITY there)
    out = torch.empty((total, 1536))
    assert mimo._row_capacity(out, "out", host=True) == total
    assert mimo._row_capacity(out, "out", host=True, perm=torch.empty(total - 1, dtype=torch.int32)) == total - 1
    # device entry points take device tensors only
    with pytest.raises(ValueError, match="CUDA"):
        mimo.preprocess_batch(params, host, torch.empty((total, 1536)))
    with pytest.raises(ValueError, match="CUDA"):
        mimo.patch_embed(torch.empty((4, 1536), dtype=torch.bfloat16), torch.empty((256, 1536), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="shape"):
        mimo.patch_embed(torch.empty((4, 1500), dtype=torch.bfloat16), torch.empty((256, 1536), dtype=torch.bfloat16))


def header_prototypes():
    """name -> list of parameter C types, from the prototypes in include/mimo.h."""
    text = open(os.path.join(ROOT, "include", "mimo.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for ret, name, params in re.findall(r"\b(int|void|const char \*)\s*(mimo_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text):
        ps = [" ".join(p.split()) for p in params.split(",") if p.strip() and p.strip() != "void"]
        protos[name] = (ret.strip(), ps)
    return protos


def _category(c_param: str) -> str:
    if "*" in c_param:
        return "pointer"
    base = c_param.replace("const ", "").split()[0]
    return {"int32_t": "i32", "uint32_t": "u32", "int64_t": "i64", "size_t": "size", "double": "f64",
            "int": "i32"}[base]


def _ctypes_category(t) -> str:
    if t is ctypes.c_void_p or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "pointer"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_double:
        return "f64"
    if t in (ctypes.c_int32, ctypes.c_int):
        return "i32"
    if t is ctypes.c_uint32:
        return "u32"
    if t is ctypes.c_int64:
        return "i64"
    raise AssertionError(f"unexpected ctypes type {t}")


def test_binding_argtypes_match_the_prototypes():
    """Every exported function's ctypes argument list has the header prototype's count, order and widths."""
    protos = header_prototypes()
    assert set(mimo.EXPORTED) <= set(protos)
    L = mimo.lib()
    restypes = {"int": ctypes.c_int, "void": None, "const char *": ctypes.c_char_p}
    for name in mimo.EXPORTED:
        ret, params = protos[name]
        want = [_category(p) for p in params]
        got = [_ctypes_category(t) for t in getattr(L, name).argtypes]
        assert got == want, (name, got, want)
        assert getattr(L, name).restype is restypes[ret], (name, ret)
