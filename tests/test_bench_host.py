"""Host-side logic of bench.py that decides what the JSON line reports (no GPU needed)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_is_reported_only_for_the_captured_kernel_source(tmp_path, monkeypatch):
    digest = bench.kernel_source_digest("preprocess")
    table = {"c5_f32": {"kernel_digest": digest, "dram_bytes_per_launch": 1000},
             "c5_bf16": {"kernel_digest": "0000000000000000", "dram_bytes_per_launch": 500},
             "pe_bf16": {"kernel_digest": bench.kernel_source_digest("patch_embed"), "dram_bytes_per_launch": 800,
                         "full_rows": 400}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the digests are computed from the sources under ROOT: point them back at the repository
    monkeypatch.setattr(bench, "kernel_source_digest",
                        lambda kernel="preprocess": table["c5_f32"]["kernel_digest"] if kernel == "preprocess"
                        else table["pe_bf16"]["kernel_digest"])
    assert bench.ncu_traffic("c5", "f32") == 1000
    assert bench.ncu_traffic("c5", "bf16") is None           # captured on another kernel source
    assert bench.ncu_traffic("c3", "f32") is None            # never captured
    assert bench.ncu_traffic("pe", "bf16", "patch_embed", rows=400) == 800
    assert bench.ncu_traffic("pe", "bf16", "patch_embed", rows=100) == 200   # scaled by rows


def test_committed_traffic_table_is_consistent():
    # entries name the kernel sources they were captured on (bench.py reports null for any other source)
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        table = json.load(f)
    for key in ("c2_f32", "c3_f32", "c4_f32", "c5_f32", "c5_bf16", "pe_bf16"):
        e = table[key]
        assert len(e["kernel_digest"]) == 16 and int(e["kernel_digest"], 16) >= 0
        if "per_image" in e:
            # two captures: the slope and offset reproduce both, and the full launch is their extrapolation
            for n, c in e["captures"].items():
                assert abs(e["per_image"] * int(n) + e["offset"] - (c["read"] + c["write"])) < 2
            assert e["dram_bytes_per_launch"] == round(e["per_image"] * e["full_images"] + e["offset"])
        else:
            assert e["dram_bytes_per_launch"] == e["read"] + e["write"]


def test_traffic_fit_is_evaluated_at_the_image_count(tmp_path, monkeypatch):
    table = {"c5_f32": {"kernel_digest": "x", "dram_bytes_per_launch": 2560, "per_image": 10.0, "offset": -5.0,
                        "full_images": 256},
             "c3_f32": {"kernel_digest": "x", "dram_bytes_per_launch": 77, "full_images": 68}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_digest", lambda kernel="preprocess": "x")
    assert bench.ncu_traffic("c5", "f32", images=16) == 155
    assert bench.ncu_traffic("c3", "f32", images=68) == 77
    assert bench.ncu_traffic("c3", "f32", images=12) is None  # a whole-workload capture applies to that workload


def test_algorithmic_bytes_of_c5():
    class Packed:
        heights = [1080] * 256
        widths = [1920] * 256
        channels = [3, 4] * 128
    nb = bench.algorithmic_bytes(Packed(), 256 * 8160, 4, True)
    assert nb["read"] == 1_857_945_600
    assert nb["write_rows"] == 12_834_570_240
    assert nb["write_perm"] == 8_355_840
    assert nb["total"] == 14_700_871_680


def test_l2_note_states_whether_inputs_outgrow_l2():
    # the default batch: 1.86 GB of uint8 inputs, 12.8 GB of fp32 rows
    assert "larger than L2" in bench.l2_note(1_857_945_600, 12_842_926_080)
    # 16 RGBA 480x640 images: 19.7 MB of inputs, below the L2 size
    note = bench.l2_note(16 * 480 * 640 * 4, 19_200 * 6_144)
    assert "smaller than the 126 MB L2" in note and "19.7 MB" in note


def test_cpu_baseline_reports_all_cores_and_one_thread():
    import workloads

    cpu = bench.image_cpu_baseline(workloads.workload("c1"), 1, 2, min_seconds=0.0, single_seconds=0.0)
    assert cpu["kind"] == "oracle" and cpu["cores"] == 2 and cpu["value"] > 0
    assert cpu["single_thread"]["cores"] == 1 and cpu["single_thread"]["value"] > 0
    assert cpu["unit"] == cpu["single_thread"]["unit"] == bench.UNIT


def test_dominant_kernel_follows_the_dispatch_rule():
    import workloads
    from vision_lm_image_b200 import mimo

    def kernel(name, dtype):
        w = workloads.workload(name, n_images=8 if name == "c5" else None)
        host = mimo.pack_images(w["images"][:8], device="cpu")
        grid, _ = mimo.plan_batch(host.heights, host.widths, mimo.make_params(w["mean"], w["std"]))
        return bench.dominant_kernel(grid, host.heights, host.widths, dtype)

    assert kernel("c5", "f32") == "preprocess_kernel"   # 1080 -> 1088 rows: heights resized
    assert kernel("c5", "bf16") == "direct_kernel"      # widths kept, bf16 rows
    assert kernel("c2", "f32") == "direct_kernel"       # identity resize
    assert kernel("c3", "f32") == "preprocess_kernel"   # widths resized, heights within 1.25 of kept
    assert kernel("c4", "f32") == "warp_kernel"         # 4096 -> 2880: every height shrunk by 1.42
    # a video clip with kept widths takes the unstaged kernel in both dtypes, resized heights or not;
    # with resized widths, the staged one
    import numpy as np

    v_grid = np.array([[32, 68, 120]])  # 1080x1920 frames -> 1088x1920
    for dtype in ("f32", "bf16"):
        assert bench.dominant_kernel(v_grid, [1080], [1920], dtype, video=True) == "direct_kernel"
        assert bench.dominant_kernel(np.array([[2, 6, 8]]), [70], [90], dtype, video=True) == "preprocess_kernel"


def test_reference_arm_config_equals_the_main_arm_config():
    # both arms print the same config for the same arguments: the reference arm computes the rows with
    # the oracle's geometry, the main arm with the library's plan
    import argparse

    import oracle
    import workloads
    from vision_lm_image_b200 import mimo

    for name in ("c1", "c3"):
        args = argparse.Namespace(workload=name, order="merge", graph=False)
        w = workloads.workload(name)
        host = mimo.pack_images(w["images"], device="cpu")
        _, offs = mimo.plan_batch(host.heights, host.widths, mimo.make_params(w["mean"], w["std"]))
        read = bench.algorithmic_bytes(host, int(offs[-1]), 4, bool(w["column_perm"]))["read"]
        ours = bench.workload_config(args, w, 1, host.n, w["dtype"], bool(w["column_perm"]), int(offs[-1]), read)
        rows = sum(oracle.get_number_of_image_patches(im.shape[0], im.shape[1]) for im in w["images"])
        ref = bench.workload_config(args, w, 1, len(w["images"]), w["dtype"], bool(w["column_perm"]), rows,
                                    sum(int(im.size) for im in w["images"]))
        assert ours == ref
        assert set(ours) >= {"workload", "images_per_gpu", "rows_per_gpu", "row_order", "out_dtype", "l2"}


def test_kernel_digest_ignores_comments_but_not_code(tmp_path, monkeypatch):
    src = tmp_path / "vision_lm_image_b200" / "csrc"
    src.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"k": ("vision_lm_image_b200/csrc/a.cu",)})

    def digest(text):
        (src / "a.cu").write_text(text)
        return bench.kernel_source_digest("k")

    base = digest("int f(int x) {\n    return x + 1;\n}\n")
    assert digest("// a note\nint f(int x) {  /* the sum */\n\n    return x + 1;  // one more\n}\n") == base
    assert digest("int f(int x) {\n    return x + 2;\n}\n") != base
