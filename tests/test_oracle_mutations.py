"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a temporary copy of oracle/oracle.c:
a dropped term, a wrong sign, index, rounding rule or loop order. The copy is
compiled, and the pin tests (tests/test_oracle_*.py) run against it. At least
one pin must fail for every mutant, and all must pass for the unmodified
copy (the control). The committed oracle is never modified. Mutants are chosen
to keep every memory access in bounds, so a caught mutant fails a comparison,
not a crash.
"""
import json
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, exact text in oracle.c, replacement)
MUTANTS = [
    # smart_resize
    ("round_ties_up", "return (fmod(lo, 2.0) == 0.0) ? lo : lo + 1.0;", "return lo + 1.0;"),
    ("aspect_guard_2000", "if (big / small > 200.0)", "if (big / small > 2000.0)"),
    ("max_branch_ceil", "h_bar = floor(h / beta / f) * f;", "h_bar = ceil(h / beta / f) * f;"),
    ("min_branch_floor", "w_bar = ceil(w * beta / f) * f;", "w_bar = floor(w * beta / f) * f;"),
    ("no_upscale_branch", "if (height < factor || width < factor) {", "if (0) {"),
    ("upscale_long_side_unrounded", "w = trunc((double)(width * factor) / (double)height);",
     "w = (double)(width * factor) / (double)height;"),
    ("max_branch_on_original_size", "double beta = sqrt((h * w) / (double)max_pixels);",
     "double beta = sqrt((h_bar * w_bar) / (double)max_pixels);"),
    # RGBA onto white
    ("flatten_truncates", "return (uint8_t)((2 * num + 255) / 510);", "return (uint8_t)(num / 255);"),
    ("flatten_onto_black", "int32_t num = (int32_t)c * (int32_t)a + 255 * (255 - (int32_t)a);",
     "int32_t num = (int32_t)c * (int32_t)a;"),
    # bilinear taps
    ("align_corners_true", "double src = ((double)d + 0.5) * scale - 0.5;",
     "double src = (out > 1) ? (double)d * (double)(in - 1) / (double)(out - 1) : 0.0;"),
    ("half_pixel_dropped", "double src = ((double)d + 0.5) * scale - 0.5;", "double src = (double)d * scale;"),
    ("x_weights_swapped", "double top = (1.0 - lx) * in[y0 * in_w + x0] + lx * in[y0 * in_w + x1];",
     "double top = lx * in[y0 * in_w + x0] + (1.0 - lx) * in[y0 * in_w + x1];"),
    ("second_row_dropped", "out[y * out_w + x] = (1.0 - ly) * top + ly * bot;",
     "out[y * out_w + x] = (1.0 - ly) * top + ly * top;"),
    # normalisation
    ("mean_sign", "planes[k * HW + i] = (planes[k * HW + i] - m) / s;",
     "planes[k * HW + i] = (planes[k * HW + i] + m) / s;"),
    ("std_not_scaled", "double s = 255.0 * stdv[k];", "double s = stdv[k];"),
    # patch rows
    ("py_px_swapped",
     "                                        int64_t y = (bh * m + mh) * p + py;\n"
     "                                        int64_t x = (bw * m + mw) * p + px;\n"
     "                                        out[row * cols + col] = (float)planes[c * Hr * Wr + y * Wr + x];",
     "                                        int64_t y = (bh * m + mh) * p + px;\n"
     "                                        int64_t x = (bw * m + mw) * p + py;\n"
     "                                        out[row * cols + col] = (float)planes[c * Hr * Wr + y * Wr + x];"),
    ("mh_mw_swapped",
     "                                        int64_t y = (bh * m + mh) * p + py;\n"
     "                                        int64_t x = (bw * m + mw) * p + px;\n"
     "                                        out[row * cols + col] = (float)planes[c * Hr * Wr + y * Wr + x];",
     "                                        int64_t y = (bh * m + mw) * p + py;\n"
     "                                        int64_t x = (bw * m + mh) * p + px;\n"
     "                                        out[row * cols + col] = (float)planes[c * Hr * Wr + y * Wr + x];"),
    ("columns_tt_before_c",
     "                        for (int64_t c = 0; c < 3; ++c)\n"
     "                            for (int64_t tt = 0; tt < T; ++tt) /* frame tt is a copy */",
     "                        for (int64_t tt = 0; tt < T; ++tt) /* frame tt is a copy */\n"
     "                            for (int64_t c = 0; c < 3; ++c)"),
    ("blocks_column_major",
     "        for (int64_t bh = 0; bh < gh / m; ++bh)\n"
     "            for (int64_t bw = 0; bw < gw / m; ++bw)\n"
     "                for (int64_t mh = 0; mh < m; ++mh)\n"
     "                    for (int64_t mw = 0; mw < m; ++mw, ++row) {\n"
     "                        int64_t col = 0;\n"
     "                        for (int64_t c = 0; c < 3; ++c)\n"
     "                            for (int64_t tt = 0; tt < T; ++tt) /* frame tt is a copy */",
     "        for (int64_t bw = 0; bw < gw / m; ++bw)\n"
     "            for (int64_t bh = 0; bh < gh / m; ++bh)\n"
     "                for (int64_t mh = 0; mh < m; ++mh)\n"
     "                    for (int64_t mw = 0; mw < m; ++mw, ++row) {\n"
     "                        int64_t col = 0;\n"
     "                        for (int64_t c = 0; c < 3; ++c)\n"
     "                            for (int64_t tt = 0; tt < T; ++tt) /* frame tt is a copy */"),
    ("sampled_value_sub_patch_swapped", "int64_t mh = sub / m, mw = sub % m;",
     "int64_t mh = sub % m, mw = sub / m;"),
    # column order and tables
    ("permutation_identity", "perm[dst++] = (int32_t)(row0 + ((t * gh2 + a) * gw2 + b) * m * m + k);",
     "perm[dst++] = (int32_t)(row0 + ((t * gw2 + b) * gh2 + a) * m * m + k);"),
    ("permutation_not_offset", "perm[dst++] = (int32_t)(row0 + ((t * gh2 + a) * gw2 + b) * m * m + k);",
     "perm[dst++] = (int32_t)(((t * gh2 + a) * gw2 + b) * m * m + k);"),
    ("positions_w_from_mh", "pos[2 * row + 1] = (int32_t)(bw * m + mw);",
     "pos[2 * row + 1] = (int32_t)(bw * m + mh);"),
    ("positions_ignore_column_order",
     "int64_t bh = column_order ? b : a;\n                        int64_t bw = column_order ? a : b;",
     "int64_t bh = a;\n                        int64_t bw = b;"),
    ("window_row_major", "win[j++] = (int32_t)(unit0 + (t * gh2 + a) * gw2 + b);",
     "win[j++] = (int32_t)(unit0 + (t * gw2 + b) * gh2 + a);"),
    ("prompt_one_short", "for (int64_t k = 0; k < counts[used]; ++k) {",
     "for (int64_t k = 0; k + 1 < counts[used]; ++k) {"),
    # video
    ("budget_without_T", "int64_t share = (total_max * temporal) / n_sampled;",
     "int64_t share = total_max / n_sampled;"),
    ("nframes_ceil_to_even", "int64_t even = (int64_t)floor(n / 2.0) * 2;",
     "int64_t even = (int64_t)ceil(n / 2.0) * 2;"),
    ("sample_frames_rounds", "int64_t i = (int64_t)v;", "int64_t i = (int64_t)(v + 0.5);"),
    ("video_one_frame_per_pair", "int64_t f = t * T + tt;", "int64_t f = t * T;"),
    ("odd_count_not_padded", "const int64_t n_pad = n + (n & 1);", "const int64_t n_pad = n - (n & 1);"),
    # patch embedding
    ("weight_transposed", "acc += (double)rows[m * K + k] * (double)w[n * K + k];",
     "acc += (double)rows[m * K + k] * (double)w[k * N + n];"),
    ("bias_dropped", "double acc = bias ? bias[n] : 0.0;", "double acc = 0.0;"),
]

# the same for the Python half of the oracle (oracle/__init__.py): batch assembly and bf16 rounding
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")
PY_MUTANTS = [
    ("pymod_perm_offset_in_units", "            row0 += gh * gw\n", "            row0 += (gh * gw) // 4\n"),
    ("pymod_window_offset_in_rows", "        unit0 += (gh // merge) * (gw // merge)\n", "        unit0 += gh * gw\n"),
    ("pymod_positions_always_merge_order", "rotary_positions(gh, gw, merge, column_order=(order == \"column\"))",
     "rotary_positions(gh, gw, merge, column_order=False)"),
    ("pymod_no_flatten", "            flat.extend(item)\n", "            flat.append(item)\n"),
    ("pymod_bf16_ties_up", "    rounding = 0x7FFF + ((bits >> 16) & 1)\n", "    rounding = 0x8000 + 0 * bits\n"),
]

CONTROL = "control"
PY_CONTROL = "pymod_control"

# Readings that no pin fixes ("parity unpinned"): their mutants are expected to pass every pin. Strict, so
# that a new pin which catches one shows up here.
UNPINNED: dict[str, str] = {}


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    # the runner tells the two kinds apart by the name's prefix
    assert not any(n.startswith("pymod_") for n, _, _ in MUTANTS)
    assert all(n.startswith("pymod_") for n, _, _ in PY_MUTANTS)
    src = open(SRC).read()
    d = tmp_path_factory.mktemp("oracle_mutants")
    builds = [(CONTROL, src)]
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, f"{name}: the text to mutate must occur once in oracle.c"
        builds.append((name, src.replace(old, new)))
    procs = []
    for name, text in builds:
        c = d / f"{name}.c"
        c.write_text(text)
        procs.append(subprocess.Popen(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(d / f"{name}.so"),
                                       str(c), "-lm"]))
    assert all(p.wait() == 0 for p in procs)
    # Python mutants: a copy of the oracle package with one changed line, built from the control library
    py_src = open(PY_SRC).read()
    py_builds = [(PY_CONTROL, py_src)]
    for name, old, new in PY_MUTANTS:
        assert py_src.count(old) == 1, f"{name}: the text to mutate must occur once in oracle/__init__.py"
        py_builds.append((name, py_src.replace(old, new)))
    for name, text in py_builds:
        pkg = d / name / "oracle"
        pkg.mkdir(parents=True)
        (pkg / "__init__.py").write_text(text)
        shutil.copy(SRC, pkg / "oracle.c")
        shutil.copy(d / f"{CONTROL}.so", pkg / "liboracle.so")  # newer than oracle.c: not rebuilt
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_oracle_mutation_runner.py"), str(d),
                        *[n for n, _ in builds], *[n for n, _ in py_builds]],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULTS ")]
    assert r.returncode == 0 and lines, r.stdout[-3000:] + r.stderr[-3000:]
    return json.loads(lines[-1][len("RESULTS "):])


def test_unmodified_copy_passes_every_pin(results):
    assert results[CONTROL] == 0
    assert results[PY_CONTROL] == 0


@pytest.mark.parametrize("name", [
    pytest.param(m[0], marks=pytest.mark.xfail(strict=True, reason=UNPINNED[m[0]])) if m[0] in UNPINNED else m[0]
    for m in MUTANTS + PY_MUTANTS])
def test_pins_catch_planted_mistake(results, name):
    # pytest exit code 1: a pin failed (0 would mean the mistake went unnoticed)
    assert results[name] == 1, f"planted mistake '{name}' passed every pin (exit code {results[name]})"
