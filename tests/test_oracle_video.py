"""Pins for the oracle's video path (docs.rs 'cortiq_engine::mimo_vision': prepare_video_frames,
video_max_pixels, smart_nframes, sample_frames).

- video_max_pixels / smart_nframes: closed forms worked by hand from the page's formulas;
- sample_frames: the page's own formula unique(int64(linspace(0, total-1, n))) and float32(idx)/fps_src,
  evaluated with numpy's linspace/unique (the routines it names);
- the pixel path: a video of two identical frames is the image path (T = 2 duplicates one frame); with
  distinct frames each temporal slot tt takes frame 2t + tt; an odd count repeats the last frame.
"""
import numpy as np
import pytest

import oracle
import workloads

M, S = workloads.IMAGENET_MEAN, workloads.IMAGENET_STD
T, P = 2, 16


def test_video_max_pixels_closed_forms():
    assert oracle.video_max_pixels(4, 100000, 2, 8192, 8388608) == 50000       # 100000*2//4
    assert oracle.video_max_pixels(1000, 100000, 2, 8192, 8388608) == 8192     # share 200 -> floor at min
    assert oracle.video_max_pixels(1, 10**7, 2, 8192, 8388608) == 8388608      # share 2e7 -> cap at max
    assert oracle.video_max_pixels(3, 100, 2, 0, 10**9) == 66                  # 200 // 3


def test_smart_nframes_closed_forms():
    assert oracle.smart_nframes(300, 30.0, 2.0, 4, 768) == 20      # 300/30*2 = 20
    assert oracle.smart_nframes(301, 30.0, 2.0, 4, 768) == 20      # 20.07 -> floor to even
    assert oracle.smart_nframes(7, 30.0, 2.0, 4, 768) == 4         # 0.47 -> min_frames 4
    assert oracle.smart_nframes(3, 30.0, 2.0, 4, 768) == 2         # min 4, capped by total 3, even 2
    assert oracle.smart_nframes(10000, 30.0, 2.0, 4, 768) == 666   # 666.67 -> 666
    assert oracle.smart_nframes(100000, 30.0, 2.0, 4, 768) == 768  # capped at max_frames
    with pytest.raises(oracle.OracleError):
        oracle.smart_nframes(1, 30.0, 2.0, 1, 768)                 # 1 frame floors to 0


@pytest.mark.parametrize("total,n,fps", [(300, 20, 30.0), (7, 4, 25.0), (1, 1, 24.0), (100, 100, 29.97),
                                         (50, 200, 30.0), (12345, 768, 59.94), (2, 7, 1.0)])
def test_sample_frames_matches_the_pages_formula(total, n, fps):
    idx, ts = oracle.sample_frames(total, n, fps)
    want = np.unique(np.linspace(0, total - 1, n).astype(np.int64))
    assert np.array_equal(idx, want)
    assert np.array_equal(ts, want.astype(np.float32) / np.float32(fps))


def test_two_identical_frames_are_the_image_path():
    img = workloads.random_small_batch(91, 1, max_side=180)[0]
    rows, g = oracle.preprocess_image(img, M, S)
    vid, gv = oracle.preprocess_video(np.stack([img, img]), M, S)
    assert gv == g and np.array_equal(vid, rows)


def test_each_temporal_slot_takes_its_frame():
    rng = workloads.rng_for(92)
    a = workloads.uniform_image(rng, 70, 90, 3)
    b = workloads.uniform_image(rng, 70, 90, 3)
    ra, _ = oracle.preprocess_image(a, M, S)
    rb, _ = oracle.preprocess_image(b, M, S)
    vid, g = oracle.preprocess_video(np.stack([a, b]), M, S)
    v = vid.reshape(-1, 3, T, P * P)
    assert np.array_equal(v[:, :, 0], ra.reshape(-1, 3, T, P * P)[:, :, 0])
    assert np.array_equal(v[:, :, 1], rb.reshape(-1, 3, T, P * P)[:, :, 1])
    # swapping the frames swaps the slots
    sw, _ = oracle.preprocess_video(np.stack([b, a]), M, S)
    s = sw.reshape(-1, 3, T, P * P)
    assert np.array_equal(s[:, :, 0], v[:, :, 1]) and np.array_equal(s[:, :, 1], v[:, :, 0])


def test_odd_count_repeats_the_last_frame():
    rng = workloads.rng_for(93)
    fr = [workloads.rgba_image(rng, 64, 96) for _ in range(3)]
    vid, g = oracle.preprocess_video(np.stack(fr), M, S)
    one, g1 = oracle.preprocess_image(fr[2], M, S)
    assert g == (2, g1[1], g1[2])
    assert np.array_equal(vid[vid.shape[0] // 2:], one)


def test_per_frame_budget_shrinks_the_grid():
    rng = workloads.rng_for(94)
    frames = np.stack([workloads.uniform_image(rng, 540, 960, 3) for _ in range(8)])
    total_max = 8 * 60000
    budget = oracle.video_max_pixels(8, total_max, 2, 8192, 8388608)
    assert budget == 120000
    _, g = oracle.preprocess_video(frames, M, S, total_max_pixels=total_max)
    hr, wr = oracle.smart_resize(540, 960, 32, 8192, budget)
    assert g == (4, hr // 16, wr // 16) and hr * wr <= budget
