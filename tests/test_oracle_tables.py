"""Pins for the oracle's column-order emission and the vision-tower index tables.

Reading (docs.rs 'cortiq_engine::mimo_vision', conventions; NeMo Automodel 'mimo_v2_flash.vision',
MiMoVisionTransformer._rotary_positions / _get_window_index): column order lists whole merge units
by (t, block col, block row); the rotary positions are each emitted row's (patch row, patch column)
and are permuted with the rows; the window index lists merge units in column-major order.
"""
import numpy as np
import torch

import oracle
import workloads


def test_positions_hand_worked_4x6():
    pos = oracle.rotary_positions(4, 6)
    want = []
    for bh in range(2):
        for bw in range(3):
            for mh in range(2):
                for mw in range(2):
                    want.append((2 * bh + mh, 2 * bw + mw))
    assert pos.tolist() == [list(w) for w in want]
    assert pos[:8].tolist() == [[0, 0], [0, 1], [1, 0], [1, 1], [0, 2], [0, 3], [1, 2], [1, 3]]


def test_positions_match_reshape_formulation():
    # hpos/wpos of a (gh, gw) grid re-ordered into merge blocks with reshape/permute
    for gh, gw in [(2, 2), (4, 6), (8, 6), (68, 120), (2, 24)]:
        h = torch.arange(gh)[:, None].expand(gh, gw)
        w = torch.arange(gw)[None, :].expand(gh, gw)
        def merge(t):
            return t.reshape(gh // 2, 2, gw // 2, 2).permute(0, 2, 1, 3).reshape(-1)
        ref = torch.stack([merge(h), merge(w)], dim=1).numpy()
        assert np.array_equal(oracle.rotary_positions(gh, gw), ref)


def test_column_order_tables_follow_the_permutation():
    for gh, gw in [(2, 2), (4, 6), (6, 4), (68, 120)]:
        perm = oracle.column_permutation(gh, gw)
        pos = oracle.rotary_positions(gh, gw)
        assert np.array_equal(oracle.rotary_positions(gh, gw, column_order=True), pos[perm])
        win = oracle.window_index(gh, gw)
        assert np.array_equal(win, perm[::4] // 4)
        assert np.array_equal(np.sort(win), np.arange(gh * gw // 4))


def test_window_index_hand_worked_and_offset():
    assert oracle.window_index(4, 6).tolist() == [0, 3, 1, 4, 2, 5]
    assert oracle.window_index(4, 6, unit0=10).tolist() == [10, 13, 11, 14, 12, 15]
    assert oracle.window_index(2, 2).tolist() == [0]


def test_column_rows_are_merge_rows_permuted():
    img = workloads.random_small_batch(81, 1, max_side=200)[0]
    rows, g = oracle.preprocess_image(img, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    col, gc = oracle.preprocess_image_column(img, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    assert g == gc
    perm = oracle.column_permutation(g[1], g[2])
    assert np.array_equal(col, rows[perm])


def test_batch_tables_are_batch_global():
    imgs = workloads.random_small_batch(82, 4, max_side=150)
    pv, grid, perm, pos, win = oracle.preprocess(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD,
                                                 column_perm=True, positions=True, window=True)
    pvc, _, _, posc, winc = oracle.preprocess(imgs, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD,
                                              column_perm=True, positions=True, window=True, order="column")
    assert np.array_equal(pvc, pv[perm])
    assert np.array_equal(posc, pos[perm])
    assert np.array_equal(win, winc)
    assert np.array_equal(win, perm[::4] // 4)
    assert pos.shape == (pv.shape[0], 2) and win.shape == (pv.shape[0] // 4,)


def test_expand_prompt_ids_hand_worked():
    PAD = 151655
    # two images: 16x192 -> grid (1, 2, 24) -> 12 tokens; 64x48 -> grid (1, 8, 6) -> 12 tokens
    counts = [oracle.get_number_of_image_patches(16, 192) // 4, oracle.get_number_of_image_patches(64, 48) // 4]
    assert counts == [12, 12]
    ids = [1, 2, PAD, 3, PAD, 4]
    out = oracle.expand_prompt_ids(ids, PAD, counts)
    assert out.tolist() == [1, 2] + [PAD] * 12 + [3] + [PAD] * 12 + [4]
    assert oracle.expand_prompt_ids([5, 6], PAD, []).tolist() == [5, 6]
    assert oracle.expand_prompt_ids([PAD], PAD, [0]).tolist() == []


def test_expand_prompt_ids_rejects_a_count_mismatch():
    import pytest
    with pytest.raises(oracle.OracleError):
        oracle.expand_prompt_ids([1, 7, 7], 7, [3])
    with pytest.raises(oracle.OracleError):
        oracle.expand_prompt_ids([1, 7], 7, [3, 4])



def test_patch_embed_is_the_conv3d_of_the_pages():
    # MiMoVisionPatchEmbed is a Conv3d with kernel = stride = (2, 16, 16): the oracle's row GEMM with the
    # weight flattened (c, tt, py, px) must equal torch's conv3d over the two duplicated frames
    import torch.nn.functional as F
    rng = np.random.Generator(np.random.PCG64(5))
    img = workloads.random_small_batch(83, 1, max_side=120)[0]
    rows, g = oracle.preprocess_image(img, workloads.IMAGENET_MEAN, workloads.IMAGENET_STD)
    N = 48
    w = rng.standard_normal((N, 3, 2, 16, 16)).astype(np.float32)
    b = rng.standard_normal(N)
    out = oracle.patch_embed(rows, w.reshape(N, -1), b)
    gh, gw = g[1], g[2]
    # rebuild the normalised frames from the rows (merge order -> planes), then convolve
    x = torch.from_numpy(rows.astype(np.float64)).reshape(gh // 2, gw // 2, 2, 2, 3, 2, 16, 16)
    x = x.permute(4, 5, 0, 2, 6, 1, 3, 7).reshape(1, 3, 2, gh * 16, gw * 16)  # (c, tt, y, x)
    conv = F.conv3d(x, torch.from_numpy(w.astype(np.float64)), torch.from_numpy(b), stride=(2, 16, 16))
    ref = conv[0, :, 0].reshape(N, gh // 2, 2, gw // 2, 2).permute(1, 3, 2, 4, 0).reshape(-1, N).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-9)


def test_patch_embed_hand_worked():
    rows = np.array([[1.0, 2.0, 3.0], [0.5, -1.0, 4.0]], np.float32)
    w = np.array([[1.0, 0.0, -1.0], [2.0, 1.0, 0.5]], np.float32)
    out = oracle.patch_embed(rows, w, [10.0, -1.0])
    assert out.tolist() == [[1 - 3 + 10, 2 + 2 + 1.5 - 1], [0.5 - 4 + 10, 1 - 1 + 2 - 1]]
