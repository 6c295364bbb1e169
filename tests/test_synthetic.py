"""The seeded input generator: shapes, layouts, determinism, subset stability (CPU)."""
import numpy as np

from prompt_conditioned_keypoint_b200 import synthetic as S


def test_subset_equals_full_batch_slice():
    full = S.make_config(2, crops=range(0, 6))
    part = S.make_config(2, crops=[4, 1])
    np.testing.assert_array_equal(part.feat, full.feat[[4, 1]])
    np.testing.assert_array_equal(part.rows, full.rows[[4, 1]])
    np.testing.assert_array_equal(part.mask, full.mask[[4, 1]])


def test_config_shapes_and_masks():
    w2 = S.make_config(2, crops=[0, 1, 2])
    assert w2.feat.shape == (3, 24, 24, 1024) and w2.feat.dtype == np.float32
    assert w2.rows.shape == (3, 2, 80, 1024) and w2.mask.shape == (3, 2, 80)
    for i in range(3):
        n = int(w2.mask[i, 0].sum())
        assert 5 <= n <= 80 and np.array_equal(w2.mask[i, 0], w2.mask[i, 1])
        assert w2.mask[i, 0, :n].all() and not w2.mask[i, 0, n:].any()
    w3 = S.make_config(3, crops=range(12))
    assert w3.C == 1280
    for i in range(12):
        mod = w3.extra["modality"][i]
        assert w3.mask[i, 0].any() == (mod in (0, 2)) and w3.mask[i, 1].any() == (mod in (1, 2))
    w1 = S.make_config(1)
    assert w1.M == 1 and w1.support.shape == (1, 24, 24, 1024) and int(w1.kmask.sum()) == 17
    assert np.all((w1.kpts >= 0) & (w1.kpts < 384))


def test_config4_is_bf16_and_shared():
    w4 = S.make_config(4, crops=[0, 5])
    assert w4.feat.dtype == np.uint16 and w4.Bk == 1 and w4.rows.shape == (1, 2, 80, 1024)
    assert int(w4.mask.sum()) == 34
    f = S.bf16_bits_to_f32(w4.feat)
    assert np.isfinite(f).all() and 0.3 < f.std() < 1.5


def test_logical_order_draw_then_nhwc():
    a = S.make_case(3, 1, 4, 5, 8, 2, 1)
    g = S._rng(3, S._FEAT, 0)
    raw = g.standard_normal((8, 4, 5), dtype=np.float32)
    np.testing.assert_array_equal(a.feat[0], raw.transpose(1, 2, 0))


def test_bf16_storage_cast_roundtrip():
    x = np.array([1.0, 1.00390625, -2.5, 3.0e-3], np.float32)
    bits = S.to_bf16_bits(x)
    back = S.bf16_bits_to_f32(bits)
    assert back[0] == 1.0 and back[2] == -2.5
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8)


def test_bf16_storage_cast_matches_torch():
    import torch
    g = np.random.default_rng(3)
    x = np.concatenate([g.standard_normal(200_000).astype(np.float32),
                        (g.standard_normal(20_000) * 1e-38).astype(np.float32),
                        np.array([0.0, -0.0, 1.00390625, 1.01171875, -1.00390625, 3.3e38, 1e-45], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(S.to_bf16_bits(x), want)


def test_image_and_boxes_are_seeded_and_inside_the_frame():
    from prompt_conditioned_keypoint_b200 import synthetic as S
    img, boxes = S.random_image_and_boxes(7, 108, 192, 16)
    img2, boxes2 = S.random_image_and_boxes(7, 108, 192, 16)
    assert img.shape == (108, 192, 3) and img.dtype == np.uint8
    assert boxes.shape == (16, 4) and boxes.dtype == np.float32
    assert np.array_equal(img, img2) and np.array_equal(boxes, boxes2)
    assert np.all(boxes[:, 0] >= 0) and np.all(boxes[:, 1] >= 0)
    assert np.all(boxes[:, 2] <= 192 + 1e-3) and np.all(boxes[:, 3] <= 108 + 1e-3)
    w, h = boxes[:, 2] - boxes[:, 0], boxes[:, 3] - boxes[:, 1]
    assert np.all(w >= 0.1 * 192 - 1e-3) and np.all(w <= 0.6 * 192 + 1e-3)
    assert np.all(h >= 0.1 * 108 - 1e-3) and np.all(h <= 0.6 * 108 + 1e-3)
