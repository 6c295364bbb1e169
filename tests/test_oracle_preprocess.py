"""Pins of the image-preprocessing oracle (oracle/preprocess.py), CPU only.

Model card (GKD_GGUF), Model section, Input bullet: longer side resized to 384,
centre-padded to 384 x 384 with (124, 116, 104), ImageNet normalisation. The
pins tie the oracle to things it does not compute itself: PyTorch's bilinear
resize where the geometry is a plain resize, closed forms (constant and affine
images, the pad value), the ROI -> image coordinate map, and a pure-Python brute
force on tiny images.
"""
import numpy as np
import pytest
import torch

from oracle import brute
from oracle import preprocess as PP
from oracle import variants as V

RNG = np.random.default_rng(17)


def _torch_resize(img, out_h, out_w):
    t = torch.from_numpy(np.asarray(img, np.float64).transpose(2, 0, 1))[None]
    r = torch.nn.functional.interpolate(t, size=(out_h, out_w), mode="bilinear", align_corners=False,
                                        antialias=False)
    return r[0].numpy()


def _normalise(v):
    return (v / 255.0 - np.asarray(PP.MEAN)[:, None, None]) / np.asarray(PP.STD)[:, None, None]


@pytest.mark.parametrize("H,W", [(384, 384), (96, 96), (500, 500), (37, 37)])
def test_square_image_equals_torch_bilinear_resize(H, W):
    img = RNG.integers(0, 256, (H, W, 3), dtype=np.uint8)
    got = PP.preprocess(img, (0, 0, W, H), 384)
    want = _normalise(_torch_resize(img, 384, 384))
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,W", [(96, 192), (192, 96), (48, 384)])
def test_integer_pad_equals_resize_plus_pad(H, W):
    """Scale 2 or 1 with integer pad offsets: the content region is PyTorch's
    resize of the image and the rest is the pad colour."""
    img = RNG.integers(0, 256, (H, W, 3), dtype=np.uint8)
    got = PP.preprocess(img, (0, 0, W, H), 384)
    s = 384 / max(H, W)
    ch, cw = int(round(H * s)), int(round(W * s))
    oy, ox = (384 - ch) // 2, (384 - cw) // 2
    want = _normalise(_torch_resize(img, ch, cw))
    np.testing.assert_allclose(got[:, oy:oy + ch, ox:ox + cw], want, rtol=0, atol=1e-12)
    pad = PP.normalised_pad()
    mask = np.ones((384, 384), bool)
    mask[oy:oy + ch, ox:ox + cw] = False
    for c in range(3):
        assert np.all(got[c][mask] == pad[c])


def test_constant_image_and_pad_values():
    img = np.full((120, 200, 3), (10, 200, 77), np.uint8)
    got = PP.preprocess(img, (0, 0, 200, 120))
    content = (np.array([10.0, 200.0, 77.0]) / 255.0 - np.array(PP.MEAN)) / np.array(PP.STD)
    pad = (np.array([124.0, 116.0, 104.0]) / 255.0 - np.array(PP.MEAN)) / np.array(PP.STD)
    # 200 wide -> scale 1.92, content 230.4 rows tall, centred: rows 77..306 hold content
    for c in range(3):
        np.testing.assert_allclose(got[c, 100, :], content[c], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got[c, 0, :], pad[c], rtol=0, atol=0)
        np.testing.assert_allclose(got[c, 383, :], pad[c], rtol=0, atol=0)
    oy = (384 - 120 * 1.92) / 2
    rows = np.nonzero(np.abs(got[0, :, 0] - content[0]) < 1e-9)[0]
    assert rows.min() == int(np.ceil(oy - 0.5)) and rows.max() == int(np.ceil(oy + 230.4 - 0.5)) - 1
    # the pad colour is close to, not exactly, the normalisation mean
    assert np.all(np.abs(pad) < 0.01) and np.all(pad != 0)


def test_affine_image_is_reproduced_away_from_the_border():
    """Bilinear sampling reproduces an affine function exactly: away from the
    clamped border each output equals the affine function at the sample position."""
    H, W = 90, 160
    yy, xx = np.mgrid[0:H, 0:W]
    ramp = np.stack([xx + yy, 2 * yy, (xx // 2) * 2], -1).astype(np.float64)   # channel 2 is not affine
    img = ramp.astype(np.uint8)
    box = (20.0, 10.0, 140.0, 80.0)
    got = PP.preprocess(img, box)
    x0, y0, s, ox, oy, bw, bh = PP.box_geometry(box)
    for Y in range(100, 300, 37):
        for X in range(20, 370, 41):
            sx, sy = PP.sample_position(box, X, Y)
            sx, sy = sx - 0.5, sy - 0.5
            if not (1 <= sx <= W - 2 and 1 <= sy <= H - 2):
                continue
            if not (ox <= X + 0.5 < ox + s * bw and oy <= Y + 0.5 < oy + s * bh):
                continue
            want0 = ((sx + sy) / 255.0 - PP.MEAN[0]) / PP.STD[0]
            want1 = ((2 * sy) / 255.0 - PP.MEAN[1]) / PP.STD[1]
            assert abs(got[0, Y, X] - want0) < 1e-12 and abs(got[1, Y, X] - want1) < 1e-12


@pytest.mark.parametrize("box", [(33, 38, 241, 310), (0, 0, 640, 480), (10.5, 20.25, 110.5, 70.25)])
def test_sample_positions_follow_the_roi_coordinate_map(box):
    """The preprocessing samples canvas pixel centre (X + 0.5, Y + 0.5) at the
    image point the ROI map sends the same canvas point to (u = 2 (X + 0.5) / 384 - 1)."""
    XY = RNG.integers(0, 384, (40, 2))
    u = (2.0 * (XY + 0.5)) / 384.0 - 1.0
    img_pts = V.roi_to_image(u, box)
    for (X, Y), p in zip(XY, img_pts):
        sx, sy = PP.sample_position(box, X, Y)
        assert abs(sx - p[0]) < 1e-9 and abs(sy - p[1]) < 1e-9


@pytest.mark.parametrize("box", [(1, 2, 7, 5), (0, 0, 6, 6), (2.5, 0.5, 4.0, 5.5), (-2, -1, 9, 4)])
def test_matches_brute_force_tiny(box):
    H, W, canvas = 5, 7, 12
    img = RNG.integers(0, 256, (H, W, 3), dtype=np.uint8)
    got = PP.preprocess(img, box, canvas)
    nested = img.astype(float).tolist()
    for c in range(3):
        for Y in range(canvas):
            for X in range(canvas):
                assert abs(got[c, Y, X] - brute.preprocess_value(nested, H, W, box, canvas, X, Y, c)) < 1e-12


def test_rejects_degenerate_boxes():
    img = np.zeros((4, 4, 3), np.uint8)
    for box in [(0, 0, 0, 4), (3, 3, 1, 4)]:
        with pytest.raises(ValueError):
            PP.preprocess(img, box)


def test_batch_is_per_box():
    img = RNG.integers(0, 256, (50, 60, 3), dtype=np.uint8)
    boxes = np.array([[0, 0, 60, 50], [5, 5, 25, 45]], np.float32)
    got = PP.preprocess_batch(img, boxes)
    assert got.shape == (2, 3, 384, 384)
    np.testing.assert_array_equal(got[1], PP.preprocess(img, boxes[1]))
