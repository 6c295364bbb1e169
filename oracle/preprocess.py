"""CPU oracle for the image preprocessing in front of the GKDT detection head.

TEST INFRASTRUCTURE ONLY (same import rule as gkd_oracle): only the tests, the
package's smoke check and the benchmark's CPU legs may import this module, and
it imports nothing from the product package.

The model card (GKD_GGUF, Model section, Input bullet) states the input
pipeline: the ROI is resized so that its longer side is 384 pixels, centre-padded
to a 384 x 384 canvas with the mean colour (124, 116, 104), and normalised with
the ImageNet mean and standard deviation. It names no interpolation filter and
no rounding. Readings (each also listed in the design notes):

  * One inverse-mapped resample with the geometry of the ROI -> image map
    (oracle/variants.py): scale s = canvas / max(box width, box height), pad
    offsets ox = (canvas - s * bw) / 2, oy = (canvas - s * bh) / 2, not rounded.
    Canvas pixel (X, Y), centred at (X + 0.5, Y + 0.5), is image content iff
    ox <= X + 0.5 < ox + s * bw and oy <= Y + 0.5 < oy + s * bh; otherwise it
    takes the pad colour.
  * Content pixels take the bilinear sample of the image at
    x = x0 + (X + 0.5 - ox) / s - 0.5, y = y0 + (Y + 0.5 - oy) / s - 0.5
    (pixel centres at integer + 0.5 in edge coordinates, as in the ROI map),
    with both taps of each axis clamped to the image (the image outside the box
    is sampled where the taps reach it). No antialiasing filter; the arithmetic
    is real-valued (no rounding back to 8 bits).
  * Normalisation (v / 255 - mean_c) / std_c with mean (0.485, 0.456, 0.406)
    and std (0.229, 0.224, 0.225), for pad pixels too. Output planes [3][H][W]
    (channel-major, as the backbone takes them); input uint8 [H][W][3] RGB.

Parity: pinned in tests/test_oracle_preprocess.py by PyTorch's bilinear
interpolation (align_corners=False) where the geometry coincides with a plain
resize, constant and affine images (bilinear sampling reproduces them exactly
away from the clamped border), the pad colour, agreement of the sample
positions with the ROI -> image coordinate map, and a pure-Python brute force
(oracle/brute.py) on tiny images.
"""
from __future__ import annotations

import math

import numpy as np

CANVAS = 384
PAD_RGB = (124.0, 116.0, 104.0)
MEAN = (0.485, 0.456, 0.406)
STD = (0.229, 0.224, 0.225)


def box_geometry(box, canvas: int = CANVAS):
    """(x0, y0, s, ox, oy, bw, bh) of a box (x0, y0, x1, y1) in image pixels."""
    x0, y0, x1, y1 = (float(v) for v in box)
    bw, bh = x1 - x0, y1 - y0
    if not (bw > 0 and bh > 0):
        raise ValueError("box must have positive width and height")
    s = canvas / max(bw, bh)
    return x0, y0, s, (canvas - s * bw) / 2.0, (canvas - s * bh) / 2.0, bw, bh


def axis_taps(n_out: int, n_in: int, origin: float, s: float, offset: float, extent: float):
    """Per output index d: (inside, i0, i1, lam) with the sample at
    origin + (d + 0.5 - offset) / s - 0.5, taps floor and floor + 1 clamped to
    [0, n_in - 1], weight lam on i1."""
    d = np.arange(n_out, dtype=np.float64)
    c = d + 0.5
    inside = (c >= offset) & (c < offset + s * extent)
    x = origin + (c - offset) / s - 0.5
    f = np.floor(x)
    lam = x - f
    i0 = np.clip(f, 0, n_in - 1).astype(np.int64)
    i1 = np.clip(f + 1, 0, n_in - 1).astype(np.int64)
    return inside, i0, i1, lam


def preprocess(img: np.ndarray, box, canvas: int = CANVAS) -> np.ndarray:
    """uint8 image [H][W][3] and a box (x0, y0, x1, y1) -> float64 [3][canvas][canvas]."""
    im = np.asarray(img, dtype=np.float64)
    H, W, _ = im.shape
    x0, y0, s, ox, oy, bw, bh = box_geometry(box, canvas)
    inx, xa, xb, lx = axis_taps(canvas, W, x0, s, ox, bw)
    iny, ya, yb, ly = axis_taps(canvas, H, y0, s, oy, bh)
    top = (1.0 - lx)[None, :, None] * im[ya][:, xa] + lx[None, :, None] * im[ya][:, xb]
    bot = (1.0 - lx)[None, :, None] * im[yb][:, xa] + lx[None, :, None] * im[yb][:, xb]
    val = (1.0 - ly)[:, None, None] * top + ly[:, None, None] * bot          # [canvas][canvas][3]
    content = iny[:, None] & inx[None, :]
    val = np.where(content[..., None], val, np.asarray(PAD_RGB)[None, None, :])
    out = (val / 255.0 - np.asarray(MEAN)) / np.asarray(STD)
    return np.ascontiguousarray(out.transpose(2, 0, 1))


def preprocess_batch(img: np.ndarray, boxes: np.ndarray, canvas: int = CANVAS) -> np.ndarray:
    """One image, B boxes -> float64 [B][3][canvas][canvas]."""
    return np.stack([preprocess(img, b, canvas) for b in np.asarray(boxes)])


def sample_position(box, X: float, Y: float, canvas: int = CANVAS):
    """Image coordinates (edge convention: pixel p spans [p, p + 1)) of the centre
    of canvas pixel (X, Y), the point whose bilinear sample it takes."""
    x0, y0, s, ox, oy, _, _ = box_geometry(box, canvas)
    return x0 + (X + 0.5 - ox) / s, y0 + (Y + 0.5 - oy) / s


def normalised_pad(canvas_unused: int = CANVAS) -> np.ndarray:
    """The normalised value of a pad pixel, per channel."""
    return (np.asarray(PAD_RGB) / 255.0 - np.asarray(MEAN)) / np.asarray(STD)


__all__ = ["CANVAS", "PAD_RGB", "MEAN", "STD", "box_geometry", "axis_taps", "preprocess", "preprocess_batch",
           "sample_position", "normalised_pad", "math"]
