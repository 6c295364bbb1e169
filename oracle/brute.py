"""Pure-Python brute force of the GKDT detection head on tiny inputs.

TEST INFRASTRUCTURE ONLY (same import rule as gkd_oracle). A second,
structurally different restatement used to pin the numpy oracle: nested lists,
Python floats (IEEE double), one output element at a time, and the upsample as
a direct 4-tap sum per pixel instead of separable interpolation matrices.
Sources as in gkd_oracle: GKD_GGUF model card, Model section (Architecture,
Prompts and Output bullets) and the GKDT summary page, pipeline paragraph.
"""
from __future__ import annotations

import math


def taps(d: int, n: int, up: int):
    """The two source indices and weights that output index d reads
    (half-pixel rule, align_corners=False, borders clamped)."""
    s = (d + 0.5) / up - 0.5
    if s < 0.0:
        s = 0.0
    i0 = int(s)                     # s >= 0, so int() is floor
    i1 = i0 + 1 if i0 + 1 < n else n - 1
    frac = s - i0
    return (i0, 1.0 - frac), (i1, frac)


def up_value(F, h: int, w: int, c: int, Y: int, X: int, up: int) -> float:
    """Upsampled feature U[Y][X][c] as the 4-tap bilinear sum. F[i][j][c]."""
    total = 0.0
    for (iy, wy) in taps(Y, h, up):
        for (ix, wx) in taps(X, w, up):
            total += wy * wx * F[iy][ix][c]
    return total


def heat_value(F, h: int, w: int, C: int, kern_row, Y: int, X: int, up: int, rnd=None) -> float:
    """sum_c kern_row[c] * U[Y][X][c]; `rnd` optionally rounds each U value first."""
    acc = 0.0
    for c in range(C):
        u = up_value(F, h, w, c, Y, X, up)
        if rnd is not None:
            u = rnd(u)
        acc += kern_row[c] * u
    return acc


def pool_row(S, h: int, w: int, C: int, x: float, y: float, sigma: float, stride: float):
    """Gaussian-weighted mean of the support patches around keypoint (x, y)."""
    d2 = [[(stride * (j + 0.5) - x) ** 2 + (stride * (i + 0.5) - y) ** 2 for j in range(w)]
          for i in range(h)]
    dmin = min(min(r) for r in d2)
    num = [0.0] * C
    den = 0.0
    for i in range(h):
        for j in range(w):
            wt = math.exp(-(d2[i][j] - dmin) / (2.0 * sigma * sigma))
            den += wt
            for c in range(C):
                num[c] += wt * S[i][j][c]
    return [v / den for v in num]


def norm_row(row, eps: float = 1e-12):
    n = math.sqrt(sum(v * v for v in row))
    n = n if n > eps else eps
    return [v / n for v in row]


def argmax_first(values) -> int:
    best = 0
    for p in range(1, len(values)):
        if values[p] > values[best]:
            best = p
    return best


def contract_first_value(F, h: int, w: int, C: int, kern_row, Y: int, X: int, up: int, rnd=None) -> float:
    """Heatmap value with the contraction on the source grid: the 4-tap bilinear
    sum of g[i][j] = sum_c kern_row[c] * F[i][j][c]; `rnd` optionally rounds
    each feature value first."""
    total = 0.0
    for (iy, wy) in taps(Y, h, up):
        for (ix, wx) in taps(X, w, up):
            g = 0.0
            for c in range(C):
                f = F[iy][ix][c]
                if rnd is not None:
                    f = rnd(f)
                g += kern_row[c] * f
            total += wy * wx * g
    return total


def mean_row(rows):
    """Elementwise mean of one or two equal-length rows."""
    if len(rows) == 1:
        return list(rows[0])
    return [(a + b) * 0.5 for a, b in zip(rows[0], rows[1])]


def preprocess_value(img, H: int, W: int, box, canvas: int, X: int, Y: int, ch: int) -> float:
    """One normalised output value of the image preprocessing (model card, Model
    section, Input bullet: longer side resized to the canvas, centre pad with
    (124, 116, 104), ImageNet normalisation), one pixel at a time: img[y][x][c]
    nested lists of 0..255 values, box (x0, y0, x1, y1)."""
    x0, y0, x1, y1 = box
    bw, bh = x1 - x0, y1 - y0
    longer = bw if bw > bh else bh
    s = canvas / longer
    ox = (canvas - s * bw) / 2.0
    oy = (canvas - s * bh) / 2.0
    cx, cy = X + 0.5, Y + 0.5
    mean = (0.485, 0.456, 0.406)[ch]
    std = (0.229, 0.224, 0.225)[ch]
    if not (ox <= cx < ox + s * bw and oy <= cy < oy + s * bh):
        v = (124.0, 116.0, 104.0)[ch]
    else:
        sx = x0 + (cx - ox) / s - 0.5
        sy = y0 + (cy - oy) / s - 0.5
        fx, fy = math.floor(sx), math.floor(sy)
        v = 0.0
        for (iy, wy) in ((fy, 1.0 - (sy - fy)), (fy + 1, sy - fy)):
            for (ix, wx) in ((fx, 1.0 - (sx - fx)), (fx + 1, sx - fx)):
                cyi = min(max(iy, 0), H - 1)
                cxi = min(max(ix, 0), W - 1)
                v += wy * wx * img[cyi][cxi][ch]
    return (v / 255.0 - mean) / std
