"""CPU oracle for variants of the GKDT detection head that sit beside the graded path.

TEST INFRASTRUCTURE ONLY (same import rule as gkd_oracle): only the tests, the
package's smoke check and the benchmark's CPU legs may import this module, and
it imports nothing from the product package.

Three variants, each written from its definition in float64 with the graded
oracle's primitives (interpolation rule, bf16 rounding, decode rule):

  fusion by linearity
     The graded head fuses the two modalities of a prompt row by averaging
     their heatmaps (masked fusion per prompt row: GKD_GGUF model card, Model
     section, Architecture bullet; text and visual prompts combined row by
     row: Prompts bullet). The heatmap is linear in the kernel row, so the
     mean of the two heatmaps equals the heatmap of the mean of the two
     normalised kernel rows. This variant contracts once per row instead of
     once per (modality, row).
  contract then upsample
     The graded order is upsample, then the 1x1 contraction (model card,
     Architecture bullet). Both steps are linear, so contracting on the h x w
     source grid and upsampling each row's map gives the same heatmaps in
     exact arithmetic, with 16x fewer multiply-adds.
  ROI -> image coordinates
     The decoded keypoint lies in the ROI's normalised -1..1 space (model
     card, Output bullet). The ROI was resized so that its longer side is 384
     pixels and centre-padded to a 384 x 384 canvas (model card, Model
     section, Input bullet); undoing the pad and the resize gives the point in
     the original image.

Readings where the pages are silent (each is also listed in the design notes):
  * fusion by linearity, bf16 operands: the mean of the two normalised rows is
    formed unrounded and rounded once to bf16. A row with one modality uses
    that modality's normalised row unchanged.
  * contract then upsample, bf16 operands: the stored features are rounded
    to bf16, as the kernel rows are. The contraction and the upsample of its
    result are unrounded (fp64 here; fp32 accumulation on the GPU).
  * ROI -> image: the -1..1 space spans the whole padded canvas, with pixel
    edges at integer canvas coordinates, so u maps to canvas pixel
    (u + 1) * 384 / 2. The resize scale is 384 / max(box width, box height),
    and the pad is exactly centred, with no rounding of the resized size or
    of the offsets.

Parity: pinned in tests/test_oracle_variants.py by the linearity identities
against the graded oracle in float64, closed forms (one-hot and constant
maps), the pure-Python brute force (oracle/brute.py), and, for the coordinate
map, its fixed points and the pages' bounding-box example.
"""
from __future__ import annotations

import numpy as np

from oracle import gkd_oracle as O

CANVAS = 384          # model input side in pixels (model card, Input bullet)


# ----------------------------------------------------------------------------
# fusion by linearity
# ----------------------------------------------------------------------------
def fused_kernel_rows(khat: np.ndarray, mask: np.ndarray, operand: str = "f32"):
    """Per prompt row, the mean of the normalised rows of the modalities present.

    khat [Bk][M][K][C] (normalised, float64, zero where masked), mask [Bk][M][K].
    Returns (kf [Bk][K][C] float64, row_valid [Bk][K] uint8). operand "bf16"
    rounds each fused row once to bf16 after the mean; rows with a single
    modality are that modality's row, rounded the same way."""
    khat = np.asarray(khat, np.float64)
    mask = np.asarray(mask)
    Bk, M, K, C = khat.shape
    kf = np.zeros((Bk, K, C), np.float64)
    valid = np.zeros((Bk, K), np.uint8)
    for b in range(Bk):
        for k in range(K):
            present = [m for m in range(M) if mask[b, m, k]]
            if not present:
                continue
            row = khat[b, present[0], k].copy()
            if len(present) == 2:
                row = (row + khat[b, present[1], k]) * 0.5
            kf[b, k] = O.bf16_round(row) if operand == "bf16" else row
            valid[b, k] = 1
    return kf, valid


def head_fused_kernels(feat: np.ndarray, rows: np.ndarray, mask: np.ndarray, *, operand: str,
                       up: int = 4, crops=None, eps: float = 1e-12):
    """The head with modality fusion moved before the contraction.

    feat [B][h][w][C] stored feature values, rows [Bk][M][K][C] raw prompt rows,
    mask [Bk][M][K]. Returns (heat [B][K][H][W] float64 with NaN on invalid rows,
    decode tuple of gkd_oracle.fuse_decode on the one fused map per row)."""
    khat = O.norm_rows(rows, mask, eps)
    kf, valid = fused_kernel_rows(khat, mask, operand)
    heat = O.heatmaps(feat, kf[:, None], valid[:, None], up, operand, crops)[:, 0]
    vsel = valid if (valid.shape[0] == 1 or crops is None) else valid[list(crops)]
    dec = O.fuse_decode(np.nan_to_num(heat, nan=0.0)[:, None], vsel[:, None])
    return heat, dec


# ----------------------------------------------------------------------------
# contract then upsample
# ----------------------------------------------------------------------------
def heatmap_crop_contract_first(feat: np.ndarray, kern: np.ndarray, mask: np.ndarray, up: int = 4,
                                operand: str = "f32") -> np.ndarray:
    """heat[m,k] = Up(G[m,k]), G[m,k,i,j] = sum_c kern[m,k,c] * F[i,j,c] on the source grid.

    feat [h][w][C], kern [M][K][C] (stored operand values). operand "bf16"
    rounds the features to bf16 before the contraction. Returns [M][K][H][W]
    float64 with NaN on invalid rows."""
    F = np.asarray(feat, np.float64)
    if operand == "bf16":
        F = O.bf16_round(F)
    h, w, C = F.shape
    M, K, _ = kern.shape
    heat = np.full((M, K, up * h, up * w), np.nan, np.float64)
    Ff = F.reshape(h * w, C)
    for m in range(M):
        for k in range(K):
            if not mask[m, k]:
                continue
            G = (Ff @ np.asarray(kern[m, k], np.float64)).reshape(h, w, 1)
            heat[m, k] = O.upsample(G, up)[:, :, 0]
    return heat


def head_contract_first(feat: np.ndarray, rows: np.ndarray, mask: np.ndarray, *, operand: str,
                        up: int = 4, eps: float = 1e-12):
    """Steps a2..a6 with the contraction on the source grid: returns the fp64
    heatmaps [B][M][K][H][W] and the decode of them (graded fusion and decode)."""
    khat = O.norm_rows(rows, mask, eps)
    if operand == "bf16":
        khat = O.bf16_round(khat)
    B = feat.shape[0]
    heat = np.stack([heatmap_crop_contract_first(feat[b], khat[0 if khat.shape[0] == 1 else b],
                                                 mask[0 if mask.shape[0] == 1 else b], up, operand)
                     for b in range(B)])
    return heat, O.fuse_decode(np.nan_to_num(heat, nan=0.0), mask)


# ----------------------------------------------------------------------------
# ROI -> image coordinates
# ----------------------------------------------------------------------------
def _box_geometry(box, canvas: int):
    x0, y0, x1, y1 = (float(v) for v in box)
    bw, bh = x1 - x0, y1 - y0
    if not (bw > 0 and bh > 0):
        raise ValueError("box must have positive width and height")
    s = canvas / max(bw, bh)                       # resize scale, longer side -> canvas
    ox, oy = (canvas - bw * s) / 2.0, (canvas - bh * s) / 2.0   # centred pad
    return x0, y0, s, ox, oy


def roi_to_image(xy: np.ndarray, box, canvas: int = CANVAS) -> np.ndarray:
    """Normalised ROI coordinates xy [..., 2] in -1..1 -> original-image pixels.

    box = (x0, y0, x1, y1) of the ROI in the original image (the whole image
    is (0, 0, width, height)). canvas pixel p = (u + 1) * canvas / 2; then the
    centred pad is removed and the resize undone."""
    x0, y0, s, ox, oy = _box_geometry(box, canvas)
    u = np.asarray(xy, np.float64)
    px = (u[..., 0] + 1.0) * canvas / 2.0
    py = (u[..., 1] + 1.0) * canvas / 2.0
    return np.stack([x0 + (px - ox) / s, y0 + (py - oy) / s], axis=-1)


def image_to_roi(pt: np.ndarray, box, canvas: int = CANVAS) -> np.ndarray:
    """Original-image pixels [..., 2] -> normalised ROI coordinates (the forward map)."""
    x0, y0, s, ox, oy = _box_geometry(box, canvas)
    p = np.asarray(pt, np.float64)
    px = (p[..., 0] - x0) * s + ox
    py = (p[..., 1] - y0) * s + oy
    return np.stack([2.0 * px / canvas - 1.0, 2.0 * py / canvas - 1.0], axis=-1)
