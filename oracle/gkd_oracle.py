"""CPU oracle for the GKDT parameter-free detection head.

TEST INFRASTRUCTURE ONLY. Only the tests, the package's smoke check and the
benchmark's CPU-baseline / reference leg may import this module; the product
path never does, and this module imports nothing from the product package.

Plain, slow, obviously-correct restatement of the head in float64 numpy. Every
step is computed from its definition, in the order the sources give, with no
blocking or fusion (a BLAS matmul serves as the contraction step):

  a1 Gaussian prototype pooling of support features at keypoints (visual
     prompts pooled with a Gaussian of sigma 14: GKD_GGUF model card, Model
     section, Prompts bullet; Gaussian weights on the support image: GKDT
     summary page, pipeline paragraph; visual keypoint prototypes: GKDT reading
     notes, Method section)
  a2 L2 normalisation of prompt rows, K padded to 80 with a validity mask
     (model card, Model section, Architecture bullet; normalised convolution:
     reading notes, Method section)
  a3 bilinear 4x upsample of the query feature map, align_corners=False
     (model card, Architecture bullet; the 96x96 grid: model card, Output
     bullet)
  a4 1x1 dynamic-kernel contraction heat = sum_c kernel[c] * U[c, p]
     (prompts applied as 1x1 kernels: model card, Architecture bullet; kernels
     convolved over the query features: summary page, pipeline paragraph)
  a5 per-row masked fusion across modalities, mean of those present
     (masked fusion per prompt row: model card, Architecture bullet; text and
     visual prompts combined row by row: Prompts bullet)
  a6 argmax decode to ROI coordinates in -1..1 plus the peak score
     (each prompt's heatmap peak on the 96x96 grid, mapped to the ROI's
     normalised -1..1 space, with a confidence score: model card, Output
     bullet)

Readings taken where the pages are silent (each is listed in the design notes):
  * pooling evaluates the Gaussian at patch centres S*(j+0.5) of the support
    grid, over the whole grid, normalised by the sum of weights; the common
    factor exp(d2_min / 2 sigma^2) is removed from every weight, which cancels
    in the ratio and keeps the largest weight at exactly 1;
  * only the prompt rows are L2-normalised; eps = 1e-12 on the norm;
  * upsample with PyTorch's half-pixel rule, negative source coordinates
    clamped to 0 and the upper neighbour clamped to the last row/column;
  * bf16 operand mode rounds the normalised rows and the upsampled features to
    bf16 (round to nearest even, directly from float64) and contracts in fp64;
  * score = raw fused peak; x = (2*col + 1 - W) / W in one fp32 division
    (= 2(col+0.5)/W - 1, correctly rounded); ties go to the lowest row-major
    index; invalid rows decode to idx -1, xy (0,0), score 0, valid 0.

Parity: pinned (see tests/test_oracle_pins.py) by closed forms, invariants,
library special cases, hand-computed golden values and a pure-Python brute
force (oracle/brute.py) on tiny inputs.
"""
from __future__ import annotations

import math

import numpy as np


# ----------------------------------------------------------------------------
# bf16 helpers (operand rounding points)
# ----------------------------------------------------------------------------
def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even, in one
    step (no intermediate fp32 rounding). bf16 keeps 8 significant bits; its
    spacing in [2^e, 2^(e+1)) is 2^(e-7), with subnormal spacing 2^-133 and
    overflow to +-inf above the largest finite bf16 value."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    m, e = np.frexp(x[nz])                     # x = m * 2^e, 0.5 <= |m| < 1
    q_exp = np.maximum(e - 8, -133)            # exponent of the bf16 spacing
    q = np.ldexp(1.0, q_exp)
    r = np.rint(x[nz] / q) * q                 # rint rounds half to even; /q exact
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = np.where(np.abs(r) > bf16_max, np.copysign(np.inf, r), r)
    out[nz] = r
    out[~nz] = x[~nz]
    return out


# ----------------------------------------------------------------------------
# a1: Gaussian prototype pooling
# ----------------------------------------------------------------------------
def pool_weights(h: int, w: int, x: float, y: float, sigma: float, stride: float) -> np.ndarray:
    """Gaussian weights [h][w] of one keypoint (x, y) (ROI pixels) at the patch
    centres X_j = stride*(j+0.5), Y_i = stride*(i+0.5), each divided by the
    largest one (common factor, cancels after normalisation)."""
    X = stride * (np.arange(w, dtype=np.float64) + 0.5)
    Y = stride * (np.arange(h, dtype=np.float64) + 0.5)
    d2 = (X[None, :] - float(x)) ** 2 + (Y[:, None] - float(y)) ** 2
    return np.exp(-(d2 - d2.min()) / (2.0 * float(sigma) ** 2))


def pool_prototypes(support: np.ndarray, kpts: np.ndarray, kmask: np.ndarray,
                    sigma: float, stride: float) -> np.ndarray:
    """proto[b,k,:] = sum_ij w_ij F[b,i,j,:] / sum_ij w_ij for valid keypoints,
    zero rows for invalid ones. support [B][h][w][C] -> float64 [B][K][C]."""
    F = np.asarray(support, dtype=np.float64)
    B, h, w, C = F.shape
    K = kpts.shape[1]
    proto = np.zeros((B, K, C), np.float64)
    for b in range(B):
        Fb = F[b].reshape(h * w, C)
        for k in range(K):
            if not kmask[b, k]:
                continue
            wts = pool_weights(h, w, kpts[b, k, 0], kpts[b, k, 1], sigma, stride).reshape(h * w)
            proto[b, k] = (wts @ Fb) / wts.sum()
    return proto


# ----------------------------------------------------------------------------
# a2: L2 normalisation of prompt rows
# ----------------------------------------------------------------------------
def norm_rows(rows: np.ndarray, mask: np.ndarray, eps: float = 1e-12) -> np.ndarray:
    """k_hat = k / max(||k||_2, eps) for valid rows; zero rows where mask == 0.
    rows [Bk][M][K][C] -> float64."""
    r = np.asarray(rows, dtype=np.float64)
    nrm = np.sqrt((r * r).sum(axis=-1, keepdims=True))
    out = r / np.maximum(nrm, eps)
    return np.where(np.asarray(mask)[..., None] != 0, out, 0.0)


# ----------------------------------------------------------------------------
# a3: bilinear upsample (align_corners=False, clamped borders)
# ----------------------------------------------------------------------------
def interp_matrix(n: int, up: int) -> np.ndarray:
    """R [up*n][n]: output index d takes source coordinate
    s = max((d + 0.5)/up - 0.5, 0), i0 = floor(s), i1 = min(i0 + 1, n - 1),
    weights (1 - (s - i0)) on i0 and (s - i0) on i1."""
    R = np.zeros((up * n, n), np.float64)
    for d in range(up * n):
        s = max((d + 0.5) / up - 0.5, 0.0)
        i0 = int(math.floor(s))
        i0 = min(i0, n - 1)
        i1 = min(i0 + 1, n - 1)
        lam1 = s - i0
        R[d, i0] += 1.0 - lam1
        R[d, i1] += lam1
    return R


def upsample(feat: np.ndarray, up: int = 4, out_rows=None) -> np.ndarray:
    """U[Y,X,c] = sum_i sum_j Ry[Y,i] Rx[X,j] F[i,j,c]; feat [h][w][C] -> [H][W][C] float64.
    `out_rows` restricts the result to those output rows Y (in that order)."""
    F = np.asarray(feat, dtype=np.float64)
    h, w, C = F.shape
    Ry = interp_matrix(h, up)
    if out_rows is not None:
        Ry = Ry[list(out_rows)]
    Rx = interp_matrix(w, up)
    tmp = np.einsum("Xj,ijc->iXc", Rx, F)       # along x
    return np.einsum("Yi,iXc->YXc", Ry, tmp)    # then along y


# ----------------------------------------------------------------------------
# a4: 1x1 dynamic-kernel contraction
# ----------------------------------------------------------------------------
def heatmap_crop(feat: np.ndarray, kern: np.ndarray, mask: np.ndarray, up: int = 4,
                 operand: str = "f32", out_rows=None) -> np.ndarray:
    """heat[m,k,Y,X] = sum_c kern[m,k,c] * U[Y,X,c] for valid rows (NaN elsewhere).

    feat [h][w][C] and kern [M][K][C] hold the stored operand values (already
    widened to float64). operand == "bf16": U is rounded to bf16 before the
    contraction (the kernel rows are bf16 already); the sum is float64.
    `out_rows` restricts the heatmaps to those output rows."""
    U = upsample(feat, up, out_rows)
    if operand == "bf16":
        U = bf16_round(U)
    H, W, C = U.shape
    M, K, _ = kern.shape
    heat = np.full((M, K, H, W), np.nan, np.float64)
    Uf = U.reshape(H * W, C)
    for m in range(M):
        ks = [k for k in range(K) if mask[m, k]]
        if ks:
            heat[m, ks] = (Uf @ np.asarray(kern[m, ks], np.float64).T).T.reshape(len(ks), H, W)
    return heat


def heatmaps(feat: np.ndarray, kern: np.ndarray, mask: np.ndarray, up: int = 4,
             operand: str = "f32", crops=None) -> np.ndarray:
    """Batched heatmap_crop; kern/mask with a leading dim of 1 are shared by all crops."""
    B = feat.shape[0]
    crops = range(B) if crops is None else crops
    out = []
    for b in crops:
        kb = 0 if kern.shape[0] == 1 else b
        out.append(heatmap_crop(feat[b], kern[kb], mask[kb], up, operand))
    return np.stack(out)


# ----------------------------------------------------------------------------
# a5 + a6: masked per-row fusion and argmax decode
# ----------------------------------------------------------------------------
def fuse_decode(heat: np.ndarray, mask: np.ndarray):
    """heat [B][M][K][H][W] (fp32 or fp64; arithmetic stays in that type),
    mask [B or 1][M][K]. Returns fused [B][K][H][W], idx int32 [B][K],
    xy float32 [B][K][2], score float32 [B][K], valid uint8 [B][K]."""
    B, M, K, H, W = heat.shape
    dt = heat.dtype.type
    fused = np.zeros((B, K, H, W), heat.dtype)
    idx = np.full((B, K), -1, np.int32)
    xy = np.zeros((B, K, 2), np.float32)
    score = np.zeros((B, K), np.float32)
    valid = np.zeros((B, K), np.uint8)
    half = dt(0.5)
    for b in range(B):
        mb = mask[0 if mask.shape[0] == 1 else b]
        for k in range(K):
            present = [m for m in range(M) if mb[m, k]]
            if not present:
                continue
            if len(present) == 2:
                f = (heat[b, 0, k] + heat[b, 1, k]) * half
            else:
                f = heat[b, present[0], k].copy()
            fused[b, k] = f
            p = int(np.argmax(f.reshape(-1)))      # first maximal index
            idx[b, k] = p
            score[b, k] = np.float32(f.reshape(-1)[p])
            col, row = p % W, p // W
            xy[b, k, 0] = np.float32(2 * col + 1 - W) / np.float32(W)
            xy[b, k, 1] = np.float32(2 * row + 1 - H) / np.float32(H)
            valid[b, k] = 1
    return fused, idx, xy, score, valid


def top2_margin(fused_row: np.ndarray) -> float:
    """Peak value minus the largest value at any other pixel of one fused row."""
    f = np.asarray(fused_row, np.float64).reshape(-1)
    p = int(np.argmax(f))
    rest = np.delete(f, p)
    return float(f[p] - rest.max()) if rest.size else float("inf")


# ----------------------------------------------------------------------------
# the whole head
# ----------------------------------------------------------------------------
def head(feat: np.ndarray, rows: np.ndarray, mask: np.ndarray, *, operand: str, up: int = 4,
         crops=None, eps: float = 1e-12):
    """Steps a2..a6 on stored operand values (feat widened to float64, rows raw
    fp32): returns the fp64 heatmaps and the fp64 decode of them."""
    khat = norm_rows(rows, mask, eps)
    if operand == "bf16":
        khat = bf16_round(khat)
    heat = heatmaps(feat, khat, mask, up, operand, crops)
    msel = mask if (mask.shape[0] == 1 or crops is None) else mask[list(crops)]
    return heat, fuse_decode(np.nan_to_num(heat, nan=0.0), msel)
