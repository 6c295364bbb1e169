"""Seeded synthetic inputs shaped like the GKDT-L detection head's workloads.

This module only draws random numbers and stores them in the documented
layouts. It holds no step of the head's arithmetic (no pooling, no
normalisation, no upsampling, no contraction, no decoding), so the CUDA path
and the CPU oracle can both consume its arrays without sharing any of the
method's code.

Layouts (row-major, last index contiguous):
  features  [B][h][w][C]      fp32, or bf16 stored as uint16 bit patterns
  support   [B][h][w][C]      fp32 (configs with visual prompts from pooling)
  kpts      [B][K][2]         fp32 (x, y) in ROI pixels
  kmask     [B][K]            uint8 0/1
  rows      [Bk][M][K][C]     fp32 raw prompt rows (modality 0 visual, 1 text)
  mask      [Bk][M][K]        uint8 0/1

Values are drawn in logical order [c][y][x] per crop and then transposed to
NHWC, so the storage layout never changes the data. Each (purpose, crop) pair
has its own PCG64 stream keyed by SeedSequence(1000 + config, spawn_key), so any
subset of crops can be regenerated alone.

The five workloads follow the GKDT-L model card: a DINOv3 ViT-L query map of
24x24 patches (384 px input, patch 16) with C=1024 channels, prompts padded to
80 rows, a 4x bilinear upsample to a 96x96 heatmap grid, and visual prompts
pooled with a Gaussian of sigma 14 px (GKD_GGUF model card, Model section).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# purposes of the independent random streams
_FEAT, _SUPPORT, _ROWS, _KPTS, _COUNTS, _PEAKS = range(6)


@dataclass
class Workload:
    """One batch of synthetic head inputs (numpy, host memory)."""
    name: str
    B: int
    h: int
    w: int
    C: int
    K: int
    M: int
    up: int
    feat: np.ndarray                 # fp32 [B][h][w][C] or uint16 bf16 bits
    feat_dtype: str                  # "f32" | "bf16"
    rows: np.ndarray | None          # fp32 [Bk][M][K][C] raw prompt rows (None for pooled-only)
    mask: np.ndarray                 # uint8 [Bk][M][K]
    Bk: int                          # B, or 1 when one prompt set is shared
    kern_dtype: str                  # operand type of the contraction: "f32" | "bf16"
    support: np.ndarray | None = None    # fp32 [B][h][w][C]
    kpts: np.ndarray | None = None       # fp32 [B][K][2]
    kmask: np.ndarray | None = None      # uint8 [B][K]
    sigma: float = 14.0
    stride: float = 16.0
    pooled_modality: int | None = None   # which modality's rows come from pooling
    extra: dict = field(default_factory=dict)

    @property
    def H(self) -> int:
        return self.up * self.h

    @property
    def W(self) -> int:
        return self.up * self.w


_SHARD = 0   # data shard of the calling process (set by make_config's `shard`)


def _rng(cfg_seed: int, purpose: int, b: int = 0) -> np.random.Generator:
    key = (purpose, b) if _SHARD == 0 else (purpose, b, _SHARD)
    ss = np.random.SeedSequence(entropy=cfg_seed, spawn_key=key)
    return np.random.Generator(np.random.PCG64(ss))


def _normal_nhwc(g: np.random.Generator, C: int, h: int, w: int, scale: float = 1.0) -> np.ndarray:
    x = g.standard_normal((C, h, w), dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return np.ascontiguousarray(x.transpose(1, 2, 0))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Store finite fp32 values as bf16 (round to nearest, ties to even),
    returned as uint16 bits. A storage cast for input preparation only: the
    upper 16 bits after adding 0x7FFF plus the lowest kept bit (the usual
    integer form of round-half-even on the dropped 16 bits)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# The five workloads
# ----------------------------------------------------------------------------
CONFIG_NAMES = {
    1: "gkdt-l single crop, fp32, visual-only 17/80 rows, pooled prompts",
    2: "gkdt-l batch 64, dual prompt, rows U{5..80}/80, bf16 operands",
    3: "wide backbone C=1280, batch 256, mixed modality, rows U{40..80}/80, bf16",
    4: "top-down batch 1024 crops, shared 17+17 prompt rows, bf16 features with planted peaks",
    5: "high-res 768px: 48x48 -> 192x192, batch 32, 80+80 rows, pooled sigma 28, bf16",
}


def _crop_list(B: int, crops) -> list[int]:
    if crops is None:
        return list(range(B))
    return [int(b) for b in crops]


def make_config(cfg: int, crops=None, shard: int = 0) -> Workload:
    """Inputs of workload `cfg` (1..5). `crops` selects a subset of crop indices
    (the selected crops get exactly the values they have in the full batch).
    `shard` > 0 draws an independent batch of the same distribution (one per
    data-parallel rank); shard 0 is the canonical batch."""
    global _SHARD
    _SHARD = int(shard)
    try:
        return _make_config(cfg, crops)
    finally:
        _SHARD = 0


def _make_config(cfg: int, crops) -> Workload:
    seed = 1000 + cfg
    if cfg == 1:
        return _pooled_workload(seed, "cfg1", B=1, h=24, w=24, C=1024, K=80, n_kpts=17,
                                roi=384.0, sigma=14.0, text=False, kern_dtype="f32", crops=crops)
    if cfg == 5:
        return _pooled_workload(seed, "cfg5", B=32, h=48, w=48, C=1024, K=80, n_kpts=80,
                                roi=768.0, sigma=28.0, text=True, kern_dtype="bf16", crops=crops)
    if cfg == 2:
        B, C, K, M = 64, 1024, 80, 2
        sel = _crop_list(B, crops)
        counts = _rng(seed, _COUNTS).integers(5, 81, size=B)
        feat = np.stack([_normal_nhwc(_rng(seed, _FEAT, b), C, 24, 24) for b in sel])
        rows = np.stack([_rng(seed, _ROWS, b).standard_normal((M, K, C), dtype=np.float32) for b in sel])
        mask = np.zeros((len(sel), M, K), np.uint8)
        for i, b in enumerate(sel):
            mask[i, :, :counts[b]] = 1
        return Workload("cfg2", len(sel), 24, 24, C, K, M, 4, feat, "f32", rows, mask, len(sel), "bf16",
                        extra={"counts": counts[sel]})
    if cfg == 3:
        B, C, K, M = 256, 1280, 80, 2
        sel = _crop_list(B, crops)
        g = _rng(seed, _COUNTS)
        counts = g.integers(40, 81, size=B)
        modality = g.integers(0, 3, size=B)       # 0 visual, 1 text, 2 both
        feat = np.stack([_normal_nhwc(_rng(seed, _FEAT, b), C, 24, 24) for b in sel])
        rows = np.stack([_rng(seed, _ROWS, b).standard_normal((M, K, C), dtype=np.float32) for b in sel])
        mask = np.zeros((len(sel), M, K), np.uint8)
        for i, b in enumerate(sel):
            if modality[b] in (0, 2):
                mask[i, 0, :counts[b]] = 1
            if modality[b] in (1, 2):
                mask[i, 1, :counts[b]] = 1
        return Workload("cfg3", len(sel), 24, 24, C, K, M, 4, feat, "f32", rows, mask, len(sel), "bf16",
                        extra={"counts": counts[sel], "modality": modality[sel]})
    if cfg == 4:
        return _topdown_workload(seed, crops)
    raise ValueError(f"unknown workload {cfg}")


def _pooled_workload(seed, name, B, h, w, C, K, n_kpts, roi, sigma, text, kern_dtype, crops):
    sel = _crop_list(B, crops)
    feat = np.stack([_normal_nhwc(_rng(seed, _FEAT, b), C, h, w) for b in sel])
    support = np.stack([_normal_nhwc(_rng(seed, _SUPPORT, b), C, h, w) for b in sel])
    kpts = np.stack([_rng(seed, _KPTS, b).uniform(0.0, roi, size=(K, 2)).astype(np.float32) for b in sel])
    kmask = np.zeros((len(sel), K), np.uint8)
    kmask[:, :n_kpts] = 1
    M = 2 if text else 1
    mask = np.zeros((len(sel), M, K), np.uint8)
    mask[:, 0, :] = kmask
    rows = None
    if text:
        rows = np.zeros((len(sel), M, K, C), np.float32)
        for i, b in enumerate(sel):
            rows[i, 1] = _rng(seed, _ROWS, b).standard_normal((K, C), dtype=np.float32)
        mask[:, 1, :n_kpts] = 1
    return Workload(name, len(sel), h, w, C, K, M, 4, feat, "f32", rows, mask, len(sel), kern_dtype,
                    support=support, kpts=kpts, kmask=kmask, sigma=sigma, stride=16.0,
                    pooled_modality=0)


def _topdown_workload(seed, crops):
    """Config 4: one shared prompt set (17 visual + 17 text rows), bf16 features
    made of N(0, 0.5^2) noise plus, per crop and keypoint k, a Gaussian bump
    (width 1 patch, amplitude 4) centred at a random (u, v) in patch units and
    pointing along d_k = (r_v[k] + r_t[k]) / sqrt(2 C), where r are the raw
    N(0,1) prompt rows (so |d_k| is close to 1)."""
    B, C, K, M, n = 1024, 1024, 80, 2, 17
    h = w = 24
    amp = 4.0
    sel = _crop_list(B, crops)
    rows = _rng(seed, _ROWS, 0).standard_normal((1, M, K, C), dtype=np.float32)
    mask = np.zeros((1, M, K), np.uint8)
    mask[0, :, :n] = 1
    d = (rows[0, 0, :n].astype(np.float64) + rows[0, 1, :n].astype(np.float64)) / math.sqrt(2.0 * C)
    jj = np.arange(w, dtype=np.float64) + 0.5
    ii = np.arange(h, dtype=np.float64) + 0.5
    feat = np.empty((len(sel), h, w, C), np.uint16)
    centres = np.empty((len(sel), n, 2), np.float64)
    for t, b in enumerate(sel):
        f = _normal_nhwc(_rng(seed, _FEAT, b), C, h, w, scale=0.5).astype(np.float64)
        uv = _rng(seed, _PEAKS, b).uniform(0.5, 23.5, size=(n, 2))
        centres[t] = uv
        gx = np.exp(-0.5 * (jj[None, :] - uv[:, 0:1]) ** 2)          # [n][w]
        gy = np.exp(-0.5 * (ii[None, :] - uv[:, 1:2]) ** 2)          # [n][h]
        bumps = (gy[:, :, None] * gx[:, None, :]).reshape(n, h * w)  # [n][h*w]
        f += amp * (bumps.T @ d).reshape(h, w, C)
        feat[t] = to_bf16_bits(f.astype(np.float32))
    return Workload("cfg4", len(sel), h, w, C, K, M, 4, feat, "bf16", rows, mask, 1, "bf16",
                    extra={"centres": centres, "amp": amp})


# ----------------------------------------------------------------------------
# Free-form cases for tests (small shapes, ragged tails, edge cases)
# ----------------------------------------------------------------------------
def make_case(seed: int, B: int, h: int, w: int, C: int, K: int, M: int, *,
              feat_dtype: str = "f32", kern_dtype: str = "bf16", shared: bool = False,
              valid: str = "prefix", feat_scale: float = 1.0) -> Workload:
    """A random head batch of any shape. `valid` picks the row mask:
    "prefix" (first n rows per crop, n ~ U{1..K}), "random" (each row 0/1 at
    p=0.6), "all", "none"."""
    g = _rng(seed, _COUNTS)
    Bk = 1 if shared else B
    feat32 = np.stack([_normal_nhwc(_rng(seed, _FEAT, b), C, h, w, feat_scale) for b in range(B)])
    feat = to_bf16_bits(feat32) if feat_dtype == "bf16" else feat32
    rows = np.stack([_rng(seed, _ROWS, b).standard_normal((M, K, C), dtype=np.float32) for b in range(Bk)])
    if valid == "prefix":
        mask = np.zeros((Bk, M, K), np.uint8)
        for b in range(Bk):
            for m in range(M):
                mask[b, m, :g.integers(1, K + 1)] = 1
    elif valid == "random":
        mask = (g.random((Bk, M, K)) < 0.6).astype(np.uint8)
    elif valid == "all":
        mask = np.ones((Bk, M, K), np.uint8)
    elif valid == "none":
        mask = np.zeros((Bk, M, K), np.uint8)
    else:
        raise ValueError(valid)
    return Workload(f"case{seed}", B, h, w, C, K, M, 4, feat, feat_dtype, rows, mask, Bk, kern_dtype)


def make_pool_case(seed: int, B: int, h: int, w: int, C: int, K: int, *, roi: float | None = None,
                   sigma: float = 14.0, stride: float = 16.0, p_valid: float = 0.7):
    """Support maps, keypoints and keypoint mask for the pooling step alone."""
    roi = roi if roi is not None else stride * max(h, w)
    support = np.stack([_normal_nhwc(_rng(seed, _SUPPORT, b), C, h, w) for b in range(B)])
    kpts = np.stack([_rng(seed, _KPTS, b).uniform(0.0, roi, size=(K, 2)).astype(np.float32) for b in range(B)])
    kmask = (_rng(seed, _COUNTS).random((B, K)) < p_valid).astype(np.uint8)
    return support, kpts, kmask


def random_bf16_rows(seed: int, shape, scale: float) -> np.ndarray:
    """N(0, scale^2) values stored as bf16 bits (operands for the contraction alone)."""
    g = _rng(seed, _ROWS, 7)
    return to_bf16_bits(g.standard_normal(shape, dtype=np.float32) * np.float32(scale))


def random_heatmaps(seed: int, B: int, M: int, K: int, H: int, W: int, *, ties: bool = True) -> np.ndarray:
    """fp32 heatmaps [B][M][K][H][W] for the fusion/decode step alone. With
    `ties`, some rows get exact repeated maxima (and +0/-0 pairs) so the
    first-index rule is exercised."""
    g = _rng(seed, _FEAT, 99)
    heat = g.standard_normal((B, M, K, H, W), dtype=np.float32)
    if ties:
        flat = heat.reshape(B * M * K, H * W)
        for r in range(0, flat.shape[0], 3):
            p1, p2 = sorted(g.choice(H * W, size=2, replace=False))
            v = np.float32(9.0 + g.integers(0, 4))
            flat[r, p1] = v
            flat[r, p2] = v
        for r in range(1, flat.shape[0], 7):
            flat[r, :] = np.float32(-1.0)
            flat[r, g.integers(0, H * W)] = np.float32(0.0)
            flat[r, g.integers(0, H * W)] = np.float32(-0.0)
    return heat


def random_image_and_boxes(seed: int, H: int, W: int, B: int) -> tuple[np.ndarray, np.ndarray]:
    """A uint8 RGB frame [H][W][3] of uniform noise and B detector boxes
    (x0, y0, x1, y1) fp32 inside it, each side 10-60% of the frame's, for the
    preprocessing step and the ROI -> image map."""
    g = _rng(seed, _FEAT, 123)
    img = g.integers(0, 256, (H, W, 3), dtype=np.uint8)
    bw = g.uniform(0.1, 0.6, B) * W
    bh = g.uniform(0.1, 0.6, B) * H
    x0 = g.uniform(0, 1, B) * (W - bw)
    y0 = g.uniform(0, 1, B) * (H - bh)
    boxes = np.stack([x0, y0, x0 + bw, y0 + bh], axis=1).astype(np.float32)
    return img, boxes
