"""Shared helpers of the GPU parity tests: upload numpy inputs, call libgkd
through the binding, and the comparison rules."""
from __future__ import annotations

import numpy as np
import torch

F32_TOL = 1e-5        # fp32 path: max|gpu - ref| <= 1e-5 * max|ref| per row
BF16_TOL = 2e-3       # bf16 operands, fp32 accumulation: <= 2e-3 * max|ref| per row


def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(a: np.ndarray, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(dev())


def bf16_dev(bits: np.ndarray):
    return to_dev(bits.view(np.int16))


def rowwise_rel_err(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """max |gpu - ref| / max |ref| over the trailing axes, per leading row."""
    g = gpu.reshape(gpu.shape[0], -1).astype(np.float64)
    r = ref.reshape(ref.shape[0], -1).astype(np.float64)
    den = np.maximum(np.abs(r).max(axis=1), 1e-30)
    return np.abs(g - r).max(axis=1) / den


def assert_rows_close(gpu: np.ndarray, ref: np.ndarray, tol: float, what: str = ""):
    err = rowwise_rel_err(gpu, ref)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= tol, f"{what}: worst row error {worst:.3e} > {tol:.1e} (row {int(err.argmax())})"
    return worst


def valid_heat_rows(heat: np.ndarray, mask: np.ndarray):
    """Stack the rows [b, m, k] with mask 1 (mask may be shared: leading dim 1)."""
    B, M, K = heat.shape[:3]
    sel = [(b, m, k) for b in range(B) for m in range(M) for k in range(K)
           if mask[0 if mask.shape[0] == 1 else b, m, k]]
    if not sel:
        return np.zeros((0,) + heat.shape[3:]), sel
    return np.stack([heat[b, m, k] for (b, m, k) in sel]), sel


def check_decode_against_margin(ref_fused: np.ndarray, ref_valid: np.ndarray, gpu_idx: np.ndarray,
                                gpu_valid: np.ndarray, tol: float, ref_heat: np.ndarray | None = None,
                                mask: np.ndarray | None = None):
    """Integer outputs bit-exact everywhere; the peak index bit-exact wherever the
    oracle's top-2 margin exceeds tol * max|ref| of that fused row.

    On the remaining near-tie rows several indices are correct. Given the
    oracle heatmaps `ref_heat` [B][M][K][H][W] and `mask` [B or 1][M][K], the
    GPU's index must then be a near-maximal pixel of the oracle's fused row:
    f[idx] >= max f - 2 (tol S + 1e-6 S), S = the largest |value| of the row's
    present modality heatmaps. This follows from heatmap rows within tol * S of
    the oracle (checked before) and the fp32 mean. Returns (rows checked
    exactly, near-tie rows checked for validity)."""
    from oracle.gkd_oracle import top2_margin
    np.testing.assert_array_equal(gpu_valid, ref_valid)
    checked = 0
    near = 0
    for b in range(ref_fused.shape[0]):
        for k in range(ref_fused.shape[1]):
            if not ref_valid[b, k]:
                assert gpu_idx[b, k] == -1
                continue
            f = ref_fused[b, k].reshape(-1)
            if top2_margin(f) > tol * np.abs(f).max():
                assert gpu_idx[b, k] == int(np.argmax(f)), (b, k)
                checked += 1
                continue
            near += 1
            if ref_heat is None:
                continue
            mb = mask[0 if mask.shape[0] == 1 else b]
            S = max(float(np.abs(ref_heat[b, m, k]).max()) for m in range(mb.shape[0]) if mb[m, k])
            i = int(gpu_idx[b, k])
            assert 0 <= i < f.size, (b, k, i)
            assert f[i] >= f.max() - 2.0 * (tol + 1e-6) * S, (b, k, i, float(f.max() - f[i]), S)
    return checked, near
