"""ctypes binding of libgkd (include/gkd.h), one Python function per C entry point.

Argument marshalling only: every function here turns tensors into device
pointers and sizes, calls the C ABI, and raises GkdError on a non-OK status.
No step of the head is computed in Python. Importing this module loads the
in-tree libgkd.so and fails loudly when it is missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgkd.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "gkd.h")

GKD_OK, GKD_ERR_ARG, GKD_ERR_SHAPE, GKD_ERR_DTYPE, GKD_ERR_ALIGN, GKD_ERR_CUDA, GKD_ERR_TIMEOUT = range(7)
GKD_F32, GKD_BF16 = 0, 1
STATUS_NAMES = {0: "GKD_OK", 1: "GKD_ERR_ARG", 2: "GKD_ERR_SHAPE", 3: "GKD_ERR_DTYPE", 4: "GKD_ERR_ALIGN",
                5: "GKD_ERR_CUDA", 6: "GKD_ERR_TIMEOUT"}
DEBUG_SKIP_PRODUCER_ARRIVE = 1


class GkdError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libgkd.so is not built at {LIB_PATH}; run `python -m prompt_conditioned_keypoint_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_ll = ctypes.c_longlong
_f = ctypes.c_float
_u = ctypes.c_uint

_SIGS = {
    "gkd_pool_prototypes": [_p, _i, _i, _i, _i, _i, _p, _p, _i, _f, _f, _p, _ll, _p],
    "gkd_norm_kernels": [_p, _p, _i, _i, _i, _i, _f, _i, _p, _p],
    "gkd_norm_fuse_kernels": [_p, _p, _i, _i, _i, _i, _f, _i, _p, _p, _p],
    "gkd_heatmap": [_p, _i, _i, _i, _i, _i, _i, _p, _i, _ll, _p, _ll, _i, _i, _p, _p],
    "gkd_fuse_decode": [_p, _p, _ll, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p],
    "gkd_heatmap_decode": [_p, _i, _i, _i, _i, _i, _i, _p, _i, _ll, _p, _ll, _i, _i, _p, _p, _p, _p, _p, _p],
    "gkd_heatmap_decode_noalloc": [_p, _i, _i, _i, _i, _i, _i, _p, _i, _ll, _p, _ll, _i, _i, _p, _p, _p, _p, _p],
    "gkd_preprocess": [_p, _i, _i, _p, _i, _i, _p, _p],
    "gkd_heatmap_contract_first": [_p, _i, _i, _i, _i, _i, _i, _p, _ll, _p, _ll, _i, _i, _p, _p, _p],
    "gkd_roi_to_image": [_p, _p, _i, _i, _i, _p, _p],
    "gkd_check_device_error": [_p],
    "gkd_set_wait_timeout_ms": [_u],
    "gkd_debug_set_flags": [_u],
    "gkd_last_error": [],
    "gkd_version": [],
}
for _name, _args in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_char_p if _name == "gkd_last_error" else ctypes.c_int


def declared_symbols() -> list[str]:
    """Entry points declared in include/gkd.h (GKD_API lines)."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"GKD_API\s+[\w\s\*]+?\b(gkd_\w+)\s*\(", text)


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s, ref=None) -> int | None:
    """cudaStream_t handle of `s`. None means torch's current stream on the
    device of `ref` (the call's first tensor, whose device runs the work), or
    on the current device when `ref` is not a CUDA tensor."""
    if s is None:
        import torch
        dev = getattr(ref, "device", None)
        if dev is None or getattr(dev, "type", None) != "cuda":
            dev = None
        return torch.cuda.current_stream(dev).cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn: str, status: int):
    if status != GKD_OK:
        raise GkdError(status, fn, gkd_last_error())


def gkd_last_error() -> str:
    return lib.gkd_last_error().decode()


def gkd_version() -> int:
    return lib.gkd_version()


def gkd_set_wait_timeout_ms(ms: int):
    _check("gkd_set_wait_timeout_ms", lib.gkd_set_wait_timeout_ms(ms))


def gkd_debug_set_flags(flags: int):
    _check("gkd_debug_set_flags", lib.gkd_debug_set_flags(flags))


def gkd_check_device_error(stream=None):
    _check("gkd_check_device_error", lib.gkd_check_device_error(_stream(stream)))


def gkd_pool_prototypes(support, sdt, B, h, w, C, kpts, kmask, K, sigma_px, stride_px, proto,
                        proto_batch_stride, stream=None):
    _check("gkd_pool_prototypes", lib.gkd_pool_prototypes(
        _ptr(support), sdt, B, h, w, C, _ptr(kpts), _ptr(kmask), K, sigma_px, stride_px, _ptr(proto),
        proto_batch_stride, _stream(stream, support)))


def gkd_norm_kernels(rows, mask, Bk, M, K, C, eps, out_dt, out, stream=None):
    _check("gkd_norm_kernels", lib.gkd_norm_kernels(
        _ptr(rows), _ptr(mask), Bk, M, K, C, eps, out_dt, _ptr(out), _stream(stream, rows)))


def gkd_norm_fuse_kernels(rows, mask, Bk, M, K, C, eps, out_dt, out, out_mask, stream=None):
    _check("gkd_norm_fuse_kernels", lib.gkd_norm_fuse_kernels(
        _ptr(rows), _ptr(mask), Bk, M, K, C, eps, out_dt, _ptr(out), _ptr(out_mask), _stream(stream, rows)))


def gkd_heatmap(feat, fdt, B, h, w, C, up, kern, kdt, kern_batch_stride, mask, mask_batch_stride, M, K, heat,
                stream=None):
    _check("gkd_heatmap", lib.gkd_heatmap(
        _ptr(feat), fdt, B, h, w, C, up, _ptr(kern), kdt, kern_batch_stride, _ptr(mask), mask_batch_stride,
        M, K, _ptr(heat), _stream(stream, feat)))


def gkd_heatmap_decode(feat, fdt, B, h, w, C, up, kern, kdt, kern_batch_stride, mask, mask_batch_stride, M, K,
                       scratch, xy, score, idx, valid, stream=None):
    _check("gkd_heatmap_decode", lib.gkd_heatmap_decode(
        _ptr(feat), fdt, B, h, w, C, up, _ptr(kern), kdt, kern_batch_stride, _ptr(mask), mask_batch_stride,
        M, K, _ptr(scratch), _ptr(xy), _ptr(score), _ptr(idx), _ptr(valid), _stream(stream, feat)))


def gkd_heatmap_decode_noalloc(feat, fdt, B, h, w, C, up, kern, kdt, kern_batch_stride, mask, mask_batch_stride,
                               M, K, xy, score, idx, valid, stream=None):
    _check("gkd_heatmap_decode_noalloc", lib.gkd_heatmap_decode_noalloc(
        _ptr(feat), fdt, B, h, w, C, up, _ptr(kern), kdt, kern_batch_stride, _ptr(mask), mask_batch_stride,
        M, K, _ptr(xy), _ptr(score), _ptr(idx), _ptr(valid), _stream(stream, feat)))


def gkd_fuse_decode(heat, mask, mask_batch_stride, B, M, K, H, W, fused, xy, score, idx, valid, stream=None):
    _check("gkd_fuse_decode", lib.gkd_fuse_decode(
        _ptr(heat), _ptr(mask), mask_batch_stride, B, M, K, H, W, _ptr(fused), _ptr(xy), _ptr(score),
        _ptr(idx), _ptr(valid), _stream(stream, heat)))


def gkd_preprocess(img, H, W, boxes, B, canvas, out, stream=None):
    _check("gkd_preprocess", lib.gkd_preprocess(_ptr(img), H, W, _ptr(boxes), B, canvas, _ptr(out),
                                                _stream(stream, img)))


def gkd_roi_to_image(xy, boxes, B, K, canvas, out, stream=None):
    _check("gkd_roi_to_image", lib.gkd_roi_to_image(_ptr(xy), _ptr(boxes), B, K, canvas, _ptr(out),
                                                    _stream(stream, xy)))


def gkd_heatmap_contract_first(feat, fdt, B, h, w, C, up, kern, kern_batch_stride, mask, mask_batch_stride, M, K,
                               scratch, heat, stream=None):
    _check("gkd_heatmap_contract_first", lib.gkd_heatmap_contract_first(
        _ptr(feat), fdt, B, h, w, C, up, _ptr(kern), kern_batch_stride, _ptr(mask), mask_batch_stride, M, K,
        _ptr(scratch), _ptr(heat), _stream(stream, feat)))
