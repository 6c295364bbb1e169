"""libgkd loads, exports every declared entry point, and rejects bad calls on
the host before touching CUDA (runs without a GPU)."""
import ctypes
import subprocess

import pytest

from prompt_conditioned_keypoint_b200 import binding as gk

L = gk.lib
OK, ARG, SHAPE, DTYPE, ALIGN = gk.GKD_OK, gk.GKD_ERR_ARG, gk.GKD_ERR_SHAPE, gk.GKD_ERR_DTYPE, gk.GKD_ERR_ALIGN
F32, BF16 = gk.GKD_F32, gk.GKD_BF16
P = 0x10000          # a 16-byte-aligned stand-in pointer value (never dereferenced: calls fail before use)
MIS = 0x10004        # misaligned stand-in


def test_header_declares_the_boundary():
    names = gk.declared_symbols()
    assert sorted(names) == sorted([
        "gkd_pool_prototypes", "gkd_norm_kernels", "gkd_norm_fuse_kernels", "gkd_heatmap", "gkd_heatmap_decode",
        "gkd_heatmap_contract_first", "gkd_heatmap_decode_noalloc", "gkd_fuse_decode",
        "gkd_preprocess", "gkd_roi_to_image", "gkd_last_error",
        "gkd_check_device_error", "gkd_set_wait_timeout_ms", "gkd_debug_set_flags", "gkd_version"])


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", gk.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in gk.declared_symbols():
        assert name in exported, name
        assert getattr(L, name) is not None
    # nothing but the C ABI is exported from our own code
    assert not [s for s in exported if s.startswith("_ZN3gkd")]


def test_version():
    assert gk.gkd_version() == 100


def _status(fn, *args):
    return getattr(L, fn)(*args)


def test_norm_validation():
    good = (P, P, 2, 2, 80, 1024, ctypes.c_float(1e-12), BF16, P, None)
    assert _status("gkd_norm_kernels", P, P, 2, 3, 80, 1024, 1e-12, BF16, P, None) == SHAPE
    assert _status("gkd_norm_kernels", P, P, 2, 2, 0, 1024, 1e-12, BF16, P, None) == SHAPE
    assert _status("gkd_norm_kernels", P, P, -1, 2, 80, 1024, 1e-12, BF16, P, None) == SHAPE
    assert _status("gkd_norm_kernels", P, P, 2, 2, 129, 1024, 1e-12, BF16, P, None) == SHAPE
    assert _status("gkd_norm_kernels", P, P, 2, 2, 80, 1020, 1e-12, BF16, P, None) == SHAPE
    assert _status("gkd_norm_kernels", P, P, 2, 2, 80, 1024, 0.0, BF16, P, None) == ARG
    assert _status("gkd_norm_kernels", P, P, 2, 2, 80, 1024, 1e-12, 7, P, None) == ARG
    assert _status("gkd_norm_kernels", None, P, 2, 2, 80, 1024, 1e-12, BF16, P, None) == ARG
    assert _status("gkd_norm_kernels", MIS, P, 2, 2, 80, 1024, 1e-12, BF16, P, None) == ALIGN
    assert _status("gkd_norm_kernels", P, P, 2, 2, 80, 1024, 1e-12, BF16, MIS, None) == ALIGN
    assert _status("gkd_norm_kernels", None, None, 0, 2, 80, 1024, 1e-12, BF16, None, None) == OK  # empty batch
    assert "aligned" in gk.gkd_last_error() or gk.gkd_last_error() == ""


def test_norm_fuse_validation():
    def nf(rows=P, mask=P, Bk=2, M=2, K=80, C=1024, eps=1e-12, odt=BF16, out=P, omask=P):
        return _status("gkd_norm_fuse_kernels", rows, mask, Bk, M, K, C, ctypes.c_float(eps), odt, out, omask, None)
    assert nf(M=3) == SHAPE and nf(K=0) == SHAPE and nf(C=12) == SHAPE and nf(Bk=-1) == SHAPE
    assert nf(eps=0.0) == ARG and nf(odt=4) == ARG
    assert nf(rows=None) == ARG and nf(omask=None) == ARG
    assert nf(rows=MIS) == ALIGN and nf(out=MIS) == ALIGN
    assert nf(Bk=0, rows=None, mask=None, out=None, omask=None) == OK


def test_heatmap_validation():
    def hm(feat=P, fdt=F32, B=2, h=24, w=24, C=1024, up=4, kern=P, kdt=BF16, kbs=2 * 80 * 1024, mask=P,
           mbs=160, M=2, K=80, heat=P):
        return _status("gkd_heatmap", feat, fdt, B, h, w, C, up, kern, kdt, kbs, mask, mbs, M, K, heat, None)
    assert hm(up=2) == SHAPE
    assert hm(fdt=BF16, kdt=F32) == DTYPE
    assert hm(fdt=5) == ARG
    assert hm(kdt=5) == ARG
    assert hm(M=2, K=81) == SHAPE                       # 2 * 88 > 160 accumulator columns
    # M * ceil8(K) = 128 fits: the call passes every host check and stops only at the
    # pointer query (no device here, or a non-device stand-in pointer on a GPU machine)
    assert hm(M=1, K=128, kbs=128 * 1024, mbs=128) in (gk.GKD_ERR_CUDA, ARG)
    assert hm(M=1, K=129, kbs=129 * 1024, mbs=129) == SHAPE and hm(M=0) == SHAPE and hm(M=3) == SHAPE
    assert hm(mbs=-1) == SHAPE
    assert hm(kdt=F32, kbs=2 * 81 * 1024, K=81) in (gk.GKD_ERR_CUDA, ARG)   # no accumulator-column limit in fp32
    assert hm(C=1028) == SHAPE
    assert hm(h=0) == SHAPE and hm(w=257) == SHAPE
    assert hm(B=-1) == SHAPE and hm(B=70000) == SHAPE
    assert hm(kbs=-8) == SHAPE
    assert hm(feat=None) == ARG and hm(kern=None) == ARG and hm(mask=None) == ARG and hm(heat=None) == ARG
    assert hm(feat=MIS) == ALIGN and hm(kern=MIS) == ALIGN and hm(heat=MIS) == ALIGN
    assert hm(kbs=3) == ALIGN                           # 6 bytes is not a 16-byte multiple
    assert hm(B=0, feat=None, kern=None, mask=None, heat=None) == OK
    assert "null" in gk.gkd_last_error() or gk.gkd_last_error() == ""


def test_heatmap_decode_validation():
    def hd(feat=P, fdt=F32, B=2, h=24, w=24, C=1024, up=4, kern=P, kdt=BF16, kbs=2 * 80 * 1024, mask=P,
           mbs=160, M=2, K=80, scratch=P, xy=P, score=P, idx=P, valid=P):
        return _status("gkd_heatmap_decode", feat, fdt, B, h, w, C, up, kern, kdt, kbs, mask, mbs, M, K, scratch,
                       xy, score, idx, valid, None)
    # the heatmap checks apply unchanged
    assert hd(up=2) == SHAPE and hd(fdt=BF16, kdt=F32) == DTYPE and hd(M=2, K=81) == SHAPE
    assert hd(feat=None) == ARG and hd(feat=MIS) == ALIGN and hd(kbs=3) == ALIGN
    # and those of the decode outputs and the scratch
    assert hd(scratch=None) == ARG and hd(xy=None) == ARG and hd(valid=None) == ARG
    assert hd(scratch=P + 4) == ALIGN and hd(idx=P + 2) == ALIGN
    assert hd(scratch=P + 8) in (gk.GKD_ERR_CUDA, ARG)  # 8-byte aligned is enough: reaches the pointer query
    assert hd(B=0, feat=None, kern=None, mask=None, scratch=None, xy=None, score=None, idx=None, valid=None) == OK


def test_contract_first_validation():
    def cf(feat=P, fdt=F32, B=2, h=24, w=24, C=1024, up=4, kern=P, kbs=2 * 80 * 1024, mask=P, mbs=160, M=2, K=80,
           scratch=P, heat=P):
        return _status("gkd_heatmap_contract_first", feat, fdt, B, h, w, C, up, kern, kbs, mask, mbs, M, K, scratch,
                       heat, None)
    assert cf(up=2) == SHAPE and cf(M=2, K=81) == SHAPE and cf(fdt=3) == ARG
    assert cf(scratch=None) == ARG and cf(heat=None) == ARG
    assert cf(heat=P + 4) == ALIGN and cf(scratch=P + 2) == ALIGN
    assert cf(B=0, feat=None, kern=None, mask=None, scratch=None, heat=None) == OK


def test_preprocess_and_roi_validation():
    def pp(img=P, H=480, W=640, boxes=P, B=4, canvas=384, out=P):
        return _status("gkd_preprocess", img, H, W, boxes, B, canvas, out, None)
    assert pp(H=0) == SHAPE and pp(W=40000) == SHAPE and pp(B=-1) == SHAPE and pp(canvas=0) == SHAPE
    assert pp(img=None) == ARG and pp(boxes=None) == ARG and pp(out=None) == ARG
    assert pp(out=P + 2) == ALIGN and pp(boxes=P + 1) == ALIGN
    assert pp(B=0, img=None, boxes=None, out=None) == OK

    def roi(xy=P, boxes=P, B=4, K=80, canvas=384, out=P):
        return _status("gkd_roi_to_image", xy, boxes, B, K, canvas, out, None)
    assert roi(K=0) == SHAPE and roi(B=70000) == SHAPE and roi(canvas=5000) == SHAPE
    assert roi(xy=None) == ARG and roi(out=None) == ARG and roi(xy=P + 2) == ALIGN
    assert roi(B=0, xy=None, boxes=None, out=None) == OK


def test_heatmap_decode_noalloc_validation():
    def hn(feat=P, fdt=F32, B=2, h=24, w=24, C=1024, up=4, kern=P, kdt=BF16, kbs=2 * 80 * 1024, mask=P,
           mbs=160, M=2, K=80, xy=P, score=P, idx=P, valid=P):
        return _status("gkd_heatmap_decode_noalloc", feat, fdt, B, h, w, C, up, kern, kdt, kbs, mask, mbs, M, K,
                       xy, score, idx, valid, None)
    assert hn(up=2) == SHAPE and hn(M=2, K=81) == SHAPE
    # more peak keys than the static buffer holds: rejected before anything runs
    assert hn(B=1639, K=80) == SHAPE and "131072" in gk.gkd_last_error()
    assert hn(B=1638, K=80) in (gk.GKD_ERR_CUDA, ARG)   # 131040 keys fit: reaches the pointer query
    assert hn(xy=None) == ARG and hn(idx=P + 2) == ALIGN
    assert hn(B=0, feat=None, kern=None, mask=None, xy=None, score=None, idx=None, valid=None) == OK


def test_pool_validation():
    def pool(support=P, sdt=F32, B=1, h=24, w=24, C=1024, kpts=P, kmask=P, K=80, sigma=14.0, stride=16.0,
             proto=P, pbs=80 * 1024):
        return _status("gkd_pool_prototypes", support, sdt, B, h, w, C, kpts, kmask, K, ctypes.c_float(sigma),
                       ctypes.c_float(stride), proto, pbs, None)
    assert pool(sdt=BF16) == DTYPE
    assert pool(sdt=9) == ARG
    assert pool(sigma=0.0) == ARG and pool(stride=-1.0) == ARG
    assert pool(pbs=80 * 1024 - 8) == SHAPE
    assert pool(K=129) == SHAPE and pool(h=0) == SHAPE and pool(C=12) == SHAPE
    assert pool(support=None) == ARG
    assert pool(proto=MIS) == ALIGN
    assert pool(B=0, support=None, kpts=None, kmask=None, proto=None) == OK


def test_fuse_decode_validation():
    def fd(heat=P, mask=P, mbs=160, B=2, M=2, K=80, H=96, W=96, fused=None, xy=P, score=P, idx=P, valid=P):
        return _status("gkd_fuse_decode", heat, mask, mbs, B, M, K, H, W, fused, xy, score, idx, valid, None)
    assert fd(M=3) == SHAPE and fd(K=0) == SHAPE and fd(H=3, W=5) == SHAPE
    assert fd(heat=None) == ARG and fd(idx=None) == ARG
    assert fd(heat=MIS) == ALIGN and fd(fused=MIS) == ALIGN and fd(xy=P + 2) == ALIGN
    assert fd(B=70000) == SHAPE and fd(mbs=-1) == SHAPE and fd(K=65536) == SHAPE
    assert fd(H=46341, W=46341) == SHAPE                 # H*W >= 2^31
    assert fd(valid=None) == ARG and fd(score=P + 1) == ALIGN
    assert fd(B=0, heat=None, mask=None, xy=None, score=None, idx=None, valid=None) == OK


def test_misc_entry_points():
    assert _status("gkd_set_wait_timeout_ms", 0) == ARG
    assert _status("gkd_set_wait_timeout_ms", 2000) == OK
    assert _status("gkd_debug_set_flags", 0x80) == ARG
    assert _status("gkd_debug_set_flags", 0) == OK
    with pytest.raises(gk.GkdError) as e:
        gk._check("x", SHAPE)
    assert e.value.status == SHAPE


def test_default_stream_follows_the_first_tensors_device(monkeypatch):
    import torch

    seen = []

    class FakeStream:
        def __init__(self, dev):
            self.cuda_stream = 1000 + (-1 if dev is None else torch.device(dev).index)

    def fake_current_stream(dev=None):
        seen.append(dev)
        return FakeStream(dev)

    monkeypatch.setattr(torch.cuda, "current_stream", fake_current_stream)

    class OnDevice:
        device = torch.device("cuda", 3)

    assert gk._stream(None, OnDevice()) == 1003 and seen[-1] == torch.device("cuda", 3)
    assert gk._stream(None, torch.zeros(4)) == 999 and seen[-1] is None       # CPU tensor
    assert gk._stream(None, 12345) == 999 and seen[-1] is None                 # raw pointer
    assert gk._stream(None) == 999
    n = len(seen)
    assert gk._stream(77, OnDevice()) == 77                                    # explicit handle wins

    class S:
        cuda_stream = 55

    assert gk._stream(S(), OnDevice()) == 55 and len(seen) == n
