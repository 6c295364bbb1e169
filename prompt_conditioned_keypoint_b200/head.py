"""The detection head as one call sequence over libgkd (device memory via torch).

`GkdHead` owns the device buffers of one batch shape and enqueues the head's
steps through the C ABI on a stream:

  [gkd_pool_prototypes]   visual rows from support maps (when keypoints are given)
  gkd_norm_kernels        L2-normalised rows (bf16 or fp32 operands)
  gkd_heatmap             fused 4x upsample + 1x1 contraction
  gkd_fuse_decode         per-row modality fusion + peak decode

or, with `fused_decode=True`, gkd_heatmap_decode in place of the last two: the
fusion and peak decode run in the heatmap kernel's epilogue and no heatmap is
written (a [B][K] uint64 scratch buffer carries the per-row peak keys).

With `fuse_rows=True` (fusion by linearity, a variant beside the graded path)
gkd_norm_fuse_kernels replaces gkd_norm_kernels: each prompt row's modalities
are averaged before the contraction, and the heatmap and decode steps run with
one modality (M = 1) over the fused rows and their mask.

torch only allocates memory, owns streams and copies host buffers; every step
of the head runs in libgkd's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import binding as gk

DTYPE_CODE = {"f32": gk.GKD_F32, "bf16": gk.GKD_BF16}


@dataclass(frozen=True)
class HeadShape:
    B: int
    h: int
    w: int
    C: int
    K: int
    M: int
    feat_dtype: str = "f32"       # "f32" | "bf16"
    kern_dtype: str = "bf16"      # operand type of the contraction: "f32" | "bf16"
    shared: bool = False          # one prompt set for all crops
    pooled: bool = False          # modality 0 rows come from Gaussian pooling
    sigma: float = 14.0
    stride: float = 16.0
    up: int = 4

    @property
    def Bk(self) -> int:
        return 1 if self.shared else self.B

    @property
    def H(self) -> int:
        return self.up * self.h

    @property
    def W(self) -> int:
        return self.up * self.w

    @staticmethod
    def of(wl) -> "HeadShape":
        return HeadShape(wl.B, wl.h, wl.w, wl.C, wl.K, wl.M, wl.feat_dtype, wl.kern_dtype, wl.Bk == 1,
                         wl.support is not None, float(wl.sigma), float(wl.stride), wl.up)

    def launches_per_step(self) -> int:
        """libgkd kernels one step launches: pool (if pooled), norm, then
        heatmap + fuse_decode, or, with the decode fused, the heatmap kernel in
        decode mode + the key finaliser (plus a cudaMemsetAsync of the scratch,
        which is not a kernel of this library)."""
        return (1 if self.pooled else 0) + 1 + 2


class GkdHead:
    def __init__(self, shape: HeadShape, device, with_fused: bool = False, fused_decode: bool = False,
                 fuse_rows: bool = False):
        s = self.shape = shape
        d = self.device = torch.device(device)
        self.fused_decode = fused_decode
        self.fuse_rows = fuse_rows
        self.Mh = 1 if fuse_rows else s.M          # modalities the contraction sees
        fdt = torch.float32 if s.feat_dtype == "f32" else torch.int16
        self.feat = torch.empty((s.B, s.h, s.w, s.C), dtype=fdt, device=d)
        self.rows = torch.zeros((s.Bk, s.M, s.K, s.C), dtype=torch.float32, device=d)
        self.mask = torch.zeros((s.Bk, s.M, s.K), dtype=torch.uint8, device=d)
        kdt = torch.float32 if s.kern_dtype == "f32" else torch.int16
        self.khat = torch.empty((s.Bk, self.Mh, s.K, s.C), dtype=kdt, device=d)
        self.rmask = torch.empty((s.Bk, 1, s.K), dtype=torch.uint8, device=d) if fuse_rows else None
        if s.pooled:
            self.support = torch.empty((s.B, s.h, s.w, s.C), dtype=torch.float32, device=d)
            self.kpts = torch.empty((s.B, s.K, 2), dtype=torch.float32, device=d)
            self.kmask = torch.empty((s.B, s.K), dtype=torch.uint8, device=d)
        self.heat = None if fused_decode else torch.empty((s.B, self.Mh, s.K, s.H, s.W), dtype=torch.float32,
                                                          device=d)
        self.scratch = torch.empty((s.B, s.K), dtype=torch.int64, device=d) if fused_decode else None
        self.fused = torch.empty((s.B, s.K, s.H, s.W), dtype=torch.float32, device=d) if with_fused else None
        self.xy = torch.empty((s.B, s.K, 2), dtype=torch.float32, device=d)
        self.score = torch.empty((s.B, s.K), dtype=torch.float32, device=d)
        self.idx = torch.empty((s.B, s.K), dtype=torch.int32, device=d)
        self.valid = torch.empty((s.B, s.K), dtype=torch.uint8, device=d)

    # ------------------------------------------------------------------ inputs
    def host_inputs(self, wl, pin: bool = True) -> dict:
        """Host tensors (pinned) of a synthetic workload, in this head's layouts."""
        s = self.shape
        feat = wl.feat.view(np.int16) if s.feat_dtype == "bf16" else wl.feat
        out = {"feat": torch.from_numpy(np.ascontiguousarray(feat)), "mask": torch.from_numpy(wl.mask)}
        if s.pooled:
            out["support"] = torch.from_numpy(wl.support)
            out["kpts"] = torch.from_numpy(wl.kpts)
            out["kmask"] = torch.from_numpy(wl.kmask)
            if s.M == 2:
                out["text_rows"] = torch.from_numpy(np.ascontiguousarray(wl.rows[:, 1]))
        else:
            out["rows"] = torch.from_numpy(wl.rows)
        if pin:
            out = {k: v.pin_memory() for k, v in out.items()}
        return out

    def upload(self, host: dict, stream=None):
        """Copy host inputs into the device buffers on `stream` (asynchronously when pinned)."""
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(st):
            self.feat.copy_(host["feat"], non_blocking=True)
            self.mask.copy_(host["mask"], non_blocking=True)
            if self.shape.pooled:
                self.support.copy_(host["support"], non_blocking=True)
                self.kpts.copy_(host["kpts"], non_blocking=True)
                self.kmask.copy_(host["kmask"], non_blocking=True)
                if "text_rows" in host:
                    self.rows[:, 1].copy_(host["text_rows"], non_blocking=True)
            else:
                self.rows.copy_(host["rows"], non_blocking=True)

    def host_input_bytes(self, host: dict) -> int:
        return sum(v.numel() * v.element_size() for v in host.values())

    # ------------------------------------------------------------------ steps
    def pool(self, stream=None):
        s = self.shape
        gk.gkd_pool_prototypes(self.support, gk.GKD_F32, s.B, s.h, s.w, s.C, self.kpts, self.kmask, s.K,
                               s.sigma, s.stride, self.rows, s.M * s.K * s.C, stream)

    def norm(self, stream=None):
        s = self.shape
        if self.fuse_rows:
            gk.gkd_norm_fuse_kernels(self.rows, self.mask, s.Bk, s.M, s.K, s.C, 1e-12, DTYPE_CODE[s.kern_dtype],
                                     self.khat, self.rmask, stream)
        else:
            gk.gkd_norm_kernels(self.rows, self.mask, s.Bk, s.M, s.K, s.C, 1e-12, DTYPE_CODE[s.kern_dtype],
                                self.khat, stream)

    def _contraction_operands(self):
        """(kernel rows, mask, modalities, kernel batch stride, mask batch stride) of the heatmap step."""
        s = self.shape
        M = self.Mh
        mask = self.rmask if self.fuse_rows else self.mask
        kbs = 0 if s.shared else M * s.K * s.C
        mbs = 0 if s.shared else M * s.K
        return self.khat, mask, M, kbs, mbs

    def heatmap(self, stream=None):
        s = self.shape
        kern, mask, M, kbs, mbs = self._contraction_operands()
        gk.gkd_heatmap(self.feat, DTYPE_CODE[s.feat_dtype], s.B, s.h, s.w, s.C, s.up, kern,
                       DTYPE_CODE[s.kern_dtype], kbs, mask, mbs, M, s.K, self.heat, stream)

    def heatmap_decode(self, stream=None):
        s = self.shape
        kern, mask, M, kbs, mbs = self._contraction_operands()
        gk.gkd_heatmap_decode(self.feat, DTYPE_CODE[s.feat_dtype], s.B, s.h, s.w, s.C, s.up, kern,
                              DTYPE_CODE[s.kern_dtype], kbs, mask, mbs, M, s.K, self.scratch, self.xy,
                              self.score, self.idx, self.valid, stream)

    def fuse_decode(self, stream=None):
        s = self.shape
        _, mask, M, _, mbs = self._contraction_operands()
        gk.gkd_fuse_decode(self.heat, mask, mbs, s.B, M, s.K, s.H, s.W, self.fused, self.xy, self.score,
                           self.idx, self.valid, stream)

    def forward(self, stream=None, heatmap_events=None):
        """Enqueue the whole head. `heatmap_events` = (start, end) CUDA events
        recorded around the heatmap launch on the same stream."""
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        if self.shape.pooled:
            self.pool(st)
        self.norm(st)
        if heatmap_events is not None:
            heatmap_events[0].record(st)
        if self.fused_decode:
            self.heatmap_decode(st)
        else:
            self.heatmap(st)
        if heatmap_events is not None:
            heatmap_events[1].record(st)
        if not self.fused_decode:
            self.fuse_decode(st)

    def outputs_to_host(self, dst: dict | None = None, stream=None) -> dict:
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        if dst is None:
            dst = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                   for k, v in (("xy", self.xy), ("score", self.score), ("idx", self.idx), ("valid", self.valid))}
        with torch.cuda.stream(st):
            dst["xy"].copy_(self.xy, non_blocking=True)
            dst["score"].copy_(self.score, non_blocking=True)
            dst["idx"].copy_(self.idx, non_blocking=True)
            dst["valid"].copy_(self.valid, non_blocking=True)
        return dst

    def output_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.xy, self.score, self.idx, self.valid))

    def run_host(self, host: dict, out: dict | None = None, stream=None) -> dict:
        """End to end through the public API: host inputs in, decoded keypoints out.

        Everything is enqueued on `stream` (default: the current stream of this
        head's device) and the copies are asynchronous. Synchronise that stream
        before reading the returned host tensors or reusing `host`."""
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.upload(host, st)
        self.forward(st)
        return self.outputs_to_host(out, st)

    def algorithmic_heatmap_flops(self, mask: np.ndarray) -> float:
        """2 * R * C * P summed over crops, R = valid rows of each crop (with
        fuse_rows, the prompt rows with any modality present)."""
        s = self.shape
        m = np.asarray(mask)
        if self.fuse_rows:
            m = m.any(axis=1)
        rows = m.reshape(m.shape[0], -1).sum(axis=1).astype(np.float64)
        total_rows = rows[0] * s.B if s.shared else rows.sum()
        return 2.0 * total_rows * s.C * s.H * s.W


class HeadPipeline:
    """Two heads of one shape for a stream of batches: the host-to-device copy
    of batch i + 1 runs on a copy stream while the head works on batch i on the
    compute stream, so each batch costs the longer of the two instead of their
    sum. Batch i's decoded outputs are copied to host on the compute stream
    right after its head."""

    def __init__(self, shape: HeadShape, device, **head_kw):
        self.device = torch.device(device)
        self.heads = [GkdHead(shape, self.device, **head_kw), GkdHead(shape, self.device, **head_kw)]
        self.copy_stream = torch.cuda.Stream(self.device)
        self._consumed = [None, None]   # per head: event after the last head that read its inputs

    def run(self, hosts, outs=None, stream=None, start_event=None) -> list:
        """Enqueue every batch of `hosts` (dicts as `GkdHead.host_inputs` gives,
        pinned) and return one host output dict per batch (`outs[i]` when
        given; a dict passed twice is overwritten by the later batch).
        `start_event`, if given, is waited on before the first copy. Keep the
        host tensors alive and synchronise `stream` before reading the outputs."""
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        if start_event is not None:
            self.copy_stream.wait_event(start_event)
        res = []
        for i, host in enumerate(hosts):
            j = i & 1
            head = self.heads[j]
            if self._consumed[j] is not None:          # the head's previous batch has been read
                self.copy_stream.wait_event(self._consumed[j])
            head.upload(host, self.copy_stream)
            landed = torch.cuda.Event()
            landed.record(self.copy_stream)
            st.wait_event(landed)
            head.forward(st)
            consumed = torch.cuda.Event()
            consumed.record(st)
            self._consumed[j] = consumed
            res.append(head.outputs_to_host(outs[i] if outs is not None else None, st))
        return res
