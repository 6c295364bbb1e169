"""GPU: HeadPipeline (two heads; the host-to-device copy of batch i + 1 overlaps
the head on batch i) returns, for every batch, exactly what GkdHead.run_host
returns for it one batch at a time. The pipeline reuses each head every other
batch, so a missing wait between a head's inputs and their next upload would
show up as a batch decoded from another batch's inputs."""
import pytest
import torch

from gpu_helpers import dev
from prompt_conditioned_keypoint_b200 import binding as gk
from prompt_conditioned_keypoint_b200 import synthetic as S
from prompt_conditioned_keypoint_b200.head import GkdHead, HeadPipeline, HeadShape

pytestmark = pytest.mark.gpu


def _same(a: dict, b: dict):
    for k in ("xy", "score", "idx", "valid"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("feat_dtype", ["f32", "bf16"])
def test_pipeline_matches_one_batch_at_a_time(feat_dtype):
    wls = [S.make_case(60 + i, 4, 12, 12, 256, 20, 2, feat_dtype=feat_dtype, valid="random") for i in range(3)]
    shape = HeadShape.of(wls[0])
    single = GkdHead(shape, dev())
    hosts = [single.host_inputs(wl, pin=True) for wl in wls]
    st = torch.cuda.current_stream(dev())
    ref = []
    for h in hosts:
        ref.append(single.run_host(h, None, st))
        st.synchronize()
    pipe = HeadPipeline(shape, dev())
    order = [0, 1, 2, 0, 2, 1]                   # every head sees more than one batch
    got = pipe.run([hosts[i] for i in order], None, st)
    st.synchronize()
    gk.gkd_check_device_error()
    for i, g in zip(order, got):
        _same(ref[i], g)


def test_pipeline_pooled_fp32_workload():
    """Workload 1's shape (pooled prototypes, fp32 kernel rows): every input the
    pipeline uploads (support map, keypoints, masks, features) goes through it."""
    wl = S.make_config(1)
    shape = HeadShape.of(wl)
    single = GkdHead(shape, dev())
    a = single.host_inputs(wl, pin=True)
    b = {k: torch.empty_like(v, pin_memory=True).copy_(v) for k, v in a.items()}
    b["feat"].neg_()                              # a second batch with other peaks
    b["support"].mul_(0.5)
    st = torch.cuda.current_stream(dev())
    ref = []
    for h in (a, b):
        ref.append(single.run_host(h, None, st))
        st.synchronize()
    pipe = HeadPipeline(shape, dev())
    got = pipe.run([a, b, b, a], None, st)
    st.synchronize()
    gk.gkd_check_device_error()
    for i, g in zip((0, 1, 1, 0), got):
        _same(ref[i], g)
