"""The call is stream-ordered and allocation-free, so it can be captured in a
CUDA graph and replayed: the replay must reproduce the eager results."""

import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, rel_l2, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_capture_and_replay(cuda_ok, mode):
    batch = synth.workload("short")
    d = to_device(batch)
    dtype = "bf16"
    dims = frnnt.dims_of(d["f"], d["g"], d["W_o"], dtype, mode, "auto", 0, batch.blank)
    out = frnnt.Outputs(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], dims)
    args = [d[k] for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        loss, grads = frnnt.fwd_bwd(*args, mode=mode, out=out, stream=stream)   # eager, also first-use setup
        stream.synchronize()
        ref_loss = loss.clone()
        ref = {k: v.clone() for k, v in grads.items()}
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            frnnt.fwd_bwd(*args, mode=mode, out=out, stream=stream, check=False)
        for k in list(out.grads().keys()):
            out.grads()[k].zero_()
        out.loss.zero_()
        g.replay()
        stream.synchronize()
    assert int(out.status[0].item()) == 0
    assert torch.allclose(out.loss, ref_loss, rtol=1e-5)
    for k in GRADS:
        assert rel_l2(out.grads()[k].float().cpu().numpy(), ref[k].float().cpu().numpy()) <= 1e-3, k
