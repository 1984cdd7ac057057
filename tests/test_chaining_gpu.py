"""The call's kernels are chained by programmatic dependent launch: each may be
launched before the one ahead of it has completed and waits on the device
before it touches that kernel's results.  With the chaining turned off
(FRNNT_CHAIN=0, read once per process, so in a child process) every launch
waits in plain stream order; both must give the same results, up to the
order of the fp32 atomic additions."""

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, rel_l2, to_device

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import to_device
batch = synth.workload({name!r})
d = to_device(batch)
w = torch.linspace(0.5, 1.5, batch.f.shape[0], device="cuda")
loss, grads = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                            d["U_len"], grad_loss=w, mode={mode!r}, chunk_cells={chunk})
torch.cuda.synchronize()
out = {{"loss": loss.float().cpu().numpy()}}
out.update({{k: v.float().cpu().numpy() for k, v in grads.items()}})
np.savez({path!r}, **out)
"""


@pytest.mark.parametrize("mode,chunk", [("untiled", 0), ("tiled", 4096)])
def test_chained_equals_plain_stream_order(cuda_ok, tmp_path, mode, chunk):
    name = "short"
    path = str(tmp_path / "plain.npz")
    env = dict(os.environ, FRNNT_CHAIN="0")
    code = CHILD.format(root=ROOT, name=name, mode=mode, chunk=chunk, path=path)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    plain = np.load(path)

    batch = synth.workload(name)
    d = to_device(batch)
    w = torch.linspace(0.5, 1.5, batch.f.shape[0], device="cuda")
    loss, grads = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                                d["U_len"], grad_loss=w, mode=mode, chunk_cells=chunk)
    torch.cuda.synchronize()
    np.testing.assert_allclose(loss.float().cpu().numpy(), plain["loss"], rtol=1e-5)
    for k in GRADS:
        assert rel_l2(grads[k].float().cpu().numpy(), plain[k]) <= 1e-3, k
