"""The sharded data-parallel call on the GPU with the CUDA library as the
per-rank compute.  One GPU is available here, so the process group has a
single NCCL rank: the exchange runs, and the result must equal the plain call."""

import socket

import pytest
import torch
import torch.distributed as dist

from rnn_joint_network_02_b200 import dist as rdist
from rnn_joint_network_02_b200 import synth
from tests.helpers import GRADS, compare, run_oracle, to_device

pytestmark = pytest.mark.gpu


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_single_rank_nccl_sharded_call_matches_oracle(cuda_ok):
    batch = synth.workload("short")
    t = to_device(batch)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        idx, loss, grads = rdist.fwd_bwd_sharded(t, rdist.gpu_compute("tiled"), 0, 1)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert idx == list(range(batch.f.shape[0]))
    # the shard was trimmed to its longest utterance: pad df / dg back to the batch's extents
    full = dict(grads)
    for k, src in (("df", t["f"]), ("dg", t["g"])):
        z = torch.zeros_like(src)
        z[:, :grads[k].shape[1]] = grads[k]
        full[k] = z
    ref = run_oracle(batch)
    compare(loss, {k: full[k] for k in GRADS}, ref, "bf16", extra_note="sharded")
