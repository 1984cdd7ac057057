"""Calls from two host threads at once, on one device and two streams.  The
untiled tensor-core path forks work onto the library's per-device side stream
and joins it back with events shared by the device's calls; each call holds a
per-device lock while it queues that work, so every call waits for its own
side work.  Both threads' results must be the oracle's."""

import threading

import numpy as np
import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import compare, run_oracle, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["untiled", "tiled"])
def test_two_threads_two_streams_one_device(cuda_ok, mode):
    batches = [synth.workload("short"), synth.workload("short", seed=4242)]
    weights = [np.linspace(0.5, 1.5, 8), np.linspace(2.0, 0.25, 8)]
    refs = [run_oracle(b, grad_loss=w) for b, w in zip(batches, weights)]
    results = [None, None]
    errors = []
    start = threading.Barrier(2)

    def worker(i):
        try:
            torch.cuda.set_device(0)
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                d = to_device(batches[i])
                w = torch.as_tensor(weights[i], dtype=torch.float32, device="cuda")
                dims = frnnt.dims_of(d["f"], d["g"], d["W_o"], "bf16", mode, "auto", 0, 0)
                out = frnnt.Outputs(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], dims)
                stream.synchronize()
                start.wait()
                for _ in range(6):
                    frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                                  d["U_len"], grad_loss=w, mode=mode, out=out, check=False, stream=stream)
                stream.synchronize()
                if int(out.status[0].item()) != 0:
                    raise RuntimeError(f"status {int(out.status[0].item())}")
                results[i] = (out.loss.clone(), {k: v.clone() for k, v in out.grads().items()})
        except Exception as e:   # reported by the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a worker thread did not finish"
    assert not errors, errors
    for i in range(2):
        loss, grads = results[i]
        compare(loss, grads, refs[i], "bf16", extra_note=f"thread {i}/{mode}")
