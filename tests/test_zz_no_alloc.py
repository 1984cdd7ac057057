"""frnnt_fwd_bwd_noalloc, the entry point for callers that cannot allocate
device memory when they run the loss (their framework's allocator owns all
device memory, or an allocation could synchronise the device).  It must give
the same result as frnnt_fwd_bwd with a caller-provided workspace, also on a
second call that finds the previous call's data in the shared scratch array.

Kept in a file that pytest collects last, so a run that stops at the first
failure has run every other test before this one."""

import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, TOL, rel_l2, to_device

pytestmark = pytest.mark.gpu


def _args(d):
    return (d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"], d["U_len"])


@pytest.mark.parametrize("name,mode,chunk", [("tiny", "tiled", 0), ("tiny", "untiled", 0),
                                             ("short", "tiled", 4096), ("short", "untiled", 0)])
def test_noalloc_matches_workspace_entry_on_two_calls(cuda_ok, name, mode, chunk):
    batch = synth.workload(name)
    d = to_device(batch)
    w = torch.linspace(0.5, 1.5, batch.f.shape[0], device="cuda")
    ref_loss, ref = frnnt.fwd_bwd(*_args(d), grad_loss=w, mode=mode, chunk_cells=chunk)
    ref_loss = ref_loss.clone()
    ref = {k: v.clone() for k, v in ref.items()}
    tol = TOL[batch.dtype]
    for _ in range(2):
        loss, grads = frnnt.fwd_bwd_noalloc(*_args(d), grad_loss=w, mode=mode, chunk_cells=chunk)
        torch.cuda.synchronize()
        lrel = ((loss - ref_loss).abs() / ref_loss.abs()).max().item()
        assert lrel <= tol["loss"], lrel
        for k in GRADS:
            err = rel_l2(grads[k].float().cpu().numpy(), ref[k].float().cpu().numpy())
            assert err <= tol["grad"], (k, err)


def test_noalloc_smaller_call_after_a_larger_one(cuda_ok):
    """A large call leaves its data all over the shared array; a following
    smaller call of other dims (other offsets for every region) must not read
    any of it."""
    big = synth.workload("short")
    db = to_device(big)
    frnnt.fwd_bwd_noalloc(*_args(db), mode="untiled")
    torch.cuda.synchronize()
    for name, mode, chunk in (("tiny", "tiled", 0), ("short", "tiled", 1024)):
        small = synth.workload(name, seed=77) if name == "short" else synth.workload(name)
        ds = to_device(small)
        w = torch.linspace(1.5, 0.5, small.f.shape[0], device="cuda")
        ref_loss, ref = frnnt.fwd_bwd(*_args(ds), grad_loss=w, mode=mode, chunk_cells=chunk)
        ref_loss = ref_loss.clone()
        ref = {k: v.clone() for k, v in ref.items()}
        loss, grads = frnnt.fwd_bwd_noalloc(*_args(ds), grad_loss=w, mode=mode, chunk_cells=chunk)
        torch.cuda.synchronize()
        tol = TOL[small.dtype]
        assert ((loss - ref_loss).abs() / ref_loss.abs()).max().item() <= tol["loss"]
        for k in GRADS:
            err = rel_l2(grads[k].float().cpu().numpy(), ref[k].float().cpu().numpy())
            assert err <= tol["grad"], (name, k, err)
        frnnt.fwd_bwd_noalloc(*_args(db), mode="untiled")    # and the large one again in between
        torch.cuda.synchronize()


def test_noalloc_rejects_dims_beyond_its_scratch(cuda_ok):
    batch = synth.workload("medium")
    d = to_device(batch)
    dims = frnnt.dims_of(d["f"], d["g"], d["W_o"], "bf16", "untiled", "auto", 0, 0)
    assert frnnt.workspace_size(dims) > frnnt.NOALLOC_MAX_BYTES
    with pytest.raises(frnnt.FrnntError) as ei:
        frnnt.fwd_bwd_noalloc(*_args(d), mode="untiled")
    assert ei.value.code == 3
