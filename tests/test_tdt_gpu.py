"""GPU parity of the token-and-duration transducer (frnnt_fwd_bwd_tdt, bf16,
tensor-core kernels) against the fp64 oracle on the same seeded inputs."""

import numpy as np
import pytest
import torch

import oracle
from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, TOL, record, rel_l2, to_device, weights_for

pytestmark = pytest.mark.gpu

TDT_GRADS = GRADS + ("dW_d", "db_d")


def _oracle(batch, W_d, b_d, D, grad_loss=None, utterances=None):
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    w = None if grad_loss is None else np.asarray(grad_loss, dtype=np.float64)
    return oracle.tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d.double().numpy(), b_d.double().numpy(),
                              batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(), D, grad_loss=w,
                              blank=batch.blank, utterances=utterances)


def _call(batch, W_d, b_d, D, mode="tiled", grad_loss=None, chunk_cells=0):
    d = to_device(batch)
    w = None if grad_loss is None else torch.as_tensor(grad_loss, dtype=torch.float32).cuda()
    out = frnnt.fwd_bwd_tdt(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], W_d.cuda(), b_d.cuda(),
                            d["labels"], d["T_len"], d["U_len"], D, grad_loss=w, mode=mode, chunk_cells=chunk_cells,
                            blank=batch.blank)
    torch.cuda.synchronize()
    return out


def _compare(loss, grads, ref, note, utterances=None):
    tol = TOL["bf16"]
    loss = loss.float().cpu().numpy().astype(np.float64)
    idx = list(range(len(ref.loss))) if utterances is None else list(utterances)
    errs = {"loss": float(np.max(np.abs(loss[idx] - ref.loss[idx]) / np.abs(ref.loss[idx])))}
    for name in TDT_GRADS:
        gpu = grads[name].float().cpu().numpy()
        r = getattr(ref, name)
        if utterances is not None and name in ("df", "dg"):
            gpu, r = gpu[idx], r[idx]
        errs[name] = rel_l2(gpu, r)
    record(note, "bf16", errs)
    bad = {k: v for k, v in errs.items() if v > (tol["loss"] if k == "loss" else tol["grad"])}
    assert not bad, f"{note}: tolerance exceeded {bad} (all {errs})"
    return errs


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
@pytest.mark.parametrize("D", [(0, 1, 2, 3, 4), (0, 1, 2, 4, 8), (0, 1)])
def test_ragged_small(cuda_ok, mode, D):
    """Several cell tiles with ragged tails, lengths down to one frame and no
    labels, weighted utterances, a bias on both heads and (tiled) several chunks."""
    batch = synth.make(B=5, T=40, U=12, D_enc=64, D_pred=32, H=128, V=256, dtype="bf16", seed=700 + len(D),
                       T_range=(1, 40), U_range=(0, 12), bias_std=0.3)
    W_d, b_d = synth.duration_head(batch, len(D), seed=71 + len(D))
    w = np.linspace(0.5, 1.5, 5)
    l, g = _call(batch, W_d, b_d, D, mode=mode, grad_loss=w, chunk_cells=512)
    _compare(l, g, _oracle(batch, W_d, b_d, D, grad_loss=w), f"tdt {D}/{mode}")


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_short_workload(cuda_ok, mode):
    batch = synth.workload("short")
    D = synth.TDT_DURATIONS
    W_d, b_d = synth.duration_head(batch, len(D), seed=5)
    l, g = _call(batch, W_d, b_d, D, mode=mode)
    _compare(l, g, _oracle(batch, W_d, b_d, D), f"tdt short/{mode}")


def test_medium_sampled_utterances(cuda_ok):
    """The medium workload in the benchmark's launch configuration (untiled),
    checked on two utterances the oracle computes one by one (the others get
    weight 0, so every weight gradient is theirs alone)."""
    batch = synth.workload("medium")
    D = synth.TDT_DURATIONS
    W_d, b_d = synth.duration_head(batch, len(D), seed=5)
    utt = [0, int(np.argmax(batch.T_len.numpy()))]
    w = weights_for(batch.f.shape[0], utt).cpu().numpy()
    l, g = _call(batch, W_d, b_d, D, mode="untiled", grad_loss=w)
    _compare(l, g, _oracle(batch, W_d, b_d, D, grad_loss=w, utterances=utt), "tdt medium", utterances=utt)


def test_modes_agree_and_padding_ignored(cuda_ok):
    """Tiled (small chunks) and untiled give the same result, and redrawn
    padding (frames past T_len, positions past U_len, labels past U_len) changes nothing."""
    batch = synth.make(B=4, T=30, U=10, D_enc=64, D_pred=64, H=128, V=256, dtype="bf16", seed=77,
                       T_range=(5, 30), U_range=(0, 10))
    D = (0, 1, 2, 3)
    W_d, b_d = synth.duration_head(batch, len(D), seed=3)
    lu, gu = _call(batch, W_d, b_d, D, mode="untiled")
    lu, gu = lu.clone(), {k: v.clone() for k, v in gu.items()}
    lt, gt = _call(synth.redraw_padding(batch, seed=9), W_d, b_d, D, mode="tiled", chunk_cells=256)
    assert torch.allclose(lu, lt, rtol=1e-4)
    for k in TDT_GRADS:
        if k in ("df", "dg"):
            continue    # padding rows of df / dg are zero on both sides; compared below
        assert rel_l2(gt[k].float().cpu().numpy(), gu[k].float().cpu().numpy()) <= 1e-2, k
    for k in ("df", "dg"):
        assert rel_l2(gt[k].float().cpu().numpy(), gu[k].float().cpu().numpy()) <= 1e-2, k


@pytest.mark.parametrize("U,D", [(300, (0, 1, 2, 3, 4)), (700, (0, 1, 2, 3, 4)), (700, (0, 1, 2, 4, 8))])
def test_wide_label_lattice(cuda_ok, U, D):
    """Label positions past 256 and 512 (the DP's 512- and 1024-thread
    instantiations, the latter with the largest duration set), both modes."""
    batch = synth.make(B=2, T=12, U=U, D_enc=64, D_pred=64, H=128, V=128, dtype="bf16", seed=900 + U,
                       T_range=(6, 12), U_range=(U - 40, U), bias_std=0.3)
    W_d, b_d = synth.duration_head(batch, len(D), seed=U)
    ref = _oracle(batch, W_d, b_d, D)
    for mode in ("untiled", "tiled"):
        l, g = _call(batch, W_d, b_d, D, mode=mode, chunk_cells=4096)
        _compare(l, g, ref, f"tdt U{U} {D}/{mode}")
