"""GPU parity of the maximum-approximation (Viterbi) loss against the fp64
oracle's Viterbi variant, through the C ABI."""

import math

import numpy as np
import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, compare, rel_l2, run_oracle, to_device, weights_for

pytestmark = pytest.mark.gpu


def _call(batch, mode="tiled", path="auto", grad_loss=None, chunk_cells=0, loss="viterbi"):
    d = to_device(batch)
    w = None if grad_loss is None else torch.as_tensor(grad_loss, dtype=torch.float32).cuda()
    out = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                        d["U_len"], grad_loss=w, mode=mode, path=path, chunk_cells=chunk_cells, blank=batch.blank,
                        loss=loss)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_tiny_fp32(cuda_ok, mode):
    batch = synth.workload("tiny")
    loss, grads = _call(batch, mode=mode)
    compare(loss, grads, run_oracle(batch, loss="viterbi"), "f32", extra_note=f"viterbi tiny/{mode}")


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_small_fp32_ragged(cuda_ok, seed):
    batch = synth.make(B=5, T=9, U=6, D_enc=12, D_pred=10, H=24, V=11, dtype="f32", seed=500 + seed,
                       T_range=(1, 9), U_range=(0, 6), bias_std=0.5)
    batch.T_len[0] = 1
    batch.U_len[1] = 0
    w = np.linspace(-1.0, 2.0, 5)
    for mode in ("tiled", "untiled"):
        loss, grads = _call(batch, mode=mode, grad_loss=w, chunk_cells=20)
        compare(loss, grads, run_oracle(batch, grad_loss=w, loss="viterbi"), "f32",
                extra_note=f"viterbi ragged/{mode}")


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
@pytest.mark.parametrize("path", ["auto", "simt"])
def test_short_bf16(cuda_ok, mode, path):
    batch = synth.workload("short")
    loss, grads = _call(batch, mode=mode, path=path)
    compare(loss, grads, run_oracle(batch, loss="viterbi"), "bf16", extra_note=f"viterbi short/{mode}/{path}")


def test_single_alignment_matches_marginal(cuda_ok):
    """U_len = 0 or T_len = 1: one alignment, so both criteria agree."""
    batch = synth.make(B=4, T=7, U=5, D_enc=8, D_pred=8, H=16, V=9, dtype="f32", seed=77,
                       T_range=(1, 7), U_range=(0, 5), bias_std=0.3)
    batch.U_len[0] = 0
    batch.U_len[1] = 0
    batch.T_len[2] = 1
    batch.T_len[3] = 1
    lv, gv = _call(batch, loss="viterbi")
    lv, gv = lv.clone(), {k: v.clone() for k, v in gv.items()}
    lm, gm = _call(batch, loss="marginal")
    assert torch.allclose(lv, lm, rtol=1e-5)
    for k in GRADS:
        assert rel_l2(gv[k].cpu().numpy(), gm[k].cpu().numpy()) <= 1e-5, k


def test_zero_logits_tie_rule(cuda_ok):
    """W_o = 0, b_o = 0: every decision ties and goes to the blank edge (the
    alignment emits every label at frame 0); the loss is (T+U) ln V."""
    batch = synth.make(B=2, T=6, U=3, D_enc=8, D_pred=8, H=16, V=7, dtype="f32", seed=78,
                       T_range=(6, 6), U_range=(3, 3))
    batch.W_o.zero_()
    batch.b_o.zero_()
    for mode in ("tiled", "untiled"):
        loss, grads = _call(batch, mode=mode)
        np.testing.assert_allclose(loss.cpu().numpy(), [9 * math.log(7)] * 2, rtol=1e-6)
        compare(loss, grads, run_oracle(batch, loss="viterbi"), "f32", extra_note=f"viterbi ties/{mode}")


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_medium_sampled(cuda_ok, mode):
    """Full medium workload in the bench's launch configuration; two utterances checked."""
    batch = synth.workload("medium")
    B = batch.f.shape[0]
    pick = [0, B - 1]
    w = weights_for(B, pick, device="cpu").numpy()
    loss, grads = _call(batch, mode=mode, grad_loss=w)
    ref = run_oracle(batch, grad_loss=w, utterances=pick, loss="viterbi")
    compare(loss, grads, ref, "bf16", utterances=pick, extra_note=f"viterbi medium/{mode}")
