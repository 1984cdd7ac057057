"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs, at the contract's tolerances."""

import json
import os

import numpy as np
import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, TOL, compare, rel_l2, run_oracle, to_device, weights_for

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _call(batch, mode="tiled", path="auto", grad_loss=None, chunk_cells=0, check=True, wgrad_f32=False):
    d = to_device(batch)
    w = None if grad_loss is None else torch.as_tensor(grad_loss, dtype=torch.float32).cuda()
    loss, grads = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                                d["U_len"], grad_loss=w, mode=mode, path=path, chunk_cells=chunk_cells,
                                blank=batch.blank, check=check, wgrad_f32=wgrad_f32)
    torch.cuda.synchronize()
    return loss, grads


# ---------------------------------------------------------------- fp32 (tiny)

@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_tiny_fp32_against_golden_and_oracle(cuda_ok, mode):
    batch = synth.workload("tiny")
    loss, grads = _call(batch, mode=mode)
    ref = run_oracle(batch)
    compare(loss, grads, ref, "f32", extra_note=f"tiny/{mode}")
    gold = json.load(open(os.path.join(HERE, "golden", "tiny_oracle.json")))
    np.testing.assert_allclose(loss.cpu().numpy(), gold["loss"], rtol=TOL["f32"]["loss"])
    for name in GRADS:
        assert rel_l2(grads[name].cpu().numpy(), np.array(gold[name])) <= TOL["f32"]["grad"]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_small_fp32_ragged(cuda_ok, seed):
    """Ragged lengths, a bias, U_len = 0 and T_len = 1 utterances, fp32."""
    batch = synth.make(B=5, T=9, U=6, D_enc=12, D_pred=10, H=24, V=11, dtype="f32", seed=200 + seed,
                       T_range=(1, 9), U_range=(0, 6), bias_std=0.5)
    batch.T_len[0] = 1
    batch.U_len[1] = 0
    w = np.linspace(-1.0, 2.0, 5)
    for mode in ("tiled", "untiled"):
        loss, grads = _call(batch, mode=mode, grad_loss=w, chunk_cells=20)
        compare(loss, grads, run_oracle(batch, grad_loss=w), "f32", extra_note=f"ragged/{mode}")


# ---------------------------------------------------------------- bf16 (short)

@pytest.mark.parametrize("mode", ["tiled", "untiled"])
@pytest.mark.parametrize("path", ["auto", "simt"])
def test_short_bf16(cuda_ok, mode, path):
    batch = synth.workload("short")
    loss, grads = _call(batch, mode=mode, path=path)
    compare(loss, grads, run_oracle(batch), "bf16", extra_note=f"short/{mode}/{path}")


def test_padding_does_not_leak(cuda_ok):
    """Redrawing every padding value (frames past T_len, positions past U_len,
    labels past U_len, here with large and out-of-range values) changes
    nothing beyond the floating-point reassociation of the fp32 atomics:
    losses are bit-exact, gradients agree to 1e-3 relative L2 (a leak would be
    O(1)), and padded gradient rows are exactly zero."""
    batch = synth.workload("short")
    other = synth.redraw_padding(batch, seed=9)
    for mode in ("tiled", "untiled"):
        l1, g1 = _call(batch, mode=mode)
        l2, g2 = _call(other, mode=mode)
        assert torch.equal(l1, l2)
        for name in GRADS:
            assert rel_l2(g1[name].float().cpu().numpy(), g2[name].float().cpu().numpy()) <= 1e-3, name
        for b in range(batch.f.shape[0]):
            Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
            assert int(torch.count_nonzero(g1["df"][b, Tb:])) == 0
            assert int(torch.count_nonzero(g1["dg"][b, Ub + 1:])) == 0
            assert int(torch.count_nonzero(g2["df"][b, Tb:])) == 0


# ---------------------------------------------------------------- status word (bit-exact)

@pytest.mark.parametrize("case,bits", [("T0", 1), ("Tbig", 1), ("Uneg", 1), ("Ubig", 1), ("blank", 2),
                                       ("label_hi", 2), ("label_neg", 2), ("both", 3)])
def test_status_bits(cuda_ok, case, bits):
    batch = synth.workload("tiny")
    if case == "T0":
        batch.T_len[0] = 0
    elif case == "Tbig":
        batch.T_len[1] = 13
    elif case == "Uneg":
        batch.U_len[0] = -1
    elif case == "Ubig":
        batch.U_len[1] = 6
    elif case == "blank":
        batch.labels[0, 2] = 0
    elif case == "label_hi":
        batch.labels[1, 4] = 8
    elif case == "label_neg":
        batch.labels[1, 0] = -2
    elif case == "both":
        batch.T_len[0] = 99
        batch.labels[1, 1] = 0
    import oracle
    expect = oracle.validate(12, 5, 8, 0, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy())
    assert expect == bits
    with pytest.raises(frnnt.FrnntStatusError) as ei:
        _call(batch)
    assert ei.value.bits == bits


def test_padding_labels_are_not_validated(cuda_ok):
    batch = synth.workload("tiny")
    batch.U_len[0] = 3
    batch.labels[0, 3] = -7          # padding: u >= U_len
    batch.labels[0, 4] = 0
    _call(batch)                     # must not raise


# ---------------------------------------------------------------- fp32 weight gradients

@pytest.mark.parametrize("mode", ["tiled", "untiled"])
@pytest.mark.parametrize("path", ["auto", "simt"])
def test_fp32_weight_gradients(cuda_ok, mode, path):
    """wgrad_f32: the weight gradients come back as the fp32 accumulators (df /
    dg stay bf16); they match the oracle, and rounding them to bf16 gives the
    default call's bf16 weight gradients up to the reassociation of the fp32
    atomics (bias sums cancel heavily, so this is checked in relative L2)."""
    batch = synth.workload("short")
    w = np.linspace(0.5, 1.5, batch.f.shape[0])
    l32, g32 = _call(batch, mode=mode, path=path, grad_loss=w, wgrad_f32=True)
    l32, g32 = l32.clone(), {k: v.clone() for k, v in g32.items()}
    for k in ("dW_f", "dW_g", "dW_o", "db_o"):
        assert g32[k].dtype == torch.float32, k
    for k in ("df", "dg"):
        assert g32[k].dtype == torch.bfloat16, k
    compare(l32, g32, run_oracle(batch, grad_loss=w), "bf16", extra_note=f"short fp32 weight grads/{mode}/{path}")
    l16, g16 = _call(batch, mode=mode, path=path, grad_loss=w)
    for k in ("dW_f", "dW_g", "dW_o", "db_o"):
        a = g32[k].to(torch.bfloat16).float().cpu().numpy()
        b = g16[k].float().cpu().numpy()
        assert rel_l2(a, b) <= 5e-3, (k, rel_l2(a, b))


def test_tiled_small_chunks_match_untiled(cuda_ok):
    """Many backward chunks (one per 4 tiles), including empty trailing chunks,
    give the untiled result up to floating-point reassociation."""
    batch = synth.workload("short")
    lt, gt = _call(batch, mode="tiled", chunk_cells=512)
    lt, gt = lt.clone(), {k: v.clone() for k, v in gt.items()}
    lu, gu = _call(batch, mode="untiled")
    assert torch.allclose(lt, lu, rtol=1e-4)
    for k in GRADS:
        assert rel_l2(gt[k].float().cpu().numpy(), gu[k].float().cpu().numpy()) <= 1e-2, k


# ---------------------------------------------------------------- joint kernel variants

@pytest.fixture
def joint_variant():
    prev = frnnt.set_joint_variant(-1)
    yield frnnt.set_joint_variant
    frnnt.set_joint_variant(prev)


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
@pytest.mark.parametrize("variant", [0, 1])
def test_joint_variants_odd_tile_count(cuda_ok, joint_variant, mode, variant):
    """Both joint kernel variants on the tensor-core path, forced, on a batch
    with an odd number of cell tiles (5: the last CTA pair holds one real tile
    and one empty one) and ragged lengths."""
    batch = synth.make(B=3, T=20, U=5, D_enc=64, D_pred=32, H=128, V=256, dtype="bf16", seed=31,
                       T_range=(13, 20), U_range=(0, 5), bias_std=0.2)
    batch.T_len[:] = torch.tensor([20, 13, 17], dtype=batch.T_len.dtype)
    joint_variant(variant)
    loss, grads = _call(batch, mode=mode, chunk_cells=256)
    compare(loss, grads, run_oracle(batch), "bf16", extra_note=f"odd/{mode}/v{variant}")


@pytest.mark.parametrize("variant", [0, 1])
def test_joint_variants_short(cuda_ok, joint_variant, variant):
    batch = synth.workload("short")
    joint_variant(variant)
    for mode in ("tiled", "untiled"):
        loss, grads = _call(batch, mode=mode)
        compare(loss, grads, run_oracle(batch), "bf16", extra_note=f"short/{mode}/v{variant}")


@pytest.mark.parametrize("loss", ["marginal", "viterbi"])
def test_wide_label_lattice(cuda_ok, loss):
    """More than 512 label positions: the DP blocks of up to 1024 threads
    (U + 1 = 701 here), both modes."""
    batch = synth.make(B=2, T=12, U=700, D_enc=64, D_pred=64, H=128, V=128, dtype="bf16", seed=77,
                       T_range=(6, 12), U_range=(660, 700), bias_std=0.3)
    ref = run_oracle(batch, loss=loss)
    for mode in ("untiled", "tiled"):
        d = to_device(batch)
        l, g = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                             d["U_len"], mode=mode, chunk_cells=4096, blank=batch.blank, loss=loss)
        torch.cuda.synchronize()
        compare(l, g, ref, "bf16", extra_note=f"wide lattice {loss}/{mode}")


@pytest.mark.parametrize("loss", ["marginal", "viterbi"])
def test_maximum_label_positions(cuda_ok, loss):
    """U+1 = 1024, the widest lattice the interface accepts (one DP thread per
    label position, a full 1024-thread block), both modes."""
    batch = synth.make(B=2, T=6, U=1023, D_enc=64, D_pred=64, H=128, V=128, dtype="bf16", seed=1023,
                       T_range=(3, 6), U_range=(1000, 1023), bias_std=0.3)
    batch.U_len[0] = 1023
    ref = run_oracle(batch, loss=loss)
    for mode in ("untiled", "tiled"):
        d = to_device(batch)
        l, g = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                             d["U_len"], mode=mode, chunk_cells=4096, blank=batch.blank, loss=loss)
        torch.cuda.synchronize()
        compare(l, g, ref, "bf16", extra_note=f"U+1 = 1024 {loss}/{mode}")
