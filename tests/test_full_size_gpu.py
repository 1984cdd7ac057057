"""GPU parity at the full sizes of the benchmark workloads, in the launch
configuration bench.py times (default chunk, both modes), against the fp64
oracle on the same seeded inputs:

* medium: every utterance's loss and the complete gradients of the whole
  batch (gradient weight 1 on all sixteen utterances);
* large and long: every utterance's loss, the gradients of two utterances
  picked by a seeded draw (another pair per mode), and exact zeros in the df /
  dg rows of every utterance whose gradient weight is 0;
* large and long with the maximum-approximation criterion, the pruned lattice
  (S = 8, a band along the diagonal) and the token-and-duration transducer
  (durations 0..4): the losses and gradients of a sampled utterance.

The transducer loss sums over every alignment of every utterance ("Sequence
Transduction with Recurrent Neural Networks", abstract), so each utterance's
loss is checked on its own.  Oracle results are cached per input, so the two
modes share them."""

import zlib

import numpy as np
import pytest
import torch

import oracle
from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, TOL, compare, record, rel_l2, run_oracle, to_device, weights_for

pytestmark = pytest.mark.gpu

_CACHE = {}


def _cached(key, fn):
    if key not in _CACHE:
        _CACHE[key] = fn()
    return _CACHE[key]


def _pick(name, tag, B, n=2):
    """n distinct utterances drawn by a generator seeded from the case's name."""
    rng = np.random.default_rng(zlib.crc32(f"{name}/{tag}".encode()))
    return sorted(int(x) for x in rng.choice(B, size=n, replace=False))


def _losses(batch, loss="marginal", bounds=None, S=0):
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    return oracle.loss_only(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                            batch.U_len.numpy(), blank=batch.blank, loss=loss,
                            bounds=None if bounds is None else np.asarray(bounds), S=S)


def _check_every_loss(loss, ref_loss, note):
    got = loss.detach().float().cpu().numpy().astype(np.float64)
    rel = np.abs(got - ref_loss) / np.abs(ref_loss)
    record(note + " (every utterance's loss)", "bf16", {"loss": float(rel.max())})
    assert np.all(np.isfinite(got)), note
    assert float(rel.max()) <= TOL["bf16"]["loss"], f"{note}: loss rel errors {rel}"


def _check_zero_rows(grads, B, pick, note):
    """Utterances with gradient weight 0 contribute nothing: their df and dg rows are exactly 0."""
    for b in range(B):
        if b in pick:
            continue
        assert int(torch.count_nonzero(grads["df"][b])) == 0, f"{note}: df rows of utterance {b}"
        assert int(torch.count_nonzero(grads["dg"][b])) == 0, f"{note}: dg rows of utterance {b}"


def _call(batch, mode, grad_loss=None, loss="marginal", bounds=None, S=0):
    d = to_device(batch)
    w = None if grad_loss is None else torch.as_tensor(grad_loss, dtype=torch.float32).cuda()
    if bounds is not None:
        bd = torch.as_tensor(np.asarray(bounds), dtype=torch.int32).contiguous().cuda()
        out = frnnt.fwd_bwd_pruned(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                                   d["U_len"], bd, S, grad_loss=w, mode=mode, blank=batch.blank, loss=loss)
    else:
        out = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                            d["U_len"], grad_loss=w, mode=mode, blank=batch.blank, loss=loss)
    torch.cuda.synchronize()
    return out


# ---------------------------------------------------------------- medium: the whole batch

@pytest.mark.parametrize("mode", ["untiled", "tiled"])
def test_medium_every_utterance(cuda_ok, mode):
    """Gradient weight 1 on every utterance: all sixteen losses and the complete
    df, dg, dW_f, dW_g, dW_o and db_o of the batch."""
    batch = synth.workload("medium")
    ref = _cached(("medium", "all"), lambda: run_oracle(batch))
    loss, grads = _call(batch, mode)
    compare(loss, grads, ref, "bf16", extra_note=f"medium whole batch/{mode}")


# ---------------------------------------------------------------- large, long: every loss, sampled gradients

@pytest.mark.parametrize("mode", ["untiled", "tiled"])
@pytest.mark.parametrize("name", ["large", "long"])
def test_every_loss_sampled_gradients(cuda_ok, name, mode):
    batch = synth.workload(name)
    B = batch.f.shape[0]
    pick = _pick(name, mode, B)
    w = weights_for(B, pick, device="cpu").numpy()
    loss, grads = _call(batch, mode, grad_loss=w)
    _check_every_loss(loss, _cached((name, "losses"), lambda: _losses(batch)), f"{name}/{mode}")
    ref = _cached((name, "grads", tuple(pick)), lambda: run_oracle(batch, grad_loss=w, utterances=pick))
    compare(loss, grads, ref, "bf16", utterances=pick, extra_note=f"{name}/{mode} utterances {pick}")
    _check_zero_rows(grads, B, pick, f"{name}/{mode}")


# ---------------------------------------------------------------- large, long: the loss variants

@pytest.mark.parametrize("mode", ["untiled", "tiled"])
@pytest.mark.parametrize("name", ["large", "long"])
def test_viterbi_sampled(cuda_ok, name, mode):
    """The maximum-approximation criterion: a sampled utterance's loss and gradients."""
    batch = synth.workload(name)
    B = batch.f.shape[0]
    pick = _pick(name, "viterbi", B, n=1)
    w = weights_for(B, pick, device="cpu").numpy()
    loss, grads = _call(batch, mode, grad_loss=w, loss="viterbi")
    ref = _cached((name, "viterbi", tuple(pick)),
                  lambda: run_oracle(batch, grad_loss=w, utterances=pick, loss="viterbi"))
    compare(loss, grads, ref, "bf16", utterances=pick, extra_note=f"viterbi {name}/{mode} utterance {pick}")
    _check_zero_rows(grads, B, pick, f"viterbi {name}/{mode}")


@pytest.mark.parametrize("mode", ["untiled", "tiled"])
@pytest.mark.parametrize("name", ["large", "long"])
def test_pruned_sampled(cuda_ok, name, mode):
    """The pruned lattice, S = 8 label positions per frame on a band along the
    diagonal: a sampled utterance's loss and gradients."""
    batch = synth.workload(name)
    B, T = batch.f.shape[:2]
    S = 8
    bounds = synth.diagonal_bounds(batch.T_len, batch.U_len, T, S).numpy()
    pick = _pick(name, "pruned", B, n=1)
    w = weights_for(B, pick, device="cpu").numpy()
    loss, grads = _call(batch, mode, grad_loss=w, bounds=bounds, S=S)
    ref = _cached((name, "pruned", tuple(pick)),
                  lambda: run_oracle(batch, grad_loss=w, utterances=pick, bounds=bounds, S=S))
    compare(loss, grads, ref, "bf16", utterances=pick, extra_note=f"pruned S8 {name}/{mode} utterance {pick}")
    _check_zero_rows(grads, B, pick, f"pruned {name}/{mode}")


@pytest.mark.parametrize("mode", ["untiled", "tiled"])
@pytest.mark.parametrize("name", ["large", "long"])
def test_tdt_sampled(cuda_ok, name, mode):
    """The token-and-duration transducer (durations 0..4): a sampled
    utterance's loss and gradients, the duration head's included.  On long the
    shortest utterance is taken (the oracle holds its whole lattice of logits)."""
    batch = synth.workload(name)
    B = batch.f.shape[0]
    D = synth.TDT_DURATIONS
    W_d, b_d = synth.duration_head(batch, len(D), seed=5)
    pick = [int(np.argmin(batch.T_len.numpy()))] if name == "long" else _pick(name, "tdt", B, n=1)
    w = weights_for(B, pick, device="cpu").numpy()
    d = to_device(batch)
    loss, grads = frnnt.fwd_bwd_tdt(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], W_d.cuda(), b_d.cuda(),
                                    d["labels"], d["T_len"], d["U_len"], D,
                                    grad_loss=torch.as_tensor(w, dtype=torch.float32).cuda(), mode=mode,
                                    blank=batch.blank)
    torch.cuda.synchronize()

    def run():
        f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
        return oracle.tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d.double().numpy(), b_d.double().numpy(),
                                  batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(), D, grad_loss=w,
                                  blank=batch.blank, utterances=pick)

    ref = _cached((name, "tdt", tuple(pick)), run)
    got = loss.float().cpu().numpy().astype(np.float64)
    errs = {"loss": float(np.max(np.abs(got[pick] - ref.loss[pick]) / np.abs(ref.loss[pick])))}
    for k in GRADS + ("dW_d", "db_d"):
        a, r = grads[k].float().cpu().numpy(), getattr(ref, k)
        if k in ("df", "dg"):
            a, r = a[pick], r[pick]
        errs[k] = rel_l2(a, r)
    note = f"tdt {name}/{mode} utterance {pick}"
    record(note, "bf16", errs)
    bad = {k: v for k, v in errs.items() if v > (TOL["bf16"]["loss"] if k == "loss" else TOL["bf16"]["grad"])}
    assert not bad, f"{note}: tolerance exceeded {bad} (all {errs})"
    _check_zero_rows(grads, B, pick, note)
