"""Shared test helpers: moving a synthetic batch to the device, running the
oracle on it, and the parity metrics with the contract's tolerances."""

from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances of the contract: fp32 loss rel <= 1e-4 and gradient rel-L2 <= 1e-4;
# bf16 loss rel <= 5e-3 and gradient rel-L2 <= 2e-2; integers bit-exact.
TOL = {"f32": dict(loss=1e-4, grad=1e-4), "bf16": dict(loss=5e-3, grad=2e-2)}
GRADS = ("df", "dg", "dW_f", "dW_g", "dW_o", "db_o")

# Every comparison's measured errors, (note, dtype, {name: error}); the test
# session's summary prints the worst error of each tensor against its tolerance.
MARGINS: list = []


def record(note: str, dtype: str, errs: dict) -> None:
    MARGINS.append((note, dtype, dict(errs)))


def margin_report() -> list:
    """Lines: per (dtype, tensor), the largest error / tolerance and where."""
    worst = {}
    for note, dtype, errs in MARGINS:
        for name, err in errs.items():
            tol = TOL[dtype]["loss" if name == "loss" else "grad"]
            key = (dtype, name)
            if key not in worst or err / tol > worst[key][0]:
                worst[key] = (err / tol, err, tol, note)
    lines = []
    for (dtype, name), (frac, err, tol, note) in sorted(worst.items()):
        lines.append(f"{dtype:5s} {name:6s} worst {err:.3e} = {frac:6.1%} of tolerance {tol:.0e}  ({note})")
    return lines


def to_device(batch, device="cuda"):
    d = {k: getattr(batch, k).to(device).contiguous()
         for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")}
    return d


def run_oracle(batch, grad_loss=None, utterances=None, keep_lattice=False, loss="marginal", bounds=None, S=0):
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    w = None if grad_loss is None else np.asarray(grad_loss, dtype=np.float64)
    return oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                          batch.U_len.numpy(), grad_loss=w, blank=batch.blank, utterances=utterances,
                          keep_lattice=keep_lattice, loss=loss,
                          bounds=None if bounds is None else np.asarray(bounds), S=S)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def compare(loss, grads, ref, dtype, utterances=None, extra_note=""):
    """Asserts the contract's tolerances; returns the measured errors."""
    tol = TOL[dtype]
    loss = loss.detach().float().cpu().numpy().astype(np.float64)
    idx = list(range(len(ref.loss))) if utterances is None else list(utterances)
    lrel = float(np.max(np.abs(loss[idx] - ref.loss[idx]) / np.abs(ref.loss[idx])))
    errs = {"loss": lrel}
    for name in GRADS:
        gpu = grads[name].detach().float().cpu().numpy()
        r = getattr(ref, name)
        if utterances is not None and name in ("df", "dg"):
            gpu = gpu[idx]
            r = r[idx]
        errs[name] = rel_l2(gpu, r)
    record(extra_note, dtype, errs)
    bad = {k: v for k, v in errs.items() if v > (tol["loss"] if k == "loss" else tol["grad"])}
    assert not bad, f"{extra_note} tolerance exceeded: {bad} (all: {errs})"
    return errs


def weights_for(B, utterances, device="cuda"):
    w = torch.zeros(B, dtype=torch.float32)
    w[list(utterances)] = 1.0
    return w.to(device)
