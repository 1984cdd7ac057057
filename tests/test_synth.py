"""The seeded input recipe that both the CUDA path and the oracle consume:
shapes, dtypes, length rules, label validity, distributions, determinism and
the padding / pruning-bound helpers.  CPU only."""

import math
import os

import pytest
import torch

import oracle
from rnn_joint_network_02_b200 import synth

NAMES = list(synth.WORKLOADS)


@pytest.mark.parametrize("name", NAMES)
def test_shapes_dtypes_and_lengths(name):
    spec = synth.WORKLOADS[name]
    b = synth.workload(name)
    B, T, U, De, Dp, H, V = (spec[k] for k in ("B", "T", "U", "D_enc", "D_pred", "H", "V"))
    ft = torch.bfloat16 if spec["dtype"] == "bf16" else torch.float32
    assert b.f.shape == (B, T, De) and b.g.shape == (B, U + 1, Dp)
    assert b.W_f.shape == (De, H) and b.W_g.shape == (Dp, H) and b.W_o.shape == (V, H) and b.b_o.shape == (V,)
    assert all(t.dtype == ft for t in b.tensors())
    assert b.labels.shape == (B, U) and b.labels.dtype == torch.int32
    assert b.T_len.dtype == torch.int32 and b.U_len.dtype == torch.int32
    lo, hi = spec["T_range"]
    assert int(b.T_len.min()) >= lo and int(b.T_len.max()) <= hi and lo >= 1 and hi <= T
    rule = spec.get("U_rule", "range")
    if rule == "full":
        assert torch.all(b.U_len == U)
    elif rule == "T/5":
        assert torch.equal(b.U_len, torch.clamp(b.T_len // 5, min=1, max=U))
    else:
        ulo, uhi = spec["U_range"]
        assert int(b.U_len.min()) >= ulo and int(b.U_len.max()) <= uhi
    assert int(b.U_len.min()) >= 0 and int(b.U_len.max()) <= U
    assert b.blank == 0 and torch.all(b.b_o == 0)


@pytest.mark.parametrize("name", NAMES)
def test_labels_are_valid_and_never_blank(name):
    b = synth.workload(name)
    V = b.W_o.shape[0]
    for i in range(b.labels.shape[0]):
        lab = b.labels[i, :int(b.U_len[i])]
        assert torch.all((lab >= 1) & (lab <= V - 1))
    assert oracle.validate(b.f.shape[1], b.g.shape[1] - 1, V, b.blank, b.labels.numpy(), b.T_len.numpy(),
                           b.U_len.numpy()) == 0


def test_seeded_and_deterministic():
    a, b = synth.workload("short"), synth.workload("short")
    for x, y in zip(a.tensors() + (a.labels, a.T_len, a.U_len), b.tensors() + (b.labels, b.T_len, b.U_len)):
        assert torch.equal(x, y)
    c = synth.workload("short", seed=12345)
    assert not torch.equal(a.f, c.f) and not torch.equal(a.labels, c.labels)
    # the seed is 1000 + the workload's index
    d = synth.make(seed=1000 + synth.WORKLOADS["short"]["index"],
                   **{k: v for k, v in synth.WORKLOADS["short"].items() if k != "index"})
    assert torch.equal(a.W_o, d.W_o)


def test_distributions():
    """N(0,1) activations and N(0, 1/fan_in) weights (the medium workload's
    samples are large enough for 3 % bands)."""
    b = synth.workload("medium")
    H = b.W_o.shape[1]
    assert abs(float(b.f.float().std()) - 1.0) < 0.03 and abs(float(b.f.float().mean())) < 0.03
    assert abs(float(b.W_o.float().std()) * math.sqrt(H) - 1.0) < 0.03
    assert abs(float(b.W_f.float().std()) * math.sqrt(b.W_f.shape[0]) - 1.0) < 0.03
    assert abs(float(b.W_g.float().std()) * math.sqrt(b.W_g.shape[0]) - 1.0) < 0.03


def test_zipf_labels_of_the_large_vocabulary():
    """P(k) proportional to k^-1.1 over 1..V-1: small ids dominate in that order."""
    b = synth.workload("large")
    counts = torch.bincount(b.labels.flatten().long(), minlength=b.W_o.shape[0]).numpy()
    assert counts[0] == 0
    assert counts[1] > counts[2] > counts[4] > counts[16]
    # ratio of the two most frequent ids close to 2^1.1
    assert abs(counts[1] / counts[2] - 2 ** 1.1) < 0.4


def test_redraw_padding_changes_only_padding():
    b = synth.workload("short")
    r = synth.redraw_padding(b, seed=3)
    for i in range(b.f.shape[0]):
        Tb, Ub = int(b.T_len[i]), int(b.U_len[i])
        assert torch.equal(r.f[i, :Tb], b.f[i, :Tb]) and torch.equal(r.g[i, :Ub + 1], b.g[i, :Ub + 1])
        assert torch.equal(r.labels[i, :Ub], b.labels[i, :Ub])
        if Tb < b.f.shape[1]:
            assert not torch.equal(r.f[i, Tb:], b.f[i, Tb:])
    assert r.W_o is b.W_o


@pytest.mark.parametrize("S", [2, 4, 8, 32])
@pytest.mark.parametrize("name", ["short", "medium"])
def test_diagonal_bounds_are_valid_bands(name, S):
    b = synth.workload(name)
    s = synth.diagonal_bounds(b.T_len, b.U_len, b.f.shape[1], S)
    assert s.dtype == torch.int32 and s.shape == (b.f.shape[0], b.f.shape[1])
    assert oracle.validate_bounds(S, s.numpy(), b.T_len.numpy(), b.U_len.numpy()) == 0


def test_duration_head():
    b = synth.workload("medium")
    W_d, b_d = synth.duration_head(b, len(synth.TDT_DURATIONS), seed=5)
    H = b.W_o.shape[1]
    assert W_d.shape == (5, H) and b_d.shape == (5,) and W_d.dtype == torch.bfloat16
    assert synth.TDT_DURATIONS[:2] == (0, 1)
    W_d2, _ = synth.duration_head(b, 5, seed=5)
    assert torch.equal(W_d, W_d2)


def test_no_method_arithmetic_in_the_generator():
    """The generator module imports neither the oracle nor the CUDA binding."""
    src = open(os.path.join(os.path.dirname(synth.__file__), "synth.py")).read()
    imports = [ln.strip() for ln in src.splitlines() if ln.strip().startswith(("import ", "from "))]
    assert all("oracle" not in ln and "frnnt" not in ln for ln in imports), imports
