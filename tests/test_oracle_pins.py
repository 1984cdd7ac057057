"""Pins for the fp64 oracle against facts that do not come from the oracle.

Each test ties one part of the oracle to something independent of its code:
brute-force enumeration of alignments, closed forms at zero / constant
logits, special cases that reduce to a library routine, finite differences,
flow-conservation invariants, and an external transducer-loss implementation
(torchaudio's CPU ``rnnt_loss``) as a cross-check.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from rnn_joint_network_02_b200 import synth


def _small_batch(B=2, T=5, U=3, D_enc=3, D_pred=4, H=5, V=6, seed=0, bias=0.5, T_range=None,
                 U_range=None):
    return synth.make(B=B, T=T, U=U, D_enc=D_enc, D_pred=D_pred, H=H, V=V, dtype="f32",
                      seed=seed, T_range=T_range or (max(1, T - 2), T),
                      U_range=U_range or (0, U), U_rule="range", bias_std=bias)


def _run(batch, w=None, keep=True, **kw):
    f, g, W_f, W_g, W_o, b_o = batch.float64()
    return oracle.fwd_bwd(f.numpy(), g.numpy(), W_f.numpy(), W_g.numpy(), W_o.numpy(), b_o.numpy(),
                          batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(),
                          grad_loss=w, keep_lattice=keep, blank=batch.blank, **kw)


def _log_probs_torch(batch, b):
    """Per-cell log-softmax computed with torch (float64), for the brute force."""
    f, g, W_f, W_g, W_o, b_o = batch.float64()
    Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
    F = f[b, :Tb] @ W_f
    G = g[b, :Ub + 1] @ W_g
    z = torch.tanh(F[:, None, :] + G[None, :, :]) @ W_o.T + b_o
    return torch.log_softmax(z, dim=-1).numpy()


def _brute_force_logp(logp, labels, Tb, Ub, blank=0):
    """log of the total probability over every alignment, by enumeration:
    every placement of the Ub label emissions among the Tb-1+Ub emissions
    that precede the final blank."""
    total = []
    n = Tb - 1 + Ub
    for pos in itertools.combinations(range(n), Ub):
        pos = set(pos)
        t = u = 0
        s = 0.0
        for i in range(n):
            if i in pos:
                s += logp[t, u, labels[u]]
                u += 1
            else:
                s += logp[t, u, blank]
                t += 1
        assert t == Tb - 1 and u == Ub
        s += logp[t, u, blank]
        total.append(s)
    m = max(total)
    return m + math.log(sum(math.exp(x - m) for x in total))


# ---------------------------------------------------------------- brute force

def test_brute_force_tiny_workload():
    batch = synth.workload("tiny")
    res = _run(batch)
    assert res.status == 0
    for b in range(batch.f.shape[0]):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        assert (Tb, Ub) == (12, 5)          # C(16, 5) = 4368 alignments
        lp = _log_probs_torch(batch, b)
        ref = _brute_force_logp(lp, batch.labels[b].tolist(), Tb, Ub)
        assert abs(-res.loss[b] - ref) <= 1e-12 * abs(ref)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_random_shapes(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(1, 7))
    U = int(rng.integers(0, 5))
    V = int(rng.integers(2, 7))
    batch = _small_batch(B=3, T=T, U=U, V=V, seed=100 + seed, T_range=(1, T), U_range=(0, U))
    res = _run(batch)
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        lp = _log_probs_torch(batch, b)
        ref = _brute_force_logp(lp, batch.labels[b].tolist(), Tb, Ub)
        assert abs(-res.loss[b] - ref) <= 1e-11 * max(1.0, abs(ref))


# ------------------------------------------------------------ closed forms

@pytest.mark.parametrize("Tb,Ub,V", [(1, 0, 2), (1, 3, 5), (4, 0, 7), (3, 2, 4), (12, 5, 8),
                                     (40, 9, 13), (200, 40, 1024)])
def test_zero_logits_closed_form(Tb, Ub, V):
    """W_o = 0, b_o = 0: every alignment has probability V^-(Tb+Ub), and
    there are C(Tb+Ub-1, Ub) of them."""
    U = max(Ub, 1)
    batch = synth.make(B=1, T=Tb, U=U, D_enc=3, D_pred=3, H=4, V=V, dtype="f32", seed=7,
                       T_range=(Tb, Tb), U_range=(Ub, Ub))
    batch.W_o.zero_()
    batch.b_o.zero_()
    res = _run(batch, keep=False)
    expect = (Tb + Ub) * math.log(V) - math.log(math.comb(Tb + Ub - 1, Ub))
    assert abs(res.loss[0] - expect) <= 1e-12 * expect + 1e-12


def test_zero_logits_bias_gradient_closed_form():
    """At zero logits every alignment visits Tb+Ub cells, emits Tb blanks and
    each label once, so db_o[k] = sum_b w_b ((Tb+Ub)/V - Tb [k=blank] - #{u: y_u=k}).
    With W_o = 0 the hidden gradient vanishes, so f, g, W_f, W_g get exactly 0."""
    batch = _small_batch(B=3, T=7, U=4, V=6, seed=11)
    batch.W_o.zero_()
    batch.b_o.zero_()
    w = np.array([1.0, 0.5, -2.0])
    res = _run(batch, w=w, keep=False)
    V = 6
    expect = np.zeros(V)
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        row = np.full(V, (Tb + Ub) / V)
        row[0] -= Tb
        for u in range(Ub):
            row[int(batch.labels[b, u])] -= 1
        expect += w[b] * row
    np.testing.assert_allclose(res.db_o, expect, rtol=0, atol=1e-12)
    for name in ("df", "dg", "dW_f", "dW_g"):
        assert np.abs(getattr(res, name)).max() == 0.0


def test_constant_logits_bias_closed_form():
    """W_o = 0, b_o != 0: z = b_o in every cell, so every alignment has the
    probability p_blank^Tb * prod_u p_{y_u} (p = softmax(b_o)), and there are
    C(Tb+Ub-1, Ub) alignments."""
    batch = _small_batch(B=2, T=6, U=3, V=5, seed=12, bias=1.0)
    batch.W_o.zero_()
    res = _run(batch, keep=False)
    b_o = batch.b_o.double()
    logp = torch.log_softmax(b_o, 0).numpy()
    for b in range(2):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        lp = Tb * logp[0] + sum(logp[int(batch.labels[b, u])] for u in range(Ub))
        lp += math.log(math.comb(Tb + Ub - 1, Ub))
        assert abs(res.loss[b] + lp) <= 1e-12 * abs(lp)


# ------------------------------------------- joint special cases (library)

def _perm_matrix(n, perm):
    P = torch.zeros(n, n)
    for i, j in enumerate(perm):
        P[i, j] = 1.0
    return P


def test_joint_orientation_encoder_only():
    """W_g = 0, W_f and W_o permutation matrices: F = f W_f picks columns of f,
    z = W_o h picks rows of h; compare with torch.log_softmax on the gathered
    tanh(f).  A transposed W_f or W_o, a missing tanh or a u-dependence fails."""
    H = V = 6
    batch = synth.make(B=1, T=4, U=2, D_enc=H, D_pred=3, H=H, V=V, dtype="f32", seed=3,
                       T_range=(4, 4), U_range=(2, 2))
    sig = [2, 0, 5, 1, 3, 4]          # W_f[i, sig[i]] = 1  ->  F[:, sig[i]] = f[:, i]
    pi = [4, 1, 0, 5, 2, 3]           # W_o[k, pi[k]] = 1   ->  z[k] = h[pi[k]]
    batch.W_f.copy_(_perm_matrix(H, sig))
    batch.W_g.zero_()
    batch.W_o.copy_(_perm_matrix(V, pi))
    batch.b_o.zero_()
    res = _run(batch)
    lat = res.lattice[0]
    f = batch.f[0].double()
    F = torch.empty_like(f)
    for i, j in enumerate(sig):
        F[:, j] = f[:, i]
    z = torch.tanh(F)[:, pi]
    logp = torch.log_softmax(z, -1).numpy()
    for u in range(3):
        np.testing.assert_allclose(lat.blank_lp[:, u], logp[:, 0], rtol=0, atol=1e-13)
        if u < 2:
            y = int(batch.labels[0, u])
            np.testing.assert_allclose(lat.label_lp[:, u], logp[:, y], rtol=0, atol=1e-13)


def test_joint_orientation_prediction_only():
    """W_f = 0, W_g a permutation, W_o = I: z depends on u only."""
    H = V = 5
    batch = synth.make(B=1, T=3, U=4, D_enc=2, D_pred=H, H=H, V=V, dtype="f32", seed=4,
                       T_range=(3, 3), U_range=(4, 4))
    sig = [3, 4, 0, 2, 1]
    batch.W_f.zero_()
    batch.W_g.copy_(_perm_matrix(H, sig))
    batch.W_o.copy_(torch.eye(V))
    batch.b_o.zero_()
    res = _run(batch)
    lat = res.lattice[0]
    g = batch.g[0].double()
    G = torch.empty_like(g)
    for i, j in enumerate(sig):
        G[:, j] = g[:, i]
    logp = torch.log_softmax(torch.tanh(G), -1).numpy()     # [U+1, V]
    for t in range(3):
        np.testing.assert_allclose(lat.blank_lp[t], logp[:, 0], rtol=0, atol=1e-13)


# --------------------------------------------------------- special cases

def test_no_labels_reduces_to_blank_sum():
    batch = _small_batch(B=2, T=6, U=3, seed=21, U_range=(0, 0))
    res = _run(batch)
    for b in range(2):
        lat = res.lattice[b]
        assert abs(res.loss[b] + lat.blank_lp[:, 0].sum()) <= 1e-12 * abs(res.loss[b])


def test_single_frame_reduces_to_label_sum():
    batch = _small_batch(B=2, T=1, U=4, seed=22, T_range=(1, 1), U_range=(1, 4))
    res = _run(batch)
    for b in range(2):
        lat = res.lattice[b]
        Ub = int(batch.U_len[b])
        expect = -(lat.label_lp[0, :Ub].sum() + lat.blank_lp[0, Ub])
        assert abs(res.loss[b] - expect) <= 1e-12 * abs(expect)


# ------------------------------------------------------------ invariants

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_flow_invariants(seed):
    batch = _small_batch(B=3, T=9, U=5, V=7, seed=30 + seed)
    res = _run(batch)
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        lat = res.lattice[b]
        # exactly one blank leaves every frame, each label is emitted once
        np.testing.assert_allclose(lat.bpost.sum(axis=1), np.ones(Tb), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lat.lpost[:, :Ub].sum(axis=0), np.ones(Ub), rtol=0, atol=1e-12)
        assert abs(lat.beta[0, 0] - lat.log_p) <= 1e-12 * abs(lat.log_p)
        assert res.loss[b] >= 0
        np.testing.assert_allclose(lat.dz.sum(axis=-1), 0.0, atol=1e-12)
    assert abs(res.db_o.sum()) <= 1e-12
    np.testing.assert_allclose(res.dW_o.sum(axis=0), 0.0, atol=1e-12)


# ---------------------------------------------------- finite differences

def _total_loss(batch, arrays, w):
    f, g, W_f, W_g, W_o, b_o = arrays
    losses = oracle.loss_only(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                              batch.U_len.numpy(), blank=batch.blank)
    return float((w * losses).sum())


def test_finite_differences_every_entry():
    batch = _small_batch(B=2, T=4, U=2, D_enc=3, D_pred=2, H=4, V=5, seed=40, bias=0.7)
    w = np.array([0.7, -1.3])
    res = _run(batch, w=w, keep=False)
    arrays = [t.numpy().copy() for t in batch.float64()]
    grads = [res.df, res.dg, res.dW_f, res.dW_g, res.dW_o, res.db_o]
    for idx, (x, gx) in enumerate(zip(arrays, grads)):
        flat = x.reshape(-1)
        for i in range(flat.size):
            step = 1e-6 * max(1.0, abs(flat[i]))
            old = flat[i]
            flat[i] = old + step
            lp = _total_loss(batch, arrays, w)
            flat[i] = old - step
            lm = _total_loss(batch, arrays, w)
            flat[i] = old
            fd = (lp - lm) / (2 * step)
            an = gx.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, i, fd, an)


def test_finite_differences_directional():
    batch = _small_batch(B=2, T=7, U=4, D_enc=6, D_pred=5, H=8, V=9, seed=41, bias=0.3)
    w = np.array([1.0, 2.0])
    res = _run(batch, w=w, keep=False)
    arrays = [t.numpy().copy() for t in batch.float64()]
    grads = [res.df, res.dg, res.dW_f, res.dW_g, res.dW_o, res.db_o]
    rng = np.random.default_rng(5)
    for idx in range(6):
        d = rng.standard_normal(arrays[idx].shape)
        if idx == 0:   # only valid frames of f matter
            for b in range(2):
                d[b, int(batch.T_len[b]):] = 0
        if idx == 1:
            for b in range(2):
                d[b, int(batch.U_len[b]) + 1:] = 0
        eps = 1e-6
        plus = [a.copy() for a in arrays]
        minus = [a.copy() for a in arrays]
        plus[idx] += eps * d
        minus[idx] -= eps * d
        fd = (_total_loss(batch, plus, w) - _total_loss(batch, minus, w)) / (2 * eps)
        an = float((grads[idx] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, fd, an)


def test_padding_rows_have_zero_gradient():
    batch = _small_batch(B=3, T=8, U=4, seed=42)
    res = _run(batch, keep=False)
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        assert np.abs(res.df[b, Tb:]).max(initial=0) == 0
        assert np.abs(res.dg[b, Ub + 1:]).max(initial=0) == 0


# ------------------------------------------------- external cross-check

def test_torchaudio_rnnt_loss_crosscheck():
    """torchaudio's CPU transducer loss on the oracle's logits: losses and the
    gradient with respect to the logits agree with the oracle (torchaudio works
    in float32)."""
    AF = pytest.importorskip("torchaudio.functional")
    batch = _small_batch(B=3, T=9, U=4, V=7, seed=50, bias=0.4, T_range=(5, 9), U_range=(1, 4))
    res = _run(batch)
    f, g, W_f, W_g, W_o, b_o = batch.float64()
    B = 3
    T = int(batch.T_len.max())          # torchaudio wants the logits sized to the longest
    U = int(batch.U_len.max())
    logits = torch.zeros(B, T, U + 1, 7, dtype=torch.float32)
    for b in range(B):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        _, z = oracle.joint_logits((f[b, :Tb] @ W_f).numpy(), (g[b, :Ub + 1] @ W_g).numpy(),
                                   W_o.numpy(), b_o.numpy())
        logits[b, :Tb, :Ub + 1] = torch.from_numpy(z).float()
    logits.requires_grad_(True)
    loss = AF.rnnt_loss(logits, batch.labels[:, :U].contiguous(), batch.T_len, batch.U_len, blank=0, reduction="none")
    loss.sum().backward()
    np.testing.assert_allclose(loss.detach().numpy(), res.loss, rtol=1e-5)
    for b in range(B):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        np.testing.assert_allclose(logits.grad[b, :Tb, :Ub + 1].numpy(), res.lattice[b].dz,
                                   rtol=0, atol=2e-5)


# ------------------------------------------------------------ validation

def test_validate_bits():
    labels = np.array([[1, 2, 0], [3, 9, 1]])
    assert oracle.validate(5, 3, 8, 0, labels, [5, 5], [2, 1]) == 0
    assert oracle.validate(5, 3, 8, 0, labels, [5, 5], [3, 1]) == oracle.STATUS_LABEL     # blank
    assert oracle.validate(5, 3, 8, 0, labels, [5, 5], [2, 2]) == oracle.STATUS_LABEL     # 9 >= V
    assert oracle.validate(5, 3, 8, 0, labels, [0, 5], [2, 1]) == oracle.STATUS_LENGTH
    assert oracle.validate(5, 3, 8, 0, labels, [6, 5], [2, 1]) == oracle.STATUS_LENGTH
    assert oracle.validate(5, 3, 8, 0, labels, [5, 5], [4, 1]) == oracle.STATUS_LENGTH
    assert oracle.validate(5, 3, 8, 0, labels, [5, 5], [-1, 2]) == (oracle.STATUS_LENGTH
                                                                   | oracle.STATUS_LABEL)


def test_golden_file_is_the_oracles_output():
    """tests/golden/tiny_oracle.json (read by the GPU parity test) is exactly
    what its generating script's oracle call produces today."""
    import json
    import os
    gold = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_oracle.json")))
    batch = synth.workload("tiny")
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    res = oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy())
    assert gold["status"] == res.status == 0
    np.testing.assert_allclose(gold["loss"], res.loss, rtol=1e-12, atol=0)
    for name in ("df", "dg", "dW_f", "dW_g", "dW_o", "db_o"):
        np.testing.assert_allclose(gold[name], getattr(res, name).reshape(-1), rtol=1e-10, atol=1e-14)
