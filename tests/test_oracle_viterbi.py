"""Pins of the oracle's maximum-approximation (Viterbi) loss: brute-force
maximisation over every alignment, the one-alignment special cases, the tie
rule, and finite differences of the loss away from ties."""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from rnn_joint_network_02_b200 import synth


def _batch(B=2, T=5, U=3, D_enc=3, D_pred=4, H=5, V=6, seed=0, bias=0.5, T_range=None, U_range=None):
    return synth.make(B=B, T=T, U=U, D_enc=D_enc, D_pred=D_pred, H=H, V=V, dtype="f32", seed=seed,
                      T_range=T_range or (max(1, T - 2), T), U_range=U_range or (0, U), U_rule="range",
                      bias_std=bias)


def _run(batch, w=None, loss="viterbi", keep=True):
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    return oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                          batch.U_len.numpy(), grad_loss=w, blank=batch.blank, keep_lattice=keep, loss=loss)


def _log_probs(batch, b):
    """Per-cell log-softmax with torch (float64), independent of the oracle's joint."""
    f, g, W_f, W_g, W_o, b_o = batch.float64()
    Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
    z = torch.tanh((f[b, :Tb] @ W_f)[:, None, :] + (g[b, :Ub + 1] @ W_g)[None, :, :]) @ W_o.T + b_o
    return torch.log_softmax(z, dim=-1).numpy()


def _alignments(Tb, Ub):
    """Every alignment as its list of edges ((t, u), 'b' | 'l'), final blank included."""
    n = Tb - 1 + Ub
    for pos in itertools.combinations(range(n), Ub):
        pos = set(pos)
        t = u = 0
        edges = []
        for i in range(n):
            if i in pos:
                edges.append(((t, u), "l"))
                u += 1
            else:
                edges.append(((t, u), "b"))
                t += 1
        edges.append(((t, u), "b"))
        yield edges


def _score(lp, labels, edges, blank=0):
    return sum(lp[t, u, blank] if kind == "b" else lp[t, u, labels[u]] for (t, u), kind in edges)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_best_alignment(seed):
    """-loss is the largest alignment log-probability, and the oracle's
    bpost / lpost are exactly that alignment's edges."""
    rng = np.random.default_rng(seed)
    T, U, V = int(rng.integers(1, 7)), int(rng.integers(0, 5)), int(rng.integers(2, 7))
    batch = _batch(B=3, T=T, U=U, V=V, seed=300 + seed, T_range=(1, T), U_range=(0, U))
    res = _run(batch)
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        lp = _log_probs(batch, b)
        labels = batch.labels[b].tolist()
        scored = [(_score(lp, labels, e), e) for e in _alignments(Tb, Ub)]
        best, edges = max(scored, key=lambda x: x[0])
        assert abs(-res.loss[b] - best) <= 1e-11 * max(1.0, abs(best))
        lat = res.lattice[b]
        bp = np.zeros((Tb, Ub + 1))
        lq = np.zeros((Tb, Ub + 1))
        for (t, u), kind in edges:
            (bp if kind == "b" else lq)[t, u] = 1.0
        np.testing.assert_array_equal(lat.bpost, bp)
        np.testing.assert_array_equal(lat.lpost, lq)


def test_tiny_workload_brute_force():
    batch = synth.workload("tiny")
    res = _run(batch)
    for b in range(batch.f.shape[0]):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        lp = _log_probs(batch, b)
        labels = batch.labels[b].tolist()
        best = max(_score(lp, labels, e) for e in _alignments(Tb, Ub))
        assert abs(-res.loss[b] - best) <= 1e-12 * abs(best)


@pytest.mark.parametrize("Tb,Ub", [(1, 0), (1, 4), (6, 0)])
def test_single_alignment_equals_marginal(Tb, Ub):
    """With no labels, or a single frame, there is one alignment: both losses
    and all gradients coincide."""
    batch = _batch(B=1, T=Tb, U=max(Ub, 1), V=7, seed=11, T_range=(Tb, Tb), U_range=(Ub, Ub))
    v = _run(batch, w=np.array([1.7]), keep=False)
    m = _run(batch, w=np.array([1.7]), loss="marginal", keep=False)
    np.testing.assert_allclose(v.loss, m.loss, rtol=1e-13)
    for k in ("df", "dg", "dW_f", "dW_g", "dW_o", "db_o"):
        np.testing.assert_allclose(getattr(v, k), getattr(m, k), rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("Tb,Ub,V", [(1, 3, 5), (4, 2, 7), (12, 5, 8)])
def test_zero_logits_tie_rule(Tb, Ub, V):
    """W_o = 0, b_o = 0: every alignment scores -(Tb+Ub) ln V, so every
    decision is a tie; ties go to the blank edge, which makes the chosen
    alignment emit all labels at frame 0 and then the blanks."""
    batch = synth.make(B=1, T=Tb, U=max(Ub, 1), D_enc=3, D_pred=3, H=4, V=V, dtype="f32", seed=8,
                       T_range=(Tb, Tb), U_range=(Ub, Ub))
    batch.W_o.zero_()
    batch.b_o.zero_()
    res = _run(batch)
    assert abs(res.loss[0] - (Tb + Ub) * math.log(V)) <= 1e-12 * (Tb + Ub) * math.log(V)
    lat = res.lattice[0]
    lq = np.zeros((Tb, Ub + 1))
    lq[0, :Ub] = 1.0
    bp = np.zeros((Tb, Ub + 1))
    bp[:, Ub] = 1.0
    np.testing.assert_array_equal(lat.lpost, lq)
    np.testing.assert_array_equal(lat.bpost, bp)


def _total(batch, arrays, w):
    f, g, W_f, W_g, W_o, b_o = arrays
    losses = oracle.loss_only(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                              batch.U_len.numpy(), blank=batch.blank, loss="viterbi")
    return float((w * losses).sum())


def test_finite_differences_directional():
    """Away from ties the loss is the log-probability of one fixed alignment,
    so central differences along random directions match the gradients."""
    batch = _batch(B=2, T=7, U=4, D_enc=6, D_pred=5, H=8, V=9, seed=61, bias=0.3)
    w = np.array([1.0, -0.6])
    res = _run(batch, w=w, keep=False)
    arrays = [t.numpy().copy() for t in batch.float64()]
    grads = [res.df, res.dg, res.dW_f, res.dW_g, res.dW_o, res.db_o]
    rng = np.random.default_rng(9)
    for idx in range(6):
        d = rng.standard_normal(arrays[idx].shape)
        if idx == 0:
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
        fd = (_total(batch, plus, w) - _total(batch, minus, w)) / (2 * eps)
        an = float((grads[idx] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, fd, an)


def test_viterbi_loss_bounds_marginal():
    """The best alignment's probability is at most the total, and at least the
    total divided by the number of alignments."""
    batch = _batch(B=3, T=6, U=3, V=5, seed=71)
    v = _run(batch, keep=False)
    m = _run(batch, loss="marginal", keep=False)
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        n = math.comb(Tb - 1 + Ub, Ub)
        assert m.loss[b] <= v.loss[b] + 1e-12
        assert v.loss[b] <= m.loss[b] + math.log(n) + 1e-12
