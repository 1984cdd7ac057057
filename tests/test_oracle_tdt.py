"""Pins of the oracle's token-and-duration transducer (TDT) loss: brute-force
summation over every alignment, a generating-function count for zero logits,
invariants of the edge posteriors, and finite differences of the gradients."""

import math

import numpy as np
import pytest
import torch

import oracle
from rnn_joint_network_02_b200 import synth

DSETS = [(0, 1), (0, 1, 2), (0, 1, 2, 3, 4), (0, 1, 3)]


def _batch(B=2, T=5, U=3, H=5, V=6, seed=0, bias=0.5):
    return synth.make(B=B, T=T, U=U, D_enc=3, D_pred=4, H=H, V=V, dtype="f32", seed=seed,
                      T_range=(max(1, T - 2), T), U_range=(0, U), U_rule="range", bias_std=bias)


def _head(batch, n_dur, seed=5, bias=0.5):
    W_d, b_d = synth.duration_head(batch, n_dur, seed=seed, bias_std=bias)
    return W_d.double(), b_d.double()


def _run(batch, W_d, b_d, D, w=None, keep=True):
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    return oracle.tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d.numpy(), b_d.numpy(), batch.labels.numpy(),
                              batch.T_len.numpy(), batch.U_len.numpy(), D, grad_loss=w, blank=batch.blank,
                              keep_lattice=keep)


def _log_probs(batch, W_d, b_d, b):
    """Token and duration log-softmax per cell with torch (float64), independent of the oracle."""
    f, g, W_f, W_g, W_o, b_o = batch.float64()
    Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
    h = torch.tanh((f[b, :Tb] @ W_f)[:, None, :] + (g[b, :Ub + 1] @ W_g)[None, :, :])
    return (torch.log_softmax(h @ W_o.T + b_o, dim=-1).numpy(),
            torch.log_softmax(h @ W_d.T + b_d, dim=-1).numpy())


def _alignment_scores(lp, ld, labels, D, Tb, Ub, blank=0):
    """log-weight of every alignment, by depth-first enumeration of the emissions."""
    out = []

    def walk(t, u, s):
        for i, d in enumerate(D):
            if d >= 1:
                w = s + lp[t, u, blank] + ld[t, u, i]
                if t + d < Tb:
                    walk(t + d, u, w)
                elif t + d == Tb and u == Ub:
                    out.append(w)
            if u < Ub and t + d < Tb:
                walk(t + d, u + 1, s + lp[t, u, labels[u]] + ld[t, u, i])

    walk(0, 0, 0.0)
    return np.array(out)


@pytest.mark.parametrize("D", DSETS)
@pytest.mark.parametrize("seed", range(3))
def test_brute_force_loss(D, seed):
    """loss = -log of the summed weight of every alignment, enumerated path by path."""
    batch = _batch(seed=seed, T=6 if len(D) < 5 else 5)
    W_d, b_d = _head(batch, len(D), seed=seed + 11)
    res = _run(batch, W_d, b_d, D)
    assert res.status == 0
    for b in range(batch.f.shape[0]):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        lp, ld = _log_probs(batch, W_d, b_d, b)
        scores = _alignment_scores(lp, ld, [int(x) for x in batch.labels[b]], D, Tb, Ub)
        assert len(scores) > 0
        ref = -math.log(np.exp(scores).sum())
        assert abs(res.loss[b] - ref) <= 1e-12 * max(1.0, abs(ref)), (b, res.loss[b], ref)


def _count_alignments_by_length(Tb, Ub, D):
    """{number of emissions: number of alignments}, from generating functions:
    Ub labels and k >= 1 blanks (the last emission a blank), the labels placed
    among the first Ub + k - 1 emissions, label durations from D and blank
    durations from D minus {0}, all durations summing to Tb."""
    def poly_pow(p, n, deg):
        out = [1] + [0] * deg
        for _ in range(n):
            nxt = [0] * (deg + 1)
            for i, a in enumerate(out):
                if a:
                    for j, c in enumerate(p):
                        if c and i + j <= deg:
                            nxt[i + j] += a * c
            out = nxt
        return out

    lab = [0] * (Tb + 1)
    blk = [0] * (Tb + 1)
    for d in D:
        if d <= Tb:
            lab[d] += 1
            if d >= 1:
                blk[d] += 1
    counts = {}
    lab_pow = poly_pow(lab, Ub, Tb)
    for k in range(1, Tb + 1):
        c = 0
        blk_pow = poly_pow(blk, k, Tb)
        for i in range(Tb + 1):
            c += lab_pow[i] * blk_pow[Tb - i]
        if c:
            counts[Ub + k] = math.comb(Ub + k - 1, Ub) * c
    return counts


@pytest.mark.parametrize("D", DSETS + [(0, 1, 2, 4, 8)])
@pytest.mark.parametrize("Tb,Ub", [(1, 0), (1, 3), (4, 2), (7, 3), (9, 5)])
def test_zero_logits_closed_form(D, Tb, Ub):
    """W_o = b_o = W_d = b_d = 0: every emission has weight 1/(V |D|), so
    P = sum_n count(n) (V |D|)^-n with the alignment counts from generating functions."""
    V = 5
    batch = synth.make(B=1, T=Tb, U=max(Ub, 1), D_enc=3, D_pred=3, H=4, V=V, dtype="f32", seed=3,
                       T_range=(Tb, Tb), U_range=(Ub, Ub), U_rule="range")
    W_d = torch.zeros(len(D), 4, dtype=torch.float64)
    b_d = torch.zeros(len(D), dtype=torch.float64)
    batch.W_o.zero_()
    res = _run(batch, W_d, b_d, D)
    counts = _count_alignments_by_length(Tb, Ub, D)
    p = sum(c * float(V * len(D)) ** -n for n, c in counts.items())
    assert abs(res.loss[0] + math.log(p)) <= 1e-12 * max(1.0, abs(math.log(p)))


@pytest.mark.parametrize("D", DSETS)
def test_posterior_invariants(D):
    """Per utterance: expected durations sum to T_len, every label is emitted
    once, each cell's gradient rows sum to zero (so do db_o and db_d), and loss >= 0."""
    batch = _batch(seed=7, T=7, U=4, V=7)
    W_d, b_d = _head(batch, len(D), seed=3)
    res = _run(batch, W_d, b_d, D)
    Dv = np.array(D, dtype=np.float64)
    for b, lat in res.lattice.items():
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        assert abs(((lat.pb + lat.pl) * Dv).sum() - Tb) < 1e-9
        for u in range(Ub):
            assert abs(lat.pl[:, u].sum() - 1.0) < 1e-9
        assert lat.pl[:, Ub].sum() == 0.0
        assert res.loss[b] >= 0
    assert abs(res.db_o.sum()) < 1e-9 and abs(res.db_d.sum()) < 1e-9
    assert np.abs(res.dW_o.sum(axis=0)).max() < 1e-9 and np.abs(res.dW_d.sum(axis=0)).max() < 1e-9


def test_duration_set_rules():
    assert oracle.validate_durations((0, 1))
    assert oracle.validate_durations((0, 1, 2, 4, 8))
    for bad in [(1, 2), (0,), (0, 2), (0, 1, 1), (0, 1, 3, 2), ()]:
        assert not oracle.validate_durations(bad)
    batch = _batch()
    W_d, b_d = _head(batch, 2)
    assert _run(batch, W_d, b_d, (0, 2)).status == oracle.STATUS_DURATIONS


@pytest.mark.parametrize("D", [(0, 1, 2), (0, 1, 3)])
def test_gradients_finite_differences(D):
    """Directional derivatives of sum_b w_b loss_b along random directions, for
    all eight parameter tensors, against fp64 central differences."""
    batch = _batch(seed=4, T=5, U=3, V=6)
    W_d, b_d = _head(batch, len(D), seed=9)
    w = np.array([0.7, -1.3])
    res = _run(batch, W_d, b_d, D, w=w, keep=False)
    base = [t.numpy().copy() for t in batch.float64()] + [W_d.numpy().copy(), b_d.numpy().copy()]
    grads = [res.df, res.dg, res.dW_f, res.dW_g, res.dW_o, res.db_o, res.dW_d, res.db_d]
    rng = np.random.default_rng(0)
    args = (batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(), D)

    def total(params):
        return float(w @ oracle.tdt_loss_only(*params, *args))

    for k in range(len(base)):
        direc = rng.standard_normal(base[k].shape)
        if k == 0:      # frames past T_len do not exist for the loss
            for b in range(2):
                direc[b, int(batch.T_len[b]):] = 0
        if k == 1:
            for b in range(2):
                direc[b, int(batch.U_len[b]) + 1:] = 0
        eps = 1e-6
        plus = [p.copy() for p in base]
        minus = [p.copy() for p in base]
        plus[k] += eps * direc
        minus[k] -= eps * direc
        fd = (total(plus) - total(minus)) / (2 * eps)
        an = float((grads[k] * direc).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (k, fd, an)
