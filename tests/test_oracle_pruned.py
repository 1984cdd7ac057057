"""Pins of the oracle's pruned (banded) lattice: the full band reproduces the
unpruned result, brute force over the alignments that stay inside the band,
finite differences, and the integer bounds checks."""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from rnn_joint_network_02_b200 import synth


def _batch(B=3, T=6, U=4, D_enc=3, D_pred=4, H=5, V=6, seed=0, bias=0.4):
    return synth.make(B=B, T=T, U=U, D_enc=D_enc, D_pred=D_pred, H=H, V=V, dtype="f32", seed=seed,
                      T_range=(2, T), U_range=(0, U), U_rule="range", bias_std=bias)


def _run(batch, bounds=None, S=0, w=None, loss="marginal"):
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    return oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                          batch.U_len.numpy(), grad_loss=w, blank=batch.blank, loss=loss,
                          bounds=None if bounds is None else np.asarray(bounds), S=S)


def _fit_lengths(batch, S):
    """Shorten U_len where no band of width S can reach it ((T_len-1)(S-1) + S-1 < U_len)."""
    for b in range(batch.f.shape[0]):
        Tb = int(batch.T_len[b])
        batch.U_len[b] = min(int(batch.U_len[b]), (Tb - 1) * (S - 1) + S - 1)
    return batch


def _random_bounds(batch, S, rng):
    """Random valid bounds: s0 = 0, steps of 0..S-1, kept reachable to U_len."""
    _fit_lengths(batch, S)
    B, T = batch.f.shape[:2]
    out = np.zeros((B, T), dtype=np.int64)
    for b in range(B):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        s = 0
        for t in range(Tb):
            lo = max(s, Ub - S + 1 - (Tb - 1 - t) * (S - 1))   # the end must stay reachable
            hi = min(s + S - 1, Ub) if t > 0 else 0
            s = int(rng.integers(max(lo, 0) if t > 0 else 0, max(hi, max(lo, 0)) + 1)) if t > 0 else 0
            out[b, t] = s
        out[b, Tb:] = out[b, Tb - 1]
    return out


def _log_probs(batch, b):
    f, g, W_f, W_g, W_o, b_o = batch.float64()
    Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
    z = torch.tanh((f[b, :Tb] @ W_f)[:, None, :] + (g[b, :Ub + 1] @ W_g)[None, :, :]) @ W_o.T + b_o
    return torch.log_softmax(z, dim=-1).numpy()


def _band_alignment_scores(lp, labels, Tb, Ub, s, S, blank=0):
    """Log-probability of every alignment whose cells all lie in the band."""
    out = []
    n = Tb - 1 + Ub
    for pos in itertools.combinations(range(n), Ub):
        pos = set(pos)
        t = u = 0
        sc = 0.0
        ok = s[0] <= 0 < s[0] + S
        for i in range(n):
            if i in pos:
                sc += lp[t, u, labels[u]]
                u += 1
            else:
                sc += lp[t, u, blank]
                t += 1
            ok = ok and s[t] <= u < s[t] + S
        sc += lp[t, u, blank]
        if ok:
            out.append(sc)
    return out


def test_full_band_equals_unpruned():
    batch = _batch(seed=1)
    B, T = batch.f.shape[:2]
    U = batch.g.shape[1] - 1
    bounds = np.zeros((B, T), dtype=np.int64)
    w = np.array([1.0, -0.5, 2.0])
    for loss in ("marginal", "viterbi"):
        p = _run(batch, bounds, U + 1, w=w, loss=loss)
        full = _run(batch, w=w, loss=loss)
        np.testing.assert_allclose(p.loss, full.loss, rtol=1e-13)
        for k in ("df", "dg", "dW_f", "dW_g", "dW_o", "db_o"):
            np.testing.assert_allclose(getattr(p, k), getattr(full, k), rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("S", [2, 3, 4])
def test_brute_force_band(seed, S):
    rng = np.random.default_rng(seed)
    batch = _batch(B=3, T=6, U=4, V=int(rng.integers(2, 7)), seed=400 + seed)
    bounds = _random_bounds(batch, S, rng)
    assert oracle.validate_bounds(S, bounds, batch.T_len.numpy(), batch.U_len.numpy()) == 0
    m = _run(batch, bounds, S)
    v = _run(batch, bounds, S, loss="viterbi")
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        scores = _band_alignment_scores(_log_probs(batch, b), batch.labels[b].tolist(), Tb, Ub,
                                        [int(x) for x in bounds[b]], S)
        assert scores, "valid bounds leave at least one alignment"
        mx = max(scores)
        ref = mx + math.log(sum(math.exp(x - mx) for x in scores))
        assert abs(-m.loss[b] - ref) <= 1e-11 * max(1.0, abs(ref))
        assert abs(-v.loss[b] - mx) <= 1e-11 * max(1.0, abs(mx))


def test_pruned_loss_not_below_full():
    batch = _batch(seed=5)
    bounds = _random_bounds(batch, 2, np.random.default_rng(3))
    p = _run(batch, bounds, 2)
    full = _run(batch)
    assert np.all(p.loss >= full.loss - 1e-12)


def test_finite_differences_directional():
    batch = _batch(B=2, T=7, U=4, D_enc=6, D_pred=5, H=8, V=9, seed=81, bias=0.3)
    S = 3
    bounds = _random_bounds(batch, S, np.random.default_rng(4))
    w = np.array([1.0, 0.7])
    res = _run(batch, bounds, S, w=w)
    arrays = [t.numpy().copy() for t in batch.float64()]
    grads = [res.df, res.dg, res.dW_f, res.dW_g, res.dW_o, res.db_o]

    def total(arr):
        f, g, W_f, W_g, W_o, b_o = arr
        losses = oracle.loss_only(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                                  batch.U_len.numpy(), blank=batch.blank, bounds=bounds, S=S)
        return float((w * losses).sum())

    rng = np.random.default_rng(10)
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
        fd = (total(plus) - total(minus)) / (2 * eps)
        an = float((grads[idx] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, fd, an)


def test_cells_outside_the_band_get_no_gradient():
    """Only band cells carry a logit gradient (pinned through dz of the oracle)."""
    batch = _batch(seed=9)
    S = 2
    bounds = _random_bounds(batch, S, np.random.default_rng(6))
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    res = oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                         batch.U_len.numpy(), keep_lattice=True, bounds=bounds, S=S)
    for b in range(3):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        mask = oracle.band_mask(bounds[b], S, Tb, Ub)
        dz = res.lattice[b].dz
        assert np.all(dz[~mask] == 0.0)


def test_bounds_checks():
    T_len = np.array([4])
    U_len = np.array([2])
    ok = np.array([[0, 1, 1, 2]])
    assert oracle.validate_bounds(2, ok, T_len, U_len) == 0
    for bad in ([[1, 1, 1, 2]],        # first frame must start at 0
                [[0, 2, 2, 2]],        # step larger than S - 1
                [[0, 1, 0, 1]],        # not monotone
                [[0, 0, 0, 0]],        # the last frame's band misses U_len
                [[0, 1, 2, 3]]):       # a start beyond U_len
        assert oracle.validate_bounds(2, np.array(bad), T_len, U_len) == oracle.STATUS_BOUNDS, bad


def test_diagonal_bounds_are_valid():
    for name in ("tiny", "short", "medium"):
        batch = synth.workload(name)
        for S in (2, 4, 8):
            s = synth.diagonal_bounds(batch.T_len, batch.U_len, batch.f.shape[1], S)
            assert oracle.validate_bounds(S, s.numpy(), batch.T_len.numpy(), batch.U_len.numpy()) == 0, (name, S)
