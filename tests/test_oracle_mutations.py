"""Mutation check of the oracle's pins (CPU only; the oracle itself is left
untouched).  Plausible mistakes are planted in a copy of the oracle's source:
a dropped term, a wrong sign, a wrong index, a transposed or swapped operand.
Each copy is run against two pins that do not come from the oracle's code:
  * the loss of every utterance against brute-force enumeration of all
    alignments over log-probabilities computed with torch;
  * every gradient against central finite differences of the weighted loss
    sum_b w_b loss_b, along a random direction, with non-uniform w.
A mutant passes unnoticed only if both pins hold for it; none may.  (A mutant
whose own internal consistency checks fail, e.g. alpha against beta, is
caught as well.)"""

import os
import sys
import types

import numpy as np
import pytest

from rnn_joint_network_02_b200 import synth
from tests.test_oracle_pins import _brute_force_logp, _log_probs_torch

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "rnnt_oracle.py")
SOURCE = open(ORACLE_PATH).read()

# (what goes wrong, exact source text, its mutated form)
MUTANTS = [
    ("tanh dropped", "h = np.tanh(F_rows[:, None, :] + G_rows[None, :, :])",
     "h = (F_rows[:, None, :] + G_rows[None, :, :])"),
    ("output bias dropped", "z = h @ W_o.T + b_o", "z = h @ W_o.T"),
    ("projection weights swapped", "return f_b @ W_f, g_b @ W_g", "return f_b @ W_g, g_b @ W_f"),
    ("max in place of log-add-exp", "return m + math.log1p(math.exp(-abs(a - b)))", "return m"),
    ("max in place of log-sum-exp", "return m + np.log(np.exp(z - m[..., None]).sum(axis=-1))", "return m"),
    ("alpha: blank edge from the wrong frame",
     "from_blank = A[t - 1, u] + blank_lp[t - 1, u] if t > 0 else NEG_INF",
     "from_blank = A[t - 1, u] + blank_lp[t, u] if t > 0 else NEG_INF"),
    ("beta: label edge weight of the wrong cell",
     "by_label = Bt[t, u + 1] + label_lp[t, u] if u < Ub else NEG_INF",
     "by_label = Bt[t, u + 1] + label_lp[t, u + 1] if u < Ub else NEG_INF"),
    ("label index off by one", "label_lp[t0:t1, u] = z[:, u, y[u]] - blk_lse[:, u]",
     "label_lp[t0:t1, u] = z[:, u, y[u - 1]] - blk_lse[:, u]"),
    ("terminal blank dropped", "beta_next_t[Tb - 1, Ub] = 0.0", "pass"),
    ("blank gradient sign", "dz[:, :, blank] -= bpost[t0:t1]", "dz[:, :, blank] += bpost[t0:t1]"),
    ("label gradient with the blank posterior", "dz[:, u, y[u]] -= lpost[t0:t1, u]",
     "dz[:, u, y[u]] -= bpost[t0:t1, u]"),
    ("utterance weight dropped", "dz *= w[b]", "pass"),
    ("bias gradient dropped", "res.db_o += dz.sum(axis=(0, 1))", "pass"),
    ("tanh derivative", "dpre = (dz @ W_o) * (1.0 - h * h)", "dpre = (dz @ W_o) * (1.0 - h)"),
    ("output-weight gradient from the pre-activation in place of h",
     "res.dW_o += dz.reshape(-1, V).T @ h.reshape(-1, H)",
     "res.dW_o += dz.reshape(-1, V).T @ np.arctanh(np.clip(h, -0.999999, 0.999999)).reshape(-1, H)"),
    ("frame gradient through W_g", "res.df[b, :Tb] = dF @ W_f.T", "res.df[b, :Tb] = dF @ W_g.T"),
    ("prediction-weight gradient assigned, not accumulated over utterances",
     "res.dW_g += g[b, :Ub + 1].T @ dG", "res.dW_g = g[b, :Ub + 1].T @ dG"),
]


def _load(source: str, name: str):
    mod = types.ModuleType(name)
    mod.__file__ = ORACLE_PATH
    sys.modules[name] = mod          # dataclasses look their module up while the class is built
    try:
        exec(compile(source, ORACLE_PATH, "exec"), mod.__dict__)
    finally:
        del sys.modules[name]
    return mod


def _batch(seed):
    # D_enc == D_pred so that swapped operands still have valid shapes
    return synth.make(B=2, T=4, U=3, D_enc=4, D_pred=4, H=5, V=6, dtype="f32", seed=seed, T_range=(2, 4),
                      U_range=(1, 3), U_rule="range", bias_std=0.5)


def _pins_hold(mod) -> bool:
    """Both pins on two seeded batches; an exception inside the module counts as caught."""
    w = np.array([0.7, 1.3])
    try:
        for seed in (0, 1):
            batch = _batch(seed)
            params = [t.numpy() for t in batch.float64()]
            ints = (batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy())
            res = mod.fwd_bwd(*params, *ints, grad_loss=w)
            for b in range(2):
                Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
                ref = -_brute_force_logp(_log_probs_torch(batch, b), batch.labels[b].tolist(), Tb, Ub)
                if not abs(res.loss[b] - ref) <= 1e-9 * abs(ref):
                    return False
            rng = np.random.default_rng(100 + seed)
            grads = [res.df, res.dg, res.dW_f, res.dW_g, res.dW_o, res.db_o]
            for i, p in enumerate(params):
                d = rng.standard_normal(p.shape)
                eps = 1e-6
                lo = [q.copy() for q in params]
                hi = [q.copy() for q in params]
                lo[i] = p - eps * d
                hi[i] = p + eps * d
                fd = (w @ mod.fwd_bwd(*hi, *ints).loss - w @ mod.fwd_bwd(*lo, *ints).loss) / (2 * eps)
                an = float((grads[i] * d).sum())
                if not abs(fd - an) <= 1e-6 * max(abs(fd), abs(an), 1e-8):
                    return False
    except (AssertionError, ValueError, IndexError, FloatingPointError):
        return False
    return True


def test_the_oracle_as_written_passes_the_pins():
    assert _pins_hold(_load(SOURCE, "_oracle_clean"))


@pytest.mark.parametrize("what,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
@pytest.mark.filterwarnings("ignore::RuntimeWarning")   # a mutant may produce inf - inf
def test_every_planted_mistake_fails_a_pin(what, old, new):
    assert SOURCE.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    mutant = _load(SOURCE.replace(old, new), "_oracle_mutant")
    assert not _pins_hold(mutant), f"the pins did not notice: {what}"


# ---------------------------------------------------------------- maximum approximation and pruned band

from tests.test_oracle_pruned import _band_alignment_scores, _random_bounds  # noqa: E402
from tests.test_oracle_viterbi import _alignments, _score  # noqa: E402

VITERBI_MUTANTS = [
    ("ties to the label edge", "            if by_blank >= by_label:\n", "            if by_blank > by_label:\n"),
    ("max-product label edge from the wrong cell",
     "by_label = A[t, u - 1] + label_lp[t, u - 1] if u > 0 else NEG_INF",
     "by_label = A[t, u - 1] + label_lp[t, u] if u > 0 else NEG_INF"),
    ("final blank left off the best alignment",
     "    bpath[t, u] = 1.0                      # the final blank", "    pass  # the final blank"),
    ("backtrack marks the blank edge at the wrong frame", "            t -= 1\n            bpath[t, u] = 1.0\n",
     "            bpath[t, u] = 1.0\n            t -= 1\n"),
]

BAND_MUTANTS = [
    ("band one position short", "M[t, s:min(Ub + 1, s + S)] = True", "M[t, s:min(Ub + 1, s + S - 1)] = True"),
    ("band start ignored", "        s = int(bounds_b[t])\n", "        s = 0\n"),
]


def _viterbi_pins_hold(mod) -> bool:
    """Brute-force maximisation (loss and the best alignment's edges) on random
    batches, and the tie rule on zero logits (every label at frame 0)."""
    try:
        for seed in range(3):
            batch = _batch(10 + seed)
            params = [t.numpy() for t in batch.float64()]
            ints = (batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy())
            res = mod.fwd_bwd(*params, *ints, loss="viterbi", keep_lattice=True)
            for b in range(2):
                Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
                lp = _log_probs_torch(batch, b)
                labels = batch.labels[b].tolist()
                best, edges = max(((_score(lp, labels, e), e) for e in _alignments(Tb, Ub)), key=lambda x: x[0])
                if not abs(-res.loss[b] - best) <= 1e-11 * max(1.0, abs(best)):
                    return False
                bp, lq = np.zeros((Tb, Ub + 1)), np.zeros((Tb, Ub + 1))
                for (t, u), kind in edges:
                    (bp if kind == "b" else lq)[t, u] = 1.0
                if not (np.array_equal(res.lattice[b].bpost, bp) and np.array_equal(res.lattice[b].lpost, lq)):
                    return False
        batch = _batch(20)
        params = [t.numpy() for t in batch.float64()]
        params[4] = np.zeros_like(params[4])
        params[5] = np.zeros_like(params[5])
        res = mod.fwd_bwd(*params, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(),
                          loss="viterbi", keep_lattice=True)
        for b in range(2):
            Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
            lat = res.lattice[b]
            want_l = np.zeros((Tb, Ub + 1))
            want_l[0, :Ub] = 1.0
            want_b = np.zeros((Tb, Ub + 1))
            want_b[:, Ub] = 1.0
            if not (np.array_equal(lat.lpost, want_l) and np.array_equal(lat.bpost, want_b)):
                return False
    except (AssertionError, ValueError, IndexError, FloatingPointError):
        return False
    return True


def _band_pins_hold(mod) -> bool:
    """Brute force over the alignments inside random valid bands."""
    try:
        for seed in range(3):
            batch = _batch(30 + seed)
            S = 2
            bounds = _random_bounds(batch, S, np.random.default_rng(seed))
            params = [t.numpy() for t in batch.float64()]
            res = mod.fwd_bwd(*params, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(),
                              bounds=bounds, S=S)
            for b in range(2):
                Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
                sc = _band_alignment_scores(_log_probs_torch(batch, b), batch.labels[b].tolist(), Tb, Ub,
                                            bounds[b], S)
                m = max(sc)
                ref = -(m + np.log(np.sum(np.exp(np.array(sc) - m))))
                if not abs(res.loss[b] - ref) <= 1e-9 * abs(ref):
                    return False
    except (AssertionError, ValueError, IndexError, FloatingPointError):
        return False
    return True


def test_the_viterbi_and_band_paths_as_written_pass_their_pins():
    clean = _load(SOURCE, "_oracle_clean2")
    assert _viterbi_pins_hold(clean) and _band_pins_hold(clean)


@pytest.mark.parametrize("what,old,new", VITERBI_MUTANTS, ids=[m[0] for m in VITERBI_MUTANTS])
@pytest.mark.filterwarnings("ignore::RuntimeWarning")   # a mutant may produce inf - inf
def test_every_planted_viterbi_mistake_fails_a_pin(what, old, new):
    assert SOURCE.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    assert not _viterbi_pins_hold(_load(SOURCE.replace(old, new), "_oracle_vmutant")), what


@pytest.mark.parametrize("what,old,new", BAND_MUTANTS, ids=[m[0] for m in BAND_MUTANTS])
@pytest.mark.filterwarnings("ignore::RuntimeWarning")   # a mutant may produce inf - inf
def test_every_planted_band_mistake_fails_a_pin(what, old, new):
    assert SOURCE.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    assert not _band_pins_hold(_load(SOURCE.replace(old, new), "_oracle_bmutant")), what
