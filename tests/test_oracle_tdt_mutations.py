"""Mutation check of the token-and-duration oracle's pins (CPU only; the
oracle itself is left untouched).  Plausible mistakes are planted in a copy of
its source and each copy is run against two pins that do not come from the
oracle's code: the loss against depth-first enumeration of every alignment
over torch log-softmaxes of both heads, and every gradient (the duration head's
included) against central finite differences of the weighted loss.  No mutant
may pass both."""

import os
import sys
import types

import numpy as np
import pytest

from rnn_joint_network_02_b200 import synth
from tests.test_oracle_tdt import _alignment_scores, _log_probs

TDT_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "tdt_oracle.py")
SOURCE = open(TDT_PATH).read()
D = (0, 1, 2)

MUTANTS = [
    ("alpha: blank edge with the duration of index 0",
     "acc = lae(acc, A[s, u] + blank_lp[s, u] + dur_lp[s, u, i])",
     "acc = lae(acc, A[s, u] + blank_lp[s, u] + dur_lp[s, u, 0])"),
    ("alpha: label edge with the duration of the wrong cell",
     "acc = lae(acc, A[s, u - 1] + label_lp[s, u - 1] + dur_lp[s, u - 1, i])",
     "acc = lae(acc, A[s, u - 1] + label_lp[s, u - 1] + dur_lp[s, u, i])"),
    ("final blank ignores its duration", "        s = Tb - d\n", "        s = Tb - 1\n"),
    ("beta: label edge keeps the label position",
     "acc = lae(acc, label_lp[t, u] + dur_lp[t, u, i] + Bt[t + d, u + 1])",
     "acc = lae(acc, label_lp[t, u] + dur_lp[t, u, i] + Bt[t + d, u])"),
    ("a blank past the last frame also ends an alignment",
     "return 0.0 if (t == Tb and u == Ub) else NEG_INF",
     "return 0.0 if (t >= Tb and u == Ub) else NEG_INF"),
    ("duration head not normalised", "dur_lp = zd - log_sum_exp_last(zd)[..., None]", "dur_lp = zd"),
    ("duration bias dropped", "return h @ W_d.T + b_d", "return h @ W_d.T"),
    ("duration gradient sign", "dzd = w[b] * (occ[:, :, None] * np.exp(dur_lp) - (pb + pl))",
     "dzd = w[b] * (occ[:, :, None] * np.exp(dur_lp) + (pb + pl))"),
    ("duration gradient without the label edges", "dzd = w[b] * (occ[:, :, None] * np.exp(dur_lp) - (pb + pl))",
     "dzd = w[b] * (occ[:, :, None] * np.exp(dur_lp) - pb)"),
    ("hidden gradient misses the duration head", "dpre = (dz @ W_o + dzd @ W_d) * (1.0 - h * h)",
     "dpre = (dz @ W_o) * (1.0 - h * h)"),
    ("duration bias gradient dropped", "res.db_d += dzd.sum(axis=(0, 1))", "pass"),
]


def _load(source: str, name: str):
    mod = types.ModuleType(f"oracle.{name}")
    mod.__file__ = TDT_PATH
    mod.__package__ = "oracle"       # its shared helpers come from the real transducer oracle
    sys.modules[mod.__name__] = mod
    try:
        exec(compile(source, TDT_PATH, "exec"), mod.__dict__)
    finally:
        del sys.modules[mod.__name__]
    return mod


def _batch(seed):
    return synth.make(B=2, T=5, U=2, D_enc=3, D_pred=4, H=5, V=6, dtype="f32", seed=seed, T_range=(3, 5),
                      U_range=(1, 2), U_rule="range", bias_std=0.5)


def _pins_hold(mod) -> bool:
    w = np.array([0.7, 1.3])
    try:
        for seed in (0, 1):
            batch = _batch(seed)
            W_d, b_d = (t.double() for t in synth.duration_head(batch, len(D), seed=5 + seed, bias_std=0.5))
            params = [t.numpy() for t in batch.float64()] + [W_d.numpy(), b_d.numpy()]
            ints = (batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(), D)
            res = mod.tdt_fwd_bwd(*params, *ints, grad_loss=w)
            for b in range(2):
                Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
                lp, ld = _log_probs(batch, W_d, b_d, b)
                s = _alignment_scores(lp, ld, batch.labels[b].tolist(), D, Tb, Ub)
                ref = -(s.max() + np.log(np.exp(s - s.max()).sum()))
                if not abs(res.loss[b] - ref) <= 1e-9 * abs(ref):
                    return False
            rng = np.random.default_rng(200 + seed)
            grads = [res.df, res.dg, res.dW_f, res.dW_g, res.dW_o, res.db_o, res.dW_d, res.db_d]
            for i, p in enumerate(params):
                d = rng.standard_normal(p.shape)
                eps = 1e-6
                lo = [q.copy() for q in params]
                hi = [q.copy() for q in params]
                lo[i] = p - eps * d
                hi[i] = p + eps * d
                fd = (w @ mod.tdt_fwd_bwd(*hi, *ints).loss - w @ mod.tdt_fwd_bwd(*lo, *ints).loss) / (2 * eps)
                an = float((grads[i] * d).sum())
                if not abs(fd - an) <= 1e-6 * max(abs(fd), abs(an), 1e-8):
                    return False
    except (AssertionError, ValueError, IndexError, FloatingPointError):
        return False
    return True


def test_the_oracle_as_written_passes_the_pins():
    assert _pins_hold(_load(SOURCE, "_tdt_clean"))


@pytest.mark.parametrize("what,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(what, old, new):
    assert SOURCE.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    mutant = _load(SOURCE.replace(old, new), "_tdt_mutant")
    assert not _pins_hold(mutant), f"the pins did not notice: {what}"
