"""fp64 CPU oracle for the token-and-duration transducer (TDT) joint and loss.

TEST INFRASTRUCTURE ONLY, like ``rnnt_oracle`` (whose joint-network helpers
it reuses): nothing on the product path may import, call or execute it, and it
shares no code with the CUDA library.

Source: "Efficient Sequence Transduction by Jointly Predicting Tokens and
Durations" (abstract).  The joint network gets a second output head, and the
two heads are normalised independently: one distribution over the label space
(blank included) and one over a set D of durations, a duration being the
number of input frames the emitted symbol covers.  The pages print nothing
beyond the abstract, so the plainest lattice reading is used:

* Heads.  h = tanh(F[t] + G[u]) as in the transducer joint;
      z  = W_o h + b_o       (V token logits)
      zd = W_d h + b_d       (|D| duration logits)
  blank_lp / label_lp = token log-softmax at blank / y_u, and
  dur_lp[i] = duration log-softmax at entry i of D.
* Edges.  From cell (t,u) (t < T_len, u <= U_len) a label y_u with duration
  d in D goes to (t+d, u+1) (u < U_len); a blank with duration d in D, d >= 1,
  goes to (t+d, u) (a blank that covers no frame would be a self-loop).  The
  weight of an edge is the product of its token and duration probabilities.
* Alignments start at (0,0) and end with a blank that lands exactly on frame
  T_len with every label emitted: (t, U_len) -> (T_len, U_len).  Landing
  anywhere else at or past T_len ends no alignment.
* loss_b = -log of the summed weight of all alignments:
      alpha(0,0) = 0
      alpha(t,u) = lae_{d in D, d>=1} alpha(t-d,u)   + blank_lp(t-d,u)   + dur_lp(t-d,u,d)
                   lae_{d in D}       alpha(t-d,u-1) + label_lp(t-d,u-1) + dur_lp(t-d,u-1,d)
      log P      = lae_{d in D, d>=1} alpha(T_len-d, U_len) + blank_lp(..) + dur_lp(.., d)
  and beta(t,u) mirrors it with beta'(T_len, U_len) = 0 for the final blank.
* D is a strictly increasing set of non-negative integers that contains 0 and
  1 (so every (T_len, U_len) has an alignment).

Gradients of sum_b w_b loss_b: with the per-edge posteriors pb_d (blank, d)
and pl_d (label, d) of cell c, bpost = sum_d pb_d, lpost = sum_d pl_d and
occ = bpost + lpost (the probability that an alignment emits at c),
      dz  = w (occ softmax(z)  - bpost e_blank - lpost e_label)
      dzd = w (occ softmax(zd) - (pb_d + pl_d))_d
and the chain rule through both heads and the tanh gives the rest.
Float64 throughout; bf16 inputs arrive already rounded.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .rnnt_oracle import NEG_INF, joint_logits, lae, log_sum_exp_last, projections, validate

STATUS_DURATIONS = 16   # host-side only: an invalid duration set


def validate_durations(durations) -> bool:
    """D strictly increasing, non-negative, containing 0 and 1."""
    d = [int(x) for x in durations]
    if len(d) < 2 or d[0] != 0 or d[1] != 1:
        return False
    return all(d[i] < d[i + 1] for i in range(len(d) - 1))


def duration_logits(h, W_d, b_d):
    """zd = W_d h + b_d over the last axis of h."""
    return h @ W_d.T + b_d


def tdt_alpha(blank_lp, label_lp, dur_lp, durations, Tb: int, Ub: int):
    """Forward variables over the (Tb, Ub+1) lattice; dur_lp has shape (Tb, Ub+1, |D|)."""
    A = np.full((Tb, Ub + 1), NEG_INF)
    A[0, 0] = 0.0
    for t in range(Tb):
        for u in range(Ub + 1):          # u ascending: duration-0 labels stay in the frame
            if t == 0 and u == 0:
                continue
            acc = NEG_INF
            for i, d in enumerate(durations):
                s = t - d
                if s < 0:
                    continue
                if d >= 1:
                    acc = lae(acc, A[s, u] + blank_lp[s, u] + dur_lp[s, u, i])
                if u >= 1:
                    acc = lae(acc, A[s, u - 1] + label_lp[s, u - 1] + dur_lp[s, u - 1, i])
            A[t, u] = acc
    return A


def tdt_log_p_from_alpha(A, blank_lp, dur_lp, durations, Tb: int, Ub: int) -> float:
    """log P: the final blank from (T_len - d, U_len) that lands on frame T_len."""
    acc = NEG_INF
    for i, d in enumerate(durations):
        s = Tb - d
        if d >= 1 and s >= 0:
            acc = lae(acc, A[s, Ub] + blank_lp[s, Ub] + dur_lp[s, Ub, i])
    return acc


def tdt_beta(blank_lp, label_lp, dur_lp, durations, Tb: int, Ub: int):
    """Backward variables beta(t,u) = log of the summed weight of the ways to
    finish an alignment that emits at (t,u) next (the emission at (t,u) included)."""
    Bt = np.full((Tb, Ub + 1), NEG_INF)

    def beta_after_blank(t, u):          # beta' at the cell a blank lands on
        if t < Tb:
            return Bt[t, u]
        return 0.0 if (t == Tb and u == Ub) else NEG_INF

    for t in range(Tb - 1, -1, -1):
        for u in range(Ub, -1, -1):      # u descending: duration-0 labels stay in the frame
            acc = NEG_INF
            for i, d in enumerate(durations):
                if d >= 1:
                    acc = lae(acc, blank_lp[t, u] + dur_lp[t, u, i] + beta_after_blank(t + d, u))
                if u < Ub and t + d < Tb:
                    acc = lae(acc, label_lp[t, u] + dur_lp[t, u, i] + Bt[t + d, u + 1])
            Bt[t, u] = acc
    return Bt


def tdt_edge_posteriors(A, Bt, blank_lp, label_lp, dur_lp, durations, Tb: int, Ub: int, log_p: float):
    """pb[t,u,i], pl[t,u,i]: posterior of the blank / label edge of duration D[i] leaving (t,u)."""
    nd = len(durations)
    pb = np.zeros((Tb, Ub + 1, nd))
    pl = np.zeros((Tb, Ub + 1, nd))
    for t in range(Tb):
        for u in range(Ub + 1):
            for i, d in enumerate(durations):
                if d >= 1:
                    if t + d < Tb:
                        nxt = Bt[t + d, u]
                    else:
                        nxt = 0.0 if (t + d == Tb and u == Ub) else NEG_INF
                    pb[t, u, i] = np.exp(A[t, u] + blank_lp[t, u] + dur_lp[t, u, i] + nxt - log_p)
                if u < Ub and t + d < Tb:
                    pl[t, u, i] = np.exp(A[t, u] + label_lp[t, u] + dur_lp[t, u, i] + Bt[t + d, u + 1] - log_p)
    return pb, pl


@dataclass
class TdtLattice:
    lse: np.ndarray
    blank_lp: np.ndarray
    label_lp: np.ndarray
    dur_lp: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    pb: np.ndarray
    pl: np.ndarray
    log_p: float


@dataclass
class TdtResult:
    status: int
    loss: np.ndarray | None = None
    df: np.ndarray | None = None
    dg: np.ndarray | None = None
    dW_f: np.ndarray | None = None
    dW_g: np.ndarray | None = None
    dW_o: np.ndarray | None = None
    db_o: np.ndarray | None = None
    dW_d: np.ndarray | None = None
    db_d: np.ndarray | None = None
    lattice: dict = field(default_factory=dict)


def _cell_log_probs(F, G, W_o, b_o, W_d, b_d, y, blank: int, Ub: int):
    h, z = joint_logits(F, G, W_o, b_o)
    lse = log_sum_exp_last(z)
    blank_lp = z[:, :, blank] - lse
    label_lp = np.full(lse.shape, NEG_INF)
    for u in range(Ub):
        label_lp[:, u] = z[:, u, y[u]] - lse[:, u]
    zd = duration_logits(h, W_d, b_d)
    dur_lp = zd - log_sum_exp_last(zd)[..., None]
    return h, z, lse, blank_lp, label_lp, dur_lp


def tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d, b_d, labels, T_len, U_len, durations, grad_loss=None,
                blank: int = 0, utterances=None, keep_lattice: bool = False) -> TdtResult:
    """Loss and gradients of sum_b w_b loss_b (float64).  W_d [|D|,H], b_d [|D|];
    the other arguments as in the transducer oracle."""
    if not validate_durations(durations):
        return TdtResult(status=STATUS_DURATIONS)
    durations = [int(x) for x in durations]
    f, g, W_f, W_g, W_o, b_o, W_d, b_d = (np.asarray(x, dtype=np.float64)
                                          for x in (f, g, W_f, W_g, W_o, b_o, W_d, b_d))
    labels, T_len, U_len = np.asarray(labels), np.asarray(T_len), np.asarray(U_len)
    B, T, _ = f.shape
    U = g.shape[1] - 1
    V, H = W_o.shape
    status = validate(T, U, V, blank, labels, T_len, U_len)
    if status:
        return TdtResult(status=status)
    w = np.ones(B) if grad_loss is None else np.asarray(grad_loss, dtype=np.float64)
    todo = range(B) if utterances is None else list(utterances)
    res = TdtResult(status=0, loss=np.full(B, np.nan), df=np.zeros_like(f), dg=np.zeros_like(g),
                    dW_f=np.zeros_like(W_f), dW_g=np.zeros_like(W_g), dW_o=np.zeros_like(W_o),
                    db_o=np.zeros_like(b_o), dW_d=np.zeros_like(W_d), db_d=np.zeros_like(b_d))
    for b in todo:
        Tb, Ub = int(T_len[b]), int(U_len[b])
        y = [int(labels[b, u]) for u in range(Ub)]
        F, G = projections(f[b, :Tb], g[b, :Ub + 1], W_f, W_g)
        h, z, lse, blank_lp, label_lp, dur_lp = _cell_log_probs(F, G, W_o, b_o, W_d, b_d, y, blank, Ub)
        A = tdt_alpha(blank_lp, label_lp, dur_lp, durations, Tb, Ub)
        Bt = tdt_beta(blank_lp, label_lp, dur_lp, durations, Tb, Ub)
        log_p = tdt_log_p_from_alpha(A, blank_lp, dur_lp, durations, Tb, Ub)
        assert abs(Bt[0, 0] - log_p) <= 1e-9 * max(1.0, abs(log_p)), (Bt[0, 0], log_p)
        res.loss[b] = -log_p
        pb, pl = tdt_edge_posteriors(A, Bt, blank_lp, label_lp, dur_lp, durations, Tb, Ub, log_p)
        bpost, lpost = pb.sum(axis=-1), pl.sum(axis=-1)
        occ = bpost + lpost
        assert np.allclose(occ, np.exp(A + Bt - log_p), rtol=1e-9, atol=1e-12)

        dz = occ[:, :, None] * np.exp(z - lse[:, :, None])
        dz[:, :, blank] -= bpost
        for u in range(Ub):
            dz[:, u, y[u]] -= lpost[:, u]
        dz *= w[b]
        dzd = w[b] * (occ[:, :, None] * np.exp(dur_lp) - (pb + pl))
        res.db_o += dz.sum(axis=(0, 1))
        res.dW_o += dz.reshape(-1, V).T @ h.reshape(-1, H)
        res.db_d += dzd.sum(axis=(0, 1))
        res.dW_d += dzd.reshape(-1, len(durations)).T @ h.reshape(-1, H)
        dpre = (dz @ W_o + dzd @ W_d) * (1.0 - h * h)
        dF, dG = dpre.sum(axis=1), dpre.sum(axis=0)
        res.df[b, :Tb] = dF @ W_f.T
        res.dW_f += f[b, :Tb].T @ dF
        res.dg[b, :Ub + 1] = dG @ W_g.T
        res.dW_g += g[b, :Ub + 1].T @ dG
        if keep_lattice:
            res.lattice[b] = TdtLattice(lse, blank_lp, label_lp, dur_lp, A, Bt, pb, pl, log_p)
    return res


def tdt_loss_only(f, g, W_f, W_g, W_o, b_o, W_d, b_d, labels, T_len, U_len, durations, blank: int = 0):
    """Per-utterance TDT losses (forward only), for finite-difference checks."""
    durations = [int(x) for x in durations]
    f, g, W_f, W_g, W_o, b_o, W_d, b_d = (np.asarray(x, dtype=np.float64)
                                          for x in (f, g, W_f, W_g, W_o, b_o, W_d, b_d))
    out = np.empty(f.shape[0])
    for b in range(f.shape[0]):
        Tb, Ub = int(T_len[b]), int(U_len[b])
        y = [int(labels[b, u]) for u in range(Ub)]
        F, G = projections(f[b, :Tb], g[b, :Ub + 1], W_f, W_g)
        _, _, _, blank_lp, label_lp, dur_lp = _cell_log_probs(F, G, W_o, b_o, W_d, b_d, y, blank, Ub)
        A = tdt_alpha(blank_lp, label_lp, dur_lp, durations, Tb, Ub)
        out[b] = -tdt_log_p_from_alpha(A, blank_lp, dur_lp, durations, Tb, Ub)
    return out
