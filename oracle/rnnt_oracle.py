"""fp64 CPU oracle for the RNN-T joint network fused with the transducer loss.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the test-suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` use it.  It shares
no code with the CUDA library (no kernels, headers, helpers or constants) and
imports nothing from the package that wraps that library.

What it computes (the definitions, written out plainly, in float64):

* Joint network.  For utterance b, frame t and label-history position u,
      h[b,t,u,:] = tanh(f[b,t,:] W_f + g[b,u,:] W_g)
      z[b,t,u,:] = W_o h[b,t,u,:] + b_o
  i.e. the encoder and prediction activations are combined by a feed-forward
  layer into a distribution over the label space for every (frame position,
  label history) pair -- "Transformer Transducer: A Streamable Speech
  Recognition Model ..." (abstract), and the transducer of "Sequence
  Transduction with Recurrent Neural Networks" (abstract).  The tanh
  composition and the shapes f[B,T,D_enc], g[B,U+1,D_pred], W_f[D_enc,H],
  W_g[D_pred,H], W_o[V,H], b_o[V] are the joint of this library's contract.
* Per-cell log-probabilities.  lse = log sum_k exp z_k,
  blank_lp = z_blank - lse, label_lp = z_{y_u} - lse (u < U_len).
* Transducer loss: -log of the probability summed over every alignment
  ("Sequence Transduction with Recurrent Neural Networks", abstract; the loss
  that learns the input/output alignment).  The pages print no recursion, so
  the textbook forward-backward over the (T_len, U_len+1) lattice is used:
      alpha(0,0) = 0
      alpha(t,u) = lae(alpha(t-1,u) + blank_lp(t-1,u),
                       alpha(t,u-1) + label_lp(t,u-1))
      log P      = alpha(T_len-1, U_len) + blank_lp(T_len-1, U_len)
      beta(T_len-1, U_len) = blank_lp(T_len-1, U_len)
      beta(t,u)  = lae(beta(t+1,u) + blank_lp(t,u), beta(t,u+1) + label_lp(t,u))
  (lae = log-add-exp; out-of-lattice terms are -inf; the final blank that
  ends the last frame is included).
* Gradients of sum_b w_b * loss_b (w_b = grad_loss[b], default 1), for the
  logits (dz = w_b (occ*softmax - bpost*e_blank - lpost*e_label)) and, by the
  chain rule through the joint, for b_o, W_o, the hidden pre-activation, f,
  g, W_f and W_g.
* Maximum approximation (``loss="viterbi"``): the sum over alignments is
  replaced by the single best alignment ("Daily Papers" page for the
  CTC/RNN-T architecture search, the RNN-transducer abstract that compares
  full marginalisation over alignments with the maximum approximation).
  The pages give no recursion, so
  the plainest reading is used: the same lattice with max in place of lae,
      alpha(t,u) = max(alpha(t-1,u) + blank_lp(t-1,u),
                       alpha(t,u-1) + label_lp(t,u-1)),
      loss = -(alpha(T_len-1,U_len) + blank_lp(T_len-1,U_len)),
  the best alignment recovered by backtracking from the last cell, and ties
  broken towards the blank edge (arriving at (t,u) from (t-1,u)).  The loss
  is -log p(best alignment), so its gradient is the marginal formula with
  bpost / lpost the 0/1 indicators of the best alignment's edges.
* Pruning bounds (``bounds`` [B,T] int, ``S``): "Pruned RNN-T for fast,
  memory-efficient ASR training" (abstract) evaluates the full non-linear
  joiner only within pruning bounds; the bounds themselves (from a linear
  joiner on the pages) are an input here.  Plainest reading: frame t of
  utterance b keeps the S label positions s[b,t] <= u < s[b,t] + S, every
  other cell is removed from the lattice (alpha = beta = -inf there, no
  logits, no gradient), and the loss sums over the alignments that stay
  inside the band.  Bounds are valid when s[b,0] = 0, s[b,t] <= U_len,
  s[b,t] <= s[b,t+1] <= s[b,t] + S - 1 and s[b,T_len-1] + S - 1 >= U_len
  (then a band alignment exists); otherwise STATUS_BOUNDS.

Every float op here is float64; inputs that the product path receives in
bf16 are handed to the oracle already rounded to bf16 (by the shared seeded
input generator), so both sides see identical values.  The work is done one
utterance and one block of frames at a time only to bound host memory; no
other blocking, fusion or reordering is applied.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# Status bits, mirroring the device-side status word of the library contract:
# a length outside its range, or a label outside the vocabulary / equal to blank.
STATUS_LENGTH = 1
STATUS_LABEL = 2
STATUS_BOUNDS = 8

NEG_INF = -math.inf


def lae(a: float, b: float) -> float:
    """log(exp(a) + exp(b)) for scalars, exact for -inf operands."""
    if a == NEG_INF:
        return b
    if b == NEG_INF:
        return a
    m = a if a > b else b
    return m + math.log1p(math.exp(-abs(a - b)))


def validate(T: int, U: int, V: int, blank: int, labels, T_len, U_len) -> int:
    """Integer checks of lengths and labels; returns the status bits.

    1 <= T_len[b] <= T, 0 <= U_len[b] <= U, and for u < U_len[b]:
    0 <= labels[b,u] < V with labels[b,u] != blank.  Label positions at or
    beyond U_len[b] are padding and are not inspected.
    """
    status = 0
    labels = np.asarray(labels)
    for b in range(len(T_len)):
        Tb, Ub = int(T_len[b]), int(U_len[b])
        if not (1 <= Tb <= T) or not (0 <= Ub <= U):
            status |= STATUS_LENGTH
            continue
        for u in range(Ub):
            y = int(labels[b, u])
            if y < 0 or y >= V or y == blank:
                status |= STATUS_LABEL
    return status


def validate_bounds(S: int, bounds, T_len, U_len) -> int:
    """STATUS_BOUNDS unless every utterance's band is valid (see the header)."""
    bounds = np.asarray(bounds)
    for b in range(len(T_len)):
        Tb, Ub = int(T_len[b]), int(U_len[b])
        s = [int(bounds[b, t]) for t in range(Tb)]
        if s[0] != 0 or s[Tb - 1] + S - 1 < Ub:
            return STATUS_BOUNDS
        for t in range(Tb):
            if s[t] < 0 or s[t] > Ub:
                return STATUS_BOUNDS
            if t + 1 < Tb and not (s[t] <= s[t + 1] <= s[t] + S - 1):
                return STATUS_BOUNDS
    return 0


def band_mask(bounds_b, S: int, Tb: int, Ub: int):
    """True for the cells (t, u) of the (Tb, Ub+1) lattice inside the band."""
    M = np.zeros((Tb, Ub + 1), dtype=bool)
    for t in range(Tb):
        s = int(bounds_b[t])
        M[t, s:min(Ub + 1, s + S)] = True
    return M


def projections(f_b, g_b, W_f, W_g):
    """F = f W_f and G = g W_g for one utterance (float64 matmuls)."""
    return f_b @ W_f, g_b @ W_g


def joint_logits(F_rows, G_rows, W_o, b_o):
    """z[t,u,:] = W_o tanh(F[t] + G[u]) + b_o for a block of frames.

    Returns (h, z) with h of shape (t, u, H) and z of shape (t, u, V).
    """
    h = np.tanh(F_rows[:, None, :] + G_rows[None, :, :])
    z = h @ W_o.T + b_o
    return h, z


def log_sum_exp_last(z):
    """Max-shifted log-sum-exp over the last axis."""
    m = z.max(axis=-1)
    return m + np.log(np.exp(z - m[..., None]).sum(axis=-1))


def alpha_lattice(blank_lp, label_lp, Tb: int, Ub: int, mask=None):
    """Forward variables alpha(t,u) over the (Tb, Ub+1) lattice (cells outside
    ``mask``, when given, are removed: -inf)."""
    A = np.full((Tb, Ub + 1), NEG_INF)
    for t in range(Tb):
        for u in range(Ub + 1):
            if mask is not None and not mask[t, u]:
                continue
            if t == 0 and u == 0:
                A[t, u] = 0.0
                continue
            from_blank = A[t - 1, u] + blank_lp[t - 1, u] if t > 0 else NEG_INF
            from_label = A[t, u - 1] + label_lp[t, u - 1] if u > 0 else NEG_INF
            A[t, u] = lae(from_blank, from_label)
    return A


def beta_lattice(blank_lp, label_lp, Tb: int, Ub: int, mask=None):
    """Backward variables beta(t,u); beta(0,0) = log P (cells outside ``mask``: -inf)."""
    Bt = np.full((Tb, Ub + 1), NEG_INF)
    for t in range(Tb - 1, -1, -1):
        for u in range(Ub, -1, -1):
            if mask is not None and not mask[t, u]:
                continue
            if t == Tb - 1 and u == Ub:
                Bt[t, u] = blank_lp[t, u]
                continue
            by_blank = Bt[t + 1, u] + blank_lp[t, u] if t + 1 < Tb else NEG_INF
            by_label = Bt[t, u + 1] + label_lp[t, u] if u < Ub else NEG_INF
            Bt[t, u] = lae(by_blank, by_label)
    return Bt


def viterbi_lattice(blank_lp, label_lp, Tb: int, Ub: int, mask=None):
    """Max-product forward variables and the best predecessor of every cell.

    Returns (A, from_blank) with from_blank[t,u] True when the best way into
    (t,u) is the blank edge from (t-1,u) (ties go to the blank edge)."""
    A = np.full((Tb, Ub + 1), NEG_INF)
    from_blank = np.zeros((Tb, Ub + 1), dtype=bool)
    for t in range(Tb):
        for u in range(Ub + 1):
            if mask is not None and not mask[t, u]:
                continue
            if t == 0 and u == 0:
                A[t, u] = 0.0
                continue
            by_blank = A[t - 1, u] + blank_lp[t - 1, u] if t > 0 else NEG_INF
            by_label = A[t, u - 1] + label_lp[t, u - 1] if u > 0 else NEG_INF
            if by_blank >= by_label:
                A[t, u] = by_blank
                from_blank[t, u] = True
            else:
                A[t, u] = by_label
    return A, from_blank


def best_alignment(from_blank, Tb: int, Ub: int):
    """0/1 indicators of the edges leaving each cell on the best alignment:
    (blank edge (t,u)->(t+1,u) incl. the final blank, label edge (t,u)->(t,u+1))."""
    bpath = np.zeros((Tb, Ub + 1))
    lpath = np.zeros((Tb, Ub + 1))
    t, u = Tb - 1, Ub
    bpath[t, u] = 1.0                      # the final blank that ends the last frame
    while (t, u) != (0, 0):
        if from_blank[t, u]:
            t -= 1
            bpath[t, u] = 1.0
        else:
            u -= 1
            lpath[t, u] = 1.0
    return bpath, lpath


@dataclass
class UtteranceLattice:
    """Per-cell quantities of one utterance, each of shape (Tb, Ub+1)."""
    lse: np.ndarray
    blank_lp: np.ndarray
    label_lp: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    bpost: np.ndarray
    lpost: np.ndarray
    log_p: float
    dz: np.ndarray | None = None   # (Tb, Ub+1, V) logit gradient, weighted by w_b


@dataclass
class OracleResult:
    status: int
    loss: np.ndarray | None = None          # [B], -log P per utterance
    df: np.ndarray | None = None
    dg: np.ndarray | None = None
    dW_f: np.ndarray | None = None
    dW_g: np.ndarray | None = None
    dW_o: np.ndarray | None = None
    db_o: np.ndarray | None = None
    lattice: dict = field(default_factory=dict)  # b -> UtteranceLattice (if kept)


def _frame_block(Ub: int, V: int, H: int, budget_bytes: int = 1 << 28) -> int:
    per_frame = (Ub + 1) * (V + H) * 8 * 3
    return max(1, budget_bytes // max(per_frame, 1))


def fwd_bwd(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss=None,
            blank: int = 0, utterances=None, keep_lattice: bool = False,
            loss: str = "marginal", bounds=None, S: int = 0) -> OracleResult:
    """Loss and gradients of sum_b w_b * loss_b, all in float64.

    f [B,T,D_enc], g [B,U+1,D_pred], W_f [D_enc,H], W_g [D_pred,H], W_o [V,H],
    b_o [V], labels [B,U] (int), T_len/U_len [B] (int), grad_loss [B] or None.
    ``utterances`` restricts the work to a subset of b (the others get loss NaN
    and contribute nothing to the weight gradients; their df/dg rows are 0).
    Gradient rows for frames t >= T_len[b] and positions u > U_len[b] are 0.
    ``loss`` is "marginal" (all alignments) or "viterbi" (the best one).
    ``bounds`` [B,T] with band width ``S`` restricts the lattice (header).
    """
    if loss not in ("marginal", "viterbi"):
        raise ValueError(f"unknown loss {loss!r}")
    f = np.asarray(f, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    W_f = np.asarray(W_f, dtype=np.float64)
    W_g = np.asarray(W_g, dtype=np.float64)
    W_o = np.asarray(W_o, dtype=np.float64)
    b_o = np.asarray(b_o, dtype=np.float64)
    labels = np.asarray(labels)
    T_len = np.asarray(T_len)
    U_len = np.asarray(U_len)
    B, T, _ = f.shape
    U = g.shape[1] - 1
    V, H = W_o.shape
    status = validate(T, U, V, blank, labels, T_len, U_len)
    if not status and bounds is not None:
        status = validate_bounds(S, bounds, T_len, U_len)
    if status:
        return OracleResult(status=status)
    w = np.ones(B) if grad_loss is None else np.asarray(grad_loss, dtype=np.float64)
    todo = range(B) if utterances is None else list(utterances)

    res = OracleResult(status=0, loss=np.full(B, np.nan),
                       df=np.zeros_like(f), dg=np.zeros_like(g),
                       dW_f=np.zeros_like(W_f), dW_g=np.zeros_like(W_g),
                       dW_o=np.zeros_like(W_o), db_o=np.zeros_like(b_o))
    for b in todo:
        Tb, Ub = int(T_len[b]), int(U_len[b])
        y = [int(labels[b, u]) for u in range(Ub)]
        F, G = projections(f[b, :Tb], g[b, :Ub + 1], W_f, W_g)
        mask = None if bounds is None else band_mask(bounds[b], S, Tb, Ub)

        # forward: per-cell log-probabilities (the band's cells only are used)
        lse = np.empty((Tb, Ub + 1))
        blank_lp = np.empty((Tb, Ub + 1))
        label_lp = np.full((Tb, Ub + 1), NEG_INF)
        step = _frame_block(Ub, V, H)
        for t0 in range(0, Tb, step):
            t1 = min(Tb, t0 + step)
            _, z = joint_logits(F[t0:t1], G, W_o, b_o)
            blk_lse = log_sum_exp_last(z)
            lse[t0:t1] = blk_lse
            blank_lp[t0:t1] = z[:, :, blank] - blk_lse
            for u in range(Ub):
                label_lp[t0:t1, u] = z[:, u, y[u]] - blk_lse[:, u]

        if loss == "viterbi":
            # best alignment: its log-probability and its edges
            A, from_blank = viterbi_lattice(blank_lp, label_lp, Tb, Ub, mask)
            log_p = A[Tb - 1, Ub] + blank_lp[Tb - 1, Ub]
            res.loss[b] = -log_p
            bpost, lpost = best_alignment(from_blank, Tb, Ub)
            Bt = np.full((Tb, Ub + 1), np.nan)              # no backward variables in this variant
        else:
            # transducer loss
            A = alpha_lattice(blank_lp, label_lp, Tb, Ub, mask)
            Bt = beta_lattice(blank_lp, label_lp, Tb, Ub, mask)
            log_p = A[Tb - 1, Ub] + blank_lp[Tb - 1, Ub]
            assert abs(Bt[0, 0] - log_p) <= 1e-9 * max(1.0, abs(log_p)), (Bt[0, 0], log_p)
            res.loss[b] = -log_p

            # alignment posteriors of each outgoing edge
            beta_next_t = np.full((Tb, Ub + 1), NEG_INF)       # beta'(t+1, u)
            beta_next_t[:-1] = Bt[1:]
            beta_next_t[Tb - 1, Ub] = 0.0                       # terminal blank
            beta_next_u = np.full((Tb, Ub + 1), NEG_INF)       # beta(t, u+1)
            beta_next_u[:, :-1] = Bt[:, 1:]
            bpost = np.exp(A + blank_lp + beta_next_t - log_p)
            lpost = np.where(np.isfinite(label_lp), np.exp(A + label_lp + beta_next_u - log_p), 0.0)
            occ = np.exp(A + Bt - log_p)
            assert np.allclose(occ, bpost + lpost, rtol=1e-9, atol=1e-12)

        # backward through the joint (logits recomputed per frame block)
        dF = np.zeros((Tb, H))
        dG = np.zeros((Ub + 1, H))
        dz_all = np.empty((Tb, Ub + 1, V)) if keep_lattice else None
        for t0 in range(0, Tb, step):
            t1 = min(Tb, t0 + step)
            h, z = joint_logits(F[t0:t1], G, W_o, b_o)
            soft = np.exp(z - lse[t0:t1, :, None])
            dz = (bpost[t0:t1] + lpost[t0:t1])[:, :, None] * soft
            dz[:, :, blank] -= bpost[t0:t1]
            for u in range(Ub):
                dz[:, u, y[u]] -= lpost[t0:t1, u]
            dz *= w[b]
            if dz_all is not None:
                dz_all[t0:t1] = dz
            res.db_o += dz.sum(axis=(0, 1))
            res.dW_o += dz.reshape(-1, V).T @ h.reshape(-1, H)
            dpre = (dz @ W_o) * (1.0 - h * h)
            dF[t0:t1] += dpre.sum(axis=1)
            dG += dpre.sum(axis=0)
        res.df[b, :Tb] = dF @ W_f.T
        res.dW_f += f[b, :Tb].T @ dF
        res.dg[b, :Ub + 1] = dG @ W_g.T
        res.dW_g += g[b, :Ub + 1].T @ dG
        if keep_lattice:
            res.lattice[b] = UtteranceLattice(lse, blank_lp, label_lp, A, Bt, bpost, lpost,
                                             log_p, dz_all)
    return res


def loss_only(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, blank: int = 0, loss: str = "marginal",
              bounds=None, S: int = 0):
    """Per-utterance losses (forward only): finite-difference checks, and the
    loss of every utterance of the full-size GPU parity checks."""
    f = np.asarray(f, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    W_f = np.asarray(W_f, dtype=np.float64)
    W_g = np.asarray(W_g, dtype=np.float64)
    W_o = np.asarray(W_o, dtype=np.float64)
    b_o = np.asarray(b_o, dtype=np.float64)
    B = f.shape[0]
    V, H = W_o.shape
    out = np.empty(B)
    for b in range(B):
        Tb, Ub = int(T_len[b]), int(U_len[b])
        F, G = projections(f[b, :Tb], g[b, :Ub + 1], W_f, W_g)
        blank_lp = np.empty((Tb, Ub + 1))
        label_lp = np.full((Tb, Ub + 1), NEG_INF)
        step = _frame_block(Ub, V, H)           # a block of frames at a time, only to bound memory
        for t0 in range(0, Tb, step):
            t1 = min(Tb, t0 + step)
            _, z = joint_logits(F[t0:t1], G, W_o, b_o)
            lse = log_sum_exp_last(z)
            blank_lp[t0:t1] = z[:, :, blank] - lse
            for u in range(Ub):
                label_lp[t0:t1, u] = z[:, u, int(labels[b, u])] - lse[:, u]
        mask = None if bounds is None else band_mask(bounds[b], S, Tb, Ub)
        if loss == "viterbi":
            A, _ = viterbi_lattice(blank_lp, label_lp, Tb, Ub, mask)
        else:
            A = alpha_lattice(blank_lp, label_lp, Tb, Ub, mask)
        out[b] = -(A[Tb - 1, Ub] + blank_lp[Tb - 1, Ub])
    return out
