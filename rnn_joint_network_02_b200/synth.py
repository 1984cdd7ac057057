"""Seeded synthetic inputs shaped like short / medium / long ASR batches.

This module holds none of the joint's or the loss's arithmetic: it only draws
lengths, labels, activations and weights from a seeded CPU generator, in a
fixed order, and rounds float inputs to bf16 once (round-to-nearest-even)
when the workload is a bf16 one.  The CUDA path and the fp64 oracle both
consume exactly these values.

Draw order (one ``torch.Generator`` seeded per workload):
lengths T_len, U_len -> labels -> f -> g -> W_f -> W_g -> W_o -> b_o.

Distributions:
* f, g ~ N(0, 1); W_f ~ N(0, 1/D_enc); W_g ~ N(0, 1/D_pred); W_o ~ N(0, 1/H);
  b_o = 0 unless ``bias_std`` > 0.
* T_len uniform on an inclusive integer range; U_len either uniform on an
  inclusive range, tied to T_len (min(U, max(1, T_len // 5))), or full.
* labels uniform on 1..V-1, or Zipf(s) over 1..V-1 (P(k) proportional to
  k^-s, label id = k).  blank = 0 never appears as a label.
* Positions past T_len / U_len hold values from the same draws (padding); the
  library must ignore them.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

# name -> (index, shape and distribution recipe).  The index fixes the seed.
WORKLOADS = {
    "tiny": dict(index=0, B=2, T=12, U=5, D_enc=16, D_pred=16, H=32, V=8, dtype="f32",
                 T_range=(12, 12), U_rule="full", labels="uniform"),
    "short": dict(index=1, B=8, T=100, U=20, D_enc=256, D_pred=256, H=256, V=128, dtype="bf16",
                  T_range=(50, 100), U_range=(10, 20), labels="uniform"),
    "medium": dict(index=2, B=16, T=400, U=80, D_enc=512, D_pred=640, H=640, V=1024, dtype="bf16",
                   T_range=(200, 400), U_rule="T/5", labels="uniform"),
    "long": dict(index=3, B=8, T=1500, U=300, D_enc=512, D_pred=640, H=640, V=1024, dtype="bf16",
                 T_range=(1000, 1500), U_rule="T/5", labels="uniform"),
    "large": dict(index=4, B=32, T=250, U=60, D_enc=1024, D_pred=1024, H=1024, V=4096, dtype="bf16",
                  T_range=(150, 250), U_range=(30, 60), labels="zipf", zipf_s=1.1),
}


@dataclass
class Batch:
    """One synthetic batch (CPU tensors).  Float tensors are float32 for an
    f32 workload and bfloat16 for a bf16 one; ints are int32."""
    f: torch.Tensor
    g: torch.Tensor
    W_f: torch.Tensor
    W_g: torch.Tensor
    W_o: torch.Tensor
    b_o: torch.Tensor
    labels: torch.Tensor
    T_len: torch.Tensor
    U_len: torch.Tensor
    dtype: str
    blank: int = 0

    @property
    def dims(self):
        B, T, D_enc = self.f.shape
        U = self.g.shape[1] - 1
        D_pred = self.g.shape[2]
        V, H = self.W_o.shape
        return dict(B=B, T=T, U=U, D_enc=D_enc, D_pred=D_pred, H=H, V=V)

    def tensors(self):
        return (self.f, self.g, self.W_f, self.W_g, self.W_o, self.b_o)

    def float64(self):
        """The same values as float64 tensors (exact: bf16/f32 embed in f64)."""
        return tuple(t.double() for t in self.tensors())

    def valid_cells(self) -> int:
        return int((self.T_len.long() * (self.U_len.long() + 1)).sum())

    def padded_cells(self) -> int:
        d = self.dims
        return d["B"] * d["T"] * (d["U"] + 1)


def _uniform_int(gen, lo: int, hi: int, n: int) -> torch.Tensor:
    return torch.randint(lo, hi + 1, (n,), generator=gen, dtype=torch.int64)


def make(B: int, T: int, U: int, D_enc: int, D_pred: int, H: int, V: int, dtype: str = "bf16",
         seed: int = 0, T_range=None, U_range=None, U_rule: str = "range", labels: str = "uniform",
         zipf_s: float = 1.1, bias_std: float = 0.0, blank: int = 0, index: int | None = None) -> Batch:
    """Draw one batch.  ``U_rule`` is "range" (uniform on ``U_range``),
    "T/5" (U_len = min(U, max(1, T_len // 5))) or "full" (U_len = U)."""
    gen = torch.Generator().manual_seed(seed)
    lo, hi = T_range if T_range is not None else (T, T)
    T_len = _uniform_int(gen, lo, hi, B)
    if U_rule == "full":
        U_len = torch.full((B,), U, dtype=torch.int64)
    elif U_rule == "T/5":
        U_len = torch.clamp(T_len // 5, min=1, max=U)
    else:
        ulo, uhi = U_range if U_range is not None else (U, U)
        U_len = _uniform_int(gen, ulo, uhi, B)
    if labels == "zipf":
        k = torch.arange(1, V, dtype=torch.float64)
        p = k.pow(-zipf_s)
        lab = torch.multinomial(p / p.sum(), B * max(U, 1), replacement=True, generator=gen) + 1
        lab = lab.view(B, max(U, 1))[:, :U]
    else:
        lab = torch.randint(1, V, (B, U), generator=gen, dtype=torch.int64)
    if blank != 0:
        # keep labels off the blank id: map blank -> 0 (0 is a label when blank != 0)
        lab = torch.where(lab == blank, torch.zeros_like(lab), lab)
    f = torch.randn(B, T, D_enc, generator=gen, dtype=torch.float32)
    g = torch.randn(B, U + 1, D_pred, generator=gen, dtype=torch.float32)
    W_f = torch.randn(D_enc, H, generator=gen, dtype=torch.float32) / D_enc ** 0.5
    W_g = torch.randn(D_pred, H, generator=gen, dtype=torch.float32) / D_pred ** 0.5
    W_o = torch.randn(V, H, generator=gen, dtype=torch.float32) / H ** 0.5
    if bias_std > 0:
        b_o = torch.randn(V, generator=gen, dtype=torch.float32) * bias_std
    else:
        b_o = torch.zeros(V, dtype=torch.float32)
    tt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return Batch(f=f.to(tt), g=g.to(tt), W_f=W_f.to(tt), W_g=W_g.to(tt), W_o=W_o.to(tt),
                 b_o=b_o.to(tt), labels=lab.to(torch.int32), T_len=T_len.to(torch.int32),
                 U_len=U_len.to(torch.int32), dtype=dtype, blank=blank)


def workload(name: str, seed: int | None = None, **overrides) -> Batch:
    """The named workload with seed 1000 + its index (or ``seed``)."""
    spec = dict(WORKLOADS[name])
    idx = spec.pop("index")
    spec.update(overrides)
    return make(seed=1000 + idx if seed is None else seed, **spec)


def redraw_padding(batch: Batch, seed: int) -> Batch:
    """Same batch with every padding position (t >= T_len, u > U_len, label
    positions u >= U_len) overwritten by other values, including labels that
    would be invalid if they were read."""
    gen = torch.Generator().manual_seed(seed)
    f = batch.f.clone()
    g = batch.g.clone()
    lab = batch.labels.clone()
    B, T, _ = f.shape
    U = g.shape[1] - 1
    V = batch.W_o.shape[0]
    for b in range(B):
        Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
        if Tb < T:
            f[b, Tb:] = (torch.randn(T - Tb, f.shape[2], generator=gen) * 7).to(f.dtype)
        if Ub < U:
            g[b, Ub + 1:] = (torch.randn(U - Ub, g.shape[2], generator=gen) * 7).to(g.dtype)
            lab[b, Ub:] = torch.randint(-3 * V, 3 * V, (U - Ub,), generator=gen).to(torch.int32)
    return Batch(f=f, g=g, W_f=batch.W_f, W_g=batch.W_g, W_o=batch.W_o, b_o=batch.b_o,
                 labels=lab, T_len=batch.T_len, U_len=batch.U_len, dtype=batch.dtype,
                 blank=batch.blank)


def diagonal_bounds(T_len, U_len, T: int, S: int) -> torch.Tensor:
    """Pruning-bound inputs: a band of S label positions per frame that follows
    the lattice's diagonal, s[b,t] = min(U_len, max(0, floor(t (U_len+1) / T_len) - S // 2)),
    int32 [B, T]; padding frames repeat the last frame's start.  (The pages
    obtain bounds from a linear joiner; here they are synthetic inputs.)"""
    B = len(T_len)
    s = torch.zeros(B, T, dtype=torch.int32)
    for b in range(B):
        Tb, Ub = int(T_len[b]), int(U_len[b])
        for t in range(T):
            tt = min(t, Tb - 1)
            s[b, t] = min(Ub, max(0, (tt * (Ub + 1)) // Tb - S // 2))
    return s


# Duration set of the token-and-duration transducer workloads: 0 .. 4 frames.
TDT_DURATIONS = (0, 1, 2, 3, 4)


def duration_head(batch: Batch, n_dur: int, seed: int, bias_std: float = 0.5):
    """Weights of a duration output head for ``batch``: W_d ~ N(0, 1/H) of shape
    [n_dur, H] and b_d ~ N(0, bias_std^2) of shape [n_dur], from their own
    generator (seeded ``seed``), rounded to the batch's float type."""
    gen = torch.Generator().manual_seed(seed)
    H = batch.W_o.shape[1]
    W_d = torch.randn(n_dur, H, generator=gen, dtype=torch.float32) / H ** 0.5
    b_d = torch.randn(n_dur, generator=gen, dtype=torch.float32) * bias_std
    tt = torch.bfloat16 if batch.dtype == "bf16" else torch.float32
    return W_d.to(tt), b_d.to(tt)
