"""Seeded synthetic inputs for the draft-sample-and-verify step.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the oracle tests and the CUDA tests / benchmark
take their inputs from here.

Recipe (the pages give no logits; the shapes stand in for their workloads):
* K+1 "core" rows per batch row, c_i[v] = N(0, base_std^2) + zeta_v with the
  Zipf(1.1) log-prior zeta_v = -1.1 * ln(v + 1) shared over rows;
* draft base logits = c_0 .. c_{K-1};
* target logits row i = c_i + N(0, sigma_i^2) for i = 0..K (row K, the bonus
  row, has no draft counterpart; it gets its own core row);
* Markov factors U [V, r], W [r, V] ~ N(0, uw_std^2);
* last committed token ~ uniform over [0, V).
Values are drawn in float32 by a seeded torch CPU generator, then rounded to
bfloat16 (round-to-nearest-even) for bf16 workloads.  Bits are identical on
every machine.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass
class Workload:
    name: str
    B: int
    K: int
    V: int
    r: int
    dtype: str            # "bf16" or "f32"
    sigma: object = 0.5   # float, or ("linear", lo, hi) over target rows 0..K
    temperature: float = 1.0
    greedy: bool = False
    seed: int = 0
    base_std: float = 2.0
    uw_std: float = 0.02
    extra: dict = field(default_factory=dict)


# The five benchmark configurations (plus the exact-distribution case).
WORKLOADS = {
    "c1": Workload("c1", B=1, K=4, V=1024, r=16, dtype="f32", sigma=0.5, temperature=1.0, seed=0),
    "c2": Workload("c2", B=8, K=8, V=32000, r=256, dtype="bf16", sigma=0.5, temperature=0.7, seed=1),
    "c3": Workload("c3", B=64, K=16, V=129280, r=256, dtype="bf16", sigma=0.5, temperature=1.0, seed=2),
    "c4": Workload("c4", B=256, K=8, V=151936, r=256, dtype="bf16", sigma=0.5, temperature=1.0, seed=3),
    "c5": Workload("c5", B=128, K=32, V=129280, r=256, dtype="bf16", sigma=("linear", 0.2, 1.5),
                   temperature=1.0, seed=4),
    # exact-distribution case: V=8, K=3; r=4 and U,W ~ N(0, 0.5^2) so the Markov term matters
    "c5b": Workload("c5b", B=1, K=3, V=8, r=4, dtype="f32", sigma=0.5, temperature=1.0, seed=5,
                    uw_std=0.5),
}


def sigmas(w: Workload) -> np.ndarray:
    if isinstance(w.sigma, tuple):
        _, lo, hi = w.sigma
        return np.array([lo + (hi - lo) * i / w.K for i in range(w.K + 1)], np.float32)
    return np.full(w.K + 1, float(w.sigma), np.float32)


def _randn(g, shape):
    return torch.randn(shape, generator=g, dtype=torch.float32)


def make(w: Workload, B: int | None = None, seed: int | None = None):
    """Return a dict of torch CPU tensors: base [B,K,V], target [B,K+1,V],
    U [V,r], W [r,V] (bf16 or f32) and last_token [B] int32."""
    B = w.B if B is None else B
    seed = w.seed if seed is None else seed
    g = torch.Generator().manual_seed(seed)
    K, V, r = w.K, w.V, w.r
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    zeta = -1.1 * torch.log(torch.arange(V, dtype=torch.float64) + 1.0)
    zeta = zeta.to(torch.float32)
    sig = torch.from_numpy(sigmas(w))
    base = torch.empty((B, K, V), dtype=tdt)
    target = torch.empty((B, K + 1, V), dtype=tdt)
    for b in range(B):  # row by row keeps peak memory small
        core = _randn(g, (K + 1, V)) * w.base_std + zeta
        noise = _randn(g, (K + 1, V)) * sig[:, None]
        base[b] = core[:K].to(tdt)
        target[b] = (core + noise).to(tdt)
    U = (_randn(g, (V, r)) * w.uw_std).to(tdt)
    W = (_randn(g, (r, V)) * w.uw_std).to(tdt)
    last = torch.randint(0, V, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    return dict(base=base, target=target, U=U, W=W, last_token=last)


def make_loop(w: Workload, n_cycles: int, B: int | None = None, seed: int | None = None,
              conf_range=(0.5, 1.0)):
    """Inputs of a multi-cycle decode loop: base [C,B,K,V] and target
    [C,B,K+1,V] (cycle c drawn as ``make`` with seed s + c), U, W and
    last_token of cycle 0, and confidence scores conf [C,B,K] float32, uniform
    over conf_range (a stand-in for a trained confidence head's outputs)."""
    seed = w.seed if seed is None else seed
    cyc = [make(w, B=B, seed=seed + 7919 * c) for c in range(n_cycles)]
    B = cyc[0]["base"].shape[0]
    g = torch.Generator().manual_seed(seed + 104729)
    lo, hi = conf_range
    conf = lo + (hi - lo) * torch.rand((n_cycles, B, w.K), generator=g, dtype=torch.float32)
    return dict(base=torch.stack([d["base"] for d in cyc]),
                target=torch.stack([d["target"] for d in cyc]),
                U=cyc[0]["U"], W=cyc[0]["W"], last_token=cyc[0]["last_token"], conf=conf)


def rnn_weights(w: Workload, scale: float | None = None, seed: int | None = None):
    """RNN head recurrence Wh [r, r] ~ N(0, scale^2) (default 1/sqrt(r)), in the
    workload's dtype."""
    g = torch.Generator().manual_seed((w.seed if seed is None else seed) + 31337)
    sc = (1.0 / np.sqrt(w.r)) if scale is None else scale
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return (_randn(g, (w.r, w.r)) * sc).to(tdt)


def to_numpy_raw(t: torch.Tensor) -> np.ndarray:
    """Raw storage for the oracle: bf16 as uint16 bit patterns, f32 as float32."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    return t.numpy()


def as_float64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()
