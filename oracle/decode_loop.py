"""Multi-cycle decode loop and the confidence-driven verify length --
TEST INFRASTRUCTURE ONLY (same rules as the rest of this package: only the
test suite, the smoke check and the benchmark's CPU-baseline leg may use it).

* aigest.pl "DeepSeek prezentuje DSpark", section "Jak działa spekulatywne
  dekodowanie DSpark?": decoding runs cycle after cycle (draft a block, verify
  it), with per-token latency L = (T_draft + T_verify) / tau.  Reading: the
  token a cycle emits last (its correction or its bonus token) is the
  committed token the next cycle's Markov head starts from, and every cycle
  draws fresh random numbers (Philox cycle counter = first cycle + c).
* same page, section "Optymalizacja weryfikacji i wydajności": a confidence
  head scores each draft position with the chance that its token survives
  verification given that its predecessors were accepted, and the scheduler
  sets each request's verify length from those scores with an early-stopping
  rule; mkdocs.reaper.mx DeepSeek-V4.1-Flash "06-extensions", DSpark table:
  the scheduler combines the prefix survival probabilities.  Reading: the
  prefix survival of position i is the product of the scores of positions
  0..i; the verify length K_b is the number of leading positions whose prefix
  survival is at least a threshold, and at least 1.  The product is taken in
  fp32, in position order (the precision the CUDA path decides it in).

Each cycle is one call of the oracle's pinned cycle (``oracle.cycle``); this
module only chains them.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import Params, cycle


def prefix_verify_len(conf, threshold) -> np.ndarray:
    """K_b per row from confidence scores conf [..., K] (float32): the number
    of leading positions i with fp32 prod(conf[..., 0..i]) >= threshold, at
    least 1.  A NaN score ends the prefix (the comparison is false)."""
    c = np.asarray(conf, dtype=np.float32)
    thr = np.float32(threshold)
    lead = c.shape[:-1]
    K = c.shape[-1]
    flat = c.reshape(-1, K)
    kb = np.empty(flat.shape[0], np.int32)
    for n in range(flat.shape[0]):
        s = np.float32(1.0)
        k = 0
        for i in range(K):
            s = np.float32(s * flat[n, i])
            if not (s >= thr):
                break
            k = i + 1
        kb[n] = max(k, 1)
    return kb.reshape(lead)


def decode_loop(P: Params, n_cycles: int, base, target, U, W, last_token, conf=None,
                threshold=0.0, verify_len=None, _plant=None):
    """Run n_cycles cycles.  base [C, B, K, V], target [C, B, K+1, V] (raw
    storage as for ``oracle.cycle``), U, W shared, last_token [B] for the
    first cycle.  The verify length of cycle c comes from conf [C, B, K] and
    the threshold, or from verify_len [C, B], or is K.

    Returns per-cycle outputs stacked on a leading axis (draft, out, tau,
    p_draft, q_draft, flag_*), kb [C, B] and next_token [B] (the last token of
    the last cycle).  ``_plant`` deliberately breaks the chaining, to show the
    pins would catch it: "no_chain" restarts every cycle from the first
    last_token, "same_cycle" reuses the first cycle's random counter."""
    assert conf is None or verify_len is None
    lt = np.ascontiguousarray(last_token, dtype=np.int32).copy()
    res = []
    kbs = []
    for c in range(n_cycles):
        if conf is not None:
            kb = prefix_verify_len(np.asarray(conf)[c], threshold)
        elif verify_len is not None:
            kb = np.ascontiguousarray(np.asarray(verify_len)[c], dtype=np.int32)
        else:
            kb = np.full(P.B, P.K, np.int32)
        cyc = P.cycle if _plant == "same_cycle" else P.cycle + c
        Pc = dataclasses.replace(P, cycle=cyc, verify_len=kb)
        o = cycle(Pc, base[c], target[c], U, W, lt)
        res.append(o)
        kbs.append(kb)
        if _plant != "no_chain":
            lt = o["out"][np.arange(P.B), o["tau"] - 1].astype(np.int32)
    out = {k: np.stack([o[k] for o in res]) for k in res[0] if k != "threads"}
    out["kb"] = np.stack(kbs)
    out["next_token"] = res[-1]["out"][np.arange(P.B), res[-1]["tau"] - 1].astype(np.int32)
    return out
