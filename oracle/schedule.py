"""Verify-length scheduler by exhaustive search -- TEST INFRASTRUCTURE ONLY.

mkdocs.reaper.mx DeepSeek-V4.1-Flash "06-extensions", DSpark table: the
scheduler combines the prefix survival probabilities estimated by the
confidence head with the engine's throughput curves measured beforehand, to
maximise the expected system throughput under the current load; aigest.pl
"Optymalizacja weryfikacji i wydajności": the curve is SPS(B), profiled once
at start-up.

Reading (the plain definition): for verify lengths k_b in 1..K,
  expected tokens E = sum_b (1 + sum_{i < k_b} S_{b,i}),
  S_{b,i} = prod_{j <= i} clamp(c_{b,j}, 0, 1)   (a NaN score counts as 0),
  throughput = E * SPS(sum_b (k_b + 1)),
SPS(m) being steps per second of a target forward over m tokens (the bonus
position included), 0 past the profiled range.  The schedule maximises the
throughput; among equal maxima the smallest total length.  Here every
allocation is enumerated (small B and K only)."""
from __future__ import annotations

import itertools

import numpy as np


def survival(conf) -> np.ndarray:
    c = np.asarray(conf, np.float64)
    c = np.where(np.isnan(c), 0.0, np.clip(c, 0.0, 1.0))
    return np.cumprod(c, axis=-1)


def throughput(conf, sps, kb) -> float:
    S = survival(conf)
    kb = np.asarray(kb)
    E = sum(1.0 + S[b, :kb[b]].sum() for b in range(len(kb)))
    m = int((kb + 1).sum())
    return E * (float(sps[m]) if m < len(sps) else 0.0)


def best(conf, sps):
    """(best throughput, smallest total length reaching it) over all allocations."""
    B, K = np.asarray(conf).shape
    top, top_m = -1.0, None
    for kb in itertools.product(range(1, K + 1), repeat=B):
        t = throughput(conf, sps, kb)
        m = sum(kb)
        if t > top * (1 + 1e-12) or (abs(t - top) <= 1e-12 * max(1.0, top) and m < top_m):
            top, top_m = t, m
    return top, top_m
