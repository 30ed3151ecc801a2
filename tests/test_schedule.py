"""Verify-length scheduler (CPU only: the scheduler is host logic).

mkdocs.reaper.mx DeepSeek-V4.1-Flash "06-extensions", DSpark table: the
scheduler combines the confidence head's prefix survival probabilities with
throughput curves measured beforehand to maximise expected throughput under
the current load; aigest.pl "DeepSeek prezentuje DSpark", "Optymalizacja
weryfikacji i wydajności": the curve is SPS(B), and idle GPUs verify more
tokens while busy ones verify fewer.

The exhaustive oracle (``oracle.schedule``) is pinned by a hand-worked case,
the two load extremes (a flat curve verifies every position with a positive
survival, a curve that drops to zero past the minimum verifies one position
per request) and the load monotonicity the pages state.  The library's
spec_schedule_verify_len is then compared with it on every small shape and on
random curves, and checked for local optimality at serving sizes."""
import math
import time

import numpy as np
import pytest

from oracle import schedule as OS

import draft_sampling_verification_head_b200 as sd


# ----------------------------------------------------------------------------- oracle pins

def test_oracle_hand_worked_case():
    """B = 2, K = 2, survivals (1, 1/2) and (1, 1/4); SPS 10, 9, 7 steps/s at
    4, 5, 6 target rows.  Allocations: (1,1) 4 * 10 = 40, (2,1) 4.5 * 9 = 40.5,
    (1,2) 4.25 * 9 = 38.25, (2,2) 4.75 * 7 = 33.25."""
    conf = [[1.0, 0.5], [1.0, 0.25]]
    sps = [0, 0, 0, 0, 10.0, 9.0, 7.0]
    assert OS.throughput(conf, sps, [1, 1]) == 40.0
    assert OS.throughput(conf, sps, [2, 1]) == 40.5
    assert OS.throughput(conf, sps, [1, 2]) == 38.25
    assert OS.throughput(conf, sps, [2, 2]) == 33.25
    assert OS.best(conf, sps) == (40.5, 3)


def test_oracle_survival_clamps_and_stops_at_nan():
    S = OS.survival([[0.5, 2.0, -1.0], [np.nan, 1.0, 1.0]])
    np.testing.assert_array_equal(S, [[0.5, 0.5, 0.0], [0.0, 0.0, 0.0]])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_oracle_load_extremes(seed):
    rng = np.random.default_rng(seed)
    B, K = 3, 4
    conf = rng.uniform(0.05, 1.0, size=(B, K))
    # idle: the cost does not grow with the batch, every positive survival pays
    flat = np.ones(B * (K + 1) + 1)
    t, m = OS.best(conf, flat)
    assert m == B * K
    assert math.isclose(t, B + OS.survival(conf).sum(), rel_tol=1e-12)
    # saturated: no capacity past one position per request
    steep = np.zeros(B * (K + 1) + 1)
    steep[2 * B] = 5.0
    t, m = OS.best(conf, steep)
    assert m == B
    assert math.isclose(t, 5.0 * (B + OS.survival(conf)[:, 0].sum()), rel_tol=1e-12)


def test_oracle_zero_survival_is_never_verified():
    """A position with survival 0 adds no expected token; with a flat curve the
    smallest-total rule leaves it out."""
    conf = [[0.9, 0.0, 0.9], [0.8, 0.8, 0.8]]
    t, m = OS.best(conf, np.ones(20))
    assert m == 1 + 3


def _sps_curve(lam, n):
    m = np.arange(n, dtype=np.float64)
    return 1.0 / (1.0 + lam * m)


def test_oracle_busier_engine_verifies_fewer():
    """SPS(m) = 1 / (1 + lam m): a larger lam is a busier engine (each extra row
    costs more).  The chosen total never grows with lam (the objective has
    decreasing differences in (total, lam))."""
    rng = np.random.default_rng(7)
    conf = rng.uniform(0.3, 1.0, size=(3, 3))
    totals = [OS.best(conf, _sps_curve(lam, 20))[1] for lam in (0.0, 0.02, 0.1, 0.3, 1.0, 5.0)]
    assert totals == sorted(totals, reverse=True)
    assert totals[0] == 9 and totals[-1] == 3


# ----------------------------------------------------------------------------- library vs oracle

def _random_conf(rng, B, K):
    c = rng.uniform(0.0, 1.0, size=(B, K))
    c[rng.random((B, K)) < 0.1] = 1.0
    c[rng.random((B, K)) < 0.05] = 0.0
    c[rng.random((B, K)) < 0.03] = 1.3      # out-of-range scores are clamped
    c[rng.random((B, K)) < 0.03] = np.nan
    return c.astype(np.float32)


def _random_sps(rng, n):
    kind = rng.integers(3)
    m = np.arange(n, dtype=np.float64)
    if kind == 0:
        return 1.0 / (1.0 + rng.uniform(0, 0.5) * m)
    if kind == 1:   # flat up to a capacity, then falling
        cap = rng.integers(0, n)
        return 1.0 / (1.0 + np.maximum(m - cap, 0))
    return rng.uniform(0.1, 1.0, size=n)    # any measured table


def _all_throughputs(conf, sps):
    B, K = conf.shape
    import itertools
    return {kb: OS.throughput(conf, sps, kb)
            for kb in itertools.product(range(1, K + 1), repeat=B)}


@pytest.mark.parametrize("B,K", [(1, 1), (1, 5), (2, 3), (3, 3), (4, 2), (3, 4)])
def test_library_matches_exhaustive_search(B, K):
    rng = np.random.default_rng(100 * B + K)
    for trial in range(25):
        conf = _random_conf(rng, B, K)
        n = int(rng.integers(2 * B, B * (K + 1) + 3))
        sps = _random_sps(rng, n)
        kb, e, t = sd.schedule_verify_len(conf, sps)
        top, top_m = OS.best(conf, sps)
        assert kb.shape == (B,) and kb.min() >= 1 and kb.max() <= K
        assert math.isclose(t, top, rel_tol=1e-12, abs_tol=1e-300), (conf, sps, kb, t, top)
        assert math.isclose(OS.throughput(conf, sps, kb), t, rel_tol=1e-12, abs_tol=1e-300)
        S = OS.survival(conf)
        assert math.isclose(e, sum(1 + S[b, :kb[b]].sum() for b in range(B)), rel_tol=1e-12)
        # the smallest total among the maxima, unless another total is within rounding
        allt = _all_throughputs(conf, sps)
        rivals = {sum(k) for k, v in allt.items()
                  if sum(k) != top_m and abs(v - top) <= 1e-9 * max(top, 1e-300)}
        if not rivals:
            assert int(kb.sum()) == top_m


def test_library_prefers_larger_survival_then_lower_row():
    """Equal objective, equal total: the position with the larger survival
    goes first, and between equal survivals the lower row."""
    sps = np.array([0, 0, 0, 0, 1.0, 1.0, 0.0])
    kb, _, _ = sd.schedule_verify_len(np.array([[1, 0.5], [1, 0.75]], np.float32), sps)
    assert kb.tolist() == [1, 2]
    kb, _, _ = sd.schedule_verify_len(np.array([[1, 0.5], [1, 0.5]], np.float32), sps)
    assert kb.tolist() == [2, 1]


@pytest.mark.parametrize("B,K", [(64, 16), (256, 8), (128, 32)])
def test_library_local_optimum_at_serving_sizes(B, K):
    """No single change of one request's length by one improves the objective,
    and the result beats every uniform length."""
    rng = np.random.default_rng(B + K)
    depth = np.linspace(0.97, 0.6, K)
    conf = np.clip(depth + rng.normal(0, 0.05, size=(B, K)), 0, 1).astype(np.float32)
    n = B * (K + 1) + 1
    m = np.arange(n, dtype=np.float64)
    sps = 1.0 / (0.02 + 2e-5 * np.maximum(m - 512, 0))  # flat to 512 rows, then linear
    kb, e, t = sd.schedule_verify_len(conf, sps)
    assert math.isclose(OS.throughput(conf, sps, kb), t, rel_tol=1e-10)
    for b in range(B):
        for d in (-1, 1):
            k2 = kb.copy()
            k2[b] += d
            if 1 <= k2[b] <= K:
                assert OS.throughput(conf, sps, k2) <= t * (1 + 1e-12)
    for k in range(1, K + 1):
        assert OS.throughput(conf, sps, np.full(B, k)) <= t * (1 + 1e-12)


def test_library_cost_at_the_largest_shape():
    B, K = 4096, 64
    rng = np.random.default_rng(3)
    conf = rng.uniform(0.5, 1.0, size=(B, K)).astype(np.float32)
    sps = 1.0 / (1.0 + 1e-4 * np.arange(B * (K + 1) + 1))
    t0 = time.perf_counter()
    kb, _, _ = sd.schedule_verify_len(conf, sps)
    dt = time.perf_counter() - t0
    assert 1 <= kb.min() and kb.max() <= K
    assert dt < 5.0


@pytest.mark.parametrize("conf,sps", [
    (np.zeros((0, 3)), np.ones(4)),
    (np.zeros((2, 0)), np.ones(4)),
    (np.ones((2, 3)), np.ones(0)),
    (np.ones((2, 3)), np.array([1.0, -1.0, 1.0])),
    (np.ones((2, 3)), np.array([1.0, np.nan])),
    (np.ones((2, 3)), np.array([1.0, np.inf])),
])
def test_library_rejects_bad_arguments(conf, sps):
    with pytest.raises(sd.SpecError) as ei:
        sd.schedule_verify_len(conf, sps)
    assert ei.value.code == sd.SPEC_ERR_INVALID_ARG
