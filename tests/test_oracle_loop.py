"""Pins of the oracle's multi-cycle decode loop and of its confidence-driven
verify length (aigest.pl "DeepSeek prezentuje DSpark": cycles of draft and
verify with L = (T_draft + T_verify) / tau, section "Jak działa spekulatywne
dekodowanie DSpark?"; per-position survival scores feeding the verify length,
section "Optymalizacja weryfikacji i wydajności").

The loop is pinned against the enumerated joint law of two chained cycles
(each cycle's law enumerated by ``oracle.exact_law``, which the single-cycle
pins fix), so a loop that does not feed each cycle's last emitted token into
the next cycle's Markov head, or that reuses the random numbers of the
previous cycle, fails.  The verify-length rule is pinned by hand-worked cases
in exactly representable binary fractions and by exact rational arithmetic."""
from fractions import Fraction

import numpy as np
import pytest
from scipy import stats

import synth
from oracle import exact_law as EL


@pytest.fixture(scope="module")
def dl(orc):
    from oracle import decode_loop
    return decode_loop


# ----------------------------------------------------------------------------- verify length

@pytest.mark.parametrize("conf,thr,kb", [
    ([1.0, 1.0, 1.0, 1.0], 0.9, 4),     # every prefix survives
    ([1.0, 0.5, 0.5, 0.5], 0.25, 3),    # survival 1, 1/2, 1/4, 1/8
    ([0.25, 1.0, 1.0, 1.0], 0.25, 4),   # equal to the threshold counts
    ([0.5, 1.0, 1.0, 1.0], 0.75, 1),    # nothing survives: one position all the same
    ([0.75, 0.5, 1.0, 1.0], 0.375, 4),  # 3/4 * 1/2 = 3/8 exactly
    ([0.75, 0.5, 1.0, 1.0], 0.3751, 1),
    ([1.0, 1.0, np.nan, 1.0], 0.5, 2),  # a NaN score ends the prefix
    ([0.1, 0.2, 0.3, 0.4], 0.0, 4),     # threshold 0: the whole block
    ([1.0, 1.0, 1.0, 1.0], 1.5, 1),     # a threshold above 1: the minimum
    ([0.5, 2.0, 0.25, 1.0], 0.5, 2),    # scores are used as given (no clamping): 1/2, 1, 1/4
])
def test_prefix_verify_len_worked_cases(dl, conf, thr, kb):
    assert int(dl.prefix_verify_len(np.array([conf], np.float32), thr)[0]) == kb


def test_prefix_verify_len_against_exact_products(dl):
    """fp32 products agree with exact rational products of the same fp32 scores
    except where the survival lies within K ulps of the threshold."""
    rng = np.random.default_rng(11)
    K = 12
    conf = rng.uniform(0.6, 1.0, size=(4000, K)).astype(np.float32)
    thr = np.float32(0.3)
    kb = dl.prefix_verify_len(conf, thr)
    T = Fraction(float(thr))
    near = 0
    for n in range(conf.shape[0]):
        s = Fraction(1)
        k = 0
        close = False
        for i in range(K):
            s *= Fraction(float(conf[n, i]))
            if abs(s - T) <= Fraction(K, 1 << 23) * T:
                close = True
            if s < T:
                break
            k = i + 1
        if close:
            near += 1
            continue
        assert kb[n] == max(k, 1), (n, kb[n], k)
    assert near < 20


def test_prefix_verify_len_monotone(dl):
    rng = np.random.default_rng(12)
    conf = rng.uniform(0.3, 1.0, size=(500, 8)).astype(np.float32)
    prev = None
    for thr in (0.0, 0.05, 0.2, 0.4, 0.7, 0.95, 1.0):
        kb = dl.prefix_verify_len(conf, thr)
        assert kb.min() >= 1 and kb.max() <= 8
        if prev is not None:
            assert np.all(kb <= prev)
        prev = kb
    # raising one score never shortens the prefix
    up = conf.copy()
    up[:, 3] = np.minimum(1.0, up[:, 3] + 0.2)
    assert np.all(dl.prefix_verify_len(up, 0.3) >= dl.prefix_verify_len(conf, 0.3))


# ----------------------------------------------------------------------------- chained law

V, K, R = 6, 2, 4
# cycle 0 verifies both positions (survival 0.9, 0.81), cycle 1 only the first
# (survival 0.6, 0.36) at threshold 0.5
CONF = np.array([[0.9, 0.9], [0.6, 0.6]], np.float32)
THR = 0.5


def _chain_inputs(seed):
    w = synth.Workload("loop", B=1, K=K, V=V, r=R, dtype="f32", sigma=0.9, seed=seed, uw_std=1.2)
    return w, synth.make_loop(w, 2)


def _chain_law(d, kbs, T=1.0):
    """Exact joint law {((tau0, out0), (tau1, out1)): prob} of two chained cycles."""
    f = synth.as_float64
    U, W = f(d["U"]), f(d["W"])
    law0 = EL.exact_law(f(d["base"][0, 0]), f(d["target"][0, 0]), U, W,
                        int(d["last_token"][0]), T, verify_len=kbs[0])
    law1 = {v: EL.exact_law(f(d["base"][1, 0]), f(d["target"][1, 0]), U, W, v, T,
                            verify_len=kbs[1]) for v in range(V)}
    joint = {}
    for (t0, o0), p0 in law0.items():
        for (t1, o1), p1 in law1[o0[-1]].items():
            joint[((t0, o0), (t1, o1))] = p0 * p1
    return joint


def _loop_draws(orc, dl, d, n, plant=None):
    base = d["base"][:, :1].expand(-1, n, -1, -1).contiguous()
    target = d["target"][:, :1].expand(-1, n, -1, -1).contiguous()
    last = d["last_token"][:1].expand(n).contiguous().numpy()
    conf = np.broadcast_to(CONF[:, None, :], (2, n, K)).copy()
    P = orc.Params(B=n, K=K, V=V, r=R, dtype="f32", temperature=1.0, seed=77, cycle=5)
    return dl.decode_loop(P, 2, synth.to_numpy_raw(base), synth.to_numpy_raw(target),
                          synth.to_numpy_raw(d["U"]), synth.to_numpy_raw(d["W"]), last,
                          conf=conf, threshold=THR, _plant=plant)


def _pooled(obs, p, n):
    e = p * n
    keep = e >= 5
    o_ = np.append(obs[keep], obs[~keep].sum())
    e_ = np.append(e[keep], e[~keep].sum())
    if e_[-1] == 0:
        o_, e_ = o_[:-1], e_[:-1]
    return stats.chisquare(o_, e_ * o_.sum() / e_.sum()).pvalue


def _chain_pvalues(orc, dl, seed, n, plant=None):
    w, d = _chain_inputs(seed)
    o = _loop_draws(orc, dl, d, n, plant)
    kbs = [int(k) for k in o["kb"][:, 0]]
    assert kbs == [2, 1]
    joint = _chain_law(d, kbs)
    assert abs(sum(joint.values()) - 1.0) < 1e-12
    # exact cell probabilities: (first token of cycle 0, first of cycle 1),
    # (last token of cycle 0, first of cycle 1), (tau0, tau1)
    ff = np.zeros((V, V))
    lf = np.zeros((V, V))
    tt = np.zeros((K + 1, K + 1))
    for ((t0, o0), (t1, o1)), p in joint.items():
        ff[o0[0], o1[0]] += p
        lf[o0[-1], o1[0]] += p
        tt[t0 - 1, t1 - 1] += p
    out, tau = o["out"], o["tau"]
    rows = np.arange(n)
    last0 = out[0, rows, tau[0] - 1]
    pv = [_pooled(np.bincount(out[0, :, 0] * V + out[1, :, 0], minlength=V * V), ff.ravel(), n),
          _pooled(np.bincount(last0 * V + out[1, :, 0], minlength=V * V), lf.ravel(), n),
          _pooled(np.bincount((tau[0] - 1) * (K + 1) + tau[1] - 1, minlength=(K + 1) ** 2),
                  tt.ravel(), n)]
    return pv, o


@pytest.mark.parametrize("seed", [31, 32])
def test_loop_samples_match_the_chained_law(orc, dl, seed):
    pv, o = _chain_pvalues(orc, dl, seed, 60000)
    assert min(pv) > 1e-3, pv
    n = o["tau"].shape[1]
    assert np.array_equal(o["next_token"], o["out"][1, np.arange(n), o["tau"][1] - 1])
    assert o["tau"][1].max() <= 2  # verify length 1 in the second cycle


@pytest.mark.parametrize("plant", ["no_chain", "same_cycle"])
def test_loop_pin_rejects_a_broken_chain(orc, dl, plant):
    """A loop that starts every cycle from the first last token, or that reuses
    the first cycle's random counter, fails the chained-law pin."""
    pv, _ = _chain_pvalues(orc, dl, 31, 60000, plant=plant)
    assert min(pv) < 1e-6, pv


def test_loop_of_one_cycle_with_full_length_is_the_cycle(orc, dl):
    """One cycle with every verify length K: the plain cycle with the same
    counters (rows, position, cycle)."""
    w = synth.Workload("loop1", B=7, K=3, V=50, r=8, dtype="f32", sigma=0.6, seed=40, uw_std=0.4)
    d = synth.make_loop(w, 1)
    P = orc.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype="f32", temperature=0.8, seed=9, cycle=12)
    raw = synth.to_numpy_raw
    lo = dl.decode_loop(P, 1, raw(d["base"]), raw(d["target"]), raw(d["U"]), raw(d["W"]),
                        d["last_token"].numpy(), conf=np.ones((1, w.B, w.K), np.float32),
                        threshold=1.0)
    one = orc.cycle(P, raw(d["base"][0]), raw(d["target"][0]), raw(d["U"]), raw(d["W"]),
                    d["last_token"].numpy())
    for k in ("draft", "out", "tau"):
        assert np.array_equal(lo[k][0], one[k]), k
