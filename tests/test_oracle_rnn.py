"""Pins of the oracle's RNN sequential head (aigest.pl "DeepSeek prezentuje
DSpark", section "Innowacje w tworzeniu tokenów": an optional RNN head tracks
the whole block prefix; the Markov head sees only the previous token).

* The enumerated law of one cycle with the recurrent state carried along each
  prefix (exact_law with Wh) is lossless, and the oracle's draws match it
  (chi-square); the oracle planted with a state that forgets the prefix fails.
  The inputs are small dyadic values, so the fp32 recurrence is exact and the
  enumeration in fp64 holds the same state.
* With Wh = 0 the head reduces to the Markov head on U' = bf16(clamp(U, -1, 1)),
  U' made by torch's bf16 conversion (round to nearest even): every output is
  equal."""
import numpy as np
import pytest
import torch
from scipy import stats

import synth
from oracle import exact_law as EL

V, K, R = 6, 3, 4


def _dyadic(g, shape, lo, hi):
    """Multiples of 1/8 in [lo, hi]."""
    n = torch.randint(int(lo * 8), int(hi * 8) + 1, shape, generator=g)
    return (n.to(torch.float32) / 8.0)


def _rnn_inputs(seed):
    w = synth.Workload("rnn", B=1, K=K, V=V, r=R, dtype="f32", sigma=0.8, seed=seed)
    d = synth.make(w)
    g = torch.Generator().manual_seed(seed + 1)
    d["U"] = _dyadic(g, (V, R), -1.25, 1.25)
    d["W"] = _dyadic(g, (R, V), -1.0, 1.0)
    Wh = _dyadic(g, (R, R), -0.5, 0.5)
    return w, d, Wh


def _law(d, Wh):
    f = synth.as_float64
    return EL.exact_law(f(d["base"])[0], f(d["target"])[0], f(d["U"]), f(d["W"]),
                        int(d["last_token"][0]), 1.0, Wh=Wh.double().numpy())


@pytest.mark.parametrize("seed", [41, 42])
def test_rnn_law_is_lossless(seed):
    w, d, Wh = _rnn_inputs(seed)
    law = _law(d, Wh)
    assert abs(sum(law.values()) - 1.0) < 1e-12
    P = [EL.softmax(synth.as_float64(d["target"])[0][i], 1.0) for i in range(K + 1)]
    for (i, prefix), (mass, dist) in EL.conditional_marginals(law, K).items():
        for v in range(V):
            assert abs(dist.get(v, 0.0) - P[i][v]) < 1e-12


def test_rnn_state_depends_on_the_whole_prefix():
    """Two prefixes ending in the same token give different draft laws at the
    next position (the Markov head could not tell them apart)."""
    w, d, Wh = _rnn_inputs(41)
    f = synth.as_float64
    U, Wn = f(d["U"]), Wh.double().numpy()
    last = int(d["last_token"][0])
    s0 = EL.rnn_state(U, Wn, last, None)
    a = EL.rnn_state(U, Wn, 2, EL.rnn_state(U, Wn, 0, s0))
    b = EL.rnn_state(U, Wn, 2, EL.rnn_state(U, Wn, 5, s0))
    assert np.abs(a - b).max() > 0.1


def _pvalues(orc, d, Wh, n, handle=None):
    base = d["base"][:1].expand(n, -1, -1).contiguous()
    target = d["target"][:1].expand(n, -1, -1).contiguous()
    last = d["last_token"][:1].expand(n).contiguous()
    P = orc.Params(B=n, K=K, V=V, r=R, dtype="f32", temperature=1.0, seed=17, cycle=2,
                   Wh=Wh.numpy())
    raw = synth.to_numpy_raw
    o = orc.cycle(P, raw(base), raw(target), raw(d["U"]), raw(d["W"]), last.numpy(), handle=handle)
    first, pair, taus = EL.cell_probs(_law(d, Wh), K, V)
    out, tau = o["out"], o["tau"]
    sel = tau >= 2

    def pooled(obs, p, m):
        e = p * m
        keep = e >= 5
        o_ = np.append(obs[keep], obs[~keep].sum())
        e_ = np.append(e[keep], e[~keep].sum())
        if e_[-1] == 0:
            o_, e_ = o_[:-1], e_[:-1]
        return stats.chisquare(o_, e_ * o_.sum() / e_.sum()).pvalue

    return [pooled(np.bincount(out[:, 0], minlength=V), first, n),
            pooled(np.bincount(out[sel, 0] * V + out[sel, 1], minlength=V * V),
                   pair.ravel() / pair.sum(), int(sel.sum())),
            pooled(np.bincount(tau - 1, minlength=K + 1), taus, n)]


@pytest.mark.parametrize("seed", [41, 42])
def test_rnn_oracle_samples_match_the_law(orc, seed):
    w, d, Wh = _rnn_inputs(seed)
    pv = _pvalues(orc, d, Wh, 100_000)
    assert min(pv) > 1e-3, pv


def test_rnn_planted_forgetful_state_is_rejected(orc, tmp_path):
    w, d, Wh = _rnn_inputs(41)
    h = orc.build_planted(4, str(tmp_path))
    pv = _pvalues(orc, d, Wh, 100_000, handle=h)
    assert min(pv) < 1e-6, pv


@pytest.mark.parametrize("greedy", [False, True])
def test_rnn_with_zero_recurrence_is_markov_on_clamped_rounded_U(orc, greedy):
    w = synth.Workload("rnn0", B=6, K=4, V=300, r=16, dtype="bf16", sigma=0.6, seed=43, uw_std=0.9)
    d = synth.make(w)
    raw = synth.to_numpy_raw
    Uc = torch.clamp(d["U"].float(), -1.0, 1.0).to(torch.bfloat16)
    assert not torch.equal(Uc, d["U"])  # the clamp and the rounding both act
    Wh0 = torch.zeros((w.r, w.r), dtype=torch.bfloat16)
    kw = dict(B=w.B, K=w.K, V=w.V, r=w.r, dtype="bf16", temperature=1.0, greedy=greedy, seed=5,
              cycle=1)
    a = orc.cycle(orc.Params(**kw, Wh=raw(Wh0)), raw(d["base"]), raw(d["target"]), raw(d["U"]),
                  raw(d["W"]), d["last_token"].numpy())
    b = orc.cycle(orc.Params(**kw), raw(d["base"]), raw(d["target"]), raw(Uc), raw(d["W"]),
                  d["last_token"].numpy())
    for k in ("draft", "out", "tau", "flag_draft", "flag_accept", "flag_final"):
        assert np.array_equal(a[k], b[k]), k
    np.testing.assert_array_equal(a["q_draft"], b["q_draft"])
