"""Exact law of one verification block by enumeration -- TEST INFRASTRUCTURE ONLY.

For tiny vocabularies (V <= 8, K <= 3) every accepted draft prefix is
enumerated with its exact probability, and every accept / reject branch is
followed, giving the exact joint law of (tau, emitted tokens).  Written with
numpy in float64 from the verification rule the oracle follows (oracle.h):

* aigest.pl "DeepSeek prezentuje DSpark", "Jak działa spekulatywne dekodowanie
  DSpark?": the longest accepted prefix plus one extra token, exactly
  preserving the target distribution;
* "Innowacje w tworzeniu tokenów": the draft at position i is biased by the
  Markov head on the previous token only.

Given that position i is reached with accepted prefix x_<i, the draft token is
d ~ q_i(.|x_{i-1}); it is accepted with probability min(1, p/q); a rejection
(total probability R = sum_v max(p_i - q_i, 0)) emits x ~ max(p_i - q_i, 0)/R,
so P(reject at i, emit x) = max(p_i(x) - q_i(x), 0).  After K acceptances the
bonus token is drawn from target row K.

``rule`` selects deliberately wrong variants used to show the lossless pin
would catch a mistake: "no_residual" resamples from p instead of the residual,
"ratio_qp" accepts with min(1, q/p).
"""
from __future__ import annotations

from collections import defaultdict

import numpy as np


def softmax(x, T):
    l = np.asarray(x, np.float64) / T
    e = np.exp(l - l.max())
    return e / e.sum()


def draft_q(base, U, W, i, prev, T):
    """q_i(. | prev) = softmax((base_i + U[prev] . W) / T)."""
    z = np.asarray(base[i], np.float64) + np.asarray(U[prev], np.float64) @ np.asarray(W, np.float64)
    return softmax(z, T)


def rnn_state(U, Wh, prev, s_old):
    """RNN head state (float64): clamp(U[prev] + Wh . s_old, -1, 1); s_old None
    at the first position.  Exact for inputs whose sums are exactly
    representable (the pins use small dyadic values)."""
    pre = np.asarray(U[prev], np.float64).copy()
    if s_old is not None:
        pre = pre + np.asarray(Wh, np.float64) @ s_old
    return np.clip(pre, -1.0, 1.0)


def exact_law(base, target, U, W, last_token, T, rule="standard", verify_len=None, Wh=None):
    """Return {(tau, out_tuple): probability} for one batch row.

    base: [K, V], target: [K+1, V], U: [V, r], W: [r, V] (float64-convertible).
    verify_len: the row's verify length K_b (1..K; default K): positions
    0..K_b-1 are drafted and verified, the bonus comes from target row K_b.
    Wh: [r, r] recurrent weights of the RNN head (the bias of position i is
    s_i . W with s_i = rnn_state(U, Wh, prev_i, s_{i-1})), or None for the
    Markov head.
    """
    base = np.asarray(base, np.float64)
    target = np.asarray(target, np.float64)
    K, V = base.shape
    if verify_len is not None:
        K = int(verify_len)
    P = [softmax(target[i], T) for i in range(K + 1)]
    law = defaultdict(float)

    def walk(i, prev, prob, prefix, s_old=None):
        if prob == 0.0:
            return
        if i == K:
            for x in range(V):
                law[(K + 1, tuple(prefix + [x]))] += prob * P[K][x]
            return
        if Wh is None:
            q = draft_q(base, U, W, i, prev, T)
            s_new = None
        else:
            s_new = rnn_state(U, Wh, prev, s_old)
            q = softmax(np.asarray(base[i], np.float64) + s_new @ np.asarray(W, np.float64), T)
        p = P[i]
        if rule == "ratio_qp":
            acc = np.minimum(1.0, np.where(p > 0, q / np.where(p > 0, p, 1.0), 1.0))
        else:
            acc = np.minimum(1.0, np.where(q > 0, p / np.where(q > 0, q, 1.0), 0.0))
        rej_total = float(np.sum(q * (1.0 - acc)))
        if rule == "no_residual":
            res = p.copy()
        else:
            res = np.maximum(p - q, 0.0)
        if res.sum() == 0.0:
            res = p.copy()
        res = res / res.sum()
        for x in range(V):
            law[(i + 1, tuple(prefix + [x]))] += prob * rej_total * res[x]
        for d in range(V):
            if q[d] > 0:
                walk(i + 1, d, prob * q[d] * acc[d], prefix + [d], s_new)

    walk(0, int(last_token), 1.0, [])
    return dict(law)


def conditional_marginals(law, K):
    """For each position i and emitted prefix x_<i (with position i reached,
    i.e. tau > i): the conditional distribution of x_i as {v: prob}."""
    joint = defaultdict(lambda: defaultdict(float))
    for (tau, out), pr in law.items():
        for i in range(tau):
            joint[(i, out[:i])][out[i]] += pr
    res = {}
    for key, dist in joint.items():
        tot = sum(dist.values())
        res[key] = (tot, {v: pv / tot for v, pv in dist.items()})
    return res


def cell_probs(law, K, V):
    """Exact cell probabilities for the chi-square pins: first token, the pair
    (x0, x1) given tau >= 2, and the tau histogram."""
    first = np.zeros(V)
    pair = np.zeros((V, V))
    taus = np.zeros(K + 1)
    for (tau, out), pr in law.items():
        first[out[0]] += pr
        taus[tau - 1] += pr
        if tau >= 2:
            pair[out[0], out[1]] += pr
    return first, pair, taus
