"""spec_cycle_kb against the oracle (needs a B200): a verify length K_b per
request (aigest.pl "DeepSeek prezentuje DSpark", "Optymalizacja weryfikacji i
wydajności": a scheduler fixes how many draft tokens of each request are
verified; the early stop keeps the method lossless).  Row b drafts and
verifies positions 0..K_b-1 and draws its bonus from target row K_b."""
import math

import numpy as np
import pytest
import torch
from scipy import stats

import oracle
import synth
from oracle import exact_law as EL
from parity import compare_cycle, note_near

import draft_sampling_verification_head_b200 as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sd.lib()
    oracle.build()


def _np(t):
    return t.cpu().numpy()


def gpu_cycle_kb(w, d, kb, greedy=False, T=None, seed=0, cyc=0, dd=None):
    T = w.temperature if T is None else T
    p = sd.Params(B=d["base"].shape[0], K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=T,
                  greedy=greedy, seed=seed, cycle=cyc)
    dd = dd or {k: v.cuda() for k, v in d.items()}
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    sd.cycle_kb(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"],
                torch.as_tensor(kb, dtype=torch.int32).cuda(), o["draft"], o["out"], o["tau"],
                o["p_draft"], o["q_draft"], ws)
    st = sd.sync_status(ws)
    return st, {k: _np(v) for k, v in o.items()}


def orc_cycle_kb(w, d, kb, greedy=False, T=None, seed=0, cyc=0):
    T = w.temperature if T is None else T
    P = oracle.Params(B=d["base"].shape[0], K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=T,
                      greedy=greedy, seed=seed, cycle=cyc, verify_len=np.asarray(kb, np.int32))
    return oracle.cycle(P, *(synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")),
                        d["last_token"].numpy())


def check_kb_invariants(g, kb, K):
    for b in range(len(kb)):
        k = int(kb[b])
        t = int(g["tau"][b])
        assert 1 <= t <= k + 1, (b, t, k)
        assert np.all(g["draft"][b, k:] == -1), (b, g["draft"][b])
        assert np.all(g["out"][b, t:] == -1)
        assert np.array_equal(g["out"][b, :t - 1], g["draft"][b, :t - 1])


CASES = [
    ("small", synth.Workload("kb", B=5, K=6, V=1000, r=64, dtype="bf16", sigma=0.4, seed=91,
                             uw_std=0.3), 1.0),
    ("two_groups", synth.Workload("kbg", B=100, K=5, V=9000, r=128, dtype="bf16", sigma=0.3,
                                  seed=92, uw_std=0.2), 0.9),    ("two_groups_n128", synth.Workload("kbg2", B=190, K=5, V=9000, r=128, dtype="bf16",
                                       sigma=0.3, seed=94, uw_std=0.2), 0.9),
]


@pytest.mark.parametrize("greedy", [False, True])
@pytest.mark.parametrize("name,w,T", CASES, ids=[c[0] for c in CASES])
def test_cycle_kb_vs_oracle(name, w, T, greedy):
    d = synth.make(w)
    rng = np.random.default_rng(5)
    total = 0
    for cyc in range(2):
        kb = rng.integers(1, w.K + 1, size=w.B).astype(np.int32)
        st, g = gpu_cycle_kb(w, d, kb, greedy=greedy, T=T, seed=19, cyc=cyc)
        assert st == sd.SPEC_OK, sd.status_string(st)
        o = orc_cycle_kb(w, d, kb, greedy=greedy, T=T, seed=19, cyc=cyc)
        f = compare_cycle(g, o, w.K)
        note_near(f"kb_{name}{'_greedy' if greedy else ''}", cyc, w.B, f)
        total += f
        check_kb_invariants(g, kb, w.K)
        assert np.array_equal(g["tau"] <= kb + 1, np.ones(w.B, bool))
    assert total <= max(1, w.B // 2)


def test_cycle_kb_full_size_config3():
    """The benchmark's configuration with a random verify length per row; every
    row against the oracle."""
    w = synth.WORKLOADS["c3"]
    d = synth.make(w)
    kb = np.random.default_rng(6).integers(1, w.K + 1, size=w.B).astype(np.int32)
    st, g = gpu_cycle_kb(w, d, kb, seed=w.seed, cyc=3)
    assert st == sd.SPEC_OK, sd.status_string(st)
    o = orc_cycle_kb(w, d, kb, seed=w.seed, cyc=3)
    f = compare_cycle(g, o, w.K)
    note_near("kb_c3", 3, w.B, f)
    check_kb_invariants(g, kb, w.K)
    assert f <= int(0.85 * w.B)


@pytest.mark.parametrize("greedy", [False, True])
def test_cycle_kb_all_k_equals_spec_cycle(greedy):
    w = CASES[1][1]
    d = synth.make(w)
    dd = {k: v.cuda() for k, v in d.items()}
    st, a = gpu_cycle_kb(w, d, np.full(w.B, w.K, np.int32), greedy=greedy, seed=3, cyc=7, dd=dd)
    assert st == sd.SPEC_OK
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                  greedy=greedy, seed=3, cycle=7)
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    sd.cycle(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"],
             o["out"], o["tau"], o["p_draft"], o["q_draft"], ws)
    assert sd.sync_status(ws) == sd.SPEC_OK
    for k in ("draft", "out", "tau"):
        assert np.array_equal(a[k], _np(o[k])), k
    np.testing.assert_array_equal(a["q_draft"], _np(o["q_draft"]))
    np.testing.assert_array_equal(a["p_draft"], _np(o["p_draft"]))


def test_cycle_kb_out_of_range_reported():
    w = CASES[0][1]
    d = synth.make(w)
    kb = np.array([1, 0, 3, w.K + 2, 2], np.int32)
    st, g = gpu_cycle_kb(w, d, kb, seed=4)
    assert st == sd.SPEC_ERR_INVALID_ARG


def test_cycle_kb_exact_distribution():
    """V = 8, K = 3, K_b = 2 (bf16 inputs, rank 64 so the tensor-core cycle
    runs): 2e5 seeded rows against the enumerated law with the verify length."""
    w = synth.Workload("kbx", B=1, K=3, V=8, r=64, dtype="bf16", sigma=0.5, seed=93, uw_std=0.3)
    d0 = synth.make(w)
    n, kb = 200_000, 2
    d = {"base": d0["base"].expand(n, -1, -1).contiguous(),
         "target": d0["target"].expand(n, -1, -1).contiguous(),
         "U": d0["U"], "W": d0["W"],
         "last_token": d0["last_token"].expand(n).contiguous()}
    st, g = gpu_cycle_kb(w, d, np.full(n, kb, np.int32), seed=321, cyc=0)
    assert st == sd.SPEC_OK
    law = EL.exact_law(synth.as_float64(d0["base"])[0], synth.as_float64(d0["target"])[0],
                       synth.as_float64(d0["U"]), synth.as_float64(d0["W"]),
                       int(d0["last_token"][0]), 1.0, verify_len=kb)
    first, pair, taus = EL.cell_probs(law, kb, w.V)
    out, tau = g["out"], g["tau"]
    assert tau.max() <= kb + 1

    def pooled(obs, p, m):
        e = p * m
        keep = e >= 5
        o_ = np.append(obs[keep], obs[~keep].sum())
        e_ = np.append(e[keep], e[~keep].sum())
        if e_[-1] == 0:
            o_, e_ = o_[:-1], e_[:-1]
        return stats.chisquare(o_, e_ * o_.sum() / e_.sum()).pvalue

    sel = tau >= 2
    pv = [pooled(np.bincount(out[:, 0], minlength=w.V), first, n),
          pooled(np.bincount(out[sel, 0] * w.V + out[sel, 1], minlength=w.V * w.V),
                 pair.ravel() / pair.sum(), int(sel.sum())),
          pooled(np.bincount(tau - 1, minlength=kb + 1), taus, n)]
    assert min(pv) > 1e-3, pv
    acc = taus[1:].sum()
    assert abs(sel.mean() - acc) < 4 * math.sqrt(acc * (1 - acc) / n)
