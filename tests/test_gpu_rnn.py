"""spec_cycle_rnn against the oracle (needs a B200): the RNN sequential head
(aigest.pl "DeepSeek prezentuje DSpark", section "Innowacje w tworzeniu
tokenów": an optional head that tracks the whole block prefix), read as
s_i = bf16(clamp(U[prev_i] + Wh s_{i-1}, -1, 1)), bias_i = s_i . W."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_invariants, compare_cycle, note_near

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


def gpu_rnn(w, d, Wh, greedy=False, T=1.0, seed=0, cyc=0, dd=None):
    p = sd.Params(B=d["base"].shape[0], K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=T,
                  greedy=greedy, seed=seed, cycle=cyc)
    dd = dd or {k: v.cuda() for k, v in d.items()}
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    sd.cycle_rnn(p, dd["base"], dd["target"], dd["U"], dd["W"], Wh.cuda(), dd["last_token"],
                 o["draft"], o["out"], o["tau"], o["p_draft"], o["q_draft"], ws)
    st = sd.sync_status(ws)
    return st, {k: _np(v) for k, v in o.items()}


def orc_rnn(w, d, Wh, greedy=False, T=1.0, seed=0, cyc=0):
    P = oracle.Params(B=d["base"].shape[0], K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=T,
                      greedy=greedy, seed=seed, cycle=cyc, Wh=synth.to_numpy_raw(Wh))
    return oracle.cycle(P, *(synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")),
                        d["last_token"].numpy())


CASES = [
    ("small", synth.Workload("rn", B=5, K=6, V=1000, r=64, dtype="bf16", sigma=0.4, seed=101,
                             uw_std=0.3), 1.0),
    ("two_groups", synth.Workload("rng", B=100, K=5, V=9000, r=128, dtype="bf16", sigma=0.3,
                                  seed=102, uw_std=0.2), 0.9),
    ("n16_rank256", synth.Workload("rn16", B=12, K=4, V=20000, r=256, dtype="bf16", sigma=0.6,
                                   seed=103, uw_std=0.08), 1.0),    ("two_groups_n128", synth.Workload("rng2", B=160, K=4, V=7000, r=128, dtype="bf16",
                                       sigma=0.4, seed=104, uw_std=0.2), 1.0),
]


@pytest.mark.parametrize("greedy", [False, True])
@pytest.mark.parametrize("name,w,T", CASES, ids=[c[0] for c in CASES])
def test_rnn_cycle_vs_oracle(name, w, T, greedy):
    d = synth.make(w)
    Wh = synth.rnn_weights(w)
    total = 0
    for cyc in range(2):
        st, g = gpu_rnn(w, d, Wh, greedy=greedy, T=T, seed=29, cyc=cyc)
        assert st == sd.SPEC_OK, sd.status_string(st)
        o = orc_rnn(w, d, Wh, greedy=greedy, T=T, seed=29, cyc=cyc)
        f = compare_cycle(g, o, w.K)
        note_near(f"rnn_{name}{'_greedy' if greedy else ''}", cyc, w.B, f)
        check_invariants(g["out"], g["tau"], g["draft"], w.K)
        total += f
    assert total <= max(1, w.B // 2)


@pytest.mark.parametrize("greedy", [False, True])
def test_rnn_full_size_config3(greedy):
    """B=64, K=16, V=129280, r=256 with a recurrence; every row against the oracle."""
    w = synth.WORKLOADS["c3"]
    d = synth.make(w)
    Wh = synth.rnn_weights(w, scale=2.0 / np.sqrt(w.r))
    st, g = gpu_rnn(w, d, Wh, greedy=greedy, seed=w.seed, cyc=4)
    assert st == sd.SPEC_OK, sd.status_string(st)
    o = orc_rnn(w, d, Wh, greedy=greedy, seed=w.seed, cyc=4)
    f = compare_cycle(g, o, w.K)
    note_near(f"rnn_c3{'_greedy' if greedy else ''}", 4, w.B, f)
    if greedy:
        assert f <= 2
    else:
        assert f <= int(0.85 * w.B)


@pytest.mark.parametrize("greedy", [False, True])
def test_rnn_zero_recurrence_equals_markov_cycle_on_clamped_U(greedy):
    """Wh = 0: the state is bf16(clamp(U[prev])), so the cycle equals spec_cycle
    with U replaced by that table (rounded by torch)."""
    w = CASES[1][1]
    d = synth.make(w)
    dd = {k: v.cuda() for k, v in d.items()}
    Wh0 = torch.zeros((w.r, w.r), dtype=torch.bfloat16)
    st, a = gpu_rnn(w, d, Wh0, greedy=greedy, T=0.9, seed=3, cyc=1, dd=dd)
    assert st == sd.SPEC_OK
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=0.9, greedy=greedy,
                  seed=3, cycle=1)
    Uc = torch.clamp(d["U"].float(), -1.0, 1.0).to(torch.bfloat16).cuda()
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    sd.cycle(p, dd["base"], dd["target"], Uc, dd["W"], dd["last_token"], o["draft"], o["out"],
             o["tau"], o["p_draft"], o["q_draft"], ws)
    assert sd.sync_status(ws) == sd.SPEC_OK
    for k in ("draft", "out", "tau", "p_draft", "q_draft"):
        np.testing.assert_array_equal(a[k], _np(o[k]), err_msg=k)


def test_rnn_recurrence_changes_the_draft():
    """A nonzero recurrence gives other drafts than the Markov head on the same
    clamped table (the state carries the prefix)."""
    w = CASES[0][1]
    d = synth.make(w)
    Wh = synth.rnn_weights(w, scale=3.0 / np.sqrt(w.r))
    _, a = gpu_rnn(w, d, Wh, greedy=True, seed=1)
    _, b = gpu_rnn(w, d, torch.zeros_like(Wh), greedy=True, seed=1)
    assert np.array_equal(a["draft"][:, 0], b["draft"][:, 0])  # position 0: no prefix yet
    assert not np.array_equal(a["draft"], b["draft"])
