"""spec_decode_loop against the oracle's decode loop (needs a B200): cycles
chained in one launch (aigest.pl "DeepSeek prezentuje DSpark", section "Jak
działa spekulatywne dekodowanie DSpark?": each cycle emits tau tokens for
T_draft + T_verify), the last emitted token of a cycle feeding the next
cycle's Markov head, and verify lengths from per-position confidence scores
(section "Optymalizacja weryfikacji i wydajności")."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import decode_loop as DL
from parity import compare_loop, note_near

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


def _params(w, B, greedy, T, seed, cyc, cls):
    return cls(B=B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=T, greedy=greedy, seed=seed,
               cycle=cyc)


def gpu_loop(w, d, C, greedy=False, T=1.0, seed=0, cyc=0, use_conf=True, thr=0.0, vlen=None,
             dd=None, in_place=False):
    B = d["base"].shape[1]
    p = _params(w, B, greedy, T, seed, cyc, sd.Params)
    dd = dd or {k: v.cuda() for k, v in d.items()}
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p, n_cycles=C)
    lt = dd["last_token"].clone()
    nt = lt if in_place else torch.full((B,), -5, dtype=torch.int32, device="cuda")
    sd.decode_loop(p, C, dd["base"], dd["target"], dd["U"], dd["W"], lt, o["draft"], o["out"],
                   o["tau"], o["p_draft"], o["q_draft"], nt, ws,
                   conf=dd["conf"] if use_conf else None, conf_threshold=thr,
                   verify_len=None if vlen is None else torch.as_tensor(vlen).cuda())
    st = sd.sync_status(ws)
    g = {k: _np(v) for k, v in o.items()}
    g["next_token"] = _np(nt)
    return st, g


def orc_loop(w, d, C, greedy=False, T=1.0, seed=0, cyc=0, use_conf=True, thr=0.0, vlen=None):
    B = d["base"].shape[1]
    P = _params(w, B, greedy, T, seed, cyc, oracle.Params)
    raw = synth.to_numpy_raw
    return DL.decode_loop(P, C, raw(d["base"]), raw(d["target"]), raw(d["U"]), raw(d["W"]),
                          d["last_token"].numpy(),
                          conf=d["conf"].numpy() if use_conf else None, threshold=thr,
                          verify_len=vlen)


def check_chain(g, C, B):
    rows = np.arange(B)
    for c in range(C):
        t = g["tau"][c]
        assert np.all((t >= 1) & (t <= g["out"].shape[2]))
    last = g["out"][C - 1][rows, g["tau"][C - 1] - 1]
    assert np.array_equal(g["next_token"], last)


CASES = [
    ("small", synth.Workload("loop", B=5, K=6, V=1000, r=64, dtype="bf16", sigma=0.4, seed=61,
                             uw_std=0.3), 3, 1.0, 0.35),
    ("two_groups", synth.Workload("loopg", B=100, K=5, V=9000, r=128, dtype="bf16", sigma=0.3,
                                  seed=62, uw_std=0.2), 3, 0.9, 0.3),
    ("n16_rank256", synth.Workload("loop16", B=12, K=4, V=20000, r=256, dtype="bf16", sigma=0.6,
                                   seed=63, uw_std=0.05), 4, 1.0, 0.5),
]


@pytest.mark.parametrize("greedy", [False, True])
@pytest.mark.parametrize("name,w,C,T,thr", CASES, ids=[c[0] for c in CASES])
def test_decode_loop_vs_oracle(name, w, C, T, thr, greedy):
    d = synth.make_loop(w, C)
    st, g = gpu_loop(w, d, C, greedy=greedy, T=T, seed=23, cyc=4, thr=thr)
    assert st == sd.SPEC_OK, sd.status_string(st)
    o = orc_loop(w, d, C, greedy=greedy, T=T, seed=23, cyc=4, thr=thr)
    f, sync = compare_loop(g, o, w.K)
    note_near(f"loop_{name}{'_greedy' if greedy else ''}", 4, C * w.B, f)
    check_chain(g, C, w.B)
    # the confidence rule picked the same verify lengths: tau never exceeds K_b + 1
    assert np.all(g["tau"] <= o["kb"] + 1)
    assert len(set(o["kb"].ravel().tolist())) > 1  # the scores made lengths differ
    assert sync.sum() >= w.B // 2


def test_decode_loop_given_verify_lengths():
    w = CASES[1][1]
    C = 4
    d = synth.make_loop(w, C, seed=64)
    vlen = np.random.default_rng(8).integers(1, w.K + 1, size=(C, w.B)).astype(np.int32)
    st, g = gpu_loop(w, d, C, seed=5, cyc=100, use_conf=False, vlen=vlen)
    assert st == sd.SPEC_OK
    o = orc_loop(w, d, C, seed=5, cyc=100, use_conf=False, vlen=vlen)
    f, _ = compare_loop(g, o, w.K)
    note_near("loop_vlen", 100, C * w.B, f)
    assert np.all(g["tau"] <= vlen + 1)


@pytest.mark.parametrize("greedy", [False, True])
def test_decode_loop_equals_chained_cycles(greedy):
    """Without scores every K_b = K: the loop equals spec_cycle called once per
    cycle with the previous call's last emitted token and the next counter."""
    w = CASES[1][1]
    C = 3
    d = synth.make_loop(w, C, seed=65)
    dd = {k: v.cuda() for k, v in d.items()}
    st, g = gpu_loop(w, d, C, greedy=greedy, T=0.8, seed=6, cyc=2**32 - 2, use_conf=False, dd=dd)
    assert st == sd.SPEC_OK
    lt = dd["last_token"].clone()
    for c in range(C):
        p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=0.8, greedy=greedy,
                      seed=6, cycle=2**32 - 2 + c)
        ws = sd.make_workspace(p)
        o = sd.alloc_outputs(p)
        sd.cycle(p, dd["base"][c], dd["target"][c], dd["U"], dd["W"], lt, o["draft"], o["out"],
                 o["tau"], o["p_draft"], o["q_draft"], ws)
        assert sd.sync_status(ws) == sd.SPEC_OK
        for k in ("draft", "out", "tau", "p_draft", "q_draft"):
            np.testing.assert_array_equal(g[k][c], _np(o[k]), err_msg=f"{k} cycle {c}")
        lt = o["out"][torch.arange(w.B, device="cuda"), o["tau"].long() - 1].to(torch.int32)
    assert np.array_equal(g["next_token"], _np(lt))


def test_decode_loop_in_place_next_token():
    """next_token may be the last_token buffer itself."""
    w = CASES[0][1]
    C = 3
    d = synth.make_loop(w, C, seed=66)
    dd = {k: v.cuda() for k, v in d.items()}
    st, a = gpu_loop(w, d, C, seed=7, thr=0.35, dd=dd)
    assert st == sd.SPEC_OK
    st, b = gpu_loop(w, d, C, seed=7, thr=0.35, dd=dd, in_place=True)
    assert st == sd.SPEC_OK
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_decode_loop_full_size_config3():
    """The benchmark's configuration over two chained cycles with confidence
    scores; every row against the oracle."""
    w = synth.WORKLOADS["c3"]
    C = 2
    d = synth.make_loop(w, C)
    st, g = gpu_loop(w, d, C, seed=w.seed, cyc=9, thr=0.3)
    assert st == sd.SPEC_OK, sd.status_string(st)
    o = orc_loop(w, d, C, seed=w.seed, cyc=9, thr=0.3)
    f, sync = compare_loop(g, o, w.K)
    note_near("loop_c3", 9, C * w.B, f)
    check_chain(g, C, w.B)
    assert f <= int(0.85 * C * w.B)


def test_decode_loop_bad_verify_length_reported():
    w = CASES[0][1]
    d = synth.make_loop(w, 2, seed=67)
    vlen = np.array([[1, 2, 3, 4, 5], [1, 0, 2, 2, 2]], np.int32)
    st, _ = gpu_loop(w, d, 2, seed=1, use_conf=False, vlen=vlen)
    assert st == sd.SPEC_ERR_INVALID_ARG


def test_decode_loop_odd_groups_odd_k():
    """Three groups of rows and an odd K over two cycles: the per-job counters
    of the target warps and the compute warps stay in step across cycles."""
    w = synth.Workload("loopodd", B=150, K=5, V=6000, r=64, dtype="bf16", sigma=0.4, seed=68,
                       uw_std=0.2)
    C = 3
    d = synth.make_loop(w, C)
    for greedy in (False, True):
        st, g = gpu_loop(w, d, C, greedy=greedy, seed=31, cyc=2, thr=0.3)
        assert st == sd.SPEC_OK, sd.status_string(st)
        o = orc_loop(w, d, C, greedy=greedy, seed=31, cyc=2, thr=0.3)
        f, sync = compare_loop(g, o, w.K)
        note_near(f"loop_odd{'_greedy' if greedy else ''}", 2, C * w.B, f)
        check_chain(g, C, w.B)
        assert sync.sum() >= w.B // 2


def test_decode_loop_wait_limit_gives_timeout_and_context_survives():
    w = CASES[0][1]
    C = 2
    d = synth.make_loop(w, C, seed=69)
    dd = {k: v.cuda() for k, v in d.items()}
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, seed=1, spin_limit=1)
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p, n_cycles=C)
    nt = torch.empty(w.B, dtype=torch.int32, device="cuda")
    sd.decode_loop(p, C, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                   o["out"], o["tau"], o["p_draft"], o["q_draft"], nt, ws, conf=dd["conf"],
                   conf_threshold=0.3)
    assert sd.sync_status(ws) == sd.SPEC_ERR_TIMEOUT
    sd.workspace_init(ws)
    st, g = gpu_loop(w, d, C, seed=1, thr=0.3, dd=dd)
    assert st == sd.SPEC_OK
    o2 = orc_loop(w, d, C, seed=1, thr=0.3)
    compare_loop(g, o2, w.K)
