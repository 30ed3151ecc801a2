"""Edge shapes of the tensor-core cycle, the decode loop and the one-launch
verification against the oracle (needs a B200): one draft position (K = 1),
one batch row, a vocabulary of one 128-token chunk (a single CTA), a ragged
last chunk, and a long block (K = 64)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import decode_loop as DL
from parity import check_invariants, compare_cycle, compare_loop, early_exit_q, note_near

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


def _cycle_pair(w, greedy, seed=3, cyc=1, kb=None):
    d = synth.make(w)
    dd = {k: v.cuda() for k, v in d.items()}
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                  greedy=greedy, seed=seed, cycle=cyc)
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    if kb is None:
        sd.cycle(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                 o["out"], o["tau"], o["p_draft"], o["q_draft"], ws)
    else:
        sd.cycle_kb(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"],
                    torch.as_tensor(kb, dtype=torch.int32).cuda(), o["draft"], o["out"], o["tau"],
                    o["p_draft"], o["q_draft"], ws)
    st = sd.sync_status(ws)
    g = {k: _np(v) for k, v in o.items()}
    P = oracle.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                      greedy=greedy, seed=seed, cycle=cyc,
                      verify_len=None if kb is None else np.asarray(kb, np.int32))
    ref = oracle.cycle(P, *(synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")),
                       d["last_token"].numpy())
    return st, g, ref


SHAPES = [
    ("k1", synth.Workload("e1", B=9, K=1, V=5000, r=64, dtype="bf16", sigma=0.5, seed=111, uw_std=0.3)),
    ("b1", synth.Workload("e2", B=1, K=6, V=3000, r=128, dtype="bf16", sigma=0.5, seed=112, uw_std=0.3)),
    ("one_cta", synth.Workload("e3", B=7, K=4, V=64, r=64, dtype="bf16", sigma=0.6, seed=113, uw_std=0.4)),
    ("ragged_v", synth.Workload("e4", B=33, K=5, V=1000 * 8 + 8, r=64, dtype="bf16", sigma=0.5, seed=114,
                                uw_std=0.3)),
    ("k64", synth.Workload("e5", B=6, K=64, V=4096, r=64, dtype="bf16", sigma=0.1, seed=115, uw_std=0.05)),
    # the first two positions' target statistics are taken at each job's start by
    # the compute warps: K = 2 leaves no position to the target warps, K = 3 one
    ("k2", synth.Workload("e6", B=20, K=2, V=6000, r=64, dtype="bf16", sigma=0.4, seed=116, uw_std=0.3)),
    ("k3_two_groups", synth.Workload("e7", B=70, K=3, V=6000, r=64, dtype="bf16", sigma=0.4, seed=117,
                                     uw_std=0.3)),
    # 128-row groups with K >= 16 take three positions at the job's start
    ("n128_k16", synth.Workload("e8", B=130, K=16, V=6000, r=64, dtype="bf16", sigma=0.3, seed=119,
                                uw_std=0.3)),
]


@pytest.mark.parametrize("greedy", [False, True])
@pytest.mark.parametrize("name,w", SHAPES, ids=[s[0] for s in SHAPES])
def test_cycle_edge_shapes(name, w, greedy):
    st, g, ref = _cycle_pair(w, greedy)
    assert st == sd.SPEC_OK, sd.status_string(st)
    f = compare_cycle(g, ref, w.K)
    note_near(f"edge_{name}{'_greedy' if greedy else ''}", 1, w.B, f)
    check_invariants(g["out"], g["tau"], g["draft"], w.K)
    assert f <= max(1, w.B // 2)


def test_cycle_kb_all_one():
    """Every verify length 1: one drafted position, the bonus from target row 1."""
    w = SHAPES[3][1]
    st, g, ref = _cycle_pair(w, False, kb=np.ones(w.B, np.int32))
    assert st == sd.SPEC_OK
    compare_cycle(g, ref, w.K)
    assert g["tau"].max() <= 2 and np.all(g["draft"][:, 1:] == -1)


def test_cycle_kb_n128_long_blocks():
    """128-row groups, K = 16, random verify lengths 1..4: bonus rows among the
    three positions taken at the job's start, and just after them."""
    w = SHAPES[-1][1]
    kb = np.random.default_rng(9).integers(1, 5, size=w.B).astype(np.int32)
    for greedy in (False, True):
        st, g, ref = _cycle_pair(w, greedy, kb=kb)
        assert st == sd.SPEC_OK
        f = compare_cycle(g, ref, w.K)
        note_near(f"edge_n128_kb{'_greedy' if greedy else ''}", 1, w.B, f)
        assert np.all(g["tau"] <= kb + 1)
        assert f <= max(1, w.B // 2)


def test_cycle_kb_short_rows_bonus_at_the_start():
    """Verify lengths 1 and 2 only, with K = 6: every row's bonus row is among
    the positions whose target statistics the compute warps take first."""
    w = SHAPES[3][1]
    kb = np.random.default_rng(8).integers(1, 3, size=w.B).astype(np.int32)
    for greedy in (False, True):
        st, g, ref = _cycle_pair(w, greedy, kb=kb)
        assert st == sd.SPEC_OK
        f = compare_cycle(g, ref, w.K)
        note_near(f"edge_kb12{'_greedy' if greedy else ''}", 1, w.B, f)
        assert np.all(g["tau"] <= kb + 1)
        assert f <= max(1, w.B // 2)


@pytest.mark.parametrize("K", [2, 3])
def test_decode_loop_short_blocks_two_groups(K):
    """Chained cycles over two batch groups with K = 2 and 3 (jobs whose target
    positions are all, or all but one, taken at the job's start)."""
    w = synth.Workload(f"el{K}", B=70, K=K, V=6000, r=64, dtype="bf16", sigma=0.4, seed=118 + K,
                       uw_std=0.3)
    C = 3
    d = synth.make_loop(w, C)
    dd = {k: v.cuda() for k, v in d.items()}
    for greedy in (False, True):
        p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, seed=4, cycle=9, greedy=greedy)
        ws = sd.make_workspace(p)
        o = sd.alloc_outputs(p, n_cycles=C)
        nt = torch.empty(w.B, dtype=torch.int32, device="cuda")
        sd.decode_loop(p, C, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"],
                       o["draft"], o["out"], o["tau"], o["p_draft"], o["q_draft"], nt, ws,
                       conf=dd["conf"], conf_threshold=0.4)
        assert sd.sync_status(ws) == sd.SPEC_OK
        g = {k: _np(v) for k, v in o.items()}
        P = oracle.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, seed=4, cycle=9, greedy=greedy)
        raw = synth.to_numpy_raw
        ref = DL.decode_loop(P, C, raw(d["base"]), raw(d["target"]), raw(d["U"]), raw(d["W"]),
                             d["last_token"].numpy(), conf=d["conf"].numpy(), threshold=0.4)
        f, _ = compare_loop(g, ref, w.K)
        note_near(f"edge_loop_k{K}{'_greedy' if greedy else ''}", 9, C * w.B, f)


def test_decode_loop_k1():
    w = SHAPES[0][1]
    C = 3
    d = synth.make_loop(w, C)
    dd = {k: v.cuda() for k, v in d.items()}
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, seed=2, cycle=5)
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p, n_cycles=C)
    nt = torch.empty(w.B, dtype=torch.int32, device="cuda")
    sd.decode_loop(p, C, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                   o["out"], o["tau"], o["p_draft"], o["q_draft"], nt, ws, conf=dd["conf"],
                   conf_threshold=0.5)
    assert sd.sync_status(ws) == sd.SPEC_OK
    g = {k: _np(v) for k, v in o.items()}
    P = oracle.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, seed=2, cycle=5)
    raw = synth.to_numpy_raw
    ref = DL.decode_loop(P, C, raw(d["base"]), raw(d["target"]), raw(d["U"]), raw(d["W"]),
                         d["last_token"].numpy(), conf=d["conf"].numpy(), threshold=0.5)
    compare_loop(g, ref, w.K)


@pytest.mark.parametrize("name,w", [SHAPES[0], SHAPES[2], SHAPES[4]], ids=["k1", "one_cta", "k64"])
def test_verify_edge_shapes(name, w):
    d = synth.make(w)
    g_ = torch.Generator().manual_seed(5)
    dl = (d["base"].float() + 0.3 * torch.randn(d["base"].shape, generator=g_)).to(torch.bfloat16)
    drafts = oracle.draft(oracle.Params(B=w.B, K=w.K, V=w.V, r=0, dtype="bf16", seed=4, cycle=2),
                          synth.to_numpy_raw(dl), np.zeros((w.V, 0), np.uint16),
                          np.zeros((0, w.V), np.uint16), d["last_token"].numpy())["draft"]
    P = oracle.Params(B=w.B, K=w.K, V=w.V, r=0, dtype="bf16", seed=4, cycle=2)
    ref = oracle.verify(P, synth.to_numpy_raw(d["target"]), synth.to_numpy_raw(dl), drafts)
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=0, dtype="bf16", seed=4, cycle=2)
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    sd.verify_block(p, d["target"].cuda(), dl.cuda(), torch.from_numpy(drafts).cuda(), o["out"],
                    o["tau"], o["p_draft"], o["q_draft"], ws)
    assert sd.sync_status(ws) == sd.SPEC_OK
    g = {k: _np(v) for k, v in o.items()}
    g["draft"] = drafts
    ref["draft"] = drafts
    ref["flag_draft"] = np.full(w.B, w.K, np.int32)
    early_exit_q(g, ref)
    compare_cycle(g, ref, w.K)
