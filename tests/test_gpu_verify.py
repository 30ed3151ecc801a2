"""spec_verify_block / spec_verify_block_kb (one persistent launch with early
exit) against the oracle's verification (needs a B200).  aigest.pl "DeepSeek
prezentuje DSpark", section "Jak działa spekulatywne dekodowanie DSpark?":
the longest accepted prefix plus one token, target distribution preserved;
section "Optymalizacja weryfikacji i wydajności": a verify length per
request."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_invariants, compare_cycle, early_exit_q, note_near

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


def make_verify_inputs(w, ddtype="bf16", T=1.0, greedy=False, seed=3, cyc=5, pert=0.3):
    """Target rows from the workload; draft logits = base + N(0, pert^2) in
    ddtype; draft tokens drawn from them by the oracle's drafting (no head)."""
    d = synth.make(w)
    g = torch.Generator().manual_seed(w.seed + 17)
    dl = d["base"].float() + pert * torch.randn(d["base"].shape, generator=g)
    dl = dl.to(torch.bfloat16 if ddtype == "bf16" else torch.float32)
    z = np.uint16 if ddtype == "bf16" else np.float32
    drafts = oracle.draft(oracle.Params(B=w.B, K=w.K, V=w.V, r=0, dtype=ddtype, temperature=T,
                                        greedy=greedy, seed=seed, cycle=cyc),
                          synth.to_numpy_raw(dl), np.zeros((w.V, 0), z), np.zeros((0, w.V), z),
                          d["last_token"].numpy())["draft"]
    return d["target"], dl, drafts


def run_both(w, target, dl, drafts, ddtype, T, greedy, seed, cyc, kb=None, row_offset=0,
             with_oracle=True):
    B, K, V = w.B, w.K, w.V
    o = {}
    if with_oracle:
        P = oracle.Params(B=B, K=K, V=V, r=0, dtype=w.dtype, draft_dtype=ddtype, temperature=T,
                          greedy=greedy, seed=seed, cycle=cyc,
                          verify_len=None if kb is None else np.asarray(kb, np.int32))
        o = oracle.verify(P, synth.to_numpy_raw(target), synth.to_numpy_raw(dl), drafts)
    p = sd.Params(B=B, K=K, V=V, r=0, dtype=w.dtype, draft_dtype=ddtype, temperature=T,
                  greedy=greedy, seed=seed, cycle=cyc, row_offset=row_offset)
    ws = sd.make_workspace(p)
    outs = sd.alloc_outputs(p)
    args = (target.cuda(), dl.cuda(), torch.from_numpy(drafts).cuda())
    if kb is None:
        sd.verify_block(p, *args, outs["out"], outs["tau"], outs["p_draft"], outs["q_draft"], ws)
    else:
        sd.verify_block_kb(p, *args, torch.as_tensor(kb, dtype=torch.int32).cuda(), outs["out"],
                           outs["tau"], outs["p_draft"], outs["q_draft"], ws)
    st = sd.sync_status(ws)
    assert sd.last_launch_count() == 1
    gpu = {k: _np(v) for k, v in outs.items()}
    gpu["draft"] = drafts
    o["draft"] = drafts
    o["flag_draft"] = np.full(B, K, np.int32)
    return st, gpu, o


CASES = [
    ("small", synth.Workload("v1", B=7, K=4, V=1000, r=8, dtype="bf16", sigma=0.7, seed=81), "bf16", 1.2),
    ("rows_over_ctas", synth.Workload("v2", B=200, K=6, V=5000, r=8, dtype="bf16", sigma=0.5, seed=82),
     "bf16", 1.0),
    ("f32_draft", synth.Workload("v3", B=16, K=9, V=20000, r=8, dtype="bf16", sigma=0.6, seed=83),
     "f32", 0.8),
    ("f32_both", synth.Workload("v4", B=5, K=3, V=512, r=8, dtype="f32", sigma=0.7, seed=84), "f32", 1.0),
    ("wide_slices", synth.Workload("v5", B=9, K=5, V=262144, r=8, dtype="bf16", sigma=0.5, seed=85),
     "bf16", 1.0),
]


@pytest.mark.parametrize("greedy", [False, True])
@pytest.mark.parametrize("name,w,ddtype,T", CASES, ids=[c[0] for c in CASES])
def test_verify_vs_oracle(name, w, ddtype, T, greedy):
    target, dl, drafts = make_verify_inputs(w, ddtype, T, greedy)
    st, gpu, o = run_both(w, target, dl, drafts, ddtype, T, greedy, seed=3, cyc=5)
    assert st == sd.SPEC_OK, sd.status_string(st)
    early_exit_q(gpu, o)
    f = compare_cycle(gpu, o, w.K)
    note_near(f"verify_{name}{'_greedy' if greedy else ''}", 5, w.B, f)
    check_invariants(gpu["out"], gpu["tau"], drafts, w.K)
    assert f <= max(1, w.B // 4)


@pytest.mark.parametrize("greedy", [False, True])
@pytest.mark.parametrize("name,w,ddtype,T", CASES[:3], ids=[c[0] for c in CASES[:3]])
def test_verify_kb_vs_oracle(name, w, ddtype, T, greedy):
    target, dl, drafts = make_verify_inputs(w, ddtype, T, greedy)
    kb = np.random.default_rng(4).integers(1, w.K + 1, size=w.B).astype(np.int32)
    st, gpu, o = run_both(w, target, dl, drafts, ddtype, T, greedy, seed=8, cyc=1, kb=kb)
    assert st == sd.SPEC_OK, sd.status_string(st)
    early_exit_q(gpu, o)
    f = compare_cycle(gpu, o, w.K)
    note_near(f"verify_kb_{name}{'_greedy' if greedy else ''}", 1, w.B, f)
    assert np.all(gpu["tau"] <= kb + 1)
    assert f <= max(1, w.B // 4)


@pytest.mark.parametrize("greedy", [False, True])
def test_verify_full_size_config3(greedy):
    """B=64, K=16, V=129280: every row against the oracle."""
    w = synth.WORKLOADS["c3"]
    target, dl, drafts = make_verify_inputs(w, "bf16", 1.0, greedy, pert=0.5)
    st, gpu, o = run_both(w, target, dl, drafts, "bf16", 1.0, greedy, seed=11, cyc=2)
    assert st == sd.SPEC_OK
    early_exit_q(gpu, o)
    f = compare_cycle(gpu, o, w.K)
    note_near(f"verify_c3{'_greedy' if greedy else ''}", 2, w.B, f)
    if greedy:
        assert f == 0
    else:
        assert f <= int(0.6 * w.B)


def test_verify_row_offset_block_equals_whole():
    """Rows 5..8 verified on their own with row_offset 5 equal the whole batch's."""
    w = CASES[0][1]
    target, dl, drafts = make_verify_inputs(w)
    _, whole, _ = run_both(w, target, dl, drafts, "bf16", 1.2, False, seed=3, cyc=5)
    b0 = 5
    w2 = synth.Workload("v1b", B=w.B - b0, K=w.K, V=w.V, r=8, dtype="bf16", sigma=0.7, seed=81)
    st, part, _ = run_both(w2, target[b0:].contiguous(), dl[b0:].contiguous(), drafts[b0:].copy(),
                           "bf16", 1.2, False, seed=3, cyc=5, row_offset=b0)
    assert st == sd.SPEC_OK
    for k in ("out", "tau"):
        assert np.array_equal(part[k], whole[k][b0:]), k


def test_verify_kb_out_of_range_reported():
    w = CASES[0][1]
    target, dl, drafts = make_verify_inputs(w)
    kb = np.array([1, 2, 0, 3, 4, 5, 1], np.int32)
    st, _, _ = run_both(w, target, dl, drafts, "bf16", 1.2, False, seed=3, cyc=5, kb=kb,
                        with_oracle=False)
    assert st == sd.SPEC_ERR_INVALID_ARG


def test_verify_kb_all_k_equals_verify_block():
    w = CASES[1][1]
    target, dl, drafts = make_verify_inputs(w)
    _, a, _ = run_both(w, target, dl, drafts, "bf16", 1.0, False, seed=21, cyc=3)
    _, b, _ = run_both(w, target, dl, drafts, "bf16", 1.0, False, seed=21, cyc=3,
                       kb=np.full(w.B, w.K, np.int32))
    for k in ("out", "tau", "p_draft", "q_draft"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_verify_wait_limit_gives_timeout_and_context_survives():
    """spin_limit = 1: the first wait of the one-launch verification gives up,
    SPEC_ERR_TIMEOUT is recorded, the copies in flight are drained, and the
    next call on the same workspace is correct."""
    w = CASES[0][1]
    target, dl, drafts = make_verify_inputs(w)
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=0, dtype="bf16", temperature=1.2, seed=3, cycle=5,
                  spin_limit=1)
    ws = sd.make_workspace(p)
    outs = sd.alloc_outputs(p)
    args = (target.cuda(), dl.cuda(), torch.from_numpy(drafts).cuda())
    sd.verify_block(p, *args, outs["out"], outs["tau"], outs["p_draft"], outs["q_draft"], ws)
    assert sd.sync_status(ws) == sd.SPEC_ERR_TIMEOUT
    sd.workspace_init(ws)
    st, gpu, o = run_both(w, target, dl, drafts, "bf16", 1.2, False, seed=3, cyc=5)
    assert st == sd.SPEC_OK
    early_exit_q(gpu, o)
    compare_cycle(gpu, o, w.K)
