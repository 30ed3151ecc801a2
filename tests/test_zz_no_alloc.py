"""spec_cycle_noalloc: the fused cycle on the library's built-in scratch array,
for callers that cannot allocate device memory when they run a cycle (their
allocations belong to a framework pool, or cudaMalloc would synchronise the
device under them).  Its outputs must equal spec_cycle's with a caller
workspace, call after call.  Collected last on purpose (file name), so a run
that stops at the first failure has run every other test first."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from parity import PROB_TOL

import draft_sampling_verification_head_b200 as sd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sd.lib()


def _with_workspace(p, dd):
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    sd.cycle(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"], o["out"],
             o["tau"], o["p_draft"], o["q_draft"], ws)
    assert sd.sync_status(ws) == sd.SPEC_OK
    return {k: v.cpu().numpy() for k, v in o.items()}


def _no_alloc(p, dd):
    o = sd.alloc_outputs(p)
    status = torch.full((1,), -99, dtype=torch.int32, device="cuda")
    sd.cycle_noalloc(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                     o["out"], o["tau"], o["p_draft"], o["q_draft"], status)
    torch.cuda.synchronize()
    assert int(status.item()) == sd.SPEC_OK
    return {k: v.cpu().numpy() for k, v in o.items()}


@pytest.mark.parametrize("w,greedy,T", [
    (synth.Workload("na", B=5, K=3, V=1000, r=64, dtype="bf16", sigma=0.6, seed=71, uw_std=0.3),
     False, 1.0),
    (synth.WORKLOADS["c2"], False, 0.7),
    (synth.WORKLOADS["c2"], True, 0.7),
])
def test_no_alloc_matches_workspace_call(w, greedy, T):
    d = synth.make(w)
    dd = {k: v.cuda() for k, v in d.items()}
    for cyc in (0, 1):  # two calls in a row: the shared array carries nothing over
        p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=T, greedy=greedy,
                      seed=13, cycle=cyc)
        ref = _with_workspace(p, dd)
        got = _no_alloc(p, dd)
        for k in ("draft", "out", "tau"):
            assert np.array_equal(got[k], ref[k]), (k, cyc)
        for k in ("p_draft", "q_draft"):
            np.testing.assert_allclose(got[k], ref[k], rtol=0, atol=PROB_TOL, equal_nan=True)


def test_no_alloc_rejects_shapes_beyond_its_buffer():
    p = sd.Params(B=64, K=64, V=129280, r=256, dtype="bf16")
    assert sd.workspace_size(p) > 8 << 20
    fake = ctypes.c_void_p(0x1000)
    rc = sd.lib().spec_cycle_noalloc(ctypes.byref(p.c()), *([fake] * 10), None, None)
    assert rc == sd.SPEC_ERR_WORKSPACE


def test_no_alloc_reports_a_device_error_and_the_next_call_starts_clean():
    """A last token outside [0, V) is caught on the device (clamped, never used
    as an address) and reported through status_out.  The shared array keeps
    that call's status; the next call clears it first, and its outputs equal
    spec_cycle's with a fresh workspace."""
    w = synth.Workload("na", B=5, K=3, V=1000, r=64, dtype="bf16", sigma=0.6, seed=72, uw_std=0.3)
    d = synth.make(w)
    dd = {k: v.cuda() for k, v in d.items()}
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=1.0, seed=14, cycle=2)
    bad = dd["last_token"].clone()
    bad[1] = w.V + 7
    o = sd.alloc_outputs(p)
    status = torch.full((1,), -99, dtype=torch.int32, device="cuda")
    sd.cycle_noalloc(p, dd["base"], dd["target"], dd["U"], dd["W"], bad, o["draft"], o["out"],
                     o["tau"], o["p_draft"], o["q_draft"], status)
    torch.cuda.synchronize()
    assert int(status.item()) == sd.SPEC_ERR_TOKEN_RANGE
    ref = _with_workspace(p, dd)
    got = _no_alloc(p, dd)
    for k in ("draft", "out", "tau"):
        assert np.array_equal(got[k], ref[k]), k
    for k in ("p_draft", "q_draft"):
        np.testing.assert_allclose(got[k], ref[k], rtol=0, atol=PROB_TOL, equal_nan=True)
