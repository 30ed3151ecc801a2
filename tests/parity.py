"""Comparison of the CUDA path with the oracle under the near-threshold rule.

The GPU decides in fp32, the oracle in fp64.  The oracle flags every decision
whose uniform lies within 1e-6 of its threshold (and greedy arg-max near-ties);
those decisions, and everything that depends on them, are counted instead of
compared.  Everything else must be bit-exact (tokens, tau) or within 1e-5
absolute (probabilities p_i(d_i), q_i(d_i)).
"""
from __future__ import annotations

import numpy as np

PROB_TOL = 1e-5

# (case, cycle, rows compared, rows with a near-threshold decision): filled by
# the GPU tests, printed in the test session's terminal summary
NEAR_THRESHOLD = []


def note_near(case: str, cycle: int, rows: int, flagged: int):
    NEAR_THRESHOLD.append((case, cycle, rows, flagged))


def compare_cycle(gpu: dict, orc: dict, K: int, rows=None, check_probs=True):
    """gpu/orc: dicts of numpy arrays (draft, out, tau, p_draft, q_draft) for the
    same batch rows.  Returns the number of rows with a flagged decision."""
    n = len(orc["tau"])
    flagged = 0
    for b in range(n):
        fd = int(orc["flag_draft"][b])
        fa = int(orc["flag_accept"][b])
        ff = int(orc["flag_final"][b])
        stop = int(orc["tau"][b]) - 1
        tag = f"row {b if rows is None else rows[b]}"
        if gpu.get("draft") is not None:
            assert np.array_equal(gpu["draft"][b, :fd], orc["draft"][b, :fd]), (
                tag, gpu["draft"][b], orc["draft"][b], fd)
        limit = min(fd, fa)
        # the outcome depends on the draft and accept decisions at 0..min(stop, K-1)
        if limit > min(stop, K - 1):
            assert int(gpu["tau"][b]) == stop + 1, (tag, gpu["tau"][b], stop + 1)
            assert np.array_equal(gpu["out"][b, :stop], orc["out"][b, :stop]), (tag, gpu["out"][b], orc["out"][b])
            assert np.all(gpu["out"][b, stop + 1:] == -1), (tag, gpu["out"][b])
            if ff:
                flagged += 1
            else:
                assert gpu["out"][b, stop] == orc["out"][b, stop], (tag, gpu["out"][b], orc["out"][b])
        else:
            flagged += 1
            assert int(gpu["tau"][b]) > limit, (tag, gpu["tau"][b], limit)
            assert np.array_equal(gpu["out"][b, :limit], orc["out"][b, :limit]), tag
        if check_probs:
            qlim = min(fd, K)
            if qlim > 0 and not np.all(np.isnan(orc["q_draft"][b, :qlim])):
                np.testing.assert_allclose(gpu["q_draft"][b, :qlim], orc["q_draft"][b, :qlim],
                                           rtol=0, atol=PROB_TOL, err_msg=tag)
            plim = min(limit, stop + 1, K)
            po, pg = orc["p_draft"][b, :plim], gpu["p_draft"][b, :plim]
            if plim > 0 and not np.all(np.isnan(po)):
                np.testing.assert_allclose(pg, po, rtol=0, atol=PROB_TOL, err_msg=tag)
            if limit > stop:
                assert np.all(np.isnan(gpu["p_draft"][b, stop + 1:])), (tag, gpu["p_draft"][b])
    return flagged


def compare_draft(gpu: dict, orc: dict, K: int):
    flagged = 0
    for b in range(len(orc["flag_draft"])):
        fd = int(orc["flag_draft"][b])
        if fd < K:
            flagged += 1
        assert np.array_equal(gpu["draft"][b, :fd], orc["draft"][b, :fd]), (b, gpu["draft"][b], orc["draft"][b], fd)
        if fd > 0 and not np.all(np.isnan(orc["q_draft"][b, :fd])):
            np.testing.assert_allclose(gpu["q_draft"][b, :fd], orc["q_draft"][b, :fd], rtol=0,
                                       atol=PROB_TOL)
    return flagged


def check_invariants(out, tau, draft, K):
    for b in range(len(tau)):
        t = int(tau[b])
        assert 1 <= t <= K + 1
        assert np.array_equal(out[b, :t - 1], draft[b, :t - 1])
        assert np.all(out[b, t:] == -1)
        assert out[b, t - 1] >= 0
        if t <= K:
            assert out[b, t - 1] != draft[b, t - 1]


def flagged_rows(orc: dict, K: int) -> np.ndarray:
    """Rows whose outcome depends on a flagged decision (compare_cycle's rule)."""
    fd, fa = orc["flag_draft"].astype(int), orc["flag_accept"].astype(int)
    stop = orc["tau"].astype(int) - 1
    return (np.minimum(fd, fa) <= np.minimum(stop, K - 1)) | (orc["flag_final"] != 0)


_KEYS = ("draft", "out", "tau", "p_draft", "q_draft")
_FLAGS = ("flag_draft", "flag_accept", "flag_final")


def compare_loop(gpu: dict, orc: dict, K: int, check_probs=True):
    """Per-cycle comparison of a decode loop ([C, B, ...] arrays).  A row stays
    compared while its inputs agree: once its last emitted token of a cycle
    differs from the oracle's (allowed only after a flagged decision), the
    next cycle starts from another token and the row leaves the comparison.
    Returns (rows with a flagged decision summed over cycles, rows still in
    step after the last cycle)."""
    C, B = orc["tau"].shape
    sync = np.ones(B, bool)
    flagged = 0
    for c in range(C):
        rows = np.nonzero(sync)[0]
        gi = {k: gpu[k][c][rows] for k in _KEYS}
        oi = {k: orc[k][c][rows] for k in _KEYS + _FLAGS}
        flagged += compare_cycle(gi, oi, K, rows=rows, check_probs=check_probs)
        gl = gi["out"][np.arange(len(rows)), gi["tau"] - 1]
        ol = oi["out"][np.arange(len(rows)), oi["tau"] - 1]
        diff = gl != ol
        assert np.all(flagged_rows(oi, K)[diff]), (c, rows[diff & ~flagged_rows(oi, K)])
        sync[rows[diff]] = False
    return flagged, sync


def early_exit_q(gpu: dict, orc: dict):
    """Verification with early exit reports q_i(d_i) only where the accept test
    ran (positions up to the row's stop, NaN after); the oracle defines it at
    every position.  Checks the GPU's NaN tail, then keeps q up to the earlier
    of the two stops on both sides for compare_cycle."""
    for b in range(len(orc["tau"])):
        sg, so = int(gpu["tau"][b]) - 1, int(orc["tau"][b]) - 1
        assert np.all(np.isnan(gpu["q_draft"][b, sg + 1:])), (b, gpu["q_draft"][b])
        m = min(sg, so)
        gpu["q_draft"][b, m + 1:] = np.nan
        orc["q_draft"][b, m + 1:] = np.nan
