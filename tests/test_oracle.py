"""Pins of the oracle against what the pages and the mathematics fix (CPU only).

Each test names the passage it follows:
* aigest.pl "DeepSeek prezentuje DSpark", "Jak działa spekulatywne dekodowanie
  DSpark?": longest accepted prefix + one extra token, target distribution
  preserved exactly (lossless);
* same page, "Innowacje w tworzeniu tokenów": parallel-core base logits plus a
  Markov-head bias on the preceding token, low-rank U[prev].W;
* same page, "Optymalizacja weryfikacji i wydajności": acceptance is governed
  by total variation (acceptance = 1 - TV(p, q));
* telemetr.me DFlash post: the accepted length counts the bonus token.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy import stats
from scipy.special import logsumexp

import synth
from oracle import exact_law as EL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- Philox / U01

def test_u01_mapping_exact(orc):
    assert orc.u01(0) == 0.0
    assert orc.u01(0xFF) == 0.0
    assert orc.u01(0x100) == 2.0 ** -24
    assert orc.u01(0xFFFFFFFF) == 1.0 - 2.0 ** -24
    xs = np.random.default_rng(0).integers(0, 2 ** 32, 1000, dtype=np.uint64)
    us = [orc.u01(int(x)) for x in sorted(xs)]
    assert all(a <= b for a, b in zip(us, us[1:]))


def test_philox_deterministic_and_keyed(orc):
    a = orc.philox([1, 2, 3, 4], [5, 6])
    assert a == orc.philox([1, 2, 3, 4], [5, 6])
    assert a != orc.philox([1, 2, 3, 5], [5, 6])
    assert a != orc.philox([1, 2, 3, 4], [5, 7])
    assert all(0 <= w < 2 ** 32 for w in a)


def test_philox_uniformity_chi2(orc):
    # 2^14 consecutive counters, all four output words, 64 bins each
    words = np.array([orc.philox([i, 7, 0, 0], [0x1234, 0x5678]) for i in range(1 << 14)],
                     dtype=np.uint64)
    for w in range(4):
        hist = np.bincount((words[:, w] >> 26).astype(np.int64), minlength=64)
        assert stats.chisquare(hist).pvalue > 1e-4
    # bit balance of word 0
    bits = ((words[:, 0][:, None] >> np.arange(32, dtype=np.uint64)) & 1).mean(axis=0)
    assert np.all(np.abs(bits - 0.5) < 5 * 0.5 / math.sqrt(len(words)))


def _curand_host_lib():
    """The CUDA toolkit's cuRAND library (its host generators need no GPU)."""
    import ctypes
    import glob
    cands = ["/usr/local/cuda/lib64/libcurand.so", "/usr/local/cuda/lib64/libcurand.so.10"]
    try:
        import nvidia.curand  # pip wheel shipped with torch
        cands += glob.glob(os.path.join(list(nvidia.curand.__path__)[0], "lib", "libcurand.so*"))
    except ImportError:
        pass
    for c in cands:
        if os.path.exists(c):
            try:
                return ctypes.CDLL(c)
            except OSError:
                pass
    return None


def test_philox_matches_curand_host_generator(orc):
    """Philox4x32-10 (Salmon et al., SC'11) as written in the oracle against an
    independent implementation of the same published generator: cuRAND's host
    generator CURAND_RNG_PSEUDO_PHILOX4_32_10, which runs on the CPU.  Its
    stream emits block j (four 32-bit words) from counter (0, 0, j, 0) under
    key (lo32(seed), hi32(seed)), and a generator offset of 4j starts at block
    j, for the first 2^15 blocks (further on its host layout is different).
    This exercises both key words, the low bits of counter word 2 and every
    round; counter words 0, 1, 3 and the high bits of word 2 are compared
    with cuRAND's device generator in the GPU suite."""
    import ctypes
    lib = _curand_host_lib()
    if lib is None:
        pytest.skip("cuRAND library not found")
    PHILOX = 161  # CURAND_RNG_PSEUDO_PHILOX4_32_10
    for seed, first_block, nblk in [(0, 0, 1 << 14), (0xF00DBEEF12345678, 0, 1024),
                                    (0xFFFFFFFF00000001, 12345, 256),
                                    (0x0123456789ABCDEF, (1 << 15) - 100, 100),
                                    (0x8000000080000000, 1 << 14, 64)]:
        gen = ctypes.c_void_p()
        assert lib.curandCreateGeneratorHost(ctypes.byref(gen), PHILOX) == 0
        try:
            assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
            assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(4 * first_block)) == 0
            ref = np.zeros(4 * nblk, np.uint32)
            assert lib.curandGenerate(gen, ref.ctypes.data_as(ctypes.c_void_p),
                                      ctypes.c_size_t(ref.size)) == 0
        finally:
            lib.curandDestroyGenerator(gen)
        key = [seed & 0xFFFFFFFF, seed >> 32]
        got = np.array([w for j in range(nblk)
                        for w in orc.philox([0, 0, first_block + j, 0], key)], np.uint32)
        assert np.array_equal(got, ref), (hex(seed), first_block)


def test_uniform_counter_layout(orc):
    seed, cyc = 0x0123456789ABCDEF, 0x0000BEEF00C0FFEE
    for (b, pos, tag) in [(0, 0, 0), (5, 3, 1), (1 << 20, 31, 2)]:
        ctr = [pos, b, cyc & 0xFFFFFFFF, tag | (((cyc >> 32) & 0xFFFF) << 16)]
        key = [seed & 0xFFFFFFFF, seed >> 32]
        assert orc.uniform(seed, cyc, b, pos, tag) == orc.u01(orc.philox(ctr, key)[0])
    # distinct streams per (b, pos, tag, cycle)
    seen = {orc.uniform(1, c, b, p, t) for c in range(3) for b in range(8) for p in range(8)
            for t in range(3)}
    assert len(seen) == 3 * 8 * 8 * 3


# ----------------------------------------------------------------------------- inverse CDF / stats

def test_icdf_matches_searchsorted(orc):
    rng = np.random.default_rng(1)
    for n in (1, 2, 7, 100):
        for _ in range(50):
            w = rng.random(n) * (rng.random(n) < 0.7)
            if w.sum() == 0:
                continue
            u = rng.random()
            idx, _ = orc.icdf(w, u)
            cs = np.cumsum(w)  # sequential prefix sums, as the definition states
            assert idx == int(np.searchsorted(cs, u * cs[-1], side="right"))


def test_icdf_special_cases(orc):
    assert orc.icdf([0, 0, 1, 0], 0.0)[0] == 2          # one-hot
    assert orc.icdf([0, 0, 1, 0], 0.999)[0] == 2
    assert orc.icdf([0, 0, 1, 1], 0.0)[0] == 2          # u = 0 -> first positive mass
    idx, near = orc.icdf([1, 1, 1, 1], 0.25)            # exact edge: strict '>' moves right
    assert idx == 1 and near
    idx, near = orc.icdf([1, 1, 1, 1], 0.3)
    assert idx == 1 and not near


def test_row_stats_vs_logsumexp(orc):
    rng = np.random.default_rng(2)
    for T in (1.0, 0.7, 2.5):
        x = rng.normal(0, 3, 5000)
        m, Z = orc.row_stats(x, T)
        assert m == pytest.approx(np.max(x / T), abs=0, rel=1e-15)
        assert m + math.log(Z) == pytest.approx(logsumexp(x / T), rel=1e-13)


def test_biased_row_vs_matmul(orc):
    w = synth.Workload("t", B=2, K=3, V=300, r=16, dtype="bf16", seed=11)
    d = synth.make(w)
    P = orc.Params(B=2, K=3, V=300, r=16, dtype="bf16")
    raw = {k: synth.to_numpy_raw(d[k]) for k in ("base", "U", "W")}
    base64, U64, W64 = (synth.as_float64(d[k]) for k in ("base", "U", "W"))
    for (b, i, prev) in [(0, 0, 5), (1, 2, 299), (1, 1, 0)]:
        z = orc.biased_row(P, raw["base"], raw["U"], raw["W"], b, i, prev)
        ref = base64[b, i] + U64[prev] @ W64
        np.testing.assert_allclose(z, ref, rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- worked examples

def _golden_cases():
    cases, cur = [], {}
    for line in open(os.path.join(GOLDEN, "verify_worked_examples.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            if cur:
                cases.append(cur)
                cur = {}
            continue
        k, v = (s.strip() for s in line.split("=", 1))
        cur[k] = v
    if cur:
        cases.append(cur)
    return cases


def _mat(s):
    return np.array([[float(x) for x in row.split()] for row in s.split(";")])


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_verify_worked_examples(orc, case):
    p, q = _mat(case["p"]), _mat(case["q"])
    d = [int(x) for x in case["d"].split()]
    r = orc.verify_probs(p, q, d, [float(x) for x in case["u_acc"].split()],
                         [float(x) for x in case["u_res"].split()])
    assert list(r["out"]) == [int(x) for x in case["out"].split()]
    assert r["tau"] == int(case["tau"])
    exp_pd = [float(x) for x in case["p_draft"].split()]
    np.testing.assert_allclose(r["p_draft"], exp_pd, rtol=0, atol=1e-15)
    assert r["flag_accept"] == int(case["flag_accept"])
    assert r["flag_final"] == int(case["flag_final"])


# ----------------------------------------------------------------------------- exact law (P1)

def _tiny_inputs(seed, V=8, K=3, r=4, uw=0.5, sigma=0.5):
    w = synth.Workload("tiny", B=1, K=K, V=V, r=r, dtype="f32", sigma=sigma, seed=seed, uw_std=uw)
    d = synth.make(w)
    return w, d


@pytest.mark.parametrize("seed,uw,T", [(5, 0.5, 1.0), (6, 0.5, 0.7), (7, 0.0, 1.0), (8, 1.5, 1.3)])
def test_lossless_by_enumeration(seed, uw, T):
    """Every emitted position, given the emitted prefix, follows target row i exactly."""
    w, d = _tiny_inputs(seed, uw=uw)
    base, target = synth.as_float64(d["base"])[0], synth.as_float64(d["target"])[0]
    U, W = synth.as_float64(d["U"]), synth.as_float64(d["W"])
    law = EL.exact_law(base, target, U, W, int(d["last_token"][0]), T)
    assert abs(sum(law.values()) - 1.0) < 1e-12
    P = [EL.softmax(target[i], T) for i in range(w.K + 1)]
    cond = EL.conditional_marginals(law, w.K)
    assert len(cond) > w.V  # prefixes of several lengths were reached
    for (i, prefix), (mass, dist) in cond.items():
        for v in range(w.V):
            assert abs(dist.get(v, 0.0) - P[i][v]) < 1e-12, (i, prefix, v)


@pytest.mark.parametrize("rule", ["no_residual", "ratio_qp"])
def test_lossless_pin_detects_wrong_rule(rule):
    """A wrong accept or resample rule breaks the lossless property."""
    w, d = _tiny_inputs(5)
    base, target = synth.as_float64(d["base"])[0], synth.as_float64(d["target"])[0]
    U, W = synth.as_float64(d["U"]), synth.as_float64(d["W"])
    law = EL.exact_law(base, target, U, W, int(d["last_token"][0]), 1.0, rule=rule)
    P = [EL.softmax(target[i], 1.0) for i in range(w.K + 1)]
    worst = max(abs(dist.get(v, 0.0) - P[i][v])
                for (i, _), (_, dist) in EL.conditional_marginals(law, w.K).items()
                for v in range(w.V))
    assert worst > 1e-3


def test_acceptance_is_one_minus_tv():
    """P(accept at 0) = sum_v min(p0, q0) = 1 - TV(p0, q0)."""
    w, d = _tiny_inputs(9)
    base, target = synth.as_float64(d["base"])[0], synth.as_float64(d["target"])[0]
    U, W = synth.as_float64(d["U"]), synth.as_float64(d["W"])
    lt = int(d["last_token"][0])
    law = EL.exact_law(base, target, U, W, lt, 1.0)
    p0 = EL.softmax(target[0], 1.0)
    q0 = EL.draft_q(base, U, W, 0, lt, 1.0)
    acc = sum(pr for (tau, _), pr in law.items() if tau >= 2)
    assert abs(acc - np.minimum(p0, q0).sum()) < 1e-12
    assert abs(acc - (1 - 0.5 * np.abs(p0 - q0).sum())) < 1e-12


# ----------------------------------------------------------------------------- oracle sampling vs exact law (P2, P3)

def _replicated(d, Bn):
    base = d["base"][:1].expand(Bn, -1, -1).contiguous()
    target = d["target"][:1].expand(Bn, -1, -1).contiguous()
    last = d["last_token"][:1].expand(Bn).contiguous()
    return base, target, last


def _pooled_chisq(obs, exp_p, n):
    exp_c = exp_p * n
    keep = exp_c >= 5
    o = np.append(obs[keep], obs[~keep].sum())
    e = np.append(exp_c[keep], exp_c[~keep].sum())
    if e[-1] == 0:
        o, e = o[:-1], e[:-1]
    return stats.chisquare(o, e * o.sum() / e.sum()).pvalue


def _law_pvalues(orc, n, seed=5, handle=None, K=3):
    """Chi-square p-values of oracle samples against the enumerated exact law:
    first token, (x0, x1 | tau >= 2), and the tau histogram."""
    w, d = _tiny_inputs(seed, K=K)
    base, target, last = _replicated(d, n)
    P = orc.Params(B=n, K=w.K, V=w.V, r=w.r, dtype="f32", temperature=1.0, seed=42, cycle=3)
    o = orc.cycle(P, synth.to_numpy_raw(base), synth.to_numpy_raw(target),
                  synth.to_numpy_raw(d["U"]), synth.to_numpy_raw(d["W"]), last.numpy(),
                  handle=handle)
    law = EL.exact_law(synth.as_float64(d["base"])[0], synth.as_float64(d["target"])[0],
                       synth.as_float64(d["U"]), synth.as_float64(d["W"]), int(last[0]), 1.0)
    first, pair, taus = EL.cell_probs(law, w.K, w.V)
    out, tau = o["out"], o["tau"]
    sel = tau >= 2
    pc = np.bincount(out[sel, 0] * w.V + out[sel, 1], minlength=w.V * w.V)
    pv = [_pooled_chisq(np.bincount(out[:, 0], minlength=w.V), first, n),
          _pooled_chisq(pc, pair.ravel() / pair.sum(), sel.sum()),
          _pooled_chisq(np.bincount(tau - 1, minlength=w.K + 1), taus, n)]
    return pv, taus, sel


def test_oracle_samples_match_exact_law(orc):
    n = 200_000
    pv, taus, sel = _law_pvalues(orc, n)
    assert min(pv) > 1e-3, pv
    # P3: acceptance at position 0 within 4 sigma of 1 - TV
    acc_exact = taus[1:].sum()
    assert abs(sel.mean() - acc_exact) < 4 * math.sqrt(acc_exact * (1 - acc_exact) / n)


@pytest.mark.parametrize("plant", [1, 2, 3])
def test_planted_oracle_mistakes_are_rejected(orc, tmp_path, plant):
    """Mistakes planted in a copy of the oracle (residual replaced by p; Markov
    head fed the wrong token; bonus from the wrong row) fail the exact-law pin."""
    h = orc.build_planted(plant, str(tmp_path))
    pv, _, _ = _law_pvalues(orc, 200_000, handle=h, K=1 if plant == 3 else 3)
    assert min(pv) < 1e-6, pv


# ----------------------------------------------------------------------------- per-row verify length K_b

# aigest.pl "DeepSeek prezentuje DSpark", "Optymalizacja weryfikacji i
# wydajności": a scheduler fixes the verify length of each request and its early
# stop keeps the method lossless.  Row b drafts and verifies positions
# 0..K_b-1 and takes the bonus from target row K_b.

@pytest.mark.parametrize("kb", [1, 2])
@pytest.mark.parametrize("seed", [3, 9])
def test_verify_length_lossless_by_enumeration(seed, kb):
    w, d = _tiny_inputs(seed)
    base, target = synth.as_float64(d["base"])[0], synth.as_float64(d["target"])[0]
    U, W = synth.as_float64(d["U"]), synth.as_float64(d["W"])
    law = EL.exact_law(base, target, U, W, int(d["last_token"][0]), 1.0, verify_len=kb)
    assert abs(sum(law.values()) - 1.0) < 1e-12
    assert max(t for t, _ in law) == kb + 1  # never more than K_b + 1 tokens
    P = [EL.softmax(target[i], 1.0) for i in range(w.K + 1)]
    for (i, prefix), (mass, dist) in EL.conditional_marginals(law, kb).items():
        for v in range(w.V):
            assert abs(dist.get(v, 0.0) - P[i][v]) < 1e-12, (i, prefix, v)


def test_oracle_verify_length_samples_match_exact_law(orc):
    """Oracle draws with K_b = 2 of K = 3 against the enumerated law (chi-square
    on the first token and the tau histogram)."""
    n, kb = 200_000, 2
    w, d = _tiny_inputs(5)
    base, target, last = _replicated(d, n)
    P = orc.Params(B=n, K=w.K, V=w.V, r=w.r, dtype="f32", temperature=1.0, seed=42, cycle=3,
                   verify_len=np.full(n, kb, np.int32))
    o = orc.cycle(P, synth.to_numpy_raw(base), synth.to_numpy_raw(target),
                  synth.to_numpy_raw(d["U"]), synth.to_numpy_raw(d["W"]), last.numpy())
    law = EL.exact_law(synth.as_float64(d["base"])[0], synth.as_float64(d["target"])[0],
                       synth.as_float64(d["U"]), synth.as_float64(d["W"]), int(last[0]), 1.0,
                       verify_len=kb)
    first, _, taus = EL.cell_probs(law, kb, w.V)
    out, tau = o["out"], o["tau"]
    assert tau.max() <= kb + 1 and np.all(out[:, kb + 1:] == -1)
    assert np.all(o["draft"][:, kb:] == -1)
    pv = [_pooled_chisq(np.bincount(out[:, 0], minlength=w.V), first, n),
          _pooled_chisq(np.bincount(tau - 1, minlength=kb + 1), taus, n)]
    assert min(pv) > 1e-3, pv


@pytest.mark.parametrize("greedy", [False, True])
def test_verify_length_k_equals_plain_cycle(orc, greedy):
    w = synth.Workload("kbk", B=12, K=5, V=300, r=16, dtype="f32", sigma=0.6, seed=81, uw_std=0.3)
    d = synth.make(w)
    raw = [synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")]
    kw = dict(B=w.B, K=w.K, V=w.V, r=w.r, dtype="f32", temperature=0.9, greedy=greedy, seed=7,
              cycle=2)
    a = orc.cycle(orc.Params(**kw), *raw, d["last_token"].numpy())
    b = orc.cycle(orc.Params(**kw, verify_len=np.full(w.B, w.K, np.int32)), *raw,
                  d["last_token"].numpy())
    for k in ("draft", "out", "tau", "flag_draft", "flag_accept", "flag_final"):
        assert np.array_equal(a[k], b[k]), k
    np.testing.assert_array_equal(a["p_draft"], b["p_draft"])


@pytest.mark.parametrize("greedy", [False, True])
def test_verify_length_is_a_prefix_of_the_full_block(orc, greedy):
    """The draws of a K_b row are the full block's first K_b draws (same random
    counters): a row that stops before K_b emits exactly what the full block
    emits; a row that accepts all K_b drafts emits them and a bonus drawn from
    target row K_b."""
    w = synth.Workload("kbp", B=64, K=6, V=400, r=16, dtype="f32", sigma=0.4, seed=82, uw_std=0.3)
    d = synth.make(w)
    raw = [synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")]
    kb = (np.arange(w.B) % w.K + 1).astype(np.int32)
    kw = dict(B=w.B, K=w.K, V=w.V, r=w.r, dtype="f32", temperature=1.0, greedy=greedy, seed=11,
              cycle=4)
    full = orc.cycle(orc.Params(**kw), *raw, d["last_token"].numpy())
    part = orc.cycle(orc.Params(**kw, verify_len=kb), *raw, d["last_token"].numpy())
    target = synth.as_float64(d["target"])
    bonus_rows = 0
    for b in range(w.B):
        k = int(kb[b])
        assert np.array_equal(part["draft"][b, :k], full["draft"][b, :k])
        assert np.all(part["draft"][b, k:] == -1)
        assert 1 <= part["tau"][b] <= k + 1 and np.all(part["out"][b, part["tau"][b]:] == -1)
        if full["tau"][b] <= k:  # stopped inside the verified prefix: the same outcome
            assert part["tau"][b] == full["tau"][b]
            assert np.array_equal(part["out"][b], full["out"][b])
        else:                    # every verified draft accepted: bonus from row K_b
            bonus_rows += 1
            assert part["tau"][b] == k + 1
            assert np.array_equal(part["out"][b, :k], full["draft"][b, :k])
            if greedy:
                assert part["out"][b, k] == int(np.argmax(target[b, k]))
            else:
                p = EL.softmax(target[b, k], 1.0)
                u = orc.uniform(11, 4, b, k, orc.TAG_RESAMPLE)
                assert part["out"][b, k] == int(np.searchsorted(np.cumsum(p), u, side="right"))
    assert bonus_rows > 5


# ----------------------------------------------------------------------------- special cases (P4) and invariants (P5)

def test_markov_off_draft_is_plain_categorical(orc):
    w, d = _tiny_inputs(12, uw=0.0)
    n = 100_000
    base, target, last = _replicated(d, n)
    P = orc.Params(B=n, K=w.K, V=w.V, r=w.r, dtype="f32", temperature=0.8, seed=3)
    o = orc.draft(P, synth.to_numpy_raw(base), synth.to_numpy_raw(d["U"]),
                  synth.to_numpy_raw(d["W"]), last.numpy())
    for i in range(w.K):
        q = EL.softmax(synth.as_float64(d["base"])[0, i], np.float32(0.8))
        assert _pooled_chisq(np.bincount(o["draft"][:, i], minlength=w.V), q, n) > 1e-3


@pytest.mark.parametrize("greedy", [False, True])
def test_target_equal_draft_accepts_all(orc, greedy):
    w = synth.Workload("eq", B=16, K=5, V=500, r=8, dtype="bf16", uw_std=0.0, seed=13)
    d = synth.make(w)
    target = torch.cat([d["base"], d["base"][:, :1]], dim=1)  # rows 0..K-1 equal the draft
    P = orc.Params(B=16, K=5, V=500, r=8, dtype="bf16", greedy=greedy, seed=1)
    o = orc.cycle(P, synth.to_numpy_raw(d["base"]), synth.to_numpy_raw(target),
                  synth.to_numpy_raw(d["U"]), synth.to_numpy_raw(d["W"]), d["last_token"].numpy())
    assert np.all(o["tau"] == w.K + 1)
    assert np.array_equal(o["out"][:, :w.K], o["draft"])
    if greedy:
        assert np.array_equal(o["draft"], synth.as_float64(d["base"]).argmax(axis=2))


def test_greedy_mismatch_at_zero(orc):
    w = synth.Workload("gm", B=8, K=4, V=200, r=8, dtype="bf16", seed=14)
    d = synth.make(w)
    P = orc.Params(B=8, K=4, V=200, r=8, dtype="bf16", greedy=True)
    raw = {k: synth.to_numpy_raw(d[k]) for k in ("base", "U", "W")}
    first = orc.draft(P, raw["base"], raw["U"], raw["W"], d["last_token"].numpy())["draft"][:, 0]
    target = d["target"].clone()
    # make row 0's arg-max a token other than the greedy draft
    other = (torch.from_numpy(first.astype(np.int64)) + 1) % w.V
    target[torch.arange(8), 0, other] = 100.0
    o = orc.cycle(P, raw["base"], synth.to_numpy_raw(target), raw["U"], raw["W"],
                  d["last_token"].numpy())
    assert np.all(o["tau"] == 1)
    assert np.array_equal(o["out"][:, 0], other.numpy())
    assert np.all(o["out"][:, 1:] == -1)


def _check_invariants(o, K):
    for b in range(len(o["tau"])):
        t = int(o["tau"][b])
        assert 1 <= t <= K + 1
        assert np.array_equal(o["out"][b, :t - 1], o["draft"][b, :t - 1])
        assert np.all(o["out"][b, t:] == -1)
        assert o["out"][b, t - 1] >= 0
        if t <= K:  # a rejection never re-emits the rejected draft
            assert o["out"][b, t - 1] != o["draft"][b, t - 1]


@pytest.mark.parametrize("greedy", [False, True])
def test_structural_invariants(orc, greedy):
    w = synth.Workload("inv", B=64, K=6, V=700, r=16, dtype="bf16", sigma=1.0, seed=15)
    d = synth.make(w)
    P = orc.Params(B=64, K=6, V=700, r=16, dtype="bf16", greedy=greedy, temperature=0.9, seed=2)
    o = orc.cycle(P, *(synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")),
                  d["last_token"].numpy())
    _check_invariants(o, w.K)
    if not greedy:
        tested = ~np.isnan(o["p_draft"])
        assert np.array_equal(tested.sum(axis=1), np.minimum(o["tau"], w.K))
        assert np.all(o["q_draft"] > 0)


def test_verify_only_matches_cycle_when_markov_off(orc):
    """With U = 0 the final draft logits equal the base logits, so verifying
    the cycle's own drafts against them must reproduce the cycle exactly."""
    w = synth.Workload("vo", B=32, K=5, V=400, r=8, dtype="bf16", uw_std=0.0, seed=16)
    d = synth.make(w)
    P = orc.Params(B=32, K=5, V=400, r=8, dtype="bf16", temperature=1.1, seed=9, cycle=2)
    raw = {k: synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")}
    c = orc.cycle(P, raw["base"], raw["target"], raw["U"], raw["W"], d["last_token"].numpy())
    v = orc.verify(P, raw["target"], raw["base"], c["draft"])
    assert np.array_equal(v["out"], c["out"]) and np.array_equal(v["tau"], c["tau"])
    np.testing.assert_array_equal(v["q_draft"], c["q_draft"])


def test_subset_rows_equal_full(orc):
    """Each row's draws are keyed on its own batch index: a row subset is exact."""
    w = synth.Workload("sub", B=12, K=4, V=300, r=8, dtype="bf16", seed=17)
    d = synth.make(w)
    P = orc.Params(B=12, K=4, V=300, r=8, dtype="bf16", seed=4)
    raw = [synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")]
    full = orc.cycle(P, *raw, d["last_token"].numpy())
    part = orc.cycle(P, *raw, d["last_token"].numpy(), b_begin=5, b_end=9)
    for k in ("draft", "out", "tau"):
        assert np.array_equal(full[k][5:9], part[k])
