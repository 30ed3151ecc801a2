"""The seeded input generator: deterministic bytes and the stated recipe."""
import numpy as np
import torch

import synth


def test_generator_deterministic_and_shaped():
    w = synth.Workload("g", B=3, K=4, V=1000, r=8, dtype="bf16", sigma=0.5, seed=21)
    a, b = synth.make(w), synth.make(w)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert a["base"].shape == (3, 4, 1000) and a["target"].shape == (3, 5, 1000)
    assert a["U"].shape == (1000, 8) and a["W"].shape == (8, 1000)
    assert a["base"].dtype == torch.bfloat16 and a["last_token"].dtype == torch.int32
    assert int(a["last_token"].min()) >= 0 and int(a["last_token"].max()) < 1000
    c = synth.make(w, seed=22)
    assert not torch.equal(a["base"], c["base"])


def test_generator_recipe_statistics():
    w = synth.Workload("g", B=4, K=8, V=20000, r=16, dtype="f32", sigma=0.5, seed=23)
    d = synth.make(w)
    zeta = -1.1 * np.log(np.arange(w.V) + 1.0)
    resid = d["base"].numpy() - zeta
    assert abs(resid.mean()) < 0.02 and abs(resid.std() - 2.0) < 0.02
    noise = d["target"][:, :w.K].numpy() - d["base"].numpy()
    assert abs(noise.std() - 0.5) < 0.01
    assert abs(d["U"].numpy().std() - 0.02) < 0.001


def test_linear_sigma_schedule():
    w = synth.WORKLOADS["c5"]
    s = synth.sigmas(w)
    assert len(s) == w.K + 1 and abs(s[0] - 0.2) < 1e-7 and abs(s[-1] - 1.5) < 1e-6
    assert np.all(np.diff(s) > 0)
