"""The seeded input generators: reproducible, regenerable by subsets (the
sampled parity checks of the large cases depend on that), and following the
stated recipes (shapes, storage types, request kinds, tables)."""
import numpy as np
import torch

from speculative_decoding_draft_sample_b200 import workloads as wl


def small(base=wl.STRESS, **kw):
    d = dict(name="wl_test", B=40, V=512, K=4)
    d.update(kw)
    return wl.scaled(base, **d)


def test_subsets_regenerate_bit_identically():
    w = small()
    full = wl.generate(w)
    reqs = [0, 7, 19, 39, 7]
    part = wl.generate(w, reqs)
    assert torch.equal(part["target"], full["target"][reqs])
    assert torch.equal(part["base"], full["base"][reqs])
    again = wl.generate(w)
    for k in ("target", "base", "U", "W"):
        assert torch.equal(again[k], full[k]), k
    for k in ("last_tok", "temp", "bias_scale", "conf_logit", "pos_temp", "step_cost"):
        assert np.array_equal(again[k], full[k]), k


def test_shapes_and_storage_types():
    for w in (small(), small(wl.TINY, V=1024)):
        g = wl.generate(w)
        dt = torch.float32 if w.dtype == wl.F32 else torch.bfloat16
        assert g["target"].shape == (w.B, w.K + 1, w.V) and g["target"].dtype == dt
        assert g["base"].shape == (w.B, w.K, w.V) and g["base"].dtype == dt
        assert g["U"].shape == (w.V, w.r) and g["W"].shape == (w.r, w.V)
        assert g["last_tok"].dtype == np.int32 and g["last_tok"].min() >= 0
        assert g["last_tok"].max() < w.V
        assert g["step_cost"].shape == (w.B * (w.K + 1),)
        assert g["conf_logit"].shape == (w.B, w.K) and g["pos_temp"].shape == (w.K,)
        assert w.V % 8 == 0


def test_request_kinds_follow_the_recipe():
    w = small()
    g = wl.generate(w)
    ident, indep = g["identical"], g["independent"]
    assert ident.sum() == round(0.05 * w.B) and indep.sum() == round(0.05 * w.B)
    assert not (ident & indep).any()
    for b in np.flatnonzero(ident):  # draft base == target rows 0..K-1, no Markov bias
        assert torch.equal(g["base"][b], g["target"][b, : w.K])
        assert g["bias_scale"][b] == 0.0
    assert (g["bias_scale"][~ident] == 1.0).all()
    assert (g["temp"] == 0.0).sum() == round(0.25 * w.B)  # greedy requests
    # ordinary requests: base = target row k-1 plus noise growing with k
    ordinary = np.flatnonzero(~ident & ~indep)
    diff = (g["base"][ordinary].float() - g["target"][ordinary, : w.K].float()).std(dim=(0, 2))
    expect = torch.tensor([w.draft_noise(k) for k in range(1, w.K + 1)])
    assert torch.allclose(diff, expect, rtol=0.1)


def test_cost_tables():
    w = wl.scaled(wl.DSPARK5, B=200, V=1024)
    c = wl.small_inputs(w)["step_cost"]
    n = np.arange(1, w.B * (w.K + 1) + 1)
    assert (c[n <= 512] == 1.0).all() and (c[n > 512] == 1.5).all()
    q = wl.small_inputs(wl.scaled(wl.QWEN3, B=16, V=1024))["step_cost"]
    assert np.all(np.diff(q) > 0) and abs(q[0] - (0.5 + 1 / q.size)) < 1e-6
    assert wl.small_inputs(wl.scaled(wl.DSPARK5, B=16, V=1024))["fixed_cost"] == 16.0


def test_zipf_targets_rank_like_the_recipe():
    w = wl.scaled(wl.QWEN3, name="zipf", B=2, K=1, V=4096)
    t = wl.generate(w)["target"][0, 0].double().numpy()
    logp = wl._zipf_logp(w)
    assert abs(np.exp(logp).sum() - 1.0) < 1e-12
    # the logits are the Zipf log-probabilities plus N(0, 0.5^2) noise
    resid = t - logp
    assert abs(resid.std() - 0.5) < 0.03 and abs(resid.mean()) < 0.03


def test_calibration_inputs():
    z, y = wl.calib_inputs(20000, K=5, seed=4)
    assert z.shape == y.shape == (20000, 5) and z.dtype == np.float32 and y.dtype == np.uint8
    assert np.all(np.diff(y.astype(int), axis=1) <= 0)  # survival is monotone along the block
    z2, y2 = wl.calib_inputs(20000, K=5, seed=4)
    assert np.array_equal(z, z2) and np.array_equal(y, y2)
