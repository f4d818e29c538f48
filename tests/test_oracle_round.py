"""The oracle's whole round on the synthetic workloads (no GPU): shapes,
emitted-token layout and the round's invariants."""
import numpy as np

from oracle import dspark as o
from speculative_decoding_draft_sample_b200 import workloads as wl


def to_oracle(inp, w):
    f = lambda t: t.double().numpy() if hasattr(t, "double") else np.asarray(t, np.float64)
    reqs = np.asarray(inp["requests"], np.int64)
    return dict(target=f(inp["target"]), base=f(inp["base"]), U=f(inp["U"]), W=f(inp["W"]),
                last_tok=np.asarray(inp["last_tok"])[reqs], bias_scale=np.asarray(inp["bias_scale"])[reqs],
                temp=np.asarray(inp["temp"], np.float64)[reqs], conf_logit=inp["conf_logit"],
                pos_temp=inp["pos_temp"], step_cost=inp["step_cost"], fixed_cost=inp["fixed_cost"],
                dtype=w.dtype, request_ids=reqs)


def check_round(r, K):
    a, L = r["verify"]["a"], r["L"]
    rid = r.get("rid")
    Lr = L if rid is None else L[rid]
    assert np.all((0 <= a) & (a <= Lr))
    out = r["verify"]["out"]
    x = r["draft"]["x"]
    for b in range(len(a)):
        assert np.array_equal(out[b, :a[b]], x[b, :a[b]])
        assert out[b, a[b]] >= 0 and np.all(out[b, a[b] + 1:] == -1)
    assert np.array_equal(r["verify"]["n_emit"], a + 1)


def test_tiny_round():
    w = wl.TINY
    inp = wl.generate(w)
    r = o.run_round(to_oracle(inp, w), wl.PHILOX_SEED, 0)
    assert r["draft"]["x"].shape == (w.B, w.K)
    check_round(r, w.K)
    assert r["S"].shape == (w.B, w.K) and np.all(np.diff(r["S"], axis=1) <= 0)


def test_sampled_requests_of_serving_shape():
    """A few requests of the B=256, K=5, V=129280 round (per-request seeding lets
    the oracle regenerate just these rows)."""
    w = wl.DSPARK5
    reqs = [0, 17, 255]
    inp = wl.generate(w, reqs)
    oi = to_oracle(inp, w)
    r = o.run_round(oi, wl.PHILOX_SEED, 3)
    r["rid"] = np.asarray(reqs)
    check_round(r, w.K)
    # identical bytes when the same rows are generated inside a larger subset
    inp2 = wl.generate(w, [5, 17])
    assert np.array_equal(inp2["target"][1].float().numpy(), inp["target"][1].float().numpy())


def test_stress_request_kinds():
    w = wl.scaled(wl.STRESS, V=4096, B=64)
    inp = wl.generate(w)
    ident = inp["identical"]
    assert ident.sum() == round(0.05 * w.B) and inp["independent"].sum() == round(0.05 * w.B)
    for b in np.nonzero(ident)[0]:
        assert np.array_equal(inp["base"][b].float().numpy(), inp["target"][b, :w.K].float().numpy())
        assert inp["bias_scale"][b] == 0
    r = o.run_round(to_oracle(inp, w), wl.PHILOX_SEED, 0)
    check_round(r, w.K)
    # identical drafts are always accepted up to the cut (the full-acceptance + bonus path)
    assert np.array_equal(r["verify"]["a"][ident], r["L"][ident])
    assert (np.asarray(inp["temp"]) == 0).sum() == round(0.25 * w.B)
