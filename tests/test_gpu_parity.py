"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Small cases span several chunks, CTA slices and a ragged tail and are checked on
every request; the full-size workloads run in the configuration the benchmark
times and are checked on sampled requests (the oracle regenerates just those
rows), the schedule on the whole batch."""
import numpy as np
import pytest
import torch

from parity import check_round, run_gpu
from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SMALL = [
    wl.TINY,
    wl.scaled(wl.DSPARK5, name="dspark5_small", B=24, V=8200),
    wl.scaled(wl.QWEN3, name="qwen3_small", B=16, V=4104, cost_kind="linear"),
    wl.scaled(wl.STRESS, name="stress_small", B=64, K=8, V=2056),
    wl.scaled(wl.sweep(16), name="sweep16_small", B=8, V=1032),
    wl.scaled(wl.DSPARK5, name="dspark5_f32_small", B=12, V=3000 // 8 * 8, dtype=wl.F32, r=32),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_round_all_requests(cuda_ok, w):
    inp = wl.generate(w)
    for round_id in (0, 1):
        rnd, _ = run_gpu(w, inp, round_id)
        stats = check_round(w, inp, rnd, list(range(w.B)), round_id)
        # decisions adopted from the GPU at flagged points stay rare
        assert stats["forced"] <= 3 + w.B * w.K // 20, stats


@pytest.mark.parametrize("mode,threshold", [(bn.CUT_NONE, 0.0), (bn.CUT_THRESHOLD, 0.3),
                                            (bn.CUT_THRESHOLD, 2.0)])
def test_cut_modes(cuda_ok, mode, threshold):
    w = wl.scaled(wl.DSPARK5, name="modes", B=32, V=4096)
    inp = wl.generate(w)
    rnd, _ = run_gpu(w, inp, 5, mode, threshold)
    check_round(w, inp, rnd, list(range(w.B)), 5, mode, threshold)
    L = rnd.cut.cpu().numpy()
    if mode == bn.CUT_NONE:
        assert np.all(L == w.K)
    if threshold > 1.0:  # nothing survives: one target token per request
        assert np.all(L == 0) and np.all(rnd.n_emit.cpu().numpy() == 1)


FULL = [wl.DSPARK5, wl.QWEN3, wl.sweep(4), wl.sweep(8), wl.sweep(12), wl.sweep(16), wl.STRESS]


def sampled_requests(w, inp, rnd, n=32, seed=0):
    """At least ``n`` requests of a full-size round: the first and last row of
    every 128-request M-tile of the draft kernel (0, 127, 128, 255, ..., B-1),
    one request of every (cut, accepted) class the round produced, the special
    request kinds of the stress mix, then random ones."""
    rng = np.random.default_rng(seed)
    reqs = {0, w.B - 1}
    for m0 in range(0, w.B, 128):
        reqs |= {m0, min(m0 + 127, w.B - 1)}
    cut = rnd.cut.cpu().numpy()
    acc = rnd.accepted.cpu().numpy()
    for c, a in sorted(set(zip(cut.tolist(), acc.tolist()))):
        reqs.add(int(rng.choice(np.nonzero((cut == c) & (acc == a))[0])))
    for kind in ("identical", "independent"):
        if np.any(inp[kind]):
            reqs.add(int(np.nonzero(inp[kind])[0][0]))
    greedy = np.nonzero(np.asarray(inp["temp"]) == 0)[0]
    if len(greedy):
        reqs.add(int(greedy[0]))
    rest = [b for b in rng.permutation(w.B).tolist() if b not in reqs]
    reqs |= set(rest[:max(0, n - len(reqs))])
    return sorted(reqs)


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled_requests(cuda_ok, w):
    inp = wl.generate(w)
    rnd, _ = run_gpu(w, inp, 0)
    reqs = sampled_requests(w, inp, rnd)
    assert len(reqs) >= min(32, w.B)
    stats = check_round(w, inp, rnd, reqs, 0)
    print(w.name, len(reqs), "requests", stats)


def test_lossless_on_gpu(cuda_ok):
    """The GPU's emitted tokens follow the target softmax (chi-square), with the
    Markov bias on and the cut off; independent of the oracle."""
    from scipy import stats
    from speculative_decoding_draft_sample_b200.spec_round import SpecRound
    B, K, V, r = 60000, 3, 64, 16
    g = torch.Generator().manual_seed(3)
    t = torch.randn(K + 1, V, generator=g) * 1.5
    base = t[:K] + torch.randn(K, V, generator=g)
    dev = dict(target=t.expand(B, K + 1, V).contiguous().cuda(),
               base=base.expand(B, K, V).contiguous().cuda(),
               U=(torch.randn(V, r, generator=g) * 0.3).cuda(),
               W=(torch.randn(r, V, generator=g) * 0.3).cuda(),
               bias_scale=None, last_tok=torch.full((B,), 5, dtype=torch.int32).cuda(),
               temp=torch.full((B,), 0.8).cuda(), conf_logit=torch.zeros(B, K).cuda(),
               pos_temp=torch.ones(K).cuda(), step_cost=torch.ones(B * (K + 1)).cuda(),
               fixed_cost=0.0)
    rnd = SpecRound(B, K, V, r, torch.float32)
    rnd.run(dev, 77, 0, bn.CUT_NONE)
    out = rnd.out.cpu().numpy()
    n = rnd.n_emit.cpu().numpy()
    assert rnd.status() == (0, -1)
    p = torch.softmax(t.double() / 0.8, dim=1).numpy()
    c1 = np.bincount(out[:, 0], minlength=V)
    assert stats.chisquare(c1, p[0] * B).pvalue > 1e-4
    sel = n >= 2
    c2 = np.bincount(out[sel, 1], minlength=V)
    assert stats.chisquare(c2, p[1] * sel.sum()).pvalue > 1e-4
