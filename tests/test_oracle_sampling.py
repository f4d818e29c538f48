"""Pins of the oracle's storage rounding, Markov bias and draft sampling (no GPU)."""
import numpy as np
import torch

from conftest import golden_path
from oracle import dspark as o


def _cases():
    for line in open(golden_path("inverse_cdf_cases.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        w, u, x = (t.strip() for t in line.split("|"))
        yield np.array([float(v) for v in w.split(",")]), float(u), int(x)


def test_inverse_cdf_hand_cases():
    for w, u, x in _cases():
        got, Z, _ = o.inverse_cdf(w[None], np.array([u]))
        assert got[0] == x, (w, u, x, got)
        assert Z[0] == w.sum()


def test_inverse_cdf_boundary_flag():
    w = np.array([[0.25, 0.5, 0.25]])
    _, _, f = o.inverse_cdf(w, np.array([0.25]))
    assert f[0]
    _, _, f = o.inverse_cdf(w, np.array([0.5]))
    assert not f[0]
    _, _, f = o.inverse_cdf(w, np.array([0.75 - 5e-7]))
    assert f[0]


def test_bf16_rounding_matches_torch():
    """fp64 -> bf16 (ties to even) against torch's fp32 -> bf16 conversion
    for values exactly representable in fp32 (where the two must agree)."""
    rng = np.random.default_rng(0)
    v32 = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 8,
        # exact midpoints and neighbours: 8 significant bits + a half
        (np.arange(1, 4000, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -6),
    ])
    got, _ = o.round_to_bf16(v32.astype(np.float64))
    want = torch.from_numpy(v32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(got, want)


def test_bf16_rounding_known_values():
    # 1 + 2^-8 is a midpoint between 1 and 1 + 2^-7: ties to even -> 1
    # 1 + 3*2^-8 is a midpoint between 1 + 2^-7 and 1 + 2^-6: ties to even -> 1 + 2^-6
    v = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -(1 + 2 ** -8)])
    got, flag = o.round_to_bf16(v)
    assert list(got) == [1.0, 1 + 2 ** -6, 1 + 2 ** -7, -1.0]
    assert list(flag) == [True, True, True, True]
    got, flag = o.round_to_bf16(np.array([1.0, 3.0, 1 + 2 ** -9]))
    assert list(got) == [1.0, 3.0, 1.0] and not flag.any()


def test_draft_logits_midpoint_window():
    base = np.array([[1.0, 1.0]])
    bias = np.array([[2 ** -8, 2 ** -8 + 2 ** -12]])
    d, f = o.draft_logits(base, bias, "bf16")
    assert list(d[0]) == [1.0, 1 + 2 ** -7]
    assert f[0, 0] and not f[0, 1]


def test_markov_bias_worked_example():
    """'Once position one samples "of", the head boosts "course" and suppresses
    "problem"' (DSpark LLM inference speedup, "The Semi-Autoregressive Trick"):
    with U[of] selecting a rank direction whose W row raises 'course' and lowers
    'problem', the draft distribution after 'of' moves that way and the bias
    depends only on the previous token."""
    OF, COURSE, PROBLEM, OTHER = range(4)
    U = np.zeros((4, 2)); U[OF, 0] = 1.0; U[OTHER, 1] = 1.0
    W = np.zeros((2, 4)); W[0, COURSE] = 2.0; W[0, PROBLEM] = -2.0; W[1, OTHER] = 0.5
    bias = o.markov_bias(U, W, np.array([OF, COURSE, OTHER]), np.array([1.0, 1.0, 2.0]))
    assert list(bias[0]) == [0.0, 2.0, -2.0, 0.0]
    assert list(bias[1]) == [0.0, 0.0, 0.0, 0.0]
    assert list(bias[2]) == [0.0, 0.0, 0.0, 1.0]
    base = np.zeros((1, 4))
    q0 = np.exp(base[0]) / np.exp(base[0]).sum()
    d, _ = o.draft_logits(base, bias[:1], "f64")
    q1 = np.exp(d[0]) / np.exp(d[0]).sum()
    assert q1[COURSE] > q0[COURSE] and q1[PROBLEM] < q0[PROBLEM]


def test_sample_position_closed_forms():
    # logits [0, ln 3] at tau 1: q = [1/4, 3/4]; at tau 1/2: weights [1, 9] -> q = [0.1, 0.9]
    d = np.array([[0.0, np.log(3.0)]] * 4)
    tau = np.array([1.0, 1.0, 0.5, 0.5])
    u = np.array([0.2, 0.3, 0.05, 0.15])
    s = o.sample_position(d, tau, u)
    assert list(s["x"]) == [0, 1, 0, 1]
    np.testing.assert_allclose(s["q_tok"], [0.25, 0.75, 0.1, 0.9], rtol=1e-14)
    np.testing.assert_allclose(s["q_lse"][:2], np.log(4.0), rtol=1e-14)
    np.testing.assert_allclose(s["q_lse"][2:], 2 * np.log(3.0) + np.log(10 / 9), rtol=1e-14)


def test_greedy_ties_lowest_index():
    s = o.sample_position(np.array([[1.0, 3.0, 3.0, 2.0]]), np.array([0.0]), np.array([0.9]))
    assert s["x"][0] == 1 and s["q_tok"][0] == 1.0 and s["q_lse"][0] == 3.0


def test_draft_frequencies_follow_q():
    """x_1 drawn by the oracle follows softmax(d/tau) (chi-square), with and
    without the Markov bias."""
    from scipy import stats
    rng = np.random.default_rng(3)
    V, N = 8, 200000
    base = rng.normal(0, 1, (V,))
    U = rng.normal(0, 0.5, (V, 3)); W = rng.normal(0, 0.5, (3, V))
    for scale in (0.0, 1.0):
        inp = dict(base=np.broadcast_to(base, (N, 1, V)), U=U, W=W,
                   last_tok=np.full(N, 2), bias_scale=np.full(N, scale),
                   temp=np.full(N, 0.8), dtype="f64")
        dr = o.draft_round(inp, 99, 5)
        z = (base + scale * (U[2] @ W)) / 0.8
        q = np.exp(z - z.max()); q /= q.sum()
        cnt = np.bincount(dr["x"][:, 0], minlength=V)
        assert stats.chisquare(cnt, q * N).pvalue > 1e-4


def test_zero_bias_reduces_to_parallel_drafter():
    """bias_scale = 0 or W = 0 gives exactly the plain parallel drafter's draw."""
    rng = np.random.default_rng(4)
    B, K, V, r = 16, 3, 32, 4
    base = rng.normal(0, 1, (B, K, V))
    U = rng.normal(0, 1, (V, r))
    common = dict(base=base, U=U, last_tok=rng.integers(0, V, B), temp=np.ones(B), dtype="bf16")
    a = o.draft_round(dict(common, W=rng.normal(0, 1, (r, V)), bias_scale=np.zeros(B)), 1, 2)
    b = o.draft_round(dict(common, W=np.zeros((r, V)), bias_scale=np.ones(B)), 1, 2)
    # the parallel drafter: every position sampled from its own stored base logits
    for k in range(K):
        dk, _ = o.round_to_bf16(base[:, k])
        s = o.sample_position(dk, np.ones(B), o.uniform(1, np.arange(B), k + 1, 0, 2))
        for r_ in (a, b):
            assert np.array_equal(r_["x"][:, k], s["x"])
            assert np.array_equal(r_["d"][:, k], dk)
