"""Pins of the oracle's recurrent sequential head (no GPU).

The pages name an optional head that tracks the whole block prefix ("DSpark
turns speculation into a scheduler", "DSpark's semi-autoregressive
compromise"; "DSpark LLM inference speedup", "The Semi-Autoregressive Trick")
and give no equations; the oracle reads it as h_0 = 0,
h_k = U[x_{k-1}] + tanh(h_{k-1} @ R), bias_k = scale_b * h_k @ W. What pins
that reading here, none of it by restating the formula:

* R = 0 is the Markov head bit for bit (tanh(0) = 0 adds nothing);
* a saturating R makes tanh exactly +-1 in fp64, so the state is the previous
  token's factor plus the sign of the previous state: values known without
  evaluating tanh;
* with that R the state at position 2 depends on the token before the block,
  which a Markov head can never see;
* U = 0 keeps the state at zero: the plain parallel drafter;
* rejection sampling stays lossless with the recurrent draft distribution,
  by exact enumeration and by Monte Carlo against that enumeration.
"""
import numpy as np
from scipy import stats

from oracle import dspark as o
from oracle.brute import output_distribution

SEED = 1234


def _inp(B, K, V, r, rng, dtype="f64", R=None, scale=1.0, peaked=False):
    base = rng.normal(0, 1.0, (B, K, V))
    if peaked:  # one token per position far above the rest: the draw ignores the bias
        base[:] = 0.0
        base[:, np.arange(K), rng.integers(0, V, K)] = 60.0
    inp = dict(base=base, U=rng.normal(0, 0.5, (V, r)), W=rng.normal(0, 0.5, (r, V)),
               last_tok=rng.integers(0, V, B), bias_scale=np.full(B, scale), temp=np.ones(B),
               dtype=dtype)
    if R is not None:
        inp["R"] = R
    return inp


def test_zero_recurrence_is_the_markov_head_bit_for_bit():
    rng = np.random.default_rng(1)
    for dtype in ("bf16", "f32", "f64"):
        inp = _inp(6, 4, 64, 8, rng, dtype)
        # factors stored in the logits' dtype, as the device reads them
        inp["U"] = o.round_to_storage(inp["U"], dtype)[0]
        inp["W"] = o.round_to_storage(inp["W"], dtype)[0]
        mk = o.draft_round(inp, SEED, 3)
        rc = o.draft_round(dict(inp, R=np.zeros((8, 8))), SEED, 3)
        for key in ("d", "x", "q_tok", "q_lse"):
            assert np.array_equal(mk[key], rc[key]), (dtype, key)
        prev = np.concatenate([inp["last_tok"][:, None], mk["x"][:, :-1]], axis=1)
        assert np.array_equal(rc["h"], inp["U"][prev])


def test_saturated_state_is_factor_plus_sign():
    """R = 100 (r = 1) with |h| >= 1/4 everywhere: tanh(100 h) is exactly +-1 in
    fp64, so h_k = U[x_{k-1}] + sign(h_{k-1}) for k >= 2 and h_1 = U[x_0]."""
    rng = np.random.default_rng(2)
    V, K, B = 4, 5, 32
    inp = _inp(B, K, V, 1, rng)
    inp["U"] = np.array([[0.5], [-0.25], [0.75], [-0.5]])
    r = o.draft_round(dict(inp, R=np.array([[100.0]])), SEED, 9)
    h = r["h"][:, :, 0]
    x = r["x"]
    assert np.array_equal(h[:, 0], inp["U"][inp["last_tok"], 0])
    for k in range(1, K):
        assert np.array_equal(h[:, k], inp["U"][x[:, k - 1], 0] + np.sign(h[:, k - 1]))
    assert set(np.unique(np.abs(h[:, 1:]))) <= {0.25, 0.5, 0.75, 1.25, 1.5, 1.75}


def test_state_sees_the_token_before_the_block():
    """Two requests with the same uniforms and base logits peaked on one token
    per position draft the same tokens, but start from last tokens whose U
    factors differ in sign. With the saturating recurrence their states at
    position 2 differ by exactly 2; the Markov head gives them equal states."""
    rng = np.random.default_rng(3)
    V, K = 4, 3
    inp = _inp(2, K, V, 1, rng, peaked=True)
    inp["base"][1] = inp["base"][0]
    inp["U"] = np.array([[0.5], [-0.25], [0.75], [-0.5]])
    inp["last_tok"] = np.array([0, 1])          # U = +0.5 and -0.25
    inp["request_ids"] = np.array([7, 7])       # the same uniforms
    rc = o.draft_round(dict(inp, R=np.array([[100.0]])), SEED, 0)
    mk = o.draft_round(dict(inp, R=np.zeros((1, 1))), SEED, 0)
    assert np.array_equal(rc["x"][0], rc["x"][1])
    assert rc["h"][0, 1, 0] - rc["h"][1, 1, 0] == 2.0
    assert np.array_equal(mk["h"][0, 1:], mk["h"][1, 1:])


def test_zero_factors_are_the_parallel_drafter():
    rng = np.random.default_rng(4)
    inp = _inp(5, 3, 32, 4, rng)
    inp["U"] = np.zeros_like(inp["U"])
    rc = o.draft_round(dict(inp, R=rng.normal(0, 2.0, (4, 4))), SEED, 1)
    plain = o.draft_round(dict(inp, bias_scale=np.zeros(5)), SEED, 1)
    assert not rc["h"].any()
    for key in ("d", "x", "q_tok"):
        assert np.array_equal(rc[key], plain[key])


def _tiny(rng, V, K, r=3):
    return dict(t=rng.normal(0, 1.2, (K + 1, V)), base=rng.normal(0, 1.2, (K, V)),
                U=rng.normal(0, 0.7, (V, r)), W=rng.normal(0, 0.7, (r, V)),
                R=rng.normal(0, 1.5, (r, r)), last=int(rng.integers(0, V)))


def test_brute_force_with_recurrent_draft_is_lossless():
    """Whatever the recurrent draft distribution, the first emitted token
    follows p of target row 0 and, given the round goes on, the next one p of
    row 1; and the recurrence does change the draft (the output distribution
    of whole sequences differs from the Markov head's)."""
    rng = np.random.default_rng(5)
    V, K = 4, 3
    for tau, L in ((1.0, 3), (0.7, 2)):
        rq = _tiny(rng, V, K)
        dist = output_distribution(rq["t"], rq["base"], rq["U"], rq["W"], rq["last"], 1.0, tau, L,
                                   R=rq["R"])
        assert abs(sum(dist.values()) - 1) < 1e-12
        p = [np.exp(rq["t"][j] / tau) / np.exp(rq["t"][j] / tau).sum() for j in range(K + 1)]
        m1 = np.zeros(V)
        for seq, pr in dist.items():
            m1[seq[0]] += pr
        np.testing.assert_allclose(m1, p[0], atol=1e-12)
        for y1 in range(V):
            cont = np.zeros(V)
            for seq, pr in dist.items():
                if len(seq) >= 2 and seq[0] == y1:
                    cont[seq[1]] += pr
            if cont.sum() > 0:
                np.testing.assert_allclose(cont / cont.sum(), p[1], atol=1e-12)
        markov = output_distribution(rq["t"], rq["base"], rq["U"], rq["W"], rq["last"], 1.0, tau, L)
        keys = set(dist) | set(markov)
        assert max(abs(dist.get(k, 0.0) - markov.get(k, 0.0)) for k in keys) > 1e-4


def test_monte_carlo_recurrent_matches_brute_force():
    """The oracle's draft (recurrent head) + verify chain against enumeration."""
    rng = np.random.default_rng(6)
    V, K, N, L, tau = 4, 3, 200000, 3, 1.0
    rq = _tiny(rng, V, K)
    dist = output_distribution(rq["t"], rq["base"], rq["U"], rq["W"], rq["last"], 1.0, tau, L,
                               R=rq["R"])
    inp = dict(base=np.broadcast_to(rq["base"], (N, K, V)), U=rq["U"], W=rq["W"], R=rq["R"],
               last_tok=np.full(N, rq["last"]), bias_scale=np.ones(N), temp=np.full(N, tau),
               dtype="f64")
    dr = o.draft_round(inp, SEED, 31)
    r = o.verify(np.broadcast_to(rq["t"], (N, K + 1, V)), dr["d"], dr["x"], np.full(N, L),
                 np.full(N, tau), SEED, 31)
    keys = sorted(dist)
    index = {k: i for i, k in enumerate(keys)}
    cnt = np.zeros(len(keys))
    for row, n in zip(r["out"], r["n_emit"]):
        cnt[index[tuple(int(v) for v in row[:n])]] += 1
    exp = np.array([dist[k] for k in keys]) * N
    big = exp >= 5
    chi = (((cnt - exp) ** 2 / exp)[big]).sum()
    assert stats.chi2.sf(chi, big.sum() - 1) > 1e-4
    assert cnt[~big].sum() <= max(30, 4 * exp[~big].sum())


def test_state_flags_mark_rounding_midpoints():
    """bf16 state: an element whose fp64 value sits on a rounding midpoint is
    flagged, one a quarter ulp away is not."""
    U = np.array([[1.0 + 2.0 ** -8, 1.0 + 2.0 ** -9]])   # midpoint 1 + 2^-8; 1 + 2^-9 (1/4 ulp)
    h, flag = o.recurrent_state(U, np.zeros((2, 2)), np.array([0]), np.zeros((1, 2)), "bf16")
    assert flag.tolist() == [[True, False]]
    assert h.tolist() == [[1.0, 1.0]]   # ties to even, then the nearest
