"""Pins of the oracle's rejection-sampling verification (no GPU).

What pins it: the closed form of the acceptance probability
(sum_x min(p, q) = 1 - TV(p, q)), the residual's support, the lossless
property of rejection sampling (emitted tokens follow the target softmax),
exact enumeration of tiny rounds (``oracle.brute``) and the deterministic
special cases (greedy exact match, d == t, L = 0)."""
import numpy as np
from scipy import stats

from oracle import dspark as o
from oracle.brute import output_distribution

SEED = 1234


def _bcast(a, n):
    return np.broadcast_to(a, (n,) + a.shape)


def test_acceptance_identity_and_residual_support():
    """p = [.5, .3, .2], q = [.2, .5, .3]: accept rate = sum min(p, q) = 0.7 = 1 - TV;
    the residual max(0, p - q) = [.3, 0, 0] puts every correction on token 0."""
    p = np.array([0.5, 0.3, 0.2]); q = np.array([0.2, 0.5, 0.3])
    assert abs(np.minimum(p, q).sum() - (1 - 0.5 * np.abs(p - q).sum())) < 1e-15
    N = 200000
    d = np.log(q)[None, None, :]
    draw = o.sample_position(np.broadcast_to(d[0], (N, 3)), np.ones(N),
                             o.uniform(SEED, np.arange(N), 1, 0, 0))
    target = np.stack([np.log(p), np.log(p)])
    r = o.verify(_bcast(target, N), _bcast(d[0], N), draw["x"][:, None], np.ones(N, np.int64),
                 np.ones(N), SEED, 0)
    rate = r["a"].mean()
    assert abs(rate - 0.7) < 5 * np.sqrt(0.7 * 0.3 / N)
    assert np.all(r["y"][r["a"] == 0] == 0)
    # accept rate per drafted token equals min(1, p/q)
    for t in range(3):
        sel = draw["x"] == t
        want = min(1.0, p[t] / q[t])
        assert abs(r["a"][sel].mean() - want) < 5 * np.sqrt(max(want * (1 - want), 1e-12) / sel.sum()) + 1e-12


def test_identical_draft_accepts_everything_and_adds_bonus():
    rng = np.random.default_rng(1)
    B, K, V = 4000, 4, 12
    t = rng.normal(0, 1.5, (K + 1, V))
    x = rng.integers(0, V, (B, K))
    L = rng.integers(0, K + 1, B)
    r = o.verify(_bcast(t, B), _bcast(t[:K], B), x, L, np.full(B, 0.7), SEED, 3)
    assert np.array_equal(r["a"], L)
    # bonus draws follow p of row L
    z = t / 0.7
    for l in range(K + 1):
        sel = L == l
        p = np.exp(z[l] - z[l].max()); p /= p.sum()
        cnt = np.bincount(r["y"][sel], minlength=V)
        assert stats.chisquare(cnt + 1e-9, p * sel.sum()).pvalue > 1e-4 or sel.sum() < 50


def test_greedy_exact_match():
    t = np.zeros((3, 4, 5))
    t[:, 0, 2] = 1.0; t[:, 1, 4] = 1.0; t[:, 2, 0] = 1.0; t[:, 3, 3] = 1.0
    t[2, 1, 1] = 1.0  # tie with index 4 -> argmax is 1 for request 2
    x = np.array([[2, 4, 0], [2, 3, 0], [2, 4, 0]])
    L = np.array([3, 3, 3])
    r = o.verify(t, np.zeros((3, 3, 5)), x, L, np.zeros(3), SEED, 0)
    assert list(r["a"]) == [3, 1, 1]
    assert list(r["y"]) == [3, 4, 1]
    assert r["out"].tolist() == [[2, 4, 0, 3], [2, 4, -1, -1], [2, 1, -1, -1]]
    assert list(r["n_emit"]) == [4, 2, 2]


def test_cut_zero_emits_one_target_token():
    rng = np.random.default_rng(2)
    N, K, V = 100000, 3, 10
    t = rng.normal(0, 1, (K + 1, V))
    r = o.verify(_bcast(t, N), _bcast(rng.normal(0, 1, (K, V)), N), np.zeros((N, K), np.int64),
                 np.zeros(N, np.int64), np.ones(N), SEED, 1)
    assert np.all(r["a"] == 0) and np.all(r["n_emit"] == 1)
    p = np.exp(t[0] - t[0].max()); p /= p.sum()
    assert stats.chisquare(np.bincount(r["y"], minlength=V), p * N).pvalue > 1e-4
    assert np.all(r["out"][:, 1:] == -1)


def _tiny_request(rng, V, K, r=3):
    return dict(t=rng.normal(0, 1.2, (K + 1, V)), base=rng.normal(0, 1.2, (K, V)),
                U=rng.normal(0, 0.7, (V, r)), W=rng.normal(0, 0.7, (r, V)),
                last=int(rng.integers(0, V)))


def test_brute_force_is_lossless():
    """The enumeration itself obeys the lossless identities exactly:
    P(out_1 = y) = p_0(y); P(out_2 = y2 | out_1 = y1, round goes on) = p_1(y2)."""
    rng = np.random.default_rng(7)
    V, K = 5, 3
    for tau, L in ((1.0, 3), (0.6, 2), (1.0, 1)):
        rq = _tiny_request(rng, V, K)
        dist = output_distribution(rq["t"], rq["base"], rq["U"], rq["W"], rq["last"], 1.0, tau, L)
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


def _oracle_rounds(rq, V, K, L, tau, N, round_id, dtype="f64"):
    inp = dict(base=_bcast(rq["base"], N), U=rq["U"], W=rq["W"],
               last_tok=np.full(N, rq["last"]), bias_scale=np.ones(N), temp=np.full(N, tau),
               dtype=dtype)
    dr = o.draft_round(inp, SEED, round_id)
    return o.verify(_bcast(rq["t"], N), dr["d"], dr["x"], np.broadcast_to(L, (N,)),
                    np.full(N, tau), SEED, round_id)


def test_monte_carlo_matches_brute_force():
    """The oracle's full draft + verify chain against exact enumeration."""
    rng = np.random.default_rng(11)
    V, K, N = 4, 3, 200000
    for tau, L in ((1.0, 3), (0.6, 2)):
        rq = _tiny_request(rng, V, K)
        dist = output_distribution(rq["t"], rq["base"], rq["U"], rq["W"], rq["last"], 1.0, tau, L)
        r = _oracle_rounds(rq, V, K, L, tau, N, 21)
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


def test_lossless_one_million_rounds():
    """10^6 rounds at V = 16: the first emitted token follows p_0, and the
    second (given the round goes on) follows p_1; Markov bias on, with and
    without a prefix cut, at tau 0.6 and 1.0."""
    rng = np.random.default_rng(13)
    V, K = 16, 3
    total = 0
    for tau, cut in ((1.0, False), (0.6, True), (1.0, True), (0.6, False)):
        rq = _tiny_request(rng, V, K, r=4)
        N = 250000
        L = rng.integers(0, K + 1, N) if cut else np.full(N, K)
        r = _oracle_rounds(rq, V, K, L, tau, N, 100 + total)
        total += N
        z = rq["t"] / tau
        p = np.exp(z - z.max(axis=1, keepdims=True)); p /= p.sum(axis=1, keepdims=True)
        c1 = np.bincount(r["out"][:, 0], minlength=V)
        assert stats.chisquare(c1, p[0] * N).pvalue > 1e-4
        sel = r["n_emit"] >= 2
        c2 = np.bincount(r["out"][sel, 1], minlength=V)
        assert stats.chisquare(c2, p[1] * sel.sum()).pvalue > 1e-4
    assert total == 10 ** 6


def test_independent_draft_rejects_and_corrects():
    rng = np.random.default_rng(17)
    V, K, N = 64, 4, 20000
    t = np.zeros((K + 1, V)); t[:, :4] = 12.0      # target mass on tokens 0..3
    base = np.zeros((K, V)); base[:, 32:36] = 12.0  # draft mass on tokens 32..35
    rq = dict(t=t, base=base, U=np.zeros((V, 2)), W=np.zeros((2, V)), last=0)
    r = _oracle_rounds(rq, V, K, K, 1.0, N, 5, dtype="bf16")
    assert r["a"].mean() < 0.005
    assert np.isin(r["y"][r["a"] == 0], [0, 1, 2, 3]).mean() > 0.99
