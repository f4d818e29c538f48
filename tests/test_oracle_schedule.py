"""Pins of the oracle's calibrated confidence, survival product and prefix cut (no GPU).

The survival product is pinned by hand products ("DSpark turns speculation
into a scheduler", "Confidence is a serving primitive", survival equation).
The early-stopping cut is pinned only as a definition: hand-worked cases
plus the structural properties the rule must have. Its parity with the
scheduler of the DSpark paper itself is unpinned (that appendix is not
among the pages)."""
import numpy as np

from conftest import golden_path
from oracle import dspark as o


def _cases():
    for line in open(golden_path("schedule_cases.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, bk, S, cost, fixed, mode, thr, L, flag = (t.strip() for t in line.split("|"))
        B, K = (int(v) for v in bk.split())
        yield (name, np.array([float(v) for v in S.split(",")]).reshape(B, K),
               np.array([float(v) for v in cost.split(",")]), float(fixed), int(mode), float(thr),
               [int(v) for v in L.split(",")], flag == "1")


def test_hand_worked_cuts():
    for name, S, cost, fixed, mode, thr, L, want_flag in _cases():
        got, flag = o.prefix_cut(S, cost, fixed, mode, thr)
        assert got.tolist() == L, name
        assert flag == want_flag, name


def test_survival_hand_product():
    # sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, sigmoid(2 ln 3 / 2) = 3/4
    z = np.array([[0.0, np.log(3.0), 2 * np.log(3.0)]])
    c, S = o.survival(z, np.array([1.0, 1.0, 2.0]))
    np.testing.assert_allclose(c[0], [0.5, 0.75, 0.75], rtol=1e-15)
    np.testing.assert_allclose(S[0], [0.5, 0.375, 0.28125], rtol=1e-15)


def _random_case(rng, B, K):
    z = rng.normal(1.0, 1.5, (B, K))
    _, S = o.survival(z, np.linspace(1.0, 1.6, K))
    n = B * (K + 1)
    cost = np.where(np.arange(1, n + 1) <= B * 2, 1.0, 1.6)
    return S, cost


def test_cut_structure():
    """Admitted drafts are per-request prefixes visited in S order; the objective
    never decreases along the admitted walk; the first rejected draft would lower it."""
    rng = np.random.default_rng(0)
    for trial in range(50):
        B, K = int(rng.integers(1, 9)), int(rng.integers(1, 7))
        S, cost = _random_case(rng, B, K)
        fixed = float(rng.uniform(0, 3 * B))
        L, _ = o.prefix_cut(S, cost, fixed)
        assert np.all((0 <= L) & (L <= K))
        admitted = np.zeros((B, K), bool)
        for b in range(B):
            admitted[b, :L[b]] = True
        if admitted.any() and (~admitted).any():
            assert S[admitted].min() >= S[~admitted].max() - 1e-15
        n = B + admitted.sum()
        A = B + S[admitted].sum()
        C = fixed + cost[:n].sum()
        if (~admitted).any():
            nxt = S[~admitted].max()
            assert (A + nxt) / (C + cost[n]) < A / C


def test_no_look_ahead():
    """Lowering the survival of drafts that were not admitted never changes the cut
    (the decision on (b, k) looks only at S_b,1..k: a stopping rule)."""
    rng = np.random.default_rng(1)
    for trial in range(50):
        B, K = int(rng.integers(1, 9)), int(rng.integers(2, 7))
        S, cost = _random_case(rng, B, K)
        L, _ = o.prefix_cut(S, cost, float(B))
        S2 = S.copy()
        for b in range(B):
            if L[b] + 1 < K:
                S2[b, L[b] + 1:] *= rng.uniform(0.0, 1.0)
        L2, _ = o.prefix_cut(S2, cost, float(B))
        assert np.array_equal(L, L2)


def test_limits():
    S = np.array([[0.99, 0.98], [0.97, 0.5]])
    L, _ = o.prefix_cut(S, np.ones(6), 0.0)            # flat cost, no fixed cost: nothing pays
    assert L.tolist() == [0, 0]
    L, _ = o.prefix_cut(S, np.ones(6), 1e6)            # huge fixed cost: every draft pays
    assert L.tolist() == [2, 2]
    L, _ = o.prefix_cut(S, np.ones(6), 0.0, mode=2)
    assert L.tolist() == [2, 2]
    L, _ = o.prefix_cut(S, np.ones(6), 0.0, mode=1, threshold=0.975)
    assert L.tolist() == [2, 0]


def test_load_trims_budget():
    """A steeper cost curve (a loaded engine) never verifies more tokens
    ("DSpark turns speculation into a scheduler", "Confidence is a serving
    primitive": the scheduler trims the budget as concurrency rises)."""
    rng = np.random.default_rng(2)
    B, K = 64, 5
    S, _ = _random_case(rng, B, K)
    n = B * (K + 1)
    prev = None
    for slope in (0.0, 0.5, 1.0, 2.0, 4.0):
        cost = 1.0 + slope * np.arange(n) / n
        L, _ = o.prefix_cut(S, cost, float(B))
        if prev is not None:
            assert L.sum() <= prev
        prev = L.sum()


def test_cost_rule_is_optimal_for_non_decreasing_costs():
    """Against brute force over every per-request prefix vector: when the step
    costs never decrease (a convex C(n), as in every cost table here), the
    early-stopping walk reaches the least cost per emitted token, max A/C, of
    the latency equation ("DSpark turns speculation into a scheduler", "The
    speculative loop"). Why it must: for a fixed count of admitted drafts the
    largest S form per-request prefixes and maximise A, and adding a draft
    moves A/C towards S/step (a mediant), which only falls along the walk, so
    A/C rises and then only falls."""
    import itertools
    rng = np.random.default_rng(5)
    for trial in range(300):
        B, K = int(rng.integers(1, 4)), int(rng.integers(1, 4))
        z = rng.normal(1.0, 2.0, (B, K))
        _, S = o.survival(z, np.linspace(1.0, 1.6, K))
        n = B * (K + 1)
        if trial % 2:
            cost = 0.2 + np.cumsum(rng.exponential(0.3, n))           # strictly rising
        else:
            at = int(rng.integers(B, n + 1))                           # one step, as DSpark-5
            cost = np.where(np.arange(1, n + 1) <= at, 1.0, float(rng.uniform(1.0, 3.0)))
        fixed = float(rng.uniform(0.0, 2.0 * B))
        L, _ = o.prefix_cut(S, cost, fixed)

        def ratio(Lv):
            m = int(np.sum(Lv))
            A = B + sum(S[b, :Lv[b]].sum() for b in range(B))
            return A / (fixed + cost[:B + m].sum())

        best = max(ratio(Lv) for Lv in itertools.product(range(K + 1), repeat=B))
        assert ratio(L) >= best * (1.0 - 1e-12), (trial, L.tolist(), ratio(L), best)
