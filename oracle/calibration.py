"""Sequential Temperature Scaling and expected calibration error, in fp64.

TEST INFRASTRUCTURE ONLY: the CUDA path never imports this module; tests,
``__graft_entry__.smoke()`` and bench.py's CPU baseline do.

[P1] "DSpark turns speculation into a scheduler", "Confidence is a serving
primitive": the confidence head's per-position outputs are calibrated with one
temperature per draft position, fitted left to right (Sequential Temperature
Scaling), because the scheduler multiplies them into survival probabilities.
[P3] "DSpark LLM inference speedup", "The Real Innovation": expected
calibration error falls from 3-8% to about 1%.

Readings (the pages give no loss, grid or binning):
- c_k = sigmoid(z_k / T_k); the quantity fitted at position k is the survival
  product S_k = prod_{i<=k} c_i against the label "drafts 1..k+1 all
  survived" (0-based k), with T_0..T_{k-1} already fixed.
- The fit minimises the negative log-likelihood of S_k over a fixed grid of
  STS_GRID temperatures, log-spaced on [STS_T_LO, STS_T_HI]; the lowest index
  wins a tie. S is clamped to [STS_EPS, 1 - STS_EPS] inside the logarithms.
- ECE uses ECE_BINS equal-width bins of S on [0, 1] (S = 1 goes to the last
  bin): sum over bins of (n_bin / N) * |mean S - mean label|.
"""
from __future__ import annotations

import numpy as np

STS_GRID = 256
STS_T_LO = 0.05
STS_T_HI = 20.0
STS_EPS = 1e-12
ECE_BINS = 15
# relative window inside which two grid losses count as tied (parity flag)
NLL_TIE_WINDOW = 1e-9


def temperature_grid() -> np.ndarray:
    """The STS_GRID candidate temperatures, log-spaced on [STS_T_LO, STS_T_HI]."""
    i = np.arange(STS_GRID, dtype=np.float64)
    return np.exp(np.log(STS_T_LO) + i * (np.log(STS_T_HI) - np.log(STS_T_LO)) / (STS_GRID - 1))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, np.float64)))


def survival(z: np.ndarray, T: np.ndarray, upto: int) -> np.ndarray:
    """S[n] = prod_{i <= upto} sigmoid(z[n, i] / T[i])."""
    z = np.asarray(z, np.float64)
    S = np.ones(z.shape[0])
    for i in range(upto + 1):
        S = S * sigmoid(z[:, i] / float(T[i]))
    return S


def nll(pred: np.ndarray, label: np.ndarray) -> float:
    """-sum(y log S + (1 - y) log(1 - S)), S clamped to [STS_EPS, 1 - STS_EPS]."""
    p = np.clip(np.asarray(pred, np.float64), STS_EPS, 1.0 - STS_EPS)
    y = np.asarray(label, np.float64)
    return float(-np.sum(y * np.log(p) + (1.0 - y) * np.log1p(-p)))


def ece(pred: np.ndarray, label: np.ndarray, nbins: int = ECE_BINS) -> float:
    """Expected calibration error of predictions in [0, 1] against 0/1 labels."""
    p = np.asarray(pred, np.float64)
    y = np.asarray(label, np.float64)
    b = np.minimum((p * nbins).astype(np.int64), nbins - 1)
    total = 0.0
    for k in range(nbins):
        m = b == k
        n = int(m.sum())
        if n:
            total += n / len(p) * abs(p[m].mean() - y[m].mean())
    return total


def sts_fit(z: np.ndarray, survived: np.ndarray):
    """Left-to-right fit of one temperature per position.

    z [N, K] confidence logits, survived [N, K] 0/1 labels (column k: drafts
    1..k+1 all accepted). Returns dict(T [K], index [K] (grid index),
    nll [K], tie [K] (the best two grid losses within NLL_TIE_WINDOW),
    ece_before [K] (T = 1), ece_after [K]).
    """
    z = np.asarray(z, np.float64)
    y = np.asarray(survived, np.float64)
    N, K = z.shape
    grid = temperature_grid()
    T = np.ones(K)
    idx = np.zeros(K, np.int64)
    best = np.zeros(K)
    tie = np.zeros(K, bool)
    for k in range(K):
        prev = survival(z, T, k - 1) if k > 0 else np.ones(N)
        losses = np.array([nll(prev * sigmoid(z[:, k] / t), y[:, k]) for t in grid])
        i = int(np.argmin(losses))  # lowest index among equal minima
        others = np.delete(losses, i)
        tie[k] = bool(np.min(np.abs(others - losses[i])) <= NLL_TIE_WINDOW * abs(losses[i]))
        idx[k], T[k], best[k] = i, grid[i], losses[i]
    ones = np.ones(K)
    before = np.array([ece(survival(z, ones, k), y[:, k]) for k in range(K)])
    after = np.array([ece(survival(z, T, k), y[:, k]) for k in range(K)])
    return dict(T=T, index=idx, nll=best, tie=tie, ece_before=before, ece_after=after)
