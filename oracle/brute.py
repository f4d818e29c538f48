"""Exact enumeration of one speculative round's output distribution (tiny V, K).

TEST INFRASTRUCTURE (see ``oracle/__init__.py`` for who may use it).

For one sampled request (temperature > 0, unrounded fp64 logits) this sums
over every draft path x_1..x_L the probability that the path is drafted
(q of each position, with the Markov bias from the previous token), that its
first m drafts are accepted (min(1, p/q) each), and that the round then emits
a given correction token (from norm(max(0, p - q))) or bonus token (from p of
row L). It uses no uniforms at all, so it is an independent check of the
Monte-Carlo oracle, and it is itself pinned by the lossless property that
rejection sampling guarantees ([P1] "Caveats"; [P3] "Speculative Decoding in
Two Sentences"): the first emitted token is distributed exactly as p of
target row 0, and, given that the round goes on, the next one as p of row 1.
Positions after L are drafted but never verified, so they do not enter.
"""
from __future__ import annotations

from collections import defaultdict
from typing import Dict, Tuple

import numpy as np


def _softmax(z: np.ndarray) -> np.ndarray:
    w = np.exp(z - z.max())
    return w / w.sum()


def output_distribution(target: np.ndarray, base: np.ndarray, U: np.ndarray, W: np.ndarray,
                        last_tok: int, scale: float, tau: float, L: int,
                        R: np.ndarray = None) -> Dict[Tuple[int, ...], float]:
    """P(emitted tokens = seq) for every emitted sequence seq of one request.

    target [K+1, V], base [K, V], U [V, r], W [r, V]; all fp64, tau > 0.
    With R [r, r] the bias comes from the recurrent state
    h_k = U[x_{k-1}] + tanh(h_{k-1} @ R) (h_0 = 0) instead of U[x_{k-1}].
    """
    target = np.asarray(target, np.float64)
    base = np.asarray(base, np.float64)
    U = np.asarray(U, np.float64)
    W = np.asarray(W, np.float64)
    V = target.shape[1]
    dist: Dict[Tuple[int, ...], float] = defaultdict(float)

    r = U.shape[1]

    def walk(k: int, prev: int, prefix: Tuple[int, ...], weight: float, h: np.ndarray) -> None:
        # ``weight`` = P(drafts x_1..x_{k-1} == prefix and all of them accepted);
        # h: the recurrent state of position k - 1
        if k > L:
            p = _softmax(target[L] / tau)
            for yv in range(V):
                dist[prefix + (yv,)] += weight * p[yv]
            return
        hk = U[prev] if R is None else U[prev] + np.tanh(h @ R)
        q = _softmax((base[k - 1] + scale * (hk @ W)) / tau)
        p = _softmax(target[k - 1] / tau)
        resid = np.maximum(0.0, p - q)
        rsum = resid.sum()
        for xv in range(V):
            if q[xv] == 0.0:
                continue
            alpha = min(1.0, p[xv] / q[xv])
            walk(k + 1, xv, prefix + (xv,), weight * q[xv] * alpha, hk)
            if alpha < 1.0 and rsum > 0:
                w_rej = weight * q[xv] * (1.0 - alpha)
                for yv in range(V):
                    if resid[yv] > 0:
                        dist[prefix + (yv,)] += w_rej * resid[yv] / rsum

    walk(1, int(last_tok), (), 1.0, np.zeros(r))
    return dict(dist)
