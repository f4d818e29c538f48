"""Plain fp64 CPU oracle of one DSpark-style speculative round.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import or call this
module. It shares no code with the CUDA path and imports nothing from it.

Sources (web pages on DSpark, cited by title and section):

* [P1] "DSpark turns speculation into a scheduler" (benebsworth.pages.dev):
  "The speculative loop" (latency equation L = (T_draft + T_verify)/tau),
  "DSpark's semi-autoregressive compromise" (parallel base logits plus a
  prefix-dependent transition bias; Markov head = low-rank signal from the
  previous sampled token), "Confidence is a serving primitive" (survival
  product P(prefix 1:k survives) = prod c_i; Sequential Temperature Scaling;
  hardware-aware prefix scheduler), "Caveats" (lossless only with the
  correct acceptance rule).
* [P2] "notes/dspark-deepseek" (skandtandon.pages.dev), "Sources": the
  acceptance rule comes from "Fast Inference from Transformers via
  Speculative Decoding" (accept x with probability min(1, p(x)/q(x));
  on rejection sample from norm(max(0, p - q))).
* [P3] "DSpark LLM inference speedup" (probackend.com): "Speculative
  Decoding in Two Sentences" (accept the longest valid prefix, append one
  bonus token), "The Semi-Autoregressive Trick" (Markov head, rank 256,
  looks only at the preceding token), "The Real Innovation:
  Confidence-Scheduled Verification" (per-position confidence, Sequential
  Temperature Scaling, prefix scheduler with an early-stopping rule).

Readings where the pages are silent (each marked R<n> below):

* R2  the Markov bias also applies at k = 1, from the last committed token.
* R3  q is the softmax of the *stored* draft logits d = round(base + bias),
      so verification uses exactly the distribution that was sampled.
* R4  inverse CDF in index order: x = min{i : sum_{j<=i} w_j > u * Z};
      if no i qualifies (rounding only), the last i with w_i > 0.
* R5  Sequential Temperature Scaling is applied as c_k = sigmoid(z_k / T_k).
* R6  the early-stopping prefix cut (see ``prefix_cut``).
* R7  acceptance is strict: accept iff u < p(x)/q(x).
* R8  a residual of exact zero (floating point only) falls back to p.
* R11 the recurrent head (the pages name an optional head that tracks the
      whole block prefix and give no equations): a state h_k in R^r,
      h_0 = 0, h_k = U[x_{k-1}] + tanh(h_{k-1} @ R), stored in the logits'
      dtype, and bias_k = scale_b * h_k @ W. With R = 0 it is the Markov head
      bit for bit.
* Greedy requests (temperature 0) draft argmax d, accept iff the draft
  equals argmax of the target row, and emit argmax of the target row;
  ties go to the lowest index.

Parity flags. Where the fp64 decision lies within the stated window of its
boundary, the CUDA path (fp32) may legitimately decide the other way; such
points are flagged, and the tests then adopt the GPU's decision there
(teacher forcing) or exempt the rest of the request.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from .philox import (PURPOSE_ACCEPT, PURPOSE_BONUS, PURPOSE_DRAFT,
                     PURPOSE_RESIDUAL, uniform)

# Window around a CDF or acceptance boundary inside which a draw is flagged.
U_WINDOW = 1e-6
# Relative window around a bf16 rounding midpoint inside which d is flagged.
BF16_MID_WINDOW = 2.0 ** -20
# Relative window for a near-tie of the scheduler's comparisons and sort keys.
CUT_WINDOW = 1e-6


# --------------------------------------------------------------------------
# storage rounding (R3)
# --------------------------------------------------------------------------

def round_to_bf16(v: np.ndarray):
    """Round fp64 values to the nearest bf16 (ties to even).

    Returns (rounded values as fp64, flag) where flag marks values within
    BF16_MID_WINDOW (relative) of a rounding midpoint.
    """
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)                 # v = m * 2**e, 0.5 <= |m| < 1
    s = m * 256.0                      # 8 significant bits
    r = np.rint(s)                     # round half to even
    out = np.ldexp(r, e - 8)
    frac = np.abs(s - np.trunc(s))
    flag = np.abs(frac - 0.5) < BF16_MID_WINDOW * np.abs(s)
    return out, flag


def round_to_storage(v: np.ndarray, dtype: str):
    """Round to the storage type ('bf16', 'f32' or 'f64'); returns (values, flags)."""
    if dtype == "bf16":
        return round_to_bf16(v)
    if dtype == "f32":
        return np.asarray(v, np.float64).astype(np.float32).astype(np.float64), np.zeros(np.shape(v), bool)
    if dtype == "f64":
        return np.asarray(v, np.float64).copy(), np.zeros(np.shape(v), bool)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# a1, a2: Markov-biased draft logits and position-by-position sampling
# --------------------------------------------------------------------------

def markov_bias(U: np.ndarray, W: np.ndarray, prev: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """bias[b, :] = scale_b * U[prev_b, :] @ W  (fp64).

    [P1] "DSpark's semi-autoregressive compromise": a low-rank transition
    signal from the previous sampled token; [P3] "The Semi-Autoregressive
    Trick": rank-256 factorisation that looks only at the preceding token.
    """
    U = np.asarray(U, np.float64)
    W = np.asarray(W, np.float64)
    rows = U[np.asarray(prev, np.int64)]                 # [B, r]
    return np.asarray(scale, np.float64)[:, None] * (rows @ W)


def draft_logits(base_k: np.ndarray, bias: np.ndarray, dtype: str,
                 bias_abs: Optional[np.ndarray] = None, r: int = 0):
    """d = round_storage(base + bias) (R3). Returns (d, midpoint flags).

    For bf16 storage an element is flagged when its fp64 value lies within
    the fp32 error of the CUDA path's sum of a rounding midpoint:
    2^-22 |v| (the final fp32 add) + r 2^-23 |scale| sum_j |U_j W_jv|
    (fp32 accumulation of r products), given as ``bias_abs`` =
    |scale| (|U[prev]| @ |W|). Without ``bias_abs`` the relative window
    BF16_MID_WINDOW is used.
    """
    v = np.asarray(base_k, np.float64) + bias
    if dtype != "bf16":
        return round_to_storage(v, dtype)
    m, e = np.frexp(v)
    s = m * 256.0
    out = np.ldexp(np.rint(s), e - 8)
    mid = np.ldexp(np.trunc(s) + np.sign(s) * 0.5, e - 8)
    if bias_abs is None:
        win = BF16_MID_WINDOW * np.abs(v)
    else:
        win = 2.0 ** -22 * np.abs(v) + r * 2.0 ** -23 * bias_abs
    with np.errstate(invalid="ignore"):  # infinite logits are never near a midpoint
        flag = np.isfinite(v) & (np.abs(v - mid) <= win)
    return out, flag


def recurrent_state(U: np.ndarray, R: np.ndarray, prev: np.ndarray, h_prev: np.ndarray,
                    dtype: str):
    """The recurrent head's state for one position (R11), every request.

    h = round_storage(U[prev] + tanh(h_prev @ R)) with h_prev [B, r] the
    previous position's stored state (zeros before the first position), so
    that the state carries the whole drafted prefix, not only the previous
    token ([P1] "DSpark's semi-autoregressive compromise": recurrent head
    machinery beside the Markov head; [P3] "The Semi-Autoregressive Trick": an
    optional head that tracks the full block prefix).

    Returns (h [B, r], flag [B, r]). For bf16 storage an element is flagged
    when its fp64 value lies within the error of a device computing it in fp32
    of a rounding midpoint. The device sums h_j R_ji with fused multiply-adds
    in ascending j, each rounding its partial sum once, so its error in a is
    at most 2^-24 sum_j |S_j| to first order (S_j the exact partial sums in
    that order); tanh adds 2^-22 |tanh a| (two units in the last place; its
    slope is at most 1, so the error in a passes through unamplified) and the
    final add 2^-23 |v|.
    """
    U = np.asarray(U, np.float64)
    R = np.asarray(R, np.float64)
    h_prev = np.asarray(h_prev, np.float64)
    h, flag, _ = recurrent_state_window(U, R, prev, h_prev, dtype)
    return h, flag


def recurrent_state_window(U: np.ndarray, R: np.ndarray, prev: np.ndarray, h_prev: np.ndarray,
                           dtype: str):
    """``recurrent_state`` plus the error window of every element (the bound
    above, in absolute terms). For fp32 storage there is no rounding point to
    flag: every element is returned flagged, and a check compares a device's
    state with this one within the window instead."""
    a = h_prev @ R
    th = np.tanh(a)
    v = U[np.asarray(prev, np.int64)] + th
    partial = np.cumsum(h_prev[:, :, None] * R[None, :, :], axis=1)   # [B, j, i]
    acc_err = 2.0 ** -24 * np.abs(partial).sum(axis=1)
    win = acc_err + 2.0 ** -22 * np.abs(th) + 2.0 ** -23 * np.abs(v)
    if dtype != "bf16":
        out, _ = round_to_storage(v, dtype)
        return out, np.ones(np.shape(v), bool), win + 2.0 ** -24 * np.abs(v)
    m, e = np.frexp(v)
    sc = m * 256.0
    out = np.ldexp(np.rint(sc), e - 8)
    mid = np.ldexp(np.trunc(sc) + np.sign(sc) * 0.5, e - 8)
    flag = np.isfinite(v) & (np.abs(v - mid) <= win)
    return out, flag, win


def inverse_cdf(w: np.ndarray, u: np.ndarray, window: float = U_WINDOW, normalized: bool = True):
    """Inverse-CDF draw from unnormalised non-negative weights, per row (R4).

    w [B, V] >= 0, u [B] in [0, 1). Returns (index [B], Z [B], flag [B]).
    The flag is raised when u lies within ``window`` of the CDF at x-1 or x:
    on the normalised CDF (``normalized``) or on the unnormalised one
    (u*Z against the running sums).
    """
    w = np.asarray(w, np.float64)
    B, V = w.shape
    csum = np.cumsum(w, axis=1)
    Z = csum[:, -1]
    thr = u * Z
    x = (csum <= thr[:, None]).sum(axis=1)               # first i with csum_i > u*Z
    none = x >= V
    if none.any():
        for b in np.nonzero(none)[0]:
            pos = np.nonzero(w[b] > 0)[0]
            x[b] = pos[-1] if len(pos) else 0
    rows = np.arange(B)
    lo = np.where(x > 0, csum[rows, np.maximum(x - 1, 0)], 0.0)
    hi = csum[rows, x]
    if normalized:
        with np.errstate(invalid="ignore", divide="ignore"):
            flag = (np.abs(u - lo / Z) < window) | (np.abs(u - hi / Z) < window)
    else:
        flag = (np.abs(thr - lo) < window) | (np.abs(thr - hi) < window)
    flag |= none
    return x.astype(np.int64), Z, flag


def softmax_parts(logits: np.ndarray, tau: np.ndarray):
    """z = logits / tau, m = max z, w = exp(z - m), Z = sum w, lse = m + log Z."""
    z = np.asarray(logits, np.float64) / np.asarray(tau, np.float64)[:, None]
    m = z.max(axis=1)
    w = np.exp(z - m[:, None])
    Z = w.sum(axis=1)
    return w, Z, m + np.log(Z)


def sample_position(d: np.ndarray, tau: np.ndarray, u: np.ndarray) -> Dict[str, np.ndarray]:
    """Sample one draft position from q = softmax(d / tau) for every request.

    Greedy requests (tau = 0) take argmax d; for them q_tok = 1 and q_lse is
    the maximum logit. Returns x, q_lse, q_tok and the flag of each draw.
    """
    d = np.asarray(d, np.float64)
    tau = np.asarray(tau, np.float64)
    B, V = d.shape
    x = np.argmax(d, axis=1).astype(np.int64)
    q_lse = d.max(axis=1)
    q_tok = np.ones(B)
    flag = np.zeros(B, bool)
    s = tau > 0
    if s.any():
        w, Z, lse = softmax_parts(d[s], tau[s])
        xs, _, fs = inverse_cdf(w, u[s])
        x[s] = xs
        q_lse[s] = lse
        q_tok[s] = w[np.arange(len(xs)), xs] / Z
        flag[s] = fs
    return dict(x=x, q_lse=q_lse, q_tok=q_tok, flag=flag)


def draft_position(base_k, U, W, prev, scale, tau, u, dtype: str,
                   h: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """One draft position for every request: bias, stored d, and the draw.

    The bias multiplies W by U[prev] (Markov head) or, when given, by the
    recurrent state h [B, r] (R11)."""
    Uf = np.asarray(U, np.float64)
    Wf = np.asarray(W, np.float64)
    if h is None:
        bias = markov_bias(Uf, Wf, prev, scale)
        rows = Uf[np.asarray(prev, np.int64)]
    else:
        rows = np.asarray(h, np.float64)
        bias = np.asarray(scale, np.float64)[:, None] * (rows @ Wf)
    babs = np.abs(np.asarray(scale, np.float64))[:, None] * (np.abs(rows) @ np.abs(Wf))
    d, d_flag = draft_logits(base_k, bias, dtype, babs, Uf.shape[1])
    s = sample_position(d, tau, u)
    return dict(d=d, d_flag=d_flag, x=s["x"], q_lse=s["q_lse"], q_tok=s["q_tok"],
                x_flag=s["flag"])


def draft_round(inp: Dict[str, np.ndarray], seed: int, round_id: int,
                teacher: Optional[Dict[str, np.ndarray]] = None) -> Dict[str, np.ndarray]:
    """All K positions of the semi-autoregressive draft (a1 + a2).

    For k = 1..K: bias from x_{k-1} (x_0 = last committed token, R2), the
    stored draft logits d_k, then x_k ~ softmax(d_k / tau). With ``inp["R"]``
    [r, r] the bias comes from the recurrent state h_k of R11 instead of
    U[x_{k-1}] alone; the states are returned as ``h`` [B, K, r].

    Teacher forcing: with ``teacher`` (the GPU's "d" [B,K,V] and "x" [B,K],
    and "h" [B,K,r] for the recurrent head), a flagged d or h element takes
    the teacher's value and a flagged draw takes the teacher's token;
    ``forced`` counts how often that changed a logit or a token, ``h_forced``
    how many state elements were adopted.
    """
    base = inp["base"]
    B, K, V = base.shape
    prev = np.asarray(inp["last_tok"], np.int64)
    tau = np.asarray(inp["temp"], np.float64)
    req = np.asarray(inp.get("request_ids", np.arange(B)), np.int64)
    d = np.empty((B, K, V))
    x = np.empty((B, K), np.int64)
    q_lse = np.empty((B, K))
    q_tok = np.empty((B, K))
    d_flag = np.zeros((B, K), bool)
    x_flag = np.zeros((B, K), bool)
    forced = 0
    Rm = inp.get("R")
    r = np.shape(inp["U"])[1]
    hs = np.zeros((B, K, r)) if Rm is not None else None
    h_flag = np.zeros((B, K), bool)
    h_forced = 0
    h_excess = 0.0  # fp32 states: the largest amount by which a device state leaves its window
    h = np.zeros((B, r))
    for k in range(1, K + 1):
        u = uniform(seed, req, k, PURPOSE_DRAFT, round_id)
        if Rm is not None:
            h, hf, hwin = recurrent_state_window(inp["U"], Rm, prev, h, inp["dtype"])
            if teacher is not None and hf.any():
                th = np.asarray(teacher["h"][:, k - 1], np.float64)
                if inp["dtype"] != "bf16":  # no rounding point: the device's state within the window
                    h_excess = max(h_excess, float((np.abs(th - h) - hwin).max()))
                h_forced += int((hf & (th != h)).sum())
                h = np.where(hf, th, h)
            hs[:, k - 1] = h
            h_flag[:, k - 1] = hf.any(axis=1) if inp["dtype"] == "bf16" else False
        st = draft_position(base[:, k - 1], inp["U"], inp["W"], prev, inp["bias_scale"],
                            tau, u, inp["dtype"], h if Rm is not None else None)
        if teacher is not None and st["d_flag"].any():
            td = np.asarray(teacher["d"][:, k - 1], np.float64)
            diff = st["d_flag"] & (td != st["d"])
            if diff.any():
                forced += int(diff.sum())
                dk = np.where(st["d_flag"], td, st["d"])
                s2 = sample_position(dk, tau, u)
                st.update(d=dk, x=s2["x"], q_lse=s2["q_lse"], q_tok=s2["q_tok"],
                          x_flag=s2["flag"])
        d_flag[:, k - 1] = st["d_flag"].any(axis=1)
        if teacher is not None:
            tx = np.asarray(teacher["x"][:, k - 1], np.int64)
            take = st["x_flag"] & (tx != st["x"])
            if take.any():
                # the adopted token's own draft probability q(x)
                forced += int(take.sum())
                st["x"] = np.where(take, tx, st["x"])
                rows = np.nonzero(take & (tau > 0))[0]
                if len(rows):
                    w, Z, _ = softmax_parts(st["d"][rows], tau[rows])
                    st["q_tok"][rows] = w[np.arange(len(rows)), st["x"][rows]] / Z
        d[:, k - 1] = st["d"]
        x[:, k - 1], q_lse[:, k - 1], q_tok[:, k - 1] = st["x"], st["q_lse"], st["q_tok"]
        x_flag[:, k - 1] = st["x_flag"]
        prev = st["x"]
    return dict(d=d, d_flag=d_flag, x=x, q_lse=q_lse, q_tok=q_tok, x_flag=x_flag,
                h=hs, h_flag=h_flag, h_forced=h_forced, h_excess=h_excess, forced=forced)


# --------------------------------------------------------------------------
# a3, a4: calibrated confidence, survival and the prefix cut
# --------------------------------------------------------------------------

def survival(conf_logit: np.ndarray, pos_temp: np.ndarray):
    """c_{b,k} = sigmoid(z_{b,k} / T_k) (R5), S_{b,k} = prod_{i<=k} c_{b,i}.

    [P1] "Confidence is a serving primitive", survival equation; per-position
    temperatures from Sequential Temperature Scaling.
    """
    z = np.asarray(conf_logit, np.float64) / np.asarray(pos_temp, np.float64)[None, :]
    c = 1.0 / (1.0 + np.exp(-z))
    return c, np.cumprod(c, axis=1)


def prefix_cut(S: np.ndarray, step_cost: np.ndarray, fixed_cost: float,
               mode: int = 0, threshold: float = 0.0):
    """Per-request verify lengths L_b from survival products (R6).

    mode 0, the early-stopping cost rule. Verifying n tokens in the batch
    costs C(n) = fixed_cost + sum_{m<=n} step_cost[m] (1-based m; every
    request always verifies one slot for its correction or bonus token, so
    n starts at B). Selected drafts D yield A(D) = B + sum_{(b,k) in D} S_bk
    expected emitted tokens; the latency equation of [P1] "The speculative
    loop" asks for the least cost per emitted token, i.e. the largest A/C.
    All B*K drafts are visited by descending S (ties: smaller k, then
    smaller b); a draft is admitted iff it does not lower A/C, i.e.
    S_j * C_{j-1} >= A_{j-1} * step_cost[B + j]; the walk stops at the first
    draft that fails and admits nothing after it. Because S is non-increasing
    along a request, every admitted set is a union of per-request prefixes,
    and whether (b, k) is admitted depends on request b only through
    S_{b,1..k}: a stopping rule, never a look at b's later positions
    ([P3] "The Real Innovation": an early-stopping rule keeps the scheduler
    lossless).

    mode 1, the static threshold ([P1] "Confidence is a serving primitive":
    "verify while confidence > x"): L_b = #{k : S_{b,k} >= threshold}.

    mode 2, no cut: L_b = K.

    Returns (L [B], flag) where the flag marks a decision within CUT_WINDOW
    (relative) of its boundary.
    """
    S = np.asarray(S, np.float64)
    B, K = S.shape
    if mode == 2:
        return np.full(B, K, np.int64), False
    if mode == 1:
        L = (S >= threshold).sum(axis=1).astype(np.int64)
        flag = bool((np.abs(S - threshold) <= CUT_WINDOW * max(abs(threshold), 1e-300)).any())
        return L, flag
    cost = np.asarray(step_cost, np.float64)
    items = sorted(((S[b, k], k, b) for b in range(B) for k in range(K)),
                   key=lambda t: (-t[0], t[1], t[2]))
    A = float(B)
    C = float(fixed_cost) + cost[:B].sum()
    L = np.zeros(B, np.int64)
    flag = False
    stop = len(items)
    for j, (s, k, b) in enumerate(items, start=1):
        c = cost[B + j - 1]
        lhs, rhs = s * C, A * c
        if abs(lhs - rhs) <= CUT_WINDOW * max(abs(lhs), abs(rhs)):
            flag = True
        if lhs >= rhs:
            A += s
            C += c
            L[b] += 1
        else:
            stop = j - 1
            break
    if 0 < stop < len(items):
        s_in, s_out = items[stop - 1][0], items[stop][0]
        if s_in - s_out <= CUT_WINDOW * s_in:
            flag = True
    return L, flag


def cut_alternatives(S: np.ndarray, step_cost: np.ndarray, fixed_cost: float,
                     mode: int = 0, threshold: float = 0.0):
    """The other cuts a flagged near-tie of ``prefix_cut`` leaves possible.

    A device that evaluates the same rule in a different rounding order may
    decide a near-tied comparison the other way, but only that comparison:
    every other decision of the walk follows from it. So each alternative
    flips exactly one flagged decision and walks on by the rule:

    * mode 0, an admission test within CUT_WINDOW of its boundary at walk
      position i: if the test admitted, the walk stops at i instead; if it
      was the stopping test, the draft is admitted and the walk goes on.
    * mode 0, survival products within CUT_WINDOW of each other on both
      sides of the stopping point (a device may order them the other way):
      the admitted draft and the first refused one trade places.
    * mode 1, a survival product within CUT_WINDOW of the threshold: that
      request's count moves by one.

    Returns a list of cut vectors [B] (empty when nothing was flagged). A
    check that adopts a device's cut only when it equals one of these still
    catches any cut that differs elsewhere.
    """
    S = np.asarray(S, np.float64)
    B, K = S.shape
    alts = []
    if mode == 2:
        return alts
    if mode == 1:
        L = (S >= threshold).sum(axis=1).astype(np.int64)
        near = np.abs(S - threshold) <= CUT_WINDOW * max(abs(threshold), 1e-300)
        for b, k in zip(*np.nonzero(near)):
            alt = L.copy()
            alt[b] = k if S[b, k] >= threshold else k + 1
            alts.append(alt)
        return alts
    cost = np.asarray(step_cost, np.float64)
    items = sorted(((S[b, k], k, b) for b in range(B) for k in range(K)),
                   key=lambda t: (-t[0], t[1], t[2]))
    n = len(items)

    def walk(order, flip):
        """Admitted count per request; the decision at walk position ``flip``
        (0-based, or -1 for none) is inverted. Also returns the stop and the
        near-tied positions seen."""
        A = float(B)
        C = float(fixed_cost) + cost[:B].sum()
        L = np.zeros(B, np.int64)
        near = []
        stop = n
        for i, (s, k, b) in enumerate(order):
            c = cost[B + i]
            lhs, rhs = s * C, A * c
            if abs(lhs - rhs) <= CUT_WINDOW * max(abs(lhs), abs(rhs)):
                near.append(i)
            admit = lhs >= rhs
            if i == flip:
                admit = not admit
            if not admit:
                stop = i
                break
            A += s
            C += c
            L[b] += 1
        return L, stop, near

    L0, stop, near = walk(items, -1)
    for i in near:
        alts.append(walk(items, i)[0])
    if 0 < stop < n:
        # near-equal survival products straddling the stopping point
        s_in = items[stop - 1][0]
        s_out = items[stop][0]
        lo = [i for i in range(stop) if items[i][0] - s_out <= CUT_WINDOW * items[i][0]]
        hi = [i for i in range(stop, n) if s_in - items[i][0] <= CUT_WINDOW * s_in]
        for i in lo:
            for j in hi:
                order = list(items)
                order[i], order[j] = order[j], order[i]
                alts.append(walk(order, -1)[0])
    return [a for a in alts if not np.array_equal(a, L0)]


def adopt_cut(L: np.ndarray, alts, L_device: np.ndarray):
    """The cut parity compares against: the oracle's own ``L``, or the
    device's cut when it equals one of the flagged alternatives ``alts``.
    Returns (cut, requests changed by adopting it)."""
    L_device = np.asarray(L_device, np.int64)
    if np.array_equal(L, L_device):
        return L, 0
    for alt in alts:
        if np.array_equal(alt, L_device):
            return L_device.copy(), int((L_device != L).sum())
    return L, 0


# --------------------------------------------------------------------------
# a5, a6, a7: lossless verification, residual / bonus, emitted tokens
# --------------------------------------------------------------------------

def verify(target: np.ndarray, d: np.ndarray, x: np.ndarray, L: np.ndarray,
           tau: np.ndarray, seed: int, round_id: int,
           request_ids: Optional[np.ndarray] = None,
           teacher: Optional[Dict[str, np.ndarray]] = None) -> Dict[str, np.ndarray]:
    """Rejection-sampling verification of every request's first L_b drafts.

    Target row j (0-based) scores draft token j+1; row L_b gives the bonus.
    For k = 1..L_b: p = softmax(t_{k-1} / tau), q = softmax(d_k / tau),
    accept x_k iff u_acc < p(x_k) / q(x_k) (R7). a_b = drafts accepted before
    the first rejection. If a_b < L_b the correction y is drawn from
    norm(max(0, p - q)) over row a_b (R8 on an exact-zero residual); else
    the bonus y is drawn from p of row L_b. Greedy requests accept iff
    x_k == argmax t_{k-1} and emit argmax t_{a_b}.

    [P1] intro and "Caveats"; [P2] "Sources" (the acceptance rule of
    "Fast Inference from Transformers via Speculative Decoding"); [P3]
    "Speculative Decoding in Two Sentences" (longest valid prefix plus one
    bonus token, exactly the target distribution).

    The residual draw is flagged on the unnormalised residual CDF (u*R
    within U_WINDOW of a running sum of max(0, p - q)), the scale on which
    the fp32 error of p and q lives; every other draw on the normalised CDF.

    Teacher forcing: with ``teacher`` (the GPU's "a" and "y"), a flagged
    acceptance test takes the teacher's decision and a flagged final draw
    the teacher's token; ``forced`` counts how often that changed anything.

    Returns a [B], y [B], out [B, K+1], n_emit [B], flags acc_flag [B, K]
    and y_flag [B], and ``forced``.
    """
    target = np.asarray(target, np.float64)
    d = np.asarray(d, np.float64)
    B, K1, V = target.shape
    x = np.asarray(x, np.int64)
    L = np.asarray(L, np.int64)
    tau = np.asarray(tau, np.float64)
    req = np.arange(B) if request_ids is None else np.asarray(request_ids, np.int64)
    greedy = tau == 0
    a = np.zeros(B, np.int64)
    rejected = np.zeros(B, bool)
    done = L == 0
    acc_flag = np.zeros((B, K1 - 1), bool)
    forced = 0
    for k in range(1, K1):
        idx = np.nonzero(~done & (k <= L))[0]
        if len(idx) == 0:
            continue
        xk = x[idx, k - 1]
        ok = np.zeros(len(idx), bool)
        g = greedy[idx]
        if g.any():
            ok[g] = xk[g] == np.argmax(target[idx[g], k - 1], axis=1)
        s = ~g
        if s.any():
            rows = idx[s]
            wp, Zp, _ = softmax_parts(target[rows, k - 1], tau[rows])
            wq, Zq, _ = softmax_parts(d[rows, k - 1], tau[rows])
            n = np.arange(len(rows))
            ratio = (wp[n, xk[s]] / Zp) / (wq[n, xk[s]] / Zq)
            u = uniform(seed, req[rows], k, PURPOSE_ACCEPT, round_id)
            oks = u < ratio
            fl = np.abs(u - ratio) < U_WINDOW
            acc_flag[rows, k - 1] = fl
            if teacher is not None and fl.any():
                t_ok = np.asarray(teacher["a"], np.int64)[rows] >= k
                forced += int((fl & (t_ok != oks)).sum())
                oks = np.where(fl, t_ok, oks)
            ok[s] = oks
        a[idx[ok]] += 1
        rejected[idx[~ok]] = True
        done[idx[~ok]] = True
        done[idx[ok & (k == L[idx])]] = True
    # the final token: correction from the residual, or the bonus
    y = np.zeros(B, np.int64)
    y_flag = np.zeros(B, bool)
    allr = np.arange(B)
    if greedy.any():
        gi = allr[greedy]
        y[gi] = np.argmax(target[gi, a[gi]], axis=1)
    si = allr[~greedy]
    if len(si):
        wp, Zp, _ = softmax_parts(target[si, a[si]], tau[si])
        p = wp / Zp[:, None]
        rj = rejected[si]
        bon = si[~rj]
        if len(bon):
            u = uniform(seed, req[bon], a[bon] + 1, PURPOSE_BONUS, round_id)
            y[bon], _, y_flag[bon] = inverse_cdf(p[~rj], u)
        res = si[rj]
        if len(res):
            wq, Zq, _ = softmax_parts(d[res, a[res]], tau[res])
            resid = np.maximum(0.0, p[rj] - wq / Zq[:, None])
            u = uniform(seed, req[res], a[res] + 1, PURPOSE_RESIDUAL, round_id)
            zero = resid.sum(axis=1) <= 0
            yr, _, fr = inverse_cdf(resid, u, normalized=False)
            if zero.any():  # R8
                yp, _, fp = inverse_cdf(p[rj][zero], u[zero])
                yr[zero], fr[zero] = yp, fp
            y[res], y_flag[res] = yr, fr
    if teacher is not None and y_flag.any():
        ty = np.asarray(teacher["y"], np.int64)
        forced += int((y_flag & (ty != y)).sum())
        y = np.where(y_flag, ty, y)
    out, n_emit = emit(x, a, y)
    return dict(a=a, y=y, out=out, n_emit=n_emit, acc_flag=acc_flag, y_flag=y_flag,
                forced=forced)


def emit(x: np.ndarray, a: np.ndarray, y: np.ndarray):
    """out[b] = x_1..x_{a_b}, then y_b, then -1; n_emit = a_b + 1 ([P3] bonus token)."""
    B, K = x.shape
    pos = np.arange(K + 1)[None, :]
    xp = np.concatenate([x, np.zeros((B, 1), np.int64)], axis=1)
    out = np.where(pos < a[:, None], xp, -1)
    out[np.arange(B), a] = y
    return out, a + 1


# --------------------------------------------------------------------------
# the whole round
# --------------------------------------------------------------------------

def run_round(inp: Dict[str, np.ndarray], seed: int, round_id: int,
              mode: int = 0, threshold: float = 0.0,
              teacher: Optional[Dict[str, np.ndarray]] = None) -> Dict[str, np.ndarray]:
    """draft -> prefix cut -> verify -> emit for one round, in fp64.

    ``inp`` holds arrays exactly convertible to fp64. The per-request ones,
    target [B',K+1,V], base [B',K,V], last_tok, bias_scale, temp [B'], may
    cover a subset of the batch, named by request_ids [B'] (their indices
    in the full batch, which key their uniforms); the schedule's inputs,
    conf_logit [B,K], pos_temp [K], step_cost [B(K+1)], fixed_cost, cover
    the whole batch. Also U [V,r], W [r,V] and dtype. ``teacher`` (the GPU's d, x, L, a, y) switches
    on teacher forcing at flagged points; without it the round runs free.
    """
    dr = draft_round(inp, seed, round_id, teacher)
    c, S = survival(inp["conf_logit"], inp["pos_temp"])
    L, cut_flag = prefix_cut(S, inp["step_cost"], inp["fixed_cost"], mode, threshold)
    forced = dr["forced"]
    cut_forced = 0
    if cut_flag and teacher is not None:
        # only a cut that one flagged decision explains is adopted
        alts = cut_alternatives(S, inp["step_cost"], inp["fixed_cost"], mode, threshold)
        L, cut_forced = adopt_cut(L, alts, teacher["L"])
        forced += cut_forced
    rid = inp.get("request_ids")
    Lr = L if rid is None else L[np.asarray(rid, np.int64)]
    vr = verify(inp["target"], dr["d"], dr["x"], Lr, inp["temp"], seed, round_id, rid, teacher)
    forced += vr["forced"]
    return dict(draft=dr, c=c, S=S, L=L, cut_flag=cut_flag, cut_forced=cut_forced, verify=vr,
                forced=forced)
