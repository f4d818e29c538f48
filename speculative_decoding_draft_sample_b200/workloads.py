"""Seeded synthetic workloads for one speculative round.

This module only draws random inputs; it holds none of the method's
arithmetic (no softmax, no sampling, no scheduling), so that the CUDA path
and the CPU oracle can both consume the very same bytes.

The shapes and value recipes follow the workloads described for the
drafter/verifier (a parallel drafter's base logits that decay along the
block, a target model's logits, a rank-256 Markov head, confidence logits
and a profiled cost-per-verified-token table). The pages measure on math,
code and chat datasets and on live traffic; none of that is available here,
so these seeded Zipf-plus-noise logits stand in for them.

Every request's rows are drawn from their own seeded stream
``(seed, request)``, so a subset of requests can be regenerated cheaply
and bit-identically (used to check sampled requests of the large cases).
"""
from __future__ import annotations

import dataclasses
import os
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic round: sizes and the recipe for every input."""

    name: str
    B: int                     # requests in the batch
    K: int                     # drafted positions per request
    V: int                     # vocabulary size
    r: int                     # Markov-head rank
    dtype: str                 # storage type of logits, U and W
    target_kind: str           # "normal" (N(0, target_std^2)) or "zipf" (Zipf log-probs + noise)
    target_std: float          # std of the target logits ("normal") or of the noise ("zipf")
    zipf_s: float              # Zipf exponent for "zipf"
    draft_noise0: float        # draft noise std at position k = 1
    draft_noise_step: float    # growth of the draft noise std per position
    uw_std: float              # std of the Markov factors U and W
    conf_mean: float           # confidence logits ~ N(conf_mean, conf_std^2)
    conf_std: float
    pos_temp_lo: float         # per-position temperatures linspace(lo, hi, K)
    pos_temp_hi: float
    temps: Sequence[float]     # per-request sampling temperatures drawn uniformly from this set
    greedy_frac: float         # fraction of requests with temperature 0
    identical_frac: float      # fraction whose draft base equals the target rows (bias scale 0)
    independent_frac: float    # fraction whose draft base is independent N(0, 2^2)
    cost_kind: str             # "flat", "linear" or "step"
    cost_step_at: int = 512    # for "step": verified-token count after which the cost rises
    cost_step_hi: float = 1.5  # for "step": per-token cost above the step
    fixed_cost: Optional[float] = None  # None: B (one slot per request is always verified)
    seed: int = 0

    @property
    def nbytes_per_logit(self) -> int:
        return 4 if self.dtype == F32 else 2

    def draft_noise(self, k: int) -> float:
        """Noise std of draft position k (1-based)."""
        return self.draft_noise0 + self.draft_noise_step * (k - 1)


def _zipf_defaults(**kw):
    d = dict(target_kind="zipf", target_std=0.5, zipf_s=1.1, draft_noise0=0.8,
             draft_noise_step=0.2, uw_std=0.05, conf_mean=1.5, conf_std=1.0,
             pos_temp_lo=1.0, pos_temp_hi=1.6, temps=(1.0,), greedy_frac=0.0,
             identical_frac=0.0, independent_frac=0.0, dtype=BF16, r=256)
    d.update(kw)
    return d


TINY = Workload(name="tiny_b4_k4_v1024_f32", B=4, K=4, V=1024, r=16, dtype=F32,
                target_kind="normal", target_std=2.0, zipf_s=0.0, draft_noise0=1.0,
                draft_noise_step=0.0, uw_std=0.1, conf_mean=1.5, conf_std=1.0,
                pos_temp_lo=1.0, pos_temp_hi=1.6, temps=(1.0,), greedy_frac=0.0,
                identical_frac=0.0, independent_frac=0.0, cost_kind="flat")

QWEN3 = Workload(name="qwen3_b64_k5_v151936", B=64, K=5, V=151936,
                 cost_kind="linear", **_zipf_defaults())

DSPARK5 = Workload(name="dspark5_b256_k5_v129280", B=256, K=5, V=129280,
                   cost_kind="step", cost_step_at=512, cost_step_hi=1.5,
                   **_zipf_defaults(temps=(0.6, 0.8, 1.0)))


def sweep(K: int) -> Workload:
    return Workload(name=f"sweep_b128_k{K}_v151936", B=128, K=K, V=151936,
                    cost_kind="flat", **_zipf_defaults(draft_noise_step=0.15))


STRESS = Workload(name="stress_b1024_k8_v151936", B=1024, K=8, V=151936,
                  cost_kind="flat",
                  **_zipf_defaults(conf_mean=0.5, conf_std=1.5, greedy_frac=0.25,
                                   identical_frac=0.05, independent_frac=0.05))

ALL = {w.name: w for w in [TINY, QWEN3, DSPARK5, sweep(4), sweep(8), sweep(12), sweep(16), STRESS]}

# Seed for the round's Philox stream (the uniforms of sampling and acceptance).
PHILOX_SEED = 1234


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some sizes changed (for small parity cases)."""
    return dataclasses.replace(w, **changes)


def _request_kinds(w: Workload) -> Dict[str, np.ndarray]:
    rng = np.random.default_rng([w.seed, 7, 0])
    perm = rng.permutation(w.B)
    n_id = int(round(w.identical_frac * w.B))
    n_ind = int(round(w.independent_frac * w.B))
    identical = np.zeros(w.B, bool)
    independent = np.zeros(w.B, bool)
    identical[perm[:n_id]] = True
    independent[perm[n_id:n_id + n_ind]] = True
    return {"identical": identical, "independent": independent}


def _zipf_logp(w: Workload) -> np.ndarray:
    rng = np.random.default_rng([w.seed, 7, 1])
    perm = rng.permutation(w.V)
    ranks = np.arange(1, w.V + 1, dtype=np.float64)
    mass = ranks ** (-w.zipf_s)
    logp = np.log(mass / mass.sum())
    out = np.empty(w.V, np.float64)
    out[perm] = logp
    return out


def _to_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t if dtype == F32 else t.to(torch.bfloat16)


def request_rows(w: Workload, b: int, zipf_logp: Optional[np.ndarray] = None,
                 kinds: Optional[Dict[str, np.ndarray]] = None):
    """Target rows [K+1, V] and draft base rows [K, V] of request ``b`` (storage dtype)."""
    if kinds is None:
        kinds = _request_kinds(w)
    rng = np.random.default_rng([w.seed, 11, b])
    V, K = w.V, w.K
    if w.target_kind == "normal":
        t = rng.standard_normal((K + 1, V), dtype=np.float32) * np.float32(w.target_std)
    else:
        if zipf_logp is None:
            zipf_logp = _zipf_logp(w)
        t = rng.standard_normal((K + 1, V), dtype=np.float32) * np.float32(w.target_std)
        t += zipf_logp.astype(np.float32)[None, :]
    t_st = _to_storage(t, w.dtype)
    if kinds["identical"][b]:
        base_st = t_st[:K].clone()
    elif kinds["independent"][b]:
        base = rng.standard_normal((K, V), dtype=np.float32) * np.float32(2.0)
        base_st = _to_storage(base, w.dtype)
    else:
        # draft position k (1-based) is scored by target row k-1
        t_f = t_st[:K].float().numpy()
        noise = rng.standard_normal((K, V), dtype=np.float32)
        scale = np.array([w.draft_noise(k) for k in range(1, K + 1)], np.float32)[:, None]
        base_st = _to_storage(t_f + noise * scale, w.dtype)
    return t_st, base_st


def small_inputs(w: Workload) -> Dict[str, object]:
    """Everything except the [B, K(+1), V] logits: factors, temperatures, tables."""
    B, K, V, r = w.B, w.K, w.V, w.r
    kinds = _request_kinds(w)
    rng = np.random.default_rng([w.seed, 13])
    U = _to_storage(rng.standard_normal((V, r), dtype=np.float32) * np.float32(w.uw_std), w.dtype)
    W = _to_storage(rng.standard_normal((r, V), dtype=np.float32) * np.float32(w.uw_std), w.dtype)
    last_tok = rng.integers(0, V, size=B).astype(np.int32)
    temps = np.asarray(w.temps, np.float32)
    temp = temps[rng.integers(0, len(temps), size=B)].astype(np.float32)
    if w.greedy_frac > 0:
        perm = rng.permutation(B)
        temp[perm[: int(round(w.greedy_frac * B))]] = 0.0
    bias_scale = np.ones(B, np.float32)
    bias_scale[kinds["identical"]] = 0.0
    conf_logit = (w.conf_mean + w.conf_std * rng.standard_normal((B, K))).astype(np.float32)
    pos_temp = np.linspace(w.pos_temp_lo, w.pos_temp_hi, K).astype(np.float32)
    step_cost, fixed_cost = cost_table(w, B)
    return dict(U=U, W=W, last_tok=last_tok, temp=temp, bias_scale=bias_scale,
                conf_logit=conf_logit, pos_temp=pos_temp, step_cost=step_cost,
                fixed_cost=fixed_cost, identical=kinds["identical"],
                independent=kinds["independent"])


def cost_table(w: Workload, B: int) -> Tuple[np.ndarray, float]:
    """The workload's cost per verified token, step_cost[n - 1] for the n-th
    verified token of a batch of B requests (B(K+1) entries), and its fixed
    cost (B unless the workload sets one: one slot per request is always
    verified). A schedule over several engines' requests takes the table of
    their combined batch."""
    n_slots = B * (w.K + 1)
    n = np.arange(1, n_slots + 1, dtype=np.float64)  # 1-based verified-token count
    if w.cost_kind == "flat":
        step_cost = np.ones(n_slots, np.float32)
    elif w.cost_kind == "linear":
        step_cost = (0.5 + n / n_slots).astype(np.float32)
    elif w.cost_kind == "step":
        step_cost = np.where(n <= w.cost_step_at, 1.0, w.cost_step_hi).astype(np.float32)
    else:
        raise ValueError(w.cost_kind)
    return step_cost, float(B if w.fixed_cost is None else w.fixed_cost)


def recurrent_factor(w: Workload, std: float = 1.0) -> torch.Tensor:
    """A seeded state matrix R [r, r] for the recurrent head, N(0, std^2), in
    the workload's storage dtype. With U ~ N(0, uw_std^2) the pre-activation
    h @ R of the first states has std sqrt(r) * uw_std * std (0.8 at r = 256,
    uw_std = 0.05, std = 1): tanh neither linear nor saturated."""
    rng = np.random.default_rng([w.seed, 17])
    return _to_storage(rng.standard_normal((w.r, w.r), dtype=np.float32) * np.float32(std), w.dtype)


def generate(w: Workload, requests: Optional[List[int]] = None) -> Dict[str, object]:
    """The full round's inputs (CPU tensors in storage dtype), or only ``requests``' rows.

    ``target`` is [B', K+1, V] and ``base`` [B', K, V] for the B' requested rows
    (all B by default); the small inputs always cover the whole batch.
    """
    out = small_inputs(w)
    reqs = list(range(w.B)) if requests is None else list(requests)
    kinds = {"identical": out["identical"], "independent": out["independent"]}
    zl = _zipf_logp(w) if w.target_kind == "zipf" else None
    tdt = torch.float32 if w.dtype == F32 else torch.bfloat16
    target = torch.empty((len(reqs), w.K + 1, w.V), dtype=tdt)
    base = torch.empty((len(reqs), w.K, w.V), dtype=tdt)

    def fill(i_b):
        i, b = i_b
        t, bs = request_rows(w, b, zl, kinds)
        target[i] = t
        base[i] = bs

    if len(reqs) >= 16:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, enumerate(reqs)))
    else:
        for ib in enumerate(reqs):
            fill(ib)
    out.update(target=target, base=base, requests=reqs)
    return out


# ---------------------------------------------------------------------------
# Calibration data for Sequential Temperature Scaling: a synthetic confidence
# head that is over-confident by a factor gamma_k at position k. Latent
# per-position survival probabilities pi = sigmoid(mu_k + 1.2 eps), labels
# survived[n, k] = survived[n, k-1] and Bernoulli(pi[n, k]), confidence
# logits z = gamma_k * logit(pi) (so that z / gamma_k is calibrated).
# ---------------------------------------------------------------------------
CALIB_GAMMAS = (1.6, 1.9, 2.2, 2.5, 2.8)


def calib_inputs(N: int, K: int = 5, gammas=CALIB_GAMMAS, seed: int = 3):
    rng = np.random.default_rng([seed, 29])
    mu = 1.0 - 0.25 * np.arange(K)
    logit_pi = mu[None, :] + 1.2 * rng.standard_normal((N, K))
    pi = 1.0 / (1.0 + np.exp(-logit_pi))
    draw = rng.random((N, K)) < pi
    survived = np.cumprod(draw, axis=1).astype(np.uint8)
    z = (np.asarray(gammas[:K], np.float64)[None, :] * logit_pi).astype(np.float32)
    return z, survived
