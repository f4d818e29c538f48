"""Helpers for comparing the CUDA path (through the C ABI) with the fp64 oracle.

Parity rules (teacher-forced mode): the oracle runs on the same inputs and,
where the CUDA path's own outputs feed a later stage (d, x, cut), on those
outputs; at a point it flags (a uniform within 1e-6 of a CDF or acceptance
boundary, a stored logit within fp32 error of a bf16 rounding midpoint, a
near-tie of the cut) it adopts the GPU's decision. Everything else must match
exactly: tokens, cuts, accepted lengths, emitted rows, and stored bf16 logits;
normalisers, probabilities and survival products within 1e-5 relative.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np
import torch

from oracle import dspark as o
from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import SpecRound, to_device

RTOL = 1e-5
SEED = wl.PHILOX_SEED


def torch_dtype(w: wl.Workload):
    return torch.float32 if w.dtype == wl.F32 else torch.bfloat16


def run_gpu(w: wl.Workload, inp: Dict[str, object], round_id: int, mode: int = bn.CUT_COST,
            threshold: float = 0.0, dev: Optional[Dict[str, object]] = None):
    """The whole round through the C ABI; returns (SpecRound, device inputs)."""
    dev = dev or to_device(inp)
    rnd = SpecRound(w.B, w.K, w.V, w.r, torch_dtype(w))
    rnd.run(dev, SEED, round_id, mode, threshold)
    torch.cuda.synchronize()
    code, first = rnd.status()
    assert code == 0, (code, first)
    return rnd, dev


def oracle_inputs(w: wl.Workload, inp: Dict[str, object], requests: List[int]) -> Dict[str, object]:
    """fp64 oracle inputs for the given requests (rows located by inp['requests'])."""
    pos = {b: i for i, b in enumerate(inp["requests"])}
    rows = [pos[b] for b in requests]
    req = np.asarray(requests, np.int64)
    f = lambda t: t.double().numpy()
    extra = {} if inp.get("R") is None else dict(R=f(inp["R"]))
    return dict(target=f(inp["target"][rows]), base=f(inp["base"][rows]), U=f(inp["U"]),
                W=f(inp["W"]), **extra, last_tok=np.asarray(inp["last_tok"])[req],
                bias_scale=np.asarray(inp["bias_scale"], np.float64)[req],
                temp=np.asarray(inp["temp"], np.float64)[req],
                conf_logit=np.asarray(inp["conf_logit"], np.float64),
                pos_temp=np.asarray(inp["pos_temp"], np.float64),
                step_cost=np.asarray(inp["step_cost"], np.float64),
                fixed_cost=float(np.float32(inp["fixed_cost"])), dtype=w.dtype, request_ids=req)


def gpu_outputs(rnd: SpecRound, requests: List[int]) -> Dict[str, np.ndarray]:
    idx = torch.as_tensor(requests, device=rnd.x.device, dtype=torch.long)
    a = rnd.accepted[idx].cpu().numpy().astype(np.int64)
    out = rnd.out[idx].cpu().numpy().astype(np.int64)
    h = None if rnd.h is None else rnd.h[idx].double().cpu().numpy()
    return dict(h=h, x=rnd.x[idx].cpu().numpy().astype(np.int64),
                d=rnd.d[idx].double().cpu().numpy(),
                q_lse=rnd.q_lse[idx].double().cpu().numpy(),
                q_tok=rnd.q_tok[idx].double().cpu().numpy(),
                a=a, out=out, y=out[np.arange(len(requests)), a],
                n_emit=rnd.n_emit[idx].cpu().numpy().astype(np.int64),
                L=rnd.cut.cpu().numpy().astype(np.int64),
                S=rnd.survival.double().cpu().numpy())


def check_round(w: wl.Workload, inp: Dict[str, object], rnd: SpecRound, requests: List[int],
                round_id: int, mode: int = bn.CUT_COST, threshold: float = 0.0) -> Dict[str, int]:
    """Teacher-forced parity of every stage on ``requests``; returns counts."""
    g = gpu_outputs(rnd, requests)
    oi = oracle_inputs(w, inp, requests)
    teacher = dict(d=g["d"], x=g["x"], L=g["L"], a=g["a"], y=g["y"], h=g["h"])
    thr = float(np.float32(threshold))
    r = o.run_round(oi, SEED, round_id, mode, thr, teacher=teacher)
    dr = r["draft"]
    # the recurrent head's states: exact in bf16 outside flagged elements (the
    # oracle adopted the GPU's state there), fp32 within rounding of tanh
    if g["h"] is not None:
        if w.dtype == wl.BF16:
            assert np.array_equal(dr["h"], g["h"]), "recurrent states differ outside flagged points"
        else:  # each fp32 state from the device's previous one, within fp32 error
            assert dr["h_excess"] <= 0.0, dr["h_excess"]
    # draft: stored logits, tokens, normalisers
    if w.dtype == wl.BF16:
        assert np.array_equal(dr["d"], g["d"]), "stored draft logits differ outside flagged points"
    else:
        np.testing.assert_allclose(g["d"], dr["d"], rtol=2.0 ** -21, atol=1e-6)
    assert np.array_equal(dr["x"], g["x"]), "drafted tokens differ"
    np.testing.assert_allclose(g["q_tok"], dr["q_tok"], rtol=RTOL)
    np.testing.assert_allclose(g["q_lse"], dr["q_lse"], rtol=RTOL, atol=1e-6)
    # schedule: the whole batch's cut. At a flagged near-tie the oracle adopts
    # the GPU's cut only if one flipped decision explains it (cut_alternatives),
    # so every request the flip does not touch is still compared with the oracle
    np.testing.assert_allclose(g["S"], r["S"], rtol=RTOL)
    assert np.array_equal(r["L"], g["L"]), "prefix cuts differ"
    # verify + emit
    vr = r["verify"]
    assert np.array_equal(vr["a"], g["a"]), "accepted lengths differ"
    assert np.array_equal(vr["out"], g["out"]), "emitted tokens differ"
    assert np.array_equal(vr["n_emit"], g["n_emit"])
    return dict(forced=int(r["forced"]), h_flags=int(dr["h_flag"].sum()),
                h_forced=int(dr["h_forced"]) if w.dtype == wl.BF16 else 0,
                cut_flag=bool(r["cut_flag"]),
                cut_forced=int(r["cut_forced"]), d_flags=int(dr["d_flag"].sum()),
                x_flags=int(dr["x_flag"].sum()), acc_flags=int(vr["acc_flag"].sum()),
                y_flags=int(vr["y_flag"].sum()), accepted=int(g["a"].sum()))
