"""The recurrent sequential head on the GPU (dspark_draft_sample_recurrent)
against the fp64 oracle's reading of it, and against the Markov head.

The reading (the pages give no equations; "DSpark turns speculation into a
scheduler", "DSpark's semi-autoregressive compromise"; "DSpark LLM inference
speedup", "The Semi-Autoregressive Trick"): h_1 = U[x_0],
h_k = round(U[x_{k-1}] + tanh(h_{k-1} @ R)), bias_k = scale_b * h_k @ W.
R = 0 must reproduce the Markov head bit for bit; otherwise the states, the
draft and the whole round are checked element by element, teacher-forced at
the points the oracle flags (a state or logit at a bf16 rounding midpoint, a
draw or acceptance at its boundary)."""
import numpy as np
import pytest
import torch

from parity import check_round, run_gpu
from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import SpecRound, to_device

pytestmark = pytest.mark.gpu

CASES = [
    wl.scaled(wl.DSPARK5, name="rnn_dspark5_small", B=24, V=8200),                  # one-launch tcgen05 path
    wl.scaled(wl.STRESS, name="rnn_stress_small", B=200, K=8, V=2056),              # two M-tiles, greedy mix
    wl.scaled(wl.DSPARK5, name="rnn_f32_small", B=12, V=3000 // 8 * 8, dtype=wl.F32, r=32),  # CUDA-core path
    wl.scaled(wl.DSPARK5, name="rnn_bf16_r512", B=10, K=3, V=2048, r=512),          # CUDA-core path, bf16
    # one-launch path with more drawn rows per CTA than its eight drawing warps
    # (10 groups of 128 requests on 140 CTAs: rows past 8 x 140 = 1120)
    wl.scaled(wl.DSPARK5, name="rnn_many_rows", B=1200, K=3, V=2048),
]


def _with_R(w, std=1.0):
    inp = wl.generate(w)
    inp["R"] = wl.recurrent_factor(w, std)
    return inp


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_recurrent_round_all_requests(cuda_ok, w):
    inp = _with_R(w)
    for round_id in (0, 1):
        rnd, _ = run_gpu(w, inp, round_id)
        stats = check_round(w, inp, rnd, list(range(w.B)), round_id)
        # decisions adopted at flagged points stay rare; fp32 states round
        # differently from the fp64 ones at about a few per thousand elements
        assert stats["forced"] <= 3 + w.B * w.K // 10, stats
        assert stats["h_forced"] <= 4 + w.B * w.K * w.r // 100, stats


def test_recurrent_full_size_sampled_requests(cuda_ok):
    w = wl.DSPARK5
    inp = _with_R(w)
    rnd, _ = run_gpu(w, inp, 0)
    reqs = sorted({0, 127, 128, 255} | set(np.random.default_rng(1).choice(w.B, 12, replace=False).tolist()))
    stats = check_round(w, inp, rnd, reqs, 0)
    print("recurrent dspark5", stats)


def test_zero_state_matrix_is_the_markov_head(cuda_ok):
    """R = 0: the draft equals dspark_draft_sample's bit for bit and the states
    are the gathered U rows."""
    w = wl.scaled(wl.DSPARK5, name="rnn_zero", B=40, V=4096)
    inp = wl.generate(w)
    dev = to_device(inp)
    mk = SpecRound(w.B, w.K, w.V, w.r)
    mk.run(dev, wl.PHILOX_SEED, 3)
    rc = SpecRound(w.B, w.K, w.V, w.r)
    rc.run(dict(dev, R=torch.zeros((w.r, w.r), dtype=torch.bfloat16, device="cuda")), wl.PHILOX_SEED, 3)
    torch.cuda.synchronize()
    assert mk.status() == (0, -1) and rc.status() == (0, -1)
    for name in ("x", "d", "q_tok", "q_lse", "out", "accepted"):
        assert torch.equal(getattr(mk, name), getattr(rc, name)), name
    prev = torch.cat([dev["last_tok"][:, None].long(), mk.x[:, :-1].long()], dim=1)
    assert torch.equal(rc.h, dev["U"][prev])
