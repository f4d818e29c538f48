"""Degenerate cases, device status reporting and argument errors of the C ABI."""
import numpy as np
import pytest
import torch

from parity import SEED, check_round, run_gpu
from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import SpecRound, to_device

pytestmark = pytest.mark.gpu


def _small(**kw):
    base = dict(name="edge", B=16, V=2048)
    base.update(kw)
    return wl.scaled(wl.DSPARK5, **base)


def test_identical_draft_full_acceptance_and_bonus(cuda_ok):
    w = _small(identical_frac=1.0)
    inp = wl.generate(w)
    rnd, _ = run_gpu(w, inp, 2, bn.CUT_NONE)
    check_round(w, inp, rnd, list(range(w.B)), 2, bn.CUT_NONE)
    assert np.all(rnd.accepted.cpu().numpy() == w.K)
    assert np.all(rnd.n_emit.cpu().numpy() == w.K + 1)


def test_independent_draft_residual_path(cuda_ok):
    w = _small(independent_frac=1.0)
    inp = wl.generate(w)
    rnd, _ = run_gpu(w, inp, 4, bn.CUT_NONE)
    check_round(w, inp, rnd, list(range(w.B)), 4, bn.CUT_NONE)
    assert rnd.accepted.float().mean().item() < 0.5


def test_greedy_exact_match(cuda_ok):
    w = _small(greedy_frac=1.0, B=32)
    inp = wl.generate(w)
    rnd, _ = run_gpu(w, inp, 0, bn.CUT_NONE)
    check_round(w, inp, rnd, list(range(w.B)), 0, bn.CUT_NONE)
    # greedy drafts are argmax d, greedy emission argmax of the target row
    d = rnd.d.float().cpu()
    assert torch.equal(rnd.x.cpu().long(), d.argmax(dim=2))


def test_zero_bias_equals_parallel_drafter(cuda_ok):
    """bias_scale = 0 gives d == round(base) exactly, and W = 0 the same draws."""
    w = _small(B=8)
    inp = wl.generate(w)
    dev = to_device(inp)
    dev["bias_scale"] = torch.zeros(w.B, device="cuda")
    rnd = SpecRound(w.B, w.K, w.V, w.r)
    rnd.run(dev, SEED, 0)
    assert torch.equal(rnd.d, dev["base"])
    dev2 = dict(dev, W=torch.zeros_like(dev["W"]), bias_scale=None)
    rnd2 = SpecRound(w.B, w.K, w.V, w.r)
    rnd2.run(dev2, SEED, 0)
    assert torch.equal(rnd2.d, rnd.d) and torch.equal(rnd2.x, rnd.x)


def test_status_bad_inputs(cuda_ok):
    w = _small(B=8)
    inp = wl.generate(w)
    dev = to_device(inp)
    rnd = SpecRound(w.B, w.K, w.V, w.r)
    # last committed token out of range
    bad = dict(dev, last_tok=dev["last_tok"].clone())
    bad["last_tok"][3] = w.V + 5
    rnd.run(bad, SEED, 0)
    code, first = rnd.status()
    assert code & bn.STATUS_BAD_TOKEN and first == 3
    # NaN in a target row of request 5 (row 0 is always read)
    bad = dict(dev, target=dev["target"].clone())
    bad["target"][5, 0, 17] = float("nan")
    rnd.run(bad, SEED, 0)
    code, first = rnd.status()
    assert code & bn.STATUS_BAD_ROW and first == 5
    assert rnd.n_emit[5].item() >= 1
    # negative temperature
    bad = dict(dev, temp=dev["temp"].clone())
    bad["temp"][6] = -1.0
    rnd.run(bad, SEED, 0)
    code, first = rnd.status()
    assert code & bn.STATUS_BAD_TEMP and first == 6
    # cut out of range, straight into verify
    rnd.run(dev, SEED, 0)
    assert rnd.status() == (0, -1)
    cut = rnd.cut.clone()
    cut[2] = w.K + 3
    bn.verify(dev["target"], rnd.d, rnd.x, rnd.q_tok, cut, dev["temp"], SEED, 0, rnd.accepted,
              rnd.out, rnd.n_emit, rnd.ws)
    code, first = rnd.status()
    assert code & bn.STATUS_BAD_CUT and first == 2
    # and a clean round afterwards reports nothing
    rnd.run(dev, SEED, 0)
    assert rnd.status() == (0, -1)


def test_argument_errors(cuda_ok):
    w = _small(B=4, V=1024)
    inp = wl.generate(w)
    dev = to_device(inp)
    rnd = SpecRound(w.B, w.K, w.V, w.r)
    # misaligned logits (2-byte offset view)
    flat = torch.empty(w.B * w.K * w.V + 8, dtype=torch.bfloat16, device="cuda")
    mis = flat[1:1 + w.B * w.K * w.V].view(w.B, w.K, w.V)
    with pytest.raises(bn.DSparkError, match="invalid argument"):
        bn.draft_sample(mis, dev["U"], dev["W"], None, dev["last_tok"], dev["temp"], SEED, 0,
                        rnd.x, rnd.d, rnd.q_lse, rnd.q_tok, rnd.ws)
    # workspace too small
    with pytest.raises(bn.DSparkError, match="workspace"):
        bn.draft_sample(dev["base"], dev["U"], dev["W"], None, dev["last_tok"], dev["temp"], SEED,
                        0, rnd.x, rnd.d, rnd.q_lse, rnd.q_tok, rnd.ws[:64])
    # V not a multiple of 8
    t = torch.zeros(w.B, w.K + 1, 1001, dtype=torch.bfloat16, device="cuda")
    dd = torch.zeros(w.B, w.K, 1001, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bn.DSparkError, match="invalid argument"):
        bn.verify(t, dd, rnd.x, rnd.q_tok, None, dev["temp"], SEED, 0, rnd.accepted, rnd.out,
                  rnd.n_emit, rnd.ws)
    # schedule larger than one CTA handles
    big = torch.zeros(4097, 4, device="cuda")   # B*K = 16388 > 16384
    with pytest.raises(bn.DSparkError, match="unsupported"):
        bn.prefix_schedule(big, torch.ones(4, device="cuda"), torch.ones(4097 * 5, device="cuda"),
                           0.0, bn.CUT_COST, 0.0, torch.empty(4097, dtype=torch.int32, device="cuda"),
                           torch.empty(4097, 4, device="cuda"), rnd.ws)
    assert rnd.status() == (0, -1)


def test_round_replay_is_deterministic(cuda_ok):
    w = _small(B=16)
    inp = wl.generate(w)
    rnd, dev = run_gpu(w, inp, 9)
    out1 = rnd.out.clone()
    rnd.run(dev, SEED, 9)
    assert torch.equal(rnd.out, out1)
    x1 = rnd.x.clone()
    rnd.run(dev, SEED, 10)  # a new round id draws new uniforms
    assert not torch.equal(rnd.x, x1)


def test_masked_vocabulary_is_not_an_error(cuda_ok):
    """Logits at -inf (masked tokens, here a quarter of the vocabulary spanning
    whole chunks and CTA slices) weigh nothing: no status bit, never drawn, and
    parity with the oracle holds."""
    w = _small(B=24, V=8192)
    inp = wl.generate(w)
    masked = torch.zeros(w.V, dtype=torch.bool)
    masked[1024:3072] = True
    masked[::7] = True
    inp["target"][:, :, masked] = float("-inf")
    inp["base"][:, :, masked] = float("-inf")
    for mode in (bn.CUT_COST, bn.CUT_NONE):
        rnd, _ = run_gpu(w, inp, 3, mode)
        check_round(w, inp, rnd, list(range(w.B)), 3, mode)
        out = rnd.out.cpu()
        emitted = out[out >= 0].long()
        assert not masked[emitted].any()
        assert not masked[rnd.x.cpu().long()].any()


@pytest.mark.parametrize("greedy_frac", [0.0, 0.5])
def test_split_draft_calls_match_draft_sample(cuda_ok, greedy_frac):
    """dspark_draft_logits(k) then dspark_draft_pick(k) for k = 1..K gives
    exactly dspark_draft_sample's outputs (tensor-core path at r = 256 and the
    CUDA-core path at r = 272)."""
    for r in (256, 272):
        w = _small(B=130, V=4096, r=r, greedy_frac=greedy_frac)
        inp = wl.generate(w)
        dev = to_device(inp)
        rnd = SpecRound(w.B, w.K, w.V, w.r)
        rnd.run(dev, SEED, 3)
        x = torch.full_like(rnd.x, -7)
        d = torch.zeros_like(rnd.d)
        q_lse = torch.zeros_like(rnd.q_lse)
        q_tok = torch.zeros_like(rnd.q_tok)
        ws = torch.zeros_like(rnd.ws)
        for k in range(1, w.K + 1):
            bn.draft_logits(dev["base"], dev["U"], dev["W"], dev["bias_scale"], dev["last_tok"], x,
                            dev["temp"], k, d, ws)
            bn.draft_pick(d, dev["last_tok"], dev["temp"], SEED, 3, k, x, q_lse, q_tok, ws)
        torch.cuda.synchronize()
        assert bn.read_status(ws) == (0, -1)
        assert torch.equal(d, rnd.d) and torch.equal(x, rnd.x)
        assert torch.equal(q_lse, rnd.q_lse) and torch.equal(q_tok, rnd.q_tok)
        with pytest.raises(bn.DSparkError):
            bn.draft_logits(dev["base"], dev["U"], dev["W"], dev["bias_scale"], dev["last_tok"], x,
                            dev["temp"], w.K + 1, d, ws)
        with pytest.raises(bn.DSparkError):
            bn.draft_pick(d, dev["last_tok"], dev["temp"], SEED, 3, 0, x, q_lse, q_tok, ws)


def test_schedule_on_side_stream_matches_one_stream(cuda_ok):
    """The prefix schedule issued on a side stream, concurrently with the draft
    (sharing the workspace), gives the same round as one stream."""
    w = _small(B=200, V=8192)
    inp = wl.generate(w)
    dev = to_device(inp)
    a = SpecRound(w.B, w.K, w.V, w.r)
    a.run(dev, SEED, 5)
    b = SpecRound(w.B, w.K, w.V, w.r)
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(main):
        b.run(dev, SEED, 5, stream=main, side_stream=side)
    torch.cuda.synchronize()
    assert a.status() == (0, -1) and b.status() == (0, -1)
    for name in ("x", "d", "q_tok", "cut", "survival", "accepted", "out", "n_emit"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_round_replayed_as_a_cuda_graph_matches_eager(cuda_ok):
    """The round captured as a CUDA graph (the one-launch draft kernel with its
    barrier-counter memset, the schedule on a forked side stream, verify) gives
    the eager round's outputs on every replay."""
    w = _small(B=150, V=8192, greedy_frac=0.2)
    inp = wl.generate(w)
    dev = to_device(inp)
    eager = SpecRound(w.B, w.K, w.V, w.r)
    eager.run(dev, SEED, 9)
    torch.cuda.synchronize()
    rnd = SpecRound(w.B, w.K, w.V, w.r)
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(main):
        rnd.run(dev, SEED, 9, stream=main, side_stream=side)  # warm-up outside capture
        main.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=main):
            rnd.run(dev, SEED, 9, stream=main, side_stream=side)
        for _ in range(3):
            rnd.out.fill_(-9)
            g.replay()
            main.synchronize()
            for name in ("x", "d", "q_tok", "cut", "accepted", "out", "n_emit"):
                assert torch.equal(getattr(rnd, name), getattr(eager, name)), name
    assert rnd.status() == (0, -1)
    del g


def test_verify_with_and_without_the_draft_normalisers(cuda_ok):
    """dspark_verify given the draws' normalisers (q_norm) and recomputing them
    (NULL) take the same decisions and emit the same tokens."""
    w = _small(B=160, V=8192, independent_frac=0.3, greedy_frac=0.1)
    inp = wl.generate(w)
    dev = to_device(inp)
    rnd = SpecRound(w.B, w.K, w.V, w.r)
    rnd.run(dev, SEED, 4)
    acc2, out2, n2 = torch.empty_like(rnd.accepted), torch.empty_like(rnd.out), torch.empty_like(rnd.n_emit)
    bn.verify(dev["target"], rnd.d, rnd.x, rnd.q_tok, rnd.cut, dev["temp"], SEED, 4, acc2, out2, n2,
              rnd.ws)
    torch.cuda.synchronize()
    assert rnd.status() == (0, -1)
    assert (rnd.accepted < rnd.cut).any()  # some residual draws happen
    assert torch.equal(acc2, rnd.accepted) and torch.equal(out2, rnd.out) and torch.equal(n2, rnd.n_emit)
    # the normalisers are those of the stored draft logits: q_tok = 2^(d_x cs - m) / s
    qn = rnd.q_norm.cpu().double().numpy()
    d = rnd.d.float().cpu().double().numpy()
    x = rnd.x.cpu().numpy()
    tau = dev["temp"].cpu().double().numpy()
    for b in range(0, w.B, 17):
        if tau[b] > 0:
            cs = 1.4426950408889634 / tau[b]
            for k in range(w.K):
                q = 2.0 ** (d[b, k, x[b, k]] * cs - qn[b, k, 0]) / qn[b, k, 1]
                assert abs(q - rnd.q_tok[b, k].item()) <= 1e-5 * max(q, 1e-30)
                # and the log normaliser: ln sum exp(d / temp) = (max + log2 sum) ln 2
                lse = (qn[b, k, 0] + np.log2(qn[b, k, 1])) * np.log(2.0)
                ql = rnd.q_lse[b, k].item()
                assert abs(lse - ql) <= 1e-5 * max(1.0, abs(ql)), (b, k, lse, ql)
