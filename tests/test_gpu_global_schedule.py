"""spec_round.GlobalSchedule on the GPU: one prefix cut over several ranks'
requests. Two ranks are emulated on one GPU by handing each GlobalSchedule a
gather that stacks both ranks' confidence logits (no process group, no
collective); the host plumbing of the real all-gather is covered with gloo
ranks in tests/test_global_schedule_gloo.py."""
import numpy as np
import pytest
import torch

from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import replicas
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import GlobalSchedule, SpecRound, to_device

pytestmark = pytest.mark.gpu

W = wl.scaled(wl.DSPARK5, name="gsched_gpu", B=200, K=5, V=4096, cost_step_at=700)


def _rank_inputs(rank):
    return wl.generate(replicas.rank_workload(W, rank))


def test_two_emulated_ranks_take_their_slices_of_one_cut(cuda_ok):
    from oracle import dspark as o
    world = 2
    confs = [torch.as_tensor(_rank_inputs(r)["conf_logit"]).cuda() for r in range(world)]
    pos_temp = torch.as_tensor(_rank_inputs(0)["pos_temp"]).cuda()
    step_cost, fixed = wl.cost_table(W, W.B * world)
    gather = lambda c: torch.cat(confs, 0)
    # the combined batch's schedule in one call
    bg = W.B * world
    ws = torch.zeros(bn.workspace_bytes(bn.OP_SCHEDULE, bg, W.K, 0, 0, 0), dtype=torch.uint8,
                     device="cuda")
    cut_all = torch.empty(bg, dtype=torch.int32, device="cuda")
    surv_all = torch.empty((bg, W.K), dtype=torch.float32, device="cuda")
    bn.prefix_schedule(torch.cat(confs, 0), pos_temp, torch.as_tensor(step_cost).cuda(), fixed,
                       bn.CUT_COST, 0.0, cut_all, surv_all, ws)
    stream = torch.cuda.current_stream()
    for r in range(world):
        g = GlobalSchedule(W.B, W.K, step_cost, fixed, r, world, gather=gather)
        cut = torch.full((W.B,), -9, dtype=torch.int32, device="cuda")
        surv = torch.zeros((W.B, W.K), dtype=torch.float32, device="cuda")
        rws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        g.run(confs[r], pos_temp, bn.CUT_COST, 0.0, cut, surv, rws, stream)
        torch.cuda.synchronize()
        assert bn.read_status(rws) == (0, -1)
        assert torch.equal(cut, cut_all[r * W.B:(r + 1) * W.B])
        assert torch.equal(surv, surv_all[r * W.B:(r + 1) * W.B])
    # the combined cut against the oracle's (a flagged near-tie may explain a difference)
    conf_all = torch.cat(confs, 0).double().cpu().numpy()
    _, S = o.survival(conf_all, pos_temp.double().cpu().numpy())
    ref, near_tie = o.prefix_cut(S, np.asarray(step_cost, np.float64), fixed)
    got = cut_all.cpu().numpy()
    if not near_tie:
        assert np.array_equal(got, ref)
    # coupled: not the two per-engine cuts
    per_engine = []
    for r in range(world):
        sc, fx = wl.cost_table(W, W.B)
        _, Sr = o.survival(confs[r].double().cpu().numpy(), pos_temp.double().cpu().numpy())
        per_engine.append(o.prefix_cut(Sr, np.asarray(sc, np.float64), fx)[0])
    assert not np.array_equal(ref, np.concatenate(per_engine))


def test_one_rank_global_schedule_is_the_engine_schedule(cuda_ok):
    inp = _rank_inputs(0)
    dev = to_device(inp)
    step_cost, fixed = wl.cost_table(W, W.B)
    a = SpecRound(W.B, W.K, W.V, W.r)
    b = SpecRound(W.B, W.K, W.V, W.r)
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(main):
        a.run(dev, wl.PHILOX_SEED, 4, stream=main, side_stream=side)
        b.run(dev, wl.PHILOX_SEED, 4, stream=main, side_stream=side,
              global_schedule=GlobalSchedule(W.B, W.K, step_cost, fixed, 0, 1))
    torch.cuda.synchronize()
    assert a.status() == (0, -1) and b.status() == (0, -1)
    for name in ("x", "d", "cut", "survival", "accepted", "out", "n_emit"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_cost_table_length_is_checked(cuda_ok):
    step_cost, fixed = wl.cost_table(W, W.B)  # one rank's table, too short for two
    with pytest.raises(bn.DSparkError):
        GlobalSchedule(W.B, W.K, step_cost, fixed, 0, 2)
