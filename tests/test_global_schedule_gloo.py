"""One prefix schedule over every rank's requests (spec_round.GlobalSchedule),
host plumbing on CPU with two gloo ranks (no GPU).

Each rank holds its own confidence logits; replicas.all_gather_rows stacks
them in rank order on every rank, the cut of the combined batch is taken
against the combined batch's cost table, and each rank keeps the slice of its
own requests. The cut here comes from the oracle (test infrastructure): the
GPU kernel that computes it in the product is checked against the oracle in
tests/test_gpu_schedule.py, and GlobalSchedule's own slicing on the GPU in
tests/test_gpu_global_schedule.py."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

from speculative_decoding_draft_sample_b200 import workloads as wl

W = wl.scaled(wl.DSPARK5, name="gsched", B=40, K=5, V=512, cost_step_at=150)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _conf(rank):
    from speculative_decoding_draft_sample_b200 import replicas
    return wl.generate(replicas.rank_workload(W, rank))["conf_logit"]


def _cut_of(conf, pos_temp, B):
    from oracle import dspark as o
    step_cost, fixed = wl.cost_table(W, B)
    _, S = o.survival(np.asarray(conf, np.float64), np.asarray(pos_temp, np.float64))
    L, _near_tie = o.prefix_cut(S, np.asarray(step_cost, np.float64), fixed)
    return L


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from speculative_decoding_draft_sample_b200 import replicas
    world_, rank_, _ = replicas.init("gloo", timeout_s=60)
    conf = torch.as_tensor(_conf(rank_))
    gathered = replicas.all_gather_rows(conf)
    pos_temp = wl.generate(W)["pos_temp"]
    cut_all = _cut_of(gathered.numpy(), pos_temp, W.B * world_)
    mine = cut_all[rank_ * W.B:(rank_ + 1) * W.B]
    replicas.finish()
    q.put((rank_, gathered.numpy(), mine))


def test_two_ranks_share_one_cut():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, g0, cut0), (r1, g1, cut1) = res
    assert (r0, r1) == (0, 1)
    # the gather is the same on both ranks and in rank order
    both = np.concatenate([_conf(0), _conf(1)], 0)
    assert np.array_equal(g0, both) and np.array_equal(g1, both)
    # each rank's slice is its part of the cut one process computes for the combined batch
    pos_temp = wl.generate(W)["pos_temp"]
    ref = _cut_of(both, pos_temp, 2 * W.B)
    assert np.array_equal(cut0, ref[:W.B]) and np.array_equal(cut1, ref[W.B:])
    # and the combined schedule is not two per-engine ones: the cost table couples the ranks
    per_engine = np.concatenate([_cut_of(_conf(0), pos_temp, W.B), _cut_of(_conf(1), pos_temp, W.B)])
    assert not np.array_equal(ref, per_engine)
