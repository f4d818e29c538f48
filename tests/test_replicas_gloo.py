"""Multi-GPU host logic on CPU with two gloo ranks (no GPU): every rank runs its
own batch with no exchange on the data path, and only the timing bookkeeping
(barrier, MAX and SUM over ranks) is collective."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from speculative_decoding_draft_sample_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _round_for(w):
    from oracle import dspark as o
    inp = wl.generate(w)
    f = lambda t: t.double().numpy()
    oi = dict(target=f(inp["target"]), base=f(inp["base"]), U=f(inp["U"]), W=f(inp["W"]),
              last_tok=np.asarray(inp["last_tok"]), bias_scale=np.asarray(inp["bias_scale"], np.float64),
              temp=np.asarray(inp["temp"], np.float64), conf_logit=np.asarray(inp["conf_logit"], np.float64),
              pos_temp=np.asarray(inp["pos_temp"], np.float64),
              step_cost=np.asarray(inp["step_cost"], np.float64), fixed_cost=float(inp["fixed_cost"]),
              dtype=w.dtype)
    r = o.run_round(oi, wl.PHILOX_SEED, 0)
    return r["verify"]["out"], float(np.asarray(inp["target"].float().sum()))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from speculative_decoding_draft_sample_b200 import replicas
    world_, rank_, _ = replicas.init("gloo", timeout_s=60)
    w = replicas.rank_workload(wl.scaled(wl.DSPARK5, name="rep", B=6, K=3, V=512), rank_)
    out, tsum = _round_for(w)          # this rank's batch, no exchange
    replicas.barrier()
    mx = replicas.max_over_ranks(float(rank_ + 1))
    sm = replicas.sum_over_ranks(float(out.sum()))
    replicas.finish()
    q.put((rank_, world_, out, tsum, mx, sm))


def test_two_gloo_ranks_independent_batches():
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
    (r0, w0, out0, t0, mx0, sm0), (r1, w1, out1, t1, mx1, sm1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert t0 != t1                    # different batches on the two ranks
    assert mx0 == mx1 == 2.0           # MAX over ranks
    assert sm0 == sm1 == float(out0.sum() + out1.sum())  # SUM over ranks
    # a rank's result is exactly what one process computes for that batch alone
    from speculative_decoding_draft_sample_b200 import replicas
    base = wl.scaled(wl.DSPARK5, name="rep", B=6, K=3, V=512)
    for r, out in ((0, out0), (1, out1)):
        ref, _ = _round_for(replicas.rank_workload(base, r))
        assert np.array_equal(out, ref)


def _worker_leaves(rank, world, port, q):
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from speculative_decoding_draft_sample_b200 import replicas
    replicas.init("gloo", timeout_s=5)
    if rank == 1:          # leaves between steps, with nothing in flight
        q.put((1, "left", 0.0))
        return
    t0 = time.monotonic()
    try:
        replicas.barrier()  # the next collective of the timing bookkeeping
        q.put((0, "no error", time.monotonic() - t0))
    except Exception as e:  # noqa: BLE001 - any error ends the wait; a hang would not
        q.put((0, type(e).__name__, time.monotonic() - t0))


def test_a_rank_that_leaves_is_detected_not_waited_for():
    """A rank that exits between steps makes the other rank's next collective
    fail within the process group's short timeout instead of hanging it."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_leaves, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (what, dt)) for r, what, dt in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
    assert res[1][0] == "left"
    what, dt = res[0]
    assert what != "no error" and dt < 60.0, res
